// h3blk_attention_noalloc: the block's document-masked attention for callers
// that cannot allocate device memory.
//
// Who needs this: code that is not allowed to call cudaMalloc at run time --
// for example a plugin living inside a host application whose own memory pool
// already owns the GPU's memory, or a latency-critical loop where the implicit
// device-wide synchronisation of cudaMalloc / cudaFree is unacceptable. The
// regular path needs a caller-provided workspace; this entry point instead
// keeps its scratch (the per-128-row tile summary the attention kernel reads,
// and the device error word) in a fixed array that lives in the library's own
// device memory.
//
// Costs and rules of that array:
//   * it is kNoAllocScratchBytes (about 128 KiB) and every GPU that loads the
//     library holds it until the process exits;
//   * sequences longer than kNoAllocMaxRows rows are rejected with
//     H3BLK_ERR_UNSUPPORTED;
//   * all calls share it and it keeps the last call's contents, so two calls
//     that overlap on the GPU (different streams, or different host threads
//     on the same device) race with each other; serialise them;
//   * the first call on each device looks up the array's device address
//     (cudaGetSymbolAddress, with that device current) and caches it; make that
//     first call before any stream capture. The cached address assumes the
//     device's primary context lives as long as the process: after a
//     cudaDeviceReset the cache is stale, and the library must not be called
//     again in that process;
//   * errors found on the device (an out-of-range tag or timestep index, a
//     pipeline wait that ran out) go to an error word inside the array;
//     h3blk_attention_noalloc_check reads it, so call it after each call (or
//     each batch of calls) whose output must be trusted.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "../../include/h3blk.h"
#include "kernels.cuh"
#include "ptx.cuh"

namespace {

constexpr int64_t kNoAllocMaxTiles = 4096;                 // 128-row tiles
constexpr int64_t kNoAllocMaxRows = kNoAllocMaxTiles * 128;  // 524,288 rows
constexpr size_t kNoAllocErrorBytes = 256;                 // error word, padded
constexpr size_t kNoAllocScratchBytes = kNoAllocErrorBytes + kNoAllocMaxTiles * sizeof(h3::TileInfo);
constexpr int kNoAllocMaxHeadChannels = 16384;             // heads * head_dim, as h3blk_create allows

// The scratch itself. In host code this name only stands for the array: its
// device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

// Device address of the scratch array on the current device (looked up once
// per device) and the driver's tensor-map encoder.
int setup(void** scratch, PFN_cuTensorMapEncodeTiled_v12000* encode) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return H3BLK_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
      return H3BLK_ERR_CUDA;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  if (!g_scratch_ptr[dev]) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return H3BLK_ERR_CUDA;
    if (major != 10 || minor != 0) return H3BLK_ERR_UNSUPPORTED;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return H3BLK_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *scratch = g_scratch_ptr[dev];
  *encode = g_encode;
  return H3BLK_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" int h3blk_attention_noalloc(int64_t n_rows, int heads, int head_dim, int n_tags, int n_t,
                                       const void* qkv, const int32_t* tag, const int32_t* tidx, void* o,
                                       void* stream) {
  if (n_rows < 1 || heads < 1 || n_tags < 1 || n_t < 1 || !qkv || !tag || !tidx || !o) return H3BLK_ERR_INVALID_ARG;
  if (!aligned16(qkv) || !aligned16(o) || !aligned16(tag) || !aligned16(tidx)) return H3BLK_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return H3BLK_ERR_UNSUPPORTED;
  if (heads > kNoAllocMaxHeadChannels / head_dim) return H3BLK_ERR_UNSUPPORTED;  // the block's own limit
  if (n_rows > kNoAllocMaxRows) return H3BLK_ERR_UNSUPPORTED;  // beyond the fixed scratch
  void* scratch = nullptr;
  PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
  const int st = setup(&scratch, &enc);
  if (st != H3BLK_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int* err = static_cast<int*>(scratch);
  h3::TileInfo* tiles = reinterpret_cast<h3::TileInfo*>(static_cast<unsigned char*>(scratch) + kNoAllocErrorBytes);
  // the error word must start at zero; the tile summary is rewritten in full
  if (cudaMemsetAsync(err, 0, sizeof(int), s) != cudaSuccess) return H3BLK_ERR_CUDA;
  if (h3::launch_tile_info(tag, tidx, n_rows, n_tags, n_t, tiles, err, s) != cudaSuccess) return H3BLK_ERR_CUDA;
  h3::AttnArgs a{};  // every field not set below (output routing among them) stays zero
  a.qkv = static_cast<const __nv_bfloat16*>(qkv);
  a.o = static_cast<__nv_bfloat16*>(o);
  a.tag = tag;
  a.tiles = tiles;
  a.n = n_rows;
  a.heads = heads;
  a.head_dim = head_dim;
  a.err = err;
  return h3::launch_attention(a, enc, s) == cudaSuccess ? H3BLK_OK : H3BLK_ERR_CUDA;
}

extern "C" int h3blk_attention_noalloc_check(void* stream, int* status) {
  if (!status) return H3BLK_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return H3BLK_ERR_CUDA;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return H3BLK_ERR_CUDA;
  int bits = 0;
  // the error word is the first int of the array; a device on which no call
  // ran yet reads the array's initial zero
  if (cudaMemcpyFromSymbol(&bits, g_noalloc_scratch, sizeof(int), 0, cudaMemcpyDeviceToHost) != cudaSuccess)
    return H3BLK_ERR_CUDA;
  if (bits & (h3::kErrTimeoutGemm | h3::kErrTimeoutAttn | h3::kErrTimeoutStream))
    *status = H3BLK_ERR_TIMEOUT;
  else if (bits & (h3::kErrBadIndex | h3::kErrBadRowIndex))
    *status = H3BLK_ERR_BAD_INDEX;
  else
    *status = H3BLK_OK;
  return H3BLK_OK;
}
