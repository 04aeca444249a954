// Block-sparse attention selection: which 128-key tiles each 256-query block
// (the two query tiles of one attention CTA) attends to, per head.
//
// Source: "HyperFlow for MiniMax-H3" (model card), summary table and
// Performance: an optional sparse attention backend, an approximation of
// dense attention; the pages do not describe its method. This library's
// reading: the score of (block B, tile J, head h) is the dot product of the
// mean query of B's valid rows and the mean key of J's valid rows; every
// (block, head) keeps the k = max(1, ceil(n_cand * m / 1024)) highest-scoring
// candidate tiles (tiles with a valid row), ties toward the lower index, m the
// density in 1/1024 units. A block without valid rows keeps its own first
// tile (its rows are padding; their attention output is discarded).
//
// Two kernels: per (tile, channel) sums of q and k over valid rows (16-byte
// loads, each row read as coalesced 2 KB runs), then per (block, head)
// the scores against every tile, the rank of each candidate, and the kept
// tiles written in ascending order as [count, tile, tile, ...].
#include <cuda_bf16.h>

#include "kernels.cuh"
#include "ptx.cuh"

namespace h3 {
namespace {

constexpr int kTileRows = 128;
constexpr int kSelThreads = 256;

// Sums over a tile's valid rows of q and k, stored as [tile][heads][head_dim]
// (= tile * HD + channel). One CTA per (128-row tile, 1024-channel window):
// threads 0..127 own 16-byte chunks of the window's q channels, threads
// 128..255 the same chunks of k, so each row is read as two coalesced 2 KB
// runs; four rows are loaded before any is added, keeping several loads in
// flight per thread.
constexpr int kPoolThreads = 256;
constexpr int kPoolWindow = 1024;  // channels per CTA (128 chunks of 8)
constexpr int kPoolUnroll = 4;

__global__ void __launch_bounds__(kPoolThreads) pool_kernel(const __nv_bfloat16* __restrict__ qkv,
                                                             const int32_t* __restrict__ tag, int64_t n, int HD,
                                                             float* __restrict__ qsum, float* __restrict__ ksum,
                                                             int32_t* __restrict__ count) {
  const int tile = blockIdx.x, part = threadIdx.x >> 7;  // part 0: q, 1: k
  const int c = blockIdx.y * kPoolWindow + (threadIdx.x & 127) * 8;  // first channel of the chunk
  const int64_t ld = 3 * (int64_t)HD;
  const int64_t r0 = (int64_t)tile * kTileRows;
  const int rows = (int)(r0 + kTileRows < n ? kTileRows : n - r0);
  const bool on = c < HD;
  const __nv_bfloat16* src = qkv + r0 * ld + (int64_t)part * HD + (on ? c : 0);
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  int valid = 0;
  for (int r = 0; r < rows; r += kPoolUnroll) {
    uint4 v[kPoolUnroll];
    bool use[kPoolUnroll];
#pragma unroll
    for (int u = 0; u < kPoolUnroll; ++u) {
      use[u] = r + u < rows && __ldg(tag + r0 + r + u) != -1;
      if (on && use[u]) v[u] = __ldg(reinterpret_cast<const uint4*>(src + (int64_t)(r + u) * ld));
    }
#pragma unroll
    for (int u = 0; u < kPoolUnroll; ++u) {
      if (!use[u]) continue;
      ++valid;
      if (!on) continue;
      const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
        acc[2 * i] += f.x;
        acc[2 * i + 1] += f.y;
      }
    }
  }
  if (on) {
    float4* dst = reinterpret_cast<float4*>((part ? ksum : qsum) + (int64_t)tile * HD + c);
    dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
  }
  if (blockIdx.y == 0 && threadIdx.x == 0) count[tile] = valid;
}

// one CTA per (query block, head)
__global__ void __launch_bounds__(kSelThreads) select_kernel(const float* __restrict__ qsum,
                                                             const float* __restrict__ ksum,
                                                             const int32_t* __restrict__ count, int n_tiles,
                                                             int heads, int D, int keep_per_1024,
                                                             int32_t* __restrict__ lists, int64_t stride) {
  extern __shared__ float sh[];
  float* qbar = sh;                                        // [D]
  float* score = sh + D;                                   // [n_tiles]
  int* flag = reinterpret_cast<int*>(score + n_tiles);     // [n_tiles]: 1 candidate / kept
  __shared__ int s_ncand, s_scan[kSelThreads + 1];
  const int b = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
  const int t0 = 2 * b, t1 = 2 * b + 1;
  const int c0 = count[t0], c1 = t1 < n_tiles ? count[t1] : 0;
  int32_t* out = lists + ((int64_t)b * heads + h) * stride;
  if (c0 + c1 == 0) {
    // a block of padding rows only: its own first tile keeps n_kv >= 1
    if (tid == 0) {
      out[0] = 1;
      out[1] = t0;
    }
    return;
  }
  const float inv = 1.f / (float)(c0 + c1);
  for (int d = tid; d < D; d += kSelThreads) {
    float v = qsum[((int64_t)t0 * heads + h) * D + d];
    if (t1 < n_tiles) v += qsum[((int64_t)t1 * heads + h) * D + d];
    qbar[d] = v * inv;
  }
  if (tid == 0) s_ncand = 0;
  __syncthreads();
  // scores: one warp per tile, lanes across the channels
  const int warp = tid >> 5, lane = tid & 31;
  for (int j = warp; j < n_tiles; j += kSelThreads / 32) {
    const int cj = count[j];
    float acc = 0.f;
    if (cj > 0) {
      const float* kj = ksum + ((int64_t)j * heads + h) * D;
      for (int d = lane; d < D; d += 32) acc = fmaf(qbar[d], kj[d], acc);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) {
      score[j] = cj > 0 ? acc / (float)cj : 0.f;
      flag[j] = cj > 0 ? 1 : 0;
    }
  }
  __syncthreads();
  int mine = 0;
  for (int j = tid; j < n_tiles; j += kSelThreads) mine += flag[j];
  atomicAdd(&s_ncand, mine);
  __syncthreads();
  const int n_cand = s_ncand;
  int k = (int)(((int64_t)n_cand * keep_per_1024 + 1023) / 1024);
  if (k < 1) k = 1;
  // rank of each candidate: higher scores first, then lower indices
  for (int j = tid; j < n_tiles; j += kSelThreads) {
    if (!flag[j]) continue;
    const float sj = score[j];
    int rank = 0;
    for (int i = 0; i < n_tiles && rank < k; ++i)
      if (flag[i] && (score[i] > sj || (score[i] == sj && i < j))) ++rank;
    flag[j] = rank < k ? 2 : 1;
  }
  __syncthreads();
  // kept tiles in ascending order: each thread owns a contiguous range
  const int per = (n_tiles + kSelThreads - 1) / kSelThreads;
  const int lo = tid * per, hi = lo + per < n_tiles ? lo + per : n_tiles;
  int cnt = 0;
  for (int j = lo; j < hi; ++j) cnt += flag[j] == 2;
  s_scan[tid + 1] = cnt;
  if (tid == 0) s_scan[0] = 0;
  __syncthreads();
  if (tid == 0)
    for (int i = 1; i <= kSelThreads; ++i) s_scan[i] += s_scan[i - 1];
  __syncthreads();
  int pos = s_scan[tid];
  for (int j = lo; j < hi; ++j)
    if (flag[j] == 2) out[1 + pos++] = j;
  if (tid == 0) out[0] = s_scan[kSelThreads];
}

}  // namespace

cudaError_t launch_sparse_select(const SparseArgs& a, cudaStream_t s) {
  const int n_tiles = (int)((a.n + kTileRows - 1) / kTileRows);
  const int n_blocks = (n_tiles + 1) / 2;
  if (a.head_dim > 256 || a.keep_per_1024 < 1 || a.keep_per_1024 > 1024) return cudaErrorInvalidValue;
  const int HD = a.heads * a.head_dim;
  if (HD % 8 != 0) return cudaErrorInvalidValue;  // whole 16-byte chunks
  pool_kernel<<<dim3((unsigned)n_tiles, (unsigned)((HD + kPoolWindow - 1) / kPoolWindow)), kPoolThreads, 0, s>>>(
      a.qkv, a.tag, a.n, HD, a.qsum, a.ksum, a.count);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t smem = (size_t)a.head_dim * 4 + (size_t)n_tiles * 8;
  if (smem > 48 * 1024) {
    e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  select_kernel<<<dim3((unsigned)n_blocks, (unsigned)a.heads), kSelThreads, smem, s>>>(
      a.qsum, a.ksum, a.count, n_tiles, a.heads, a.head_dim, a.keep_per_1024, a.lists, a.list_stride);
  return cudaGetLastError();
}

}  // namespace h3
