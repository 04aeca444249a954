// h3blk_selftest_wait: runs the bounded mbarrier wait that every pipeline of
// the library uses (mbar_wait_for in ptx.cuh) on a barrier whose phase either
// completes or never does, so a test can check on a real GPU that a wait
// which runs out ends the kernel with an error status the host reads, and
// that the CUDA context stays usable afterwards. Nothing faults: the expired
// wait simply returns false after its time limit.
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/h3blk.h"
#include "ptx.cuh"

namespace {

__global__ void wait_selftest_kernel(int complete, unsigned long long limit_ns, int* word) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    h3::mbar_init(&bar, 1);
    h3::fence_mbar_init();
  }
  __syncthreads();
  if (complete && threadIdx.x == 0) h3::mbar_arrive(&bar);  // the phase's one arrival
  __syncthreads();
  const bool ok = h3::mbar_wait_for(&bar, 0, nullptr, limit_ns);
  if (!ok && threadIdx.x == 0) atomicOr(word, h3::kErrTimeoutStream);
}

}  // namespace

extern "C" int h3blk_selftest_wait(int complete, int limit_ms, void* word, void* stream, int* status) {
  if (!word || !status || limit_ms < 1 || limit_ms > 2000) return H3BLK_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(word) % 4 != 0) return H3BLK_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int* w = static_cast<int*>(word);
  if (cudaMemsetAsync(w, 0, sizeof(int), s) != cudaSuccess) return H3BLK_ERR_CUDA;
  wait_selftest_kernel<<<1, 32, 0, s>>>(complete ? 1 : 0, (unsigned long long)limit_ms * 1000000ull, w);
  if (cudaGetLastError() != cudaSuccess) return H3BLK_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return H3BLK_ERR_CUDA;
  int bits = 0;
  if (cudaMemcpy(&bits, w, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return H3BLK_ERR_CUDA;
  *status = (bits & h3::kErrTimeoutStream) ? H3BLK_ERR_TIMEOUT : H3BLK_OK;
  return H3BLK_OK;
}
