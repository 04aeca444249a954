// Shared between the C-ABI translation units of libh3blk (not installed).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "../../include/h3blk.h"
#include "kernels.cuh"

struct h3blk_ctx {
  h3blk_config cfg;
  h3::RopeTable rope;
  cudaEvent_t events[H3BLK_TIMING_POINTS];
  bool timing;
};

namespace h3api {

// Current device's SM count and the driver's tensor-map encoder; UNSUPPORTED
// unless the device is sm_100.
int device_info(int* num_sms, PFN_cuTensorMapEncodeTiled_v12000* encode);
bool aligned16(const void* p);
size_t align256(size_t v);
int cuda_status(cudaError_t e);

// Non-null, 16-byte aligned block weights (and int8 scales in W8A8 mode).
int check_block_weights(const h3blk_config& c, const h3blk_weights* w);

// Bytes of one block forward's workspace over n rows (error word at offset 0).
size_t block_workspace_bytes(const h3blk_config& c, int64_t n);

// The block forward's launch sequence on validated arguments. clear_err resets
// the error word (offset 0 of the workspace) first; timing records the
// handle's events.
int block_forward(const h3blk_ctx* h, int64_t n_rows, const void* x, const int32_t* tag, const int32_t* tidx,
                  const int32_t* pos, const float* mod_table, const h3blk_weights* w, void* out, void* workspace,
                  int num_sms, PFN_cuTensorMapEncodeTiled_v12000 enc, cudaStream_t s, bool clear_err, bool timing);

// Size limits of the modulation producer's weights for this handle.
int mod_check(const h3blk_ctx* h, const h3blk_mod_weights* w);

}  // namespace h3api
