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
  int keep_per_1024;  // 1024: dense attention; below: block-sparse
  // test-only dump of one int8 GEMM's s32 accumulators (-1: off)
  int dbg_gemm;
  int32_t* dbg_buf;
  size_t dbg_bytes;
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

// Bytes of one block forward's workspace over n rows (error word at offset 0);
// keep_per_1024 < 1024 adds the block-sparse selection buffers.
size_t block_workspace_bytes(const h3blk_config& c, int64_t n, int keep_per_1024);

// Buffers of one block forward (W8A8 ones null in bf16 mode and vice versa).
struct BlockBufs {
  int* err = nullptr;
  h3::TileInfo* tiles = nullptr;
  float4* modt = nullptr;  // the pre-norm vectors rearranged for the row passes
  float2* rope_tab = nullptr;  // (sin, cos) of this call's rows' rotary angles, [rows, head_dim / 2]
  // block-sparse selection (null when dense)
  float *sp_qsum = nullptr, *sp_ksum = nullptr;
  int32_t *sp_count = nullptr, *sp_lists = nullptr;
  __nv_bfloat16 *h1 = nullptr, *qkv = nullptr, *o = nullptr, *x1 = nullptr, *h2 = nullptr, *a = nullptr;
  int8_t *h1_q = nullptr, *o_q = nullptr, *h2_q = nullptr, *a_q = nullptr;
  float *h1_s = nullptr, *o_s = nullptr, *h2_s = nullptr, *a_s = nullptr;
};

// This call's rows [row0, row0 + n_local) of a packed sequence of n_total rows.
struct Span {
  int64_t n_local, row0, n_total;
};

// Head-group routing of the QKV projection: head h goes to dst[h / hg], a
// [n_total, 3 * hg * head_dim] buffer, at its global row.
struct QkvRoute {
  int ranks, hg;
  void* dst[h3::kMaxRanks];
};

// Row routing of the attention output: global row r goes to
// dst[r / rows] at row r % rows of a [rows, ld] buffer, columns from
// (head0 + head) * head_dim.
struct ORoute {
  int ranks, head0;
  int64_t rows, ld;
  void* dst[h3::kMaxRanks];
};

// The block in three phases: tile summary + pre-norm + QKV (x = this call's
// rows; tag / tidx / pos cover the whole sequence), attention over the whole
// sequence for `heads` heads, and out-projection through the FFN for this
// call's rows.
int phase_qkv(const h3blk_ctx* h, const Span& sp, const void* x, const int32_t* tag, const int32_t* tidx,
              const int32_t* pos, const float* mod_table, const h3blk_weights* w, const BlockBufs& b,
              const QkvRoute* route, int sms, PFN_cuTensorMapEncodeTiled_v12000 enc, cudaStream_t s, bool clear_err,
              bool timing);
int phase_attention(const h3blk_ctx* h, int64_t n_total, int heads, const int32_t* tag, const BlockBufs& b,
                    const ORoute* route, PFN_cuTensorMapEncodeTiled_v12000 enc, cudaStream_t s, bool timing);
int phase_out(const h3blk_ctx* h, const Span& sp, const void* x, const int32_t* tag, const int32_t* tidx,
              const float* mod_table, const h3blk_weights* w, const BlockBufs& b, void* out, int sms,
              PFN_cuTensorMapEncodeTiled_v12000 enc, cudaStream_t s, bool timing);

// The block forward's launch sequence on validated arguments. clear_err resets
// the error word (offset 0 of the workspace) first; timing records the
// handle's events.
int block_forward(const h3blk_ctx* h, int64_t n_rows, const void* x, const int32_t* tag, const int32_t* tidx,
                  const int32_t* pos, const float* mod_table, const h3blk_weights* w, void* out, void* workspace,
                  int num_sms, PFN_cuTensorMapEncodeTiled_v12000 enc, cudaStream_t s, bool clear_err, bool timing);

// Size limits of the modulation producer's weights for this handle.
int mod_check(const h3blk_ctx* h, const h3blk_mod_weights* w);

}  // namespace h3api
