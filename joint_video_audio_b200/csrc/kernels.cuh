// Launch interfaces of the block's kernels (internal to libh3blk).
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

namespace h3 {

constexpr int kMaxRopePairs = 128;  // head_dim <= 256
constexpr int kMaxRanks = 8;        // ranks of a sequence-parallel (Ulysses) group

// Rotary table of one head: for pair j, which position axis drives it
// (0 t, 1 h, 2 w, 3 none) and its frequency.
struct RopeTable {
  float freq[kMaxRopePairs];
  int8_t axis[kMaxRopePairs];
};

// Per 128-row tile of the packed sequence: number of rows present, number of
// padding rows among them, and a padding bit per row.
struct TileInfo {
  int32_t rows;
  int32_t npad;
  uint32_t padbits[4];
  int32_t _unused[2];
};
static_assert(sizeof(TileInfo) == 32, "TileInfo is 32 bytes");

// ---------------------------------------------------------------- prep
// Validates tag / tidx and fills one TileInfo per 128 rows.
cudaError_t launch_tile_info(const int32_t* tag, const int32_t* tidx, int64_t n, int n_tags, int n_t,
                             TileInfo* info, int* err, cudaStream_t s);

// ---------------------------------------------------------------- K1
// h[r] = rmsnorm(x[r]) * (1 + table[tag][tidx][scale_idx]) + table[..][shift_idx]
// bf16 output, or (quant) Hadamard-rotated per-token int8 + fp32 scale.
struct ModNormArgs {
  const __nv_bfloat16* x;
  const int32_t* tag;
  const int32_t* tidx;
  const float* table;
  int64_t n;
  int C, n_tags, n_t, shift_idx, scale_idx;
  float eps;
  __nv_bfloat16* out_bf16;  // used when out_q == nullptr
  int8_t* out_q;
  float* out_scale;
  int* err = nullptr;  // device error word (a load that never landed), may be null
  // the table's shift / (1 + scale) vectors rearranged by launch_modt, and
  // which pair this pass applies (0: shift1 / scale1, 2: shift2 / scale2)
  const float4* modt = nullptr;
  int modt_v0 = 0;
};
cudaError_t launch_modnorm(const ModNormArgs& a, cudaStream_t s);
// Rearranges the table's pre-norm vectors (shift1, 1 + scale1, shift2,
// 1 + scale2 of every (tag, tidx)) for the row passes: n_tags * n_t * 4 * K
// floats at `modt`.
cudaError_t launch_modt(const float* table, int n_tags, int n_t, int K, float4* modt, cudaStream_t s);
inline size_t modt_bytes(int n_tags, int n_t, int K) { return (size_t)n_tags * n_t * 4 * K * sizeof(float); }

// ---------------------------------------------------------------- K4
// Rows of a bf16 matrix [rows, K] -> block-128 Hadamard rotation ->
// symmetric per-row int8 with fp32 scale.
cudaError_t launch_rotate_quant(const __nv_bfloat16* in, int64_t rows, int K, int8_t* out_q, float* out_scale,
                                int* err, cudaStream_t s);

// ---------------------------------------------------------------- GEMM
enum GemmEpilogue : int {
  kEpiStoreBf16 = 0,  // out = acc (+ bias[col])
  kEpiQKV = 1,        // q/k: per-head RMSNorm * gain + RoPE; v: plain
  kEpiResid = 2,      // out = resid + gate * acc
  kEpiSwiGLU = 3,     // out[:, j] = silu(acc_gate[:, j]) * acc_up[:, j]
  kEpiStoreS32 = 4,   // raw int32 accumulators (int8 GEMM only)
};

struct GemmArgs {
  // operands: A [M, K] row-major, B [Nb, K] row-major (the weight), both K-major
  const void* A;
  const void* B;
  int64_t M;
  int N;  // logical output columns (SwiGLU: F)
  int K;
  int Nb;  // rows of B
  bool int8;
  int epi;
  // outputs
  void* out;
  int64_t ld_out;  // elements
  // kEpiResid
  const __nv_bfloat16* resid;
  const float* table;
  const int32_t* tag;
  const int32_t* tidx;
  int n_tags, n_t, gate_idx;
  // kEpiQKV
  const __nv_bfloat16* q_gain;
  const __nv_bfloat16* k_gain;
  int head_dim, hd;
  float qk_eps;
  RopeTable rope;
  // (sin, cos) of every rotary pair's angle per output row, [M, head_dim / 2]
  // (launch_rope_table); required by kEpiQKV
  const float2* rope_tab = nullptr;
  // kEpiStoreBf16: optional fp32 bias added per column
  const float* bias;
  // int8 dequantisation: acc * s_a[row] * s_b[col]
  const float* s_a;
  const float* s_b;
  int* err;
  // kEpiQKV routing by head group (route_ranks > 0): head h of region q / k / v
  // goes to route_dst[h / route_hg], a [rows, 3 * route_hg * head_dim] buffer,
  // at row route_row0 + row
  int route_ranks = 0, route_hg = 0;
  int64_t route_row0 = 0;
  void* route_dst[kMaxRanks] = {};
  // int8 mode, test-only: when set, the epilogue also writes every raw s32
  // accumulator it reads to acc_dump[row * ld_dump + b_row] (b_row = the
  // weight row the value belongs to)
  int32_t* acc_dump = nullptr;
  int64_t ld_dump = 0;
};
cudaError_t launch_gemm(const GemmArgs& a, PFN_cuTensorMapEncodeTiled_v12000 encode, int num_sms, cudaStream_t s);

// (sin, cos) of the rotary angle pos[row][axis(pair)] * freq[pair] for every
// row and pair, tab[row * pairs + pair]; pairs without an axis get (0, 1).
// Evaluated once per row here instead of once per query / key head in the
// QKV epilogue, with the same reduction and hardware sine / cosine.
cudaError_t launch_rope_table(const int32_t* pos, int64_t n, const RopeTable& rope, int pairs, float2* tab,
                              cudaStream_t s);
inline size_t rope_table_bytes(int64_t n, int pairs) { return (size_t)n * pairs * sizeof(float2); }

// ---------------------------------------------------------------- attention
struct AttnArgs {
  const __nv_bfloat16* qkv;  // [N, 3*H*D]: q heads, k heads, v heads
  __nv_bfloat16* o;          // [N, H*D]
  const int32_t* tag;
  const TileInfo* tiles;
  int64_t n;
  int heads, head_dim;
  int* err;
  // output routing by row (route_ranks > 0): row r goes to
  // route_dst[r / route_rows] at row r % route_rows of a [route_rows, route_ld]
  // buffer, columns from (route_head0 + head) * head_dim
  int route_ranks = 0, route_head0 = 0;
  int64_t route_rows = 0, route_ld = 0;
  __nv_bfloat16* route_dst[kMaxRanks] = {};
  // block-sparse mode (kv_list != nullptr): the KV tiles of CTA (pair, head)
  // are kv_list[(pair * heads + head) * kv_list_stride + 1 ..][0 .. count),
  // count at offset 0, ascending
  const int32_t* kv_list = nullptr;
  int64_t kv_list_stride = 0;
};
cudaError_t launch_attention(const AttnArgs& a, PFN_cuTensorMapEncodeTiled_v12000 encode, cudaStream_t s);

// ---------------------------------------------------------------- sparse selection
// Per 256-query block and head, the 128-key tiles block-sparse attention keeps
// (see sparse.cu): lists [n_blocks][heads][1 + n_tiles] as count, tiles.
struct SparseArgs {
  const __nv_bfloat16* qkv;  // [n, 3 * heads * head_dim], q and k final (normed, rotated)
  const int32_t* tag;
  int64_t n;
  int heads, head_dim, keep_per_1024;
  float* qsum;               // [n_tiles][heads][head_dim]
  float* ksum;               // [n_tiles][heads][head_dim]
  int32_t* count;            // [n_tiles] valid rows
  int32_t* lists;
  int64_t list_stride;       // 1 + n_tiles
};
cudaError_t launch_sparse_select(const SparseArgs& a, cudaStream_t s);

// ---------------------------------------------------------------- modulation table
constexpr int kMaxModSets = 8;  // timestep sets (the table's n_t) per call

struct ModTimes {
  int count;                 // 0: no embedding (the input comes from memory)
  float t[kMaxModSets];      // used when dev == nullptr
  const float* dev;          // device array of count timesteps (graph-replayable)
};

struct ModTableArgs {
  int n_sets, n_tags, hidden, freq_dim, time_hidden, time_dim;
  int n_vec;                 // vectors per (tag, set): 6 for a block, 2 for norm_out
  ModTimes t_now, t_end;     // per set
  float gate;                // two-time blend weight of the t_end embedding
  const float *w1, *b1, *w2, *b2;
  const float *w1_r, *b1_r, *w2_r, *b2_r;
  const __nv_bfloat16* adaln_w;  // [n_tags][n_vec * hidden][time_dim]
  const float* adaln_b;          // [n_tags][n_vec * hidden]
  float* table;              // [n_tags][n_sets][n_vec * hidden]
  float* scratch;            // n_sets * (time_hidden + time_dim) floats: hidden layer, then E
};
// Time embedding E (into scratch + n_sets * time_hidden) and the projection.
cudaError_t launch_modulation_table(const ModTableArgs& a, int num_sms, cudaStream_t s);
// The two halves on their own: E = time MLP(s) of the sets' timesteps ...
cudaError_t launch_time_embedding(const ModTableArgs& a, int num_sms, cudaStream_t s);
// ... and table = A_tag silu(E) + a_tag from an E already in scratch.
cudaError_t launch_adaln_projection(const ModTableArgs& a, int num_sms, cudaStream_t s);

// ---------------------------------------------------------------- model shell
// out[idx[m]] = bf16(W x[m] + b) for the M fp32 rows x [M][K]; W fp32 [C][K].
cudaError_t launch_embed_rows(const float* x, int64_t M, int K, const float* W, const float* b, int C,
                              const int32_t* idx, int64_t n_rows, __nv_bfloat16* out, int* err, cudaStream_t s);
// out[idx[m]] = bf16(rmsnorm(r[m]) * gain) over C channels.
cudaError_t launch_norm_scatter(const __nv_bfloat16* r, int64_t M, int C, const __nv_bfloat16* gain, float eps,
                                const int32_t* idx, int64_t n_rows, __nv_bfloat16* out, int* err, cudaStream_t s);
// y[m] = W (rmsnorm(x[idx[m]]) (1 + scale) + shift) + b, (shift, scale) =
// table[tag][tidx][0..1] (zero for padding); W fp32 [n_out][C], y fp32.
struct HeadArgs {
  const __nv_bfloat16* x;
  const int32_t* idx;
  int64_t M, n_rows;
  int C, n_out;
  const int32_t* tag;
  const int32_t* tidx;
  const float* table;  // [n_tags][n_t][2][C]
  int n_tags, n_t;
  float eps;
  const float* W;
  const float* b;
  float* y;
  int* err;
};
cudaError_t launch_head(const HeadArgs& a, int num_sms, cudaStream_t s);
// out_*[m] = in_*[idx[m]]
cudaError_t launch_gather_meta(const int32_t* idx, int64_t M, int64_t n_rows, const int32_t* tag,
                               const int32_t* tidx, const int32_t* pos, int32_t* out_tag, int32_t* out_tidx,
                               int32_t* out_pos, int* err, cudaStream_t s);

}  // namespace h3
