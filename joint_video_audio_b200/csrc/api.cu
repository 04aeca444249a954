// C-ABI of libh3blk: argument validation, workspace layout and the launch
// sequence of one MiniMax-H3 block forward (see include/h3blk.h).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstring>
#include <mutex>
#include <new>

#include "api_internal.h"
#include "ptx.cuh"

using h3::GemmArgs;

namespace {
constexpr int kVersion = 100;  // 0.1.0

// ------------------------------------------------------------------ device info
struct DeviceInfo {
  bool ready = false;
  int num_sms = 0;
};
constexpr int kMaxDevices = 64;
DeviceInfo g_dev[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::mutex g_mu;
}  // namespace

namespace h3api {

int device_info(int* num_sms, PFN_cuTensorMapEncodeTiled_v12000* encode) {
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
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return H3BLK_ERR_CUDA;
    if (major != 10 || minor != 0) return H3BLK_ERR_UNSUPPORTED;  // built for sm_100a only
    d.num_sms = sms;
    d.ready = true;
  }
  *num_sms = d.num_sms;
  *encode = g_encode;
  return H3BLK_OK;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? H3BLK_OK : H3BLK_ERR_CUDA; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

}  // namespace h3api

namespace {
using h3api::aligned16;
using h3api::align256;
using h3api::cuda_status;
using h3api::device_info;

bool overlap(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

// Workspace layout: every stage buffer at a 256-byte aligned offset.
struct Layout {
  size_t off[H3BLK_STAGE_COUNT];
  size_t len[H3BLK_STAGE_COUNT];
  size_t tiles_off;
  size_t modt_off;
  size_t rope_off;
  size_t sp_qsum, sp_ksum, sp_count;  // block-sparse pooling buffers (0 when dense)
  size_t total;
};

Layout make_layout(const h3blk_config& c, int64_t n, int keep_per_1024) {
  Layout L;
  std::memset(&L, 0, sizeof(L));
  const size_t N = (size_t)n, C = c.hidden, HD = (size_t)c.heads * c.head_dim, F = c.ffn;
  size_t o = 0;
  auto put = [&](int stage, size_t bytes) {
    L.off[stage] = o;
    L.len[stage] = bytes;
    o = align256(o + bytes);
  };
  put(H3BLK_STAGE_ERROR, 4);
  L.tiles_off = o;
  o = align256(o + ((N + 127) / 128) * sizeof(h3::TileInfo));
  const bool q = c.quant != 0;
  L.modt_off = o;
  if (q) o = align256(o + h3::modt_bytes(c.n_tags, c.n_t, c.hidden));
  L.rope_off = o;
  o = align256(o + h3::rope_table_bytes(n, c.head_dim / 2));
  if (!q) put(H3BLK_STAGE_H1, N * C * 2);
  put(H3BLK_STAGE_QKV, N * 3 * HD * 2);
  put(H3BLK_STAGE_O, N * HD * 2);
  put(H3BLK_STAGE_X1, N * C * 2);
  if (!q) put(H3BLK_STAGE_H2, N * C * 2);
  put(H3BLK_STAGE_A, N * F * 2);
  if (q) {
    put(H3BLK_STAGE_H1_Q8, N * C);
    put(H3BLK_STAGE_H1_SCALE, N * 4);
    put(H3BLK_STAGE_O_Q8, N * HD);
    put(H3BLK_STAGE_O_SCALE, N * 4);
    put(H3BLK_STAGE_H2_Q8, N * C);
    put(H3BLK_STAGE_H2_SCALE, N * 4);
    put(H3BLK_STAGE_A_Q8, N * F);
    put(H3BLK_STAGE_A_SCALE, N * 4);
  }
  if (keep_per_1024 < 1024) {
    const size_t n_tiles = (N + 127) / 128, n_blocks = (n_tiles + 1) / 2, H = c.heads;
    const size_t pool = n_tiles * H * (size_t)c.head_dim * 4;
    L.sp_qsum = o;
    o = align256(o + pool);
    L.sp_ksum = o;
    o = align256(o + pool);
    L.sp_count = o;
    o = align256(o + n_tiles * 4);
    put(H3BLK_STAGE_KV_LIST, n_blocks * H * (1 + n_tiles) * 4);
  }
  L.total = o;
  return L;
}

// Int8 weight blob layout.
struct BlobLayout {
  size_t wqkv, wo, w13, w2, s_qkv, s_o, s_13, s_2, q_gain, k_gain, total;
};

BlobLayout make_blob(const h3blk_config& c) {
  const size_t C = c.hidden, HD = (size_t)c.heads * c.head_dim, F = c.ffn, D = c.head_dim;
  BlobLayout b;
  size_t o = 0;
  auto put = [&](size_t bytes) {
    const size_t at = o;
    o = align256(o + bytes);
    return at;
  };
  b.wqkv = put(3 * HD * C);
  b.wo = put(C * HD);
  b.w13 = put(2 * F * C);
  b.w2 = put(C * F);
  b.s_qkv = put(3 * HD * 4);
  b.s_o = put(C * 4);
  b.s_13 = put(2 * F * 4);
  b.s_2 = put(C * 4);
  b.q_gain = put(D * 2);
  b.k_gain = put(D * 2);
  b.total = o;
  return b;
}

GemmArgs base_gemm(const h3blk_ctx* h, int* err) {
  GemmArgs g;
  std::memset(&g, 0, sizeof(g));
  g.n_tags = h->cfg.n_tags;
  g.n_t = h->cfg.n_t;
  g.head_dim = h->cfg.head_dim;
  g.hd = h->cfg.heads * h->cfg.head_dim;
  g.qk_eps = h->cfg.qk_norm_eps;
  g.rope = h->rope;
  g.err = err;
  g.int8 = h->cfg.quant != 0;
  return g;
}

}  // namespace

namespace h3api {

int check_block_weights(const h3blk_config& c, const h3blk_weights* w) {
  if (!w || !w->wqkv || !w->q_gain || !w->k_gain || !w->wo || !w->w13 || !w->w2) return H3BLK_ERR_INVALID_ARG;
  if (c.quant != 0 && (!w->s_qkv || !w->s_o || !w->s_13 || !w->s_2)) return H3BLK_ERR_INVALID_ARG;
  // the GEMM epilogues read the gains and the int8 scales 16 bytes at a time
  const void* ptrs[] = {w->wqkv, w->wo, w->w13, w->w2, w->q_gain, w->k_gain};
  for (const void* p : ptrs)
    if (!aligned16(p)) return H3BLK_ERR_INVALID_ARG;
  if (c.quant != 0) {
    const void* sc[] = {w->s_qkv, w->s_o, w->s_13, w->s_2};
    for (const void* p : sc)
      if (!aligned16(p)) return H3BLK_ERR_INVALID_ARG;
  }
  return H3BLK_OK;
}

size_t block_workspace_bytes(const h3blk_config& c, int64_t n, int keep_per_1024) {
  return make_layout(c, n, keep_per_1024).total;
}

#define H3_TRY(expr)                              \
  do {                                            \
    cudaError_t e_ = (expr);                      \
    if (e_ != cudaSuccess) return H3BLK_ERR_CUDA; \
  } while (0)

namespace {
// Test-only: routes the s32 accumulators of int8 GEMM `which` (0 QKV, 1
// out-projection, 2 FFN up, 3 FFN down) to the caller's buffer when that dump
// is switched on; INVALID_ARG if the buffer cannot hold [M, Nb] int32.
int attach_dump(const h3blk_ctx* h, int which, GemmArgs& g) {
  if (h->dbg_gemm != which || !g.int8) return H3BLK_OK;
  if ((size_t)g.M * (size_t)g.Nb * sizeof(int32_t) > h->dbg_bytes) return H3BLK_ERR_INVALID_ARG;
  g.acc_dump = h->dbg_buf;
  g.ld_dump = g.Nb;
  return H3BLK_OK;
}

cudaError_t mark(const h3blk_ctx* h, bool timing, int i, cudaStream_t s) {
  return timing ? cudaEventRecord(h->events[i], s) : cudaSuccess;
}
}  // namespace

int phase_qkv(const h3blk_ctx* h, const Span& sp, const void* x, const int32_t* tag, const int32_t* tidx,
              const int32_t* pos, const float* mod_table, const h3blk_weights* w, const BlockBufs& b,
              const QkvRoute* route, int sms, PFN_cuTensorMapEncodeTiled_v12000 enc, cudaStream_t s, bool clear_err,
              bool timing) {
  const h3blk_config& c = h->cfg;
  const bool q = c.quant != 0;
  const size_t HD = (size_t)c.heads * c.head_dim;
  H3_TRY(mark(h, timing, 0, s));
  if (clear_err) H3_TRY(cudaMemsetAsync(b.err, 0, sizeof(int), s));
  // the tile summary covers the whole sequence: attention reads every row
  H3_TRY(h3::launch_tile_info(tag, tidx, sp.n_total, c.n_tags, c.n_t, b.tiles, b.err, s));
  // W8A8: the table's pre-norm vectors in the row passes' layout (both pre-norms)
  if (q) H3_TRY(h3::launch_modt(mod_table, c.n_tags, c.n_t, c.hidden, b.modt, s));

  // ---- pre-attention AdaLN + RMSNorm of this call's rows
  h3::ModNormArgs mn;
  std::memset(&mn, 0, sizeof(mn));
  mn.x = static_cast<const __nv_bfloat16*>(x);
  mn.tag = tag + sp.row0;
  mn.tidx = tidx + sp.row0;
  mn.table = mod_table;
  mn.n = sp.n_local;
  mn.C = c.hidden;
  mn.n_tags = c.n_tags;
  mn.n_t = c.n_t;
  mn.shift_idx = 0;
  mn.scale_idx = 1;
  mn.modt = b.modt;
  mn.modt_v0 = 0;
  mn.eps = c.norm_eps;
  mn.out_q = b.h1_q;
  mn.out_scale = b.h1_s;
  mn.out_bf16 = b.h1;
  if (q) mn.out_bf16 = nullptr;
  H3_TRY(mark(h, timing, 1, s));
  mn.err = b.err;
  H3_TRY(h3::launch_modnorm(mn, s));

  // ---- QKV projection + QK-RMSNorm + RoPE (optionally routed by head group)
  GemmArgs g = base_gemm(h, b.err);
  g.A = q ? (const void*)b.h1_q : (const void*)b.h1;
  g.B = w->wqkv;
  g.M = sp.n_local;
  g.N = (int)(3 * HD);
  g.Nb = (int)(3 * HD);
  g.K = c.hidden;
  g.epi = h3::kEpiQKV;
  g.out = b.qkv;
  g.ld_out = 3 * HD;
  g.q_gain = static_cast<const __nv_bfloat16*>(w->q_gain);
  g.k_gain = static_cast<const __nv_bfloat16*>(w->k_gain);
  g.s_a = q ? b.h1_s : nullptr;
  g.s_b = w->s_qkv;
  if (route) {
    g.route_ranks = route->ranks;
    g.route_hg = route->hg;
    g.route_row0 = sp.row0;
    for (int r = 0; r < route->ranks; ++r) g.route_dst[r] = route->dst[r];
  }
  g.rope_tab = b.rope_tab;
  if (int st = attach_dump(h, 0, g)) return st;
  H3_TRY(mark(h, timing, 2, s));
  H3_TRY(h3::launch_rope_table(pos + 3 * sp.row0, sp.n_local, h->rope, c.head_dim / 2, b.rope_tab, s));
  H3_TRY(h3::launch_gemm(g, enc, sms, s));
  return H3BLK_OK;
}

int phase_attention(const h3blk_ctx* h, int64_t n_total, int heads, const int32_t* tag, const BlockBufs& b,
                    const ORoute* route, PFN_cuTensorMapEncodeTiled_v12000 enc, cudaStream_t s, bool timing) {
  h3::AttnArgs at;
  std::memset(&at, 0, sizeof(at));
  at.qkv = b.qkv;
  at.o = b.o;
  at.tag = tag;
  at.tiles = b.tiles;
  at.n = n_total;
  at.heads = heads;
  at.head_dim = h->cfg.head_dim;
  at.err = b.err;
  if (route) {
    at.route_ranks = route->ranks;
    at.route_head0 = route->head0;
    at.route_rows = route->rows;
    at.route_ld = route->ld;
    for (int r = 0; r < route->ranks; ++r) at.route_dst[r] = static_cast<__nv_bfloat16*>(route->dst[r]);
  }
  H3_TRY(mark(h, timing, 3, s));
  if (b.sp_lists) {
    // block-sparse: pool q and k per tile, rank the tiles per block and head
    h3::SparseArgs sa;
    std::memset(&sa, 0, sizeof(sa));
    sa.qkv = b.qkv;
    sa.tag = tag;
    sa.n = n_total;
    sa.heads = heads;
    sa.head_dim = h->cfg.head_dim;
    sa.keep_per_1024 = h->keep_per_1024;
    sa.qsum = b.sp_qsum;
    sa.ksum = b.sp_ksum;
    sa.count = b.sp_count;
    sa.lists = b.sp_lists;
    sa.list_stride = 1 + (n_total + 127) / 128;
    H3_TRY(h3::launch_sparse_select(sa, s));
    at.kv_list = b.sp_lists;
    at.kv_list_stride = sa.list_stride;
  }
  H3_TRY(h3::launch_attention(at, enc, s));
  H3_TRY(mark(h, timing, 4, s));
  return H3BLK_OK;
}

int phase_out(const h3blk_ctx* h, const Span& sp, const void* x, const int32_t* tag, const int32_t* tidx,
              const float* mod_table, const h3blk_weights* w, const BlockBufs& b, void* out, int sms,
              PFN_cuTensorMapEncodeTiled_v12000 enc, cudaStream_t s, bool timing) {
  const h3blk_config& c = h->cfg;
  const bool q = c.quant != 0;
  const size_t C = c.hidden, HD = (size_t)c.heads * c.head_dim, F = c.ffn;
  const int64_t n = sp.n_local;
  auto* xb = static_cast<const __nv_bfloat16*>(x);
  const int32_t* tg = tag + sp.row0;
  const int32_t* ti = tidx + sp.row0;

  // ---- out-projection + gated residual
  if (q) H3_TRY(h3::launch_rotate_quant(b.o, n, (int)HD, b.o_q, b.o_s, b.err, s));
  GemmArgs g = base_gemm(h, b.err);
  g.A = q ? (const void*)b.o_q : (const void*)b.o;
  g.B = w->wo;
  g.M = n;
  g.N = c.hidden;
  g.Nb = c.hidden;
  g.K = (int)HD;
  g.epi = h3::kEpiResid;
  g.out = b.x1;
  g.ld_out = C;
  g.resid = xb;
  g.table = mod_table;
  g.tag = tg;
  g.tidx = ti;
  g.gate_idx = 2;
  g.s_a = q ? b.o_s : nullptr;
  g.s_b = w->s_o;
  if (int st = attach_dump(h, 1, g)) return st;
  H3_TRY(mark(h, timing, 5, s));
  H3_TRY(h3::launch_gemm(g, enc, sms, s));
  H3_TRY(mark(h, timing, 6, s));

  // ---- pre-FFN AdaLN + RMSNorm
  h3::ModNormArgs mn;
  std::memset(&mn, 0, sizeof(mn));
  mn.x = b.x1;
  mn.tag = tg;
  mn.tidx = ti;
  mn.table = mod_table;
  mn.n = n;
  mn.C = c.hidden;
  mn.n_tags = c.n_tags;
  mn.n_t = c.n_t;
  mn.shift_idx = 3;
  mn.scale_idx = 4;
  mn.modt = b.modt;
  mn.modt_v0 = 2;
  mn.eps = c.norm_eps;
  mn.out_q = b.h2_q;
  mn.out_scale = b.h2_s;
  mn.out_bf16 = q ? nullptr : b.h2;
  mn.err = b.err;
  H3_TRY(h3::launch_modnorm(mn, s));

  // ---- FFN up (W1 | W3) + SwiGLU
  g = base_gemm(h, b.err);
  g.A = q ? (const void*)b.h2_q : (const void*)b.h2;
  g.B = w->w13;
  g.M = n;
  g.N = c.ffn;
  g.Nb = 2 * c.ffn;
  g.K = c.hidden;
  g.epi = h3::kEpiSwiGLU;
  g.out = b.a;
  g.ld_out = F;
  g.s_a = q ? b.h2_s : nullptr;
  g.s_b = w->s_13;
  if (int st = attach_dump(h, 2, g)) return st;
  H3_TRY(mark(h, timing, 7, s));
  H3_TRY(h3::launch_gemm(g, enc, sms, s));
  H3_TRY(mark(h, timing, 8, s));

  // ---- FFN down + gated residual
  if (q) H3_TRY(h3::launch_rotate_quant(b.a, n, (int)F, b.a_q, b.a_s, b.err, s));
  g = base_gemm(h, b.err);
  g.A = q ? (const void*)b.a_q : (const void*)b.a;
  g.B = w->w2;
  g.M = n;
  g.N = c.hidden;
  g.Nb = c.hidden;
  g.K = c.ffn;
  g.epi = h3::kEpiResid;
  g.out = out;
  g.ld_out = C;
  g.resid = b.x1;
  g.table = mod_table;
  g.tag = tg;
  g.tidx = ti;
  g.gate_idx = 5;
  g.s_a = q ? b.a_s : nullptr;
  g.s_b = w->s_2;
  if (int st = attach_dump(h, 3, g)) return st;
  H3_TRY(mark(h, timing, 9, s));
  H3_TRY(h3::launch_gemm(g, enc, sms, s));
  H3_TRY(mark(h, timing, 10, s));
  return H3BLK_OK;
}

int block_forward(const h3blk_ctx* h, int64_t n_rows, const void* x, const int32_t* tag, const int32_t* tidx,
                  const int32_t* pos, const float* mod_table, const h3blk_weights* w, void* out, void* workspace,
                  int sms, PFN_cuTensorMapEncodeTiled_v12000 enc, cudaStream_t s, bool clear_err, bool timing) {
  const Layout L = make_layout(h->cfg, n_rows, h->keep_per_1024);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  auto buf = [&](int stage) { return L.len[stage] ? ws + L.off[stage] : nullptr; };
  BlockBufs b{};
  b.err = reinterpret_cast<int*>(buf(H3BLK_STAGE_ERROR));
  b.tiles = reinterpret_cast<h3::TileInfo*>(ws + L.tiles_off);
  b.modt = reinterpret_cast<float4*>(ws + L.modt_off);
  b.rope_tab = reinterpret_cast<float2*>(ws + L.rope_off);
  const bool sparse = h->keep_per_1024 < 1024;
  b.sp_qsum = sparse ? reinterpret_cast<float*>(ws + L.sp_qsum) : nullptr;
  b.sp_ksum = sparse ? reinterpret_cast<float*>(ws + L.sp_ksum) : nullptr;
  b.sp_count = sparse ? reinterpret_cast<int32_t*>(ws + L.sp_count) : nullptr;
  b.sp_lists = reinterpret_cast<int32_t*>(buf(H3BLK_STAGE_KV_LIST));
  b.h1 = reinterpret_cast<__nv_bfloat16*>(buf(H3BLK_STAGE_H1));
  b.qkv = reinterpret_cast<__nv_bfloat16*>(buf(H3BLK_STAGE_QKV));
  b.o = reinterpret_cast<__nv_bfloat16*>(buf(H3BLK_STAGE_O));
  b.x1 = reinterpret_cast<__nv_bfloat16*>(buf(H3BLK_STAGE_X1));
  b.h2 = reinterpret_cast<__nv_bfloat16*>(buf(H3BLK_STAGE_H2));
  b.a = reinterpret_cast<__nv_bfloat16*>(buf(H3BLK_STAGE_A));
  b.h1_q = reinterpret_cast<int8_t*>(buf(H3BLK_STAGE_H1_Q8));
  b.o_q = reinterpret_cast<int8_t*>(buf(H3BLK_STAGE_O_Q8));
  b.h2_q = reinterpret_cast<int8_t*>(buf(H3BLK_STAGE_H2_Q8));
  b.a_q = reinterpret_cast<int8_t*>(buf(H3BLK_STAGE_A_Q8));
  b.h1_s = reinterpret_cast<float*>(buf(H3BLK_STAGE_H1_SCALE));
  b.o_s = reinterpret_cast<float*>(buf(H3BLK_STAGE_O_SCALE));
  b.h2_s = reinterpret_cast<float*>(buf(H3BLK_STAGE_H2_SCALE));
  b.a_s = reinterpret_cast<float*>(buf(H3BLK_STAGE_A_SCALE));
  const Span sp{n_rows, 0, n_rows};
  int st = phase_qkv(h, sp, x, tag, tidx, pos, mod_table, w, b, nullptr, sms, enc, s, clear_err, timing);
  if (st != H3BLK_OK) return st;
  st = phase_attention(h, n_rows, h->cfg.heads, tag, b, nullptr, enc, s, timing);
  if (st != H3BLK_OK) return st;
  return phase_out(h, sp, x, tag, tidx, mod_table, w, b, out, sms, enc, s, timing);
}

}  // namespace h3api

int h3api::mod_check(const h3blk_ctx* h, const h3blk_mod_weights* w) {
  if (!h || !w) return H3BLK_ERR_INVALID_ARG;
  if (w->freq_dim <= 0 || w->freq_dim % 16 || w->freq_dim > 1024 || w->time_hidden <= 0 || w->time_hidden % 8 ||
      w->time_dim <= 0 || w->time_dim % 8 || h->cfg.n_t > h3::kMaxModSets)
    return H3BLK_ERR_UNSUPPORTED;
  const size_t biggest = (size_t)h->cfg.n_t * (size_t)(w->time_hidden > w->time_dim ? w->time_hidden : w->time_dim);
  if (biggest * sizeof(float) > 200 * 1024) return H3BLK_ERR_UNSUPPORTED;
  return H3BLK_OK;
}

extern "C" {

const char* h3blk_error_string(int status) {
  switch (status) {
    case H3BLK_OK: return "ok";
    case H3BLK_ERR_INVALID_ARG: return "invalid argument (null or misaligned pointer, bad size, or aliasing)";
    case H3BLK_ERR_UNSUPPORTED: return "unsupported dimension or device";
    case H3BLK_ERR_CUDA: return "CUDA runtime or driver error";
    case H3BLK_ERR_TIMEOUT: return "a kernel pipeline wait timed out";
    case H3BLK_ERR_BAD_INDEX: return "a modality tag or timestep index lies outside the modulation table, or a row index outside the packed sequence";
    default: return "unknown status";
  }
}

int h3blk_version(void) { return kVersion; }

int h3blk_create(const h3blk_config* cfg, h3blk_handle* out) {
  if (!cfg || !out) return H3BLK_ERR_INVALID_ARG;
  *out = nullptr;
  const h3blk_config& c = *cfg;
  if (c.hidden <= 0 || c.heads <= 0 || c.head_dim <= 0 || c.ffn <= 0 || c.n_tags <= 0 || c.n_t <= 0 ||
      c.rope_pairs_t < 0 || c.rope_pairs_h < 0 || c.rope_pairs_w < 0 || !(c.rope_theta > 0.f) ||
      !(c.norm_eps >= 0.f) || !(c.qk_norm_eps >= 0.f) || (c.quant != 0 && c.quant != 1))
    return H3BLK_ERR_INVALID_ARG;
  if (c.hidden % 128 || c.ffn % 128 || (c.head_dim != 64 && c.head_dim != 128) || (c.heads * c.head_dim) % 128 ||
      c.rope_pairs_t + c.rope_pairs_h + c.rope_pairs_w > c.head_dim / 2 || c.hidden > 6144 || c.ffn > 16384 ||
      c.heads * c.head_dim > 16384)
    return H3BLK_ERR_UNSUPPORTED;
  h3blk_ctx* h = new (std::nothrow) h3blk_ctx;
  if (!h) return H3BLK_ERR_INVALID_ARG;
  h->cfg = c;
  h->timing = false;
  h->keep_per_1024 = 1024;
  h->dbg_gemm = -1;
  h->dbg_buf = nullptr;
  h->dbg_bytes = 0;
  for (auto& e : h->events) e = nullptr;
  const int pairs[3] = {c.rope_pairs_t, c.rope_pairs_h, c.rope_pairs_w};
  int j = 0;
  for (int axis = 0; axis < 3; ++axis)
    for (int i = 0; i < pairs[axis]; ++i, ++j) {
      h->rope.axis[j] = (int8_t)axis;
      h->rope.freq[j] = (float)std::pow((double)c.rope_theta, -(double)i / (double)pairs[axis]);
    }
  for (; j < h3::kMaxRopePairs; ++j) {
    h->rope.axis[j] = 3;
    h->rope.freq[j] = 0.f;
  }
  *out = h;
  return H3BLK_OK;
}

void h3blk_destroy(h3blk_handle h) { delete h; }

int h3blk_set_kernel_events(h3blk_handle h, void* const* events, int n_events) {
  if (!h) return H3BLK_ERR_INVALID_ARG;
  if (n_events == 0 || !events) {
    h->timing = false;
    return H3BLK_OK;
  }
  if (n_events != H3BLK_TIMING_POINTS) return H3BLK_ERR_INVALID_ARG;
  for (int i = 0; i < n_events; ++i) {
    if (!events[i]) return H3BLK_ERR_INVALID_ARG;
    h->events[i] = reinterpret_cast<cudaEvent_t>(events[i]);
  }
  h->timing = true;
  return H3BLK_OK;
}

int h3blk_set_debug_accumulators(h3blk_handle h, int gemm, void* buf, size_t bytes) {
  if (!h || gemm < -1 || gemm > 3) return H3BLK_ERR_INVALID_ARG;
  if (gemm == -1) {
    h->dbg_gemm = -1;
    h->dbg_buf = nullptr;
    h->dbg_bytes = 0;
    return H3BLK_OK;
  }
  if (h->cfg.quant == 0) return H3BLK_ERR_UNSUPPORTED;
  if (!buf || !aligned16(buf) || bytes == 0) return H3BLK_ERR_INVALID_ARG;
  h->dbg_gemm = gemm;
  h->dbg_buf = static_cast<int32_t*>(buf);
  h->dbg_bytes = bytes;
  return H3BLK_OK;
}

int h3blk_set_attention_density(h3blk_handle h, float density) {
  if (!h || !(density > 0.f && density <= 1.f)) return H3BLK_ERR_INVALID_ARG;
  int m = (int)std::lround((double)density * 1024.0);
  if (m < 1) m = 1;
  if (m > 1024) m = 1024;
  h->keep_per_1024 = m;
  return H3BLK_OK;
}

int h3blk_workspace_bytes(h3blk_handle h, int64_t n_rows, size_t* bytes) {
  if (!h || !bytes || n_rows < 1) return H3BLK_ERR_INVALID_ARG;
  *bytes = make_layout(h->cfg, n_rows, h->keep_per_1024).total;
  return H3BLK_OK;
}

int h3blk_stage_view(h3blk_handle h, int64_t n_rows, int stage, size_t* offset, size_t* bytes) {
  if (!h || !offset || !bytes || n_rows < 1 || stage < 0 || stage >= H3BLK_STAGE_COUNT) return H3BLK_ERR_INVALID_ARG;
  const Layout L = make_layout(h->cfg, n_rows, h->keep_per_1024);
  if (L.len[stage] == 0) return H3BLK_ERR_UNSUPPORTED;  // stage not produced in this mode
  *offset = L.off[stage];
  *bytes = L.len[stage];
  return H3BLK_OK;
}

int h3blk_forward(h3blk_handle h, int64_t n_rows, const void* x, const int32_t* tag, const int32_t* tidx,
                  const int32_t* pos, const float* mod_table, const h3blk_weights* w, void* out, void* workspace,
                  size_t workspace_bytes, void* stream) {
  if (!h || !w || n_rows < 1 || !x || !tag || !tidx || !pos || !mod_table || !out || !workspace)
    return H3BLK_ERR_INVALID_ARG;
  const h3blk_config& c = h->cfg;
  if (h3api::check_block_weights(c, w) != H3BLK_OK) return H3BLK_ERR_INVALID_ARG;
  const void* ptrs[] = {x, tag, tidx, pos, mod_table, out, workspace};
  for (const void* p : ptrs)
    if (!aligned16(p)) return H3BLK_ERR_INVALID_ARG;
  const Layout L = make_layout(c, n_rows, h->keep_per_1024);
  if (workspace_bytes < L.total) return H3BLK_ERR_INVALID_ARG;
  const size_t N = (size_t)n_rows, C = c.hidden;
  if (overlap(out, N * C * 2, x, N * C * 2) || overlap(out, N * C * 2, workspace, L.total) ||
      overlap(x, N * C * 2, workspace, L.total))
    return H3BLK_ERR_INVALID_ARG;
  int sms = 0;
  PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
  int st = device_info(&sms, &enc);
  if (st != H3BLK_OK) return st;

  return h3api::block_forward(h, n_rows, x, tag, tidx, pos, mod_table, w, out, workspace, sms, enc,
                              reinterpret_cast<cudaStream_t>(stream), true, h->timing);
}

int h3blk_check(h3blk_handle h, int64_t n_rows, const void* workspace, void* stream, int* status) {
  if (!h || !workspace || !status || n_rows < 1) return H3BLK_ERR_INVALID_ARG;
  const Layout L = make_layout(h->cfg, n_rows, h->keep_per_1024);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return H3BLK_ERR_CUDA;
  int bits = 0;
  if (cudaMemcpy(&bits, static_cast<const uint8_t*>(workspace) + L.off[H3BLK_STAGE_ERROR], sizeof(int),
                 cudaMemcpyDeviceToHost) != cudaSuccess)
    return H3BLK_ERR_CUDA;
  if (bits & (h3::kErrTimeoutGemm | h3::kErrTimeoutAttn | h3::kErrTimeoutStream))
    *status = H3BLK_ERR_TIMEOUT;
  else if (bits & (h3::kErrBadIndex | h3::kErrBadRowIndex))
    *status = H3BLK_ERR_BAD_INDEX;
  else
    *status = H3BLK_OK;
  return H3BLK_OK;
}

int h3blk_int8_weights_bytes(h3blk_handle h, size_t* bytes) {
  if (!h || !bytes) return H3BLK_ERR_INVALID_ARG;
  *bytes = make_blob(h->cfg).total;
  return H3BLK_OK;
}

int h3blk_prepare_int8_weights(h3blk_handle h, const h3blk_weights* in, void* blob, size_t blob_bytes,
                               h3blk_weights* out, void* stream) {
  if (!h || !in || !blob || !out) return H3BLK_ERR_INVALID_ARG;
  if (!in->wqkv || !in->q_gain || !in->k_gain || !in->wo || !in->w13 || !in->w2) return H3BLK_ERR_INVALID_ARG;
  const h3blk_config& c = h->cfg;
  const BlobLayout b = make_blob(c);
  if (blob_bytes < b.total || !aligned16(blob)) return H3BLK_ERR_INVALID_ARG;
  const void* ptrs[] = {in->wqkv, in->wo, in->w13, in->w2};
  for (const void* p : ptrs)
    if (!aligned16(p)) return H3BLK_ERR_INVALID_ARG;
  int sms = 0;
  PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
  int st = device_info(&sms, &enc);
  if (st != H3BLK_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* bl = static_cast<uint8_t*>(blob);
  const int64_t C = c.hidden, HD = (int64_t)c.heads * c.head_dim, F = c.ffn;
  auto rq = [&](const void* w, int64_t rows, int K, size_t qo, size_t so) {
    return h3::launch_rotate_quant(static_cast<const __nv_bfloat16*>(w), rows, K,
                                   reinterpret_cast<int8_t*>(bl + qo), reinterpret_cast<float*>(bl + so), nullptr, s);
  };
  if (rq(in->wqkv, 3 * HD, (int)C, b.wqkv, b.s_qkv) != cudaSuccess) return H3BLK_ERR_CUDA;
  if (rq(in->wo, C, (int)HD, b.wo, b.s_o) != cudaSuccess) return H3BLK_ERR_CUDA;
  if (rq(in->w13, 2 * F, (int)C, b.w13, b.s_13) != cudaSuccess) return H3BLK_ERR_CUDA;
  if (rq(in->w2, C, (int)F, b.w2, b.s_2) != cudaSuccess) return H3BLK_ERR_CUDA;
  if (cudaMemcpyAsync(bl + b.q_gain, in->q_gain, c.head_dim * 2, cudaMemcpyDeviceToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(bl + b.k_gain, in->k_gain, c.head_dim * 2, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return H3BLK_ERR_CUDA;
  out->wqkv = bl + b.wqkv;
  out->wo = bl + b.wo;
  out->w13 = bl + b.w13;
  out->w2 = bl + b.w2;
  out->s_qkv = reinterpret_cast<const float*>(bl + b.s_qkv);
  out->s_o = reinterpret_cast<const float*>(bl + b.s_o);
  out->s_13 = reinterpret_cast<const float*>(bl + b.s_13);
  out->s_2 = reinterpret_cast<const float*>(bl + b.s_2);
  out->q_gain = bl + b.q_gain;
  out->k_gain = bl + b.k_gain;
  return H3BLK_OK;
}


int h3blk_modulation_scratch_bytes(h3blk_handle h, const h3blk_mod_weights* w, size_t* bytes) {
  const int st = h3api::mod_check(h, w);
  if (st != H3BLK_OK) return st;
  if (!bytes) return H3BLK_ERR_INVALID_ARG;
  *bytes = (size_t)h->cfg.n_t * (size_t)(w->time_hidden + w->time_dim) * sizeof(float);
  return H3BLK_OK;
}

int h3blk_modulation_table(h3blk_handle h, const h3blk_mod_weights* w, const float* t_now, const float* t_end,
                           float gate, float* table, void* scratch, size_t scratch_bytes, void* stream) {
  int st = h3api::mod_check(h, w);
  if (st != H3BLK_OK) return st;
  const int V = h->cfg.n_t;
  if (!t_now || !table || !scratch || !w->w1 || !w->b1 || !w->w2 || !w->b2 || !w->adaln_w || !w->adaln_b)
    return H3BLK_ERR_INVALID_ARG;
  if (!(gate >= 0.f && gate <= 1.f)) return H3BLK_ERR_INVALID_ARG;
  if (gate != 0.f && (!t_end || !w->w1_r || !w->b1_r || !w->w2_r || !w->b2_r)) return H3BLK_ERR_INVALID_ARG;
  if (scratch_bytes < (size_t)V * (size_t)(w->time_hidden + w->time_dim) * sizeof(float)) return H3BLK_ERR_INVALID_ARG;
  const void* ptrs[] = {w->w1, w->w2, w->adaln_w, table, scratch};
  for (const void* p : ptrs)
    if (!aligned16(p)) return H3BLK_ERR_INVALID_ARG;
  if (gate != 0.f && (!aligned16(w->w1_r) || !aligned16(w->w2_r))) return H3BLK_ERR_INVALID_ARG;
  int sms = 0;
  PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
  st = device_info(&sms, &enc);
  if (st != H3BLK_OK) return st;
  h3::ModTableArgs m;
  std::memset(&m, 0, sizeof(m));
  m.n_sets = V;
  m.n_vec = 6;
  m.n_tags = h->cfg.n_tags;
  m.hidden = h->cfg.hidden;
  m.freq_dim = w->freq_dim;
  m.time_hidden = w->time_hidden;
  m.time_dim = w->time_dim;
  m.t_now.count = V;
  m.t_end.count = V;
  for (int k = 0; k < V; ++k) {
    m.t_now.t[k] = t_now[k];
    m.t_end.t[k] = t_end ? t_end[k] : t_now[k];
  }
  m.gate = gate;
  m.w1 = w->w1;
  m.b1 = w->b1;
  m.w2 = w->w2;
  m.b2 = w->b2;
  m.w1_r = w->w1_r;
  m.b1_r = w->b1_r;
  m.w2_r = w->w2_r;
  m.b2_r = w->b2_r;
  m.adaln_w = static_cast<const __nv_bfloat16*>(w->adaln_w);
  m.adaln_b = w->adaln_b;
  m.table = table;
  m.scratch = static_cast<float*>(scratch);
  return cuda_status(h3::launch_modulation_table(m, sms, reinterpret_cast<cudaStream_t>(stream)));
}

int h3blk_rotate_quantize(int64_t rows, int K, const void* in_bf16, int8_t* out_q, float* out_scale, void* stream) {
  if (rows < 0 || K <= 0 || K % 128 || K > 16384 || !in_bf16 || !out_q || !out_scale) return H3BLK_ERR_INVALID_ARG;
  if (!aligned16(in_bf16) || !aligned16(out_q) || !aligned16(out_scale)) return H3BLK_ERR_INVALID_ARG;
  int sms = 0;
  PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
  int st = device_info(&sms, &enc);
  if (st != H3BLK_OK) return st;
  return cuda_status(h3::launch_rotate_quant(static_cast<const __nv_bfloat16*>(in_bf16), rows, K, out_q, out_scale,
                                             nullptr, reinterpret_cast<cudaStream_t>(stream)));
}

static int plain_gemm(int64_t M, int N, int K, const void* A, const void* B, void* C, void* stream, bool int8) {
  if (M < 0 || N <= 0 || K <= 0 || !A || !B || !C) return H3BLK_ERR_INVALID_ARG;
  if (N % 128 || K % (int8 ? 128 : 64)) return H3BLK_ERR_INVALID_ARG;
  if (!aligned16(A) || !aligned16(B) || !aligned16(C)) return H3BLK_ERR_INVALID_ARG;
  int sms = 0;
  PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
  int st = device_info(&sms, &enc);
  if (st != H3BLK_OK) return st;
  GemmArgs g;
  std::memset(&g, 0, sizeof(g));
  g.A = A;
  g.B = B;
  g.M = M;
  g.N = N;
  g.Nb = N;
  g.K = K;
  g.int8 = int8;
  g.epi = int8 ? h3::kEpiStoreS32 : h3::kEpiStoreBf16;
  g.out = C;
  g.ld_out = N;
  g.err = nullptr;  // a standalone GEMM that times out just stops; C is then incomplete
  return cuda_status(h3::launch_gemm(g, enc, sms, reinterpret_cast<cudaStream_t>(stream)));
}

int h3blk_gemm_s8_s32(int64_t M, int N, int K, const int8_t* A, const int8_t* B, int32_t* C, void* stream) {
  return plain_gemm(M, N, K, A, B, C, stream, true);
}

int h3blk_gemm_bf16(int64_t M, int N, int K, const void* A, const void* B, void* C, void* stream) {
  return plain_gemm(M, N, K, A, B, C, stream, false);
}

}  // extern "C"
