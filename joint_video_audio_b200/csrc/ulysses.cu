// C-ABI of the sequence-parallel (Ulysses) block forward: G ranks each hold a
// contiguous 1/G of the packed rows; attention is the only step that needs
// every row, so it runs head-parallel instead (H/G heads per rank over all
// rows). Sources: "MiniMaxH3Transformer3DModel" (diffusers API page),
// introduction (full self-attention over the one packed sequence), and
// "HyperFlow for MiniMax-H3" (model card): its summary table, Usage (several
// GPUs) and Performance (Ulysses degree 4 on four GPUs) name Ulysses context
// parallelism over up to four GPUs.
//
// The two exchanges of the method (rows -> head groups before attention,
// head groups -> rows after it) are not separate all-to-all collectives here:
// the QKV projection's epilogue writes each head's q / k / v straight into the
// buffer of the rank that owns the head's group, and the attention epilogue
// writes each output row straight into the buffer of the rank that owns the
// row. With peer pointers those stores cross NVLink tile by tile while the
// math runs; with the rank's own send buffers the same kernels feed an
// all-to-all instead. The caller orders the three phases across the group
// (every rank's QKV phase before any rank's attention, every attention before
// any output phase): one stream on one device, or a group barrier.
#include <cuda_runtime.h>

#include <cstring>

#include "api_internal.h"
#include "ptx.cuh"

namespace {

using h3api::align256;
using h3api::aligned16;

struct ULayout {
  size_t err, tiles, modt, rope, h1, h1_q, h1_s, x1, h2, h2_q, h2_s, a, o_q, o_s, a_q, a_s, total;
};

ULayout u_layout(const h3blk_config& c, int64_t n_total, int world) {
  ULayout L;
  std::memset(&L, 0, sizeof(L));
  const size_t nl = (size_t)(n_total / world), C = c.hidden, HD = (size_t)c.heads * c.head_dim, F = c.ffn;
  const bool q = c.quant != 0;
  size_t o = 0;
  auto put = [&](size_t bytes) {
    const size_t at = o;
    o = align256(o + bytes);
    return at;
  };
  L.err = put(4);
  L.tiles = put((size_t)((n_total + 127) / 128) * sizeof(h3::TileInfo));
  L.modt = put(q ? h3::modt_bytes(c.n_tags, c.n_t, c.hidden) : 0);
  L.rope = put(h3::rope_table_bytes((int64_t)nl, c.head_dim / 2));
  if (q) {
    L.h1_q = put(nl * C);
    L.h1_s = put(nl * 4);
    L.h2_q = put(nl * C);
    L.h2_s = put(nl * 4);
    L.o_q = put(nl * HD);
    L.o_s = put(nl * 4);
    L.a_q = put(nl * F);
    L.a_s = put(nl * 4);
  } else {
    L.h1 = put(nl * C * 2);
    L.h2 = put(nl * C * 2);
  }
  L.x1 = put(nl * C * 2);
  L.a = put(nl * F * 2);
  L.total = o;
  return L;
}

int check_group(const h3blk_ctx* h, int64_t n_rows, const h3blk_ulysses* u) {
  if (!h || !u || n_rows < 1) return H3BLK_ERR_INVALID_ARG;
  if (u->world < 1 || u->world > H3BLK_MAX_RANKS || u->rank < 0 || u->rank >= u->world) return H3BLK_ERR_INVALID_ARG;
  if (h->cfg.heads % u->world || n_rows % u->world) return H3BLK_ERR_UNSUPPORTED;
  if (h->keep_per_1024 < 1024) return H3BLK_ERR_UNSUPPORTED;  // block-sparse attention is single-device
  return H3BLK_OK;
}

h3api::BlockBufs bufs(const h3blk_ctx* h, int64_t n_rows, const h3blk_ulysses* u, void* workspace) {
  const ULayout L = u_layout(h->cfg, n_rows, u->world);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  auto at = [&](size_t off, bool used) { return used ? ws + off : nullptr; };
  const bool q = h->cfg.quant != 0;
  h3api::BlockBufs b{};  // sparse buffers and anything unset stay null
  b.err = reinterpret_cast<int*>(ws + L.err);
  b.tiles = reinterpret_cast<h3::TileInfo*>(ws + L.tiles);
  b.modt = reinterpret_cast<float4*>(ws + L.modt);
  b.rope_tab = reinterpret_cast<float2*>(ws + L.rope);
  b.h1 = reinterpret_cast<__nv_bfloat16*>(at(L.h1, !q));
  b.h2 = reinterpret_cast<__nv_bfloat16*>(at(L.h2, !q));
  b.x1 = reinterpret_cast<__nv_bfloat16*>(ws + L.x1);
  b.a = reinterpret_cast<__nv_bfloat16*>(ws + L.a);
  b.h1_q = reinterpret_cast<int8_t*>(at(L.h1_q, q));
  b.h2_q = reinterpret_cast<int8_t*>(at(L.h2_q, q));
  b.o_q = reinterpret_cast<int8_t*>(at(L.o_q, q));
  b.a_q = reinterpret_cast<int8_t*>(at(L.a_q, q));
  b.h1_s = reinterpret_cast<float*>(at(L.h1_s, q));
  b.h2_s = reinterpret_cast<float*>(at(L.h2_s, q));
  b.o_s = reinterpret_cast<float*>(at(L.o_s, q));
  b.a_s = reinterpret_cast<float*>(at(L.a_s, q));
  b.qkv = static_cast<__nv_bfloat16*>(u->qkv[u->rank]);
  b.o = static_cast<__nv_bfloat16*>(u->o[u->rank]);
  return b;
}

int prologue(const h3blk_ctx* h, int64_t n_rows, const h3blk_ulysses* u, const void* workspace, size_t ws_bytes,
             int* sms, PFN_cuTensorMapEncodeTiled_v12000* enc) {
  int st = check_group(h, n_rows, u);
  if (st != H3BLK_OK) return st;
  if (!workspace || !aligned16(workspace) || ws_bytes < u_layout(h->cfg, n_rows, u->world).total)
    return H3BLK_ERR_INVALID_ARG;
  return h3api::device_info(sms, enc);
}

}  // namespace

extern "C" {

int h3blk_ulysses_buffer_bytes(h3blk_handle h, int64_t n_rows, int world, size_t* qkv_bytes, size_t* o_bytes) {
  h3blk_ulysses u;
  std::memset(&u, 0, sizeof(u));
  u.world = world;
  const int st = check_group(h, n_rows, &u);
  if (st != H3BLK_OK) return st;
  if (!qkv_bytes || !o_bytes) return H3BLK_ERR_INVALID_ARG;
  const size_t hd = (size_t)h->cfg.heads * h->cfg.head_dim;
  *qkv_bytes = (size_t)n_rows * 3 * (hd / world) * 2;
  *o_bytes = (size_t)(n_rows / world) * hd * 2;
  return H3BLK_OK;
}

int h3blk_ulysses_workspace_bytes(h3blk_handle h, int64_t n_rows, int world, size_t* bytes) {
  h3blk_ulysses u;
  std::memset(&u, 0, sizeof(u));
  u.world = world;
  const int st = check_group(h, n_rows, &u);
  if (st != H3BLK_OK) return st;
  if (!bytes) return H3BLK_ERR_INVALID_ARG;
  *bytes = u_layout(h->cfg, n_rows, world).total;
  return H3BLK_OK;
}

int h3blk_ulysses_qkv(h3blk_handle h, int64_t n_rows, const h3blk_ulysses* u, const void* x_local,
                      const int32_t* tag, const int32_t* tidx, const int32_t* pos, const float* mod_table,
                      const h3blk_weights* w, void* workspace, size_t workspace_bytes, void* stream) {
  int sms = 0;
  PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
  if (!x_local || !tag || !tidx || !pos || !mod_table || !w) return H3BLK_ERR_INVALID_ARG;
  int st = check_group(h, n_rows, u);
  if (st != H3BLK_OK) return st;
  if (h3api::check_block_weights(h->cfg, w) != H3BLK_OK) return H3BLK_ERR_INVALID_ARG;
  const void* ptrs[] = {x_local, tag, tidx, pos, mod_table};
  for (const void* p : ptrs)
    if (!aligned16(p)) return H3BLK_ERR_INVALID_ARG;
  for (int d = 0; d < u->world; ++d)
    if (!u->qkv[d] || !aligned16(u->qkv[d])) return H3BLK_ERR_INVALID_ARG;
  st = prologue(h, n_rows, u, workspace, workspace_bytes, &sms, &enc);
  if (st != H3BLK_OK) return st;
  const int64_t nl = n_rows / u->world;
  const h3api::Span sp{nl, u->rank * nl, n_rows};
  h3api::QkvRoute route;
  std::memset(&route, 0, sizeof(route));
  route.ranks = u->world;
  route.hg = h->cfg.heads / u->world;
  for (int d = 0; d < u->world; ++d) route.dst[d] = u->qkv[d];
  return h3api::phase_qkv(h, sp, x_local, tag, tidx, pos, mod_table, w, bufs(h, n_rows, u, workspace), &route, sms,
                          enc, reinterpret_cast<cudaStream_t>(stream), true, false);
}

int h3blk_ulysses_attention(h3blk_handle h, int64_t n_rows, const h3blk_ulysses* u, const int32_t* tag,
                            void* workspace, size_t workspace_bytes, void* stream) {
  int sms = 0;
  PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
  if (!tag || !aligned16(tag)) return H3BLK_ERR_INVALID_ARG;
  int st = check_group(h, n_rows, u);
  if (st != H3BLK_OK) return st;
  if (!u->qkv[u->rank] || !aligned16(u->qkv[u->rank])) return H3BLK_ERR_INVALID_ARG;
  for (int d = 0; d < u->world; ++d)
    if (!u->o[d] || !aligned16(u->o[d])) return H3BLK_ERR_INVALID_ARG;
  st = prologue(h, n_rows, u, workspace, workspace_bytes, &sms, &enc);
  if (st != H3BLK_OK) return st;
  const int hg = h->cfg.heads / u->world;
  h3api::ORoute route;
  std::memset(&route, 0, sizeof(route));
  route.ranks = u->world;
  route.head0 = u->rank * hg;
  route.rows = n_rows / u->world;
  route.ld = (int64_t)h->cfg.heads * h->cfg.head_dim;
  for (int d = 0; d < u->world; ++d) route.dst[d] = u->o[d];
  return h3api::phase_attention(h, n_rows, hg, tag, bufs(h, n_rows, u, workspace), &route, enc,
                                reinterpret_cast<cudaStream_t>(stream), false);
}

int h3blk_ulysses_out(h3blk_handle h, int64_t n_rows, const h3blk_ulysses* u, const void* x_local,
                      const int32_t* tag, const int32_t* tidx, const float* mod_table, const h3blk_weights* w,
                      void* out_local, void* workspace, size_t workspace_bytes, void* stream) {
  int sms = 0;
  PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
  if (!x_local || !tag || !tidx || !mod_table || !w || !out_local) return H3BLK_ERR_INVALID_ARG;
  int st = check_group(h, n_rows, u);
  if (st != H3BLK_OK) return st;
  if (h3api::check_block_weights(h->cfg, w) != H3BLK_OK) return H3BLK_ERR_INVALID_ARG;
  const void* ptrs[] = {x_local, tag, tidx, mod_table, out_local, u->o[u->rank]};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return H3BLK_ERR_INVALID_ARG;
  const int64_t nl = n_rows / u->world;
  const size_t row_bytes = (size_t)h->cfg.hidden * 2;
  const uintptr_t xo = reinterpret_cast<uintptr_t>(out_local), xi = reinterpret_cast<uintptr_t>(x_local);
  if (xo < xi + nl * row_bytes && xi < xo + nl * row_bytes) return H3BLK_ERR_INVALID_ARG;  // out aliases x
  st = prologue(h, n_rows, u, workspace, workspace_bytes, &sms, &enc);
  if (st != H3BLK_OK) return st;
  const h3api::Span sp{nl, u->rank * nl, n_rows};
  return h3api::phase_out(h, sp, x_local, tag, tidx, mod_table, w, bufs(h, n_rows, u, workspace), out_local, sms,
                          enc, reinterpret_cast<cudaStream_t>(stream), false);
}

}  // extern "C"
