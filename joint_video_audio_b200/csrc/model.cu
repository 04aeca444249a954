// C-ABI of the model shell: the launch sequence of a whole transformer forward
// around the block (input projections, token refiner, the block stack with
// each layer's AdaLN table produced just before it, norm_out and the two
// heads), and its capture into a CUDA graph (see include/h3blk.h).
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstring>
#include <new>

#include "api_internal.h"
#include "ptx.cuh"

namespace {

using h3api::align256;
using h3api::aligned16;

// Model workspace: the block workspace first, so the error word every kernel
// reports into sits at offset 0 for the refiner's and the stack's layers alike.
struct ModelLayout {
  size_t block, xa, xb, table, table_o, time, ra, rb, ttag, ttidx, tpos, total;
};

h3blk_config refiner_config(const h3blk_config& c) {
  h3blk_config r = c;
  r.quant = 0;  // the refiner stays bf16
  return r;
}

ModelLayout model_layout(const h3blk_config& c, const h3blk_mod_weights& t, int64_t n, int64_t nt, int keep) {
  ModelLayout L;
  std::memset(&L, 0, sizeof(L));
  const size_t C = c.hidden, N = (size_t)n, NT = (size_t)nt;
  size_t blk = h3api::block_workspace_bytes(c, n, keep);
  if (nt > 0) {
    const size_t r = h3api::block_workspace_bytes(refiner_config(c), nt, keep);
    if (r > blk) blk = r;
  }
  size_t o = 0;
  auto put = [&](size_t bytes) {
    const size_t at = o;
    o = align256(o + bytes);
    return at;
  };
  L.block = put(blk);
  L.xa = put(N * C * 2);
  L.xb = put(N * C * 2);
  L.table = put((size_t)c.n_tags * c.n_t * 6 * C * 4);
  L.table_o = put((size_t)c.n_tags * c.n_t * 2 * C * 4);
  L.time = put((size_t)c.n_t * (size_t)(t.time_hidden + t.time_dim) * 4);
  if (nt > 0) {
    L.ra = put(NT * C * 2);
    L.rb = put(NT * C * 2);
    L.ttag = put(NT * 4);
    L.ttidx = put(NT * 4);
    L.tpos = put(NT * 12);
  }
  L.total = o;
  return L;
}

int check_model(const h3blk_ctx* h, const h3blk_model_config* mc, const h3blk_mod_weights* t) {
  if (!h || !mc || !t) return H3BLK_ERR_INVALID_ARG;
  if (mc->n_layers < 0 || mc->n_refiner < 0 || !(mc->final_norm_eps >= 0.f)) return H3BLK_ERR_INVALID_ARG;
  if (mc->video_in <= 0 || mc->video_in % 4 || mc->video_in > 128 || mc->audio_in <= 0 || mc->audio_in % 4 ||
      mc->audio_in > 128 || mc->text_dim <= 0 || mc->text_dim % 64)
    return H3BLK_ERR_UNSUPPORTED;
  return h3api::mod_check(h, t);
}

// Host-side validation of weights and inputs shared by the eager forward and
// the graph capture.
int check_forward(const h3blk_ctx* h, const h3blk_model_config* mc, const h3blk_model_weights* w,
                  const h3blk_model_inputs* in, const float* video_out, const float* audio_out, const void* ws,
                  size_t ws_bytes) {
  if (!w || !in) return H3BLK_ERR_INVALID_ARG;
  int st = check_model(h, mc, &w->time);
  if (st != H3BLK_OK) return st;
  const h3blk_config& c = h->cfg;
  const h3blk_config rc = refiner_config(c);
  if (in->n_rows < 1 || in->n_video < 0 || in->n_audio < 0 || in->n_text < 0 ||
      in->n_video + in->n_audio + in->n_text > in->n_rows)
    return H3BLK_ERR_INVALID_ARG;
  if (!in->tag || !in->tidx || !in->pos || !in->t_now || !ws) return H3BLK_ERR_INVALID_ARG;
  if (!(in->gate >= 0.f && in->gate <= 1.f)) return H3BLK_ERR_INVALID_ARG;
  if (in->gate != 0.f && (!in->t_end || !w->time.w1_r || !w->time.b1_r || !w->time.w2_r || !w->time.b2_r))
    return H3BLK_ERR_INVALID_ARG;
  if (!w->time.w1 || !w->time.b1 || !w->time.w2 || !w->time.b2 || !w->out_adaln_w || !w->out_adaln_b)
    return H3BLK_ERR_INVALID_ARG;
  if (in->n_video > 0 && (!in->video_idx || !in->video || !video_out || !w->proj_in_w || !w->proj_in_b ||
                          !w->proj_out_w || !w->proj_out_b))
    return H3BLK_ERR_INVALID_ARG;
  if (in->n_audio > 0 && (!in->audio_idx || !in->audio || !audio_out || !w->audio_in_w || !w->audio_in_b ||
                          !w->audio_out_w || !w->audio_out_b))
    return H3BLK_ERR_INVALID_ARG;
  if (in->n_text > 0 && (!in->text_idx || !in->text || !w->ctx_w || !w->ctx_b || !w->refiner_gain))
    return H3BLK_ERR_INVALID_ARG;
  if ((mc->n_layers > 0 && !w->layers) || (mc->n_refiner > 0 && in->n_text > 0 && !w->refiner))
    return H3BLK_ERR_INVALID_ARG;
  for (int l = 0; l < mc->n_layers; ++l)
    if (h3api::check_block_weights(c, &w->layers[l].w) != H3BLK_OK || !w->layers[l].adaln_w ||
        !w->layers[l].adaln_b || !aligned16(w->layers[l].adaln_w))
      return H3BLK_ERR_INVALID_ARG;
  if (in->n_text > 0)
    for (int l = 0; l < mc->n_refiner; ++l)
      if (h3api::check_block_weights(rc, &w->refiner[l].w) != H3BLK_OK || !w->refiner[l].adaln_w ||
          !w->refiner[l].adaln_b || !aligned16(w->refiner[l].adaln_w))
        return H3BLK_ERR_INVALID_ARG;
  const void* ptrs[] = {in->tag, in->tidx, in->pos, in->video, in->audio, in->text, video_out, audio_out, ws,
                        w->time.w1, w->time.w2, w->time.w1_r, w->time.w2_r, w->out_adaln_w, w->proj_in_w,
                        w->audio_in_w, w->ctx_w, w->ctx_b, w->proj_in_b, w->audio_in_b, w->proj_out_w,
                        w->audio_out_w, w->refiner_gain};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return H3BLK_ERR_INVALID_ARG;
  if (ws_bytes < model_layout(c, w->time, in->n_rows, in->n_text, h->keep_per_1024).total) return H3BLK_ERR_INVALID_ARG;
  return H3BLK_OK;
}

#define H3_TRY(expr)                                \
  do {                                              \
    cudaError_t e_ = (expr);                        \
    if (e_ != cudaSuccess) return H3BLK_ERR_CUDA;   \
  } while (0)

// The launch sequence (arguments already validated).
int run_forward(const h3blk_ctx* h, const h3blk_model_config* mc, const h3blk_model_weights* w,
                const h3blk_model_inputs* in, float* video_out, float* audio_out, void* workspace, cudaStream_t s) {
  int sms = 0;
  PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
  int st = h3api::device_info(&sms, &enc);
  if (st != H3BLK_OK) return st;
  const h3blk_config& c = h->cfg;
  const int64_t N = in->n_rows, NT = in->n_text;
  const ModelLayout L = model_layout(c, w->time, N, NT, h->keep_per_1024);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int* err = reinterpret_cast<int*>(ws + L.block);  // the block workspace's error word
  auto* xa = reinterpret_cast<__nv_bfloat16*>(ws + L.xa);
  auto* xb = reinterpret_cast<__nv_bfloat16*>(ws + L.xb);
  float* table = reinterpret_cast<float*>(ws + L.table);
  float* table_o = reinterpret_cast<float*>(ws + L.table_o);
  const int C = c.hidden;

  H3_TRY(cudaMemsetAsync(err, 0, sizeof(int), s));

  // ---- time embedding of the forward's timestep sets (device timesteps)
  h3::ModTableArgs m;
  std::memset(&m, 0, sizeof(m));
  m.n_sets = c.n_t;
  m.n_tags = c.n_tags;
  m.hidden = C;
  m.freq_dim = w->time.freq_dim;
  m.time_hidden = w->time.time_hidden;
  m.time_dim = w->time.time_dim;
  m.t_now.count = c.n_t;
  m.t_now.dev = in->t_now;
  m.t_end.count = c.n_t;
  m.t_end.dev = in->t_end ? in->t_end : in->t_now;
  m.gate = in->gate;
  m.w1 = w->time.w1;
  m.b1 = w->time.b1;
  m.w2 = w->time.w2;
  m.b2 = w->time.b2;
  m.w1_r = w->time.w1_r;
  m.b1_r = w->time.b1_r;
  m.w2_r = w->time.w2_r;
  m.b2_r = w->time.b2_r;
  m.scratch = reinterpret_cast<float*>(ws + L.time);
  H3_TRY(h3::launch_time_embedding(m, sms, s));
  auto project = [&](const void* aw, const float* ab, int n_vec, float* dst) {
    h3::ModTableArgs p = m;
    p.n_vec = n_vec;
    p.adaln_w = static_cast<const __nv_bfloat16*>(aw);
    p.adaln_b = ab;
    p.table = dst;
    return h3::launch_adaln_projection(p, sms, s);
  };
  H3_TRY(project(w->out_adaln_w, w->out_adaln_b, 2, table_o));

  // ---- packed input sequence: padding rows zero, video and audio rows projected
  H3_TRY(cudaMemsetAsync(xa, 0, (size_t)N * C * 2, s));
  H3_TRY(h3::launch_embed_rows(in->video, in->n_video, mc->video_in, w->proj_in_w, w->proj_in_b, C, in->video_idx,
                               N, xa, err, s));
  H3_TRY(h3::launch_embed_rows(in->audio, in->n_audio, mc->audio_in, w->audio_in_w, w->audio_in_b, C, in->audio_idx,
                               N, xa, err, s));

  // ---- text rows: context embedder, token refiner over the text rows alone, output norm
  if (NT > 0) {
    auto* ra = reinterpret_cast<__nv_bfloat16*>(ws + L.ra);
    auto* rb = reinterpret_cast<__nv_bfloat16*>(ws + L.rb);
    auto* ttag = reinterpret_cast<int32_t*>(ws + L.ttag);
    auto* ttidx = reinterpret_cast<int32_t*>(ws + L.ttidx);
    auto* tpos = reinterpret_cast<int32_t*>(ws + L.tpos);
    H3_TRY(h3::launch_gather_meta(in->text_idx, NT, N, in->tag, in->tidx, in->pos, ttag, ttidx, tpos, err, s));
    h3::GemmArgs g;
    std::memset(&g, 0, sizeof(g));
    g.A = in->text;
    g.B = w->ctx_w;
    g.M = NT;
    g.N = C;
    g.Nb = C;
    g.K = mc->text_dim;
    g.epi = h3::kEpiStoreBf16;
    g.out = ra;
    g.ld_out = C;
    g.bias = w->ctx_b;
    g.err = err;
    H3_TRY(h3::launch_gemm(g, enc, sms, s));
    h3blk_ctx rh = *h;
    rh.cfg = refiner_config(c);
    rh.timing = false;
    for (int l = 0; l < mc->n_refiner; ++l) {
      H3_TRY(project(w->refiner[l].adaln_w, w->refiner[l].adaln_b, 6, table));
      st = h3api::block_forward(&rh, NT, ra, ttag, ttidx, tpos, table, &w->refiner[l].w, rb, ws + L.block, sms, enc,
                                s, false, false);
      if (st != H3BLK_OK) return st;
      auto* t = ra;
      ra = rb;
      rb = t;
    }
    H3_TRY(h3::launch_norm_scatter(ra, NT, C, static_cast<const __nv_bfloat16*>(w->refiner_gain),
                                   mc->final_norm_eps, in->text_idx, N, xa, err, s));
  }

  // ---- the block stack: each layer's table just before the layer
  for (int l = 0; l < mc->n_layers; ++l) {
    H3_TRY(project(w->layers[l].adaln_w, w->layers[l].adaln_b, 6, table));
    st = h3api::block_forward(h, N, xa, in->tag, in->tidx, in->pos, table, &w->layers[l].w, xb, ws + L.block, sms,
                              enc, s, false, false);
    if (st != H3BLK_OK) return st;
    auto* t = xa;
    xa = xb;
    xb = t;
  }

  // ---- norm_out + heads
  h3::HeadArgs hd;
  std::memset(&hd, 0, sizeof(hd));
  hd.x = xa;
  hd.n_rows = N;
  hd.C = C;
  hd.tag = in->tag;
  hd.tidx = in->tidx;
  hd.table = table_o;
  hd.n_tags = c.n_tags;
  hd.n_t = c.n_t;
  hd.eps = mc->final_norm_eps;
  hd.err = err;
  hd.idx = in->video_idx;
  hd.M = in->n_video;
  hd.n_out = mc->video_in;
  hd.W = w->proj_out_w;
  hd.b = w->proj_out_b;
  hd.y = video_out;
  H3_TRY(h3::launch_head(hd, sms, s));
  hd.idx = in->audio_idx;
  hd.M = in->n_audio;
  hd.n_out = mc->audio_in;
  hd.W = w->audio_out_w;
  hd.b = w->audio_out_b;
  hd.y = audio_out;
  H3_TRY(h3::launch_head(hd, sms, s));
  return H3BLK_OK;
}

}  // namespace

struct h3blk_graph_s {
  cudaGraphExec_t exec;
  int kernel_nodes, other_nodes;
};

extern "C" {

int h3blk_model_workspace_bytes(h3blk_handle h, const h3blk_model_config* mc, const h3blk_mod_weights* time,
                                int64_t n_rows, int64_t n_text, size_t* bytes) {
  const int st = check_model(h, mc, time);
  if (st != H3BLK_OK) return st;
  if (!bytes || n_rows < 1 || n_text < 0 || n_text > n_rows) return H3BLK_ERR_INVALID_ARG;
  *bytes = model_layout(h->cfg, *time, n_rows, n_text, h->keep_per_1024).total;
  return H3BLK_OK;
}

int h3blk_model_forward(h3blk_handle h, const h3blk_model_config* mc, const h3blk_model_weights* w,
                        const h3blk_model_inputs* in, float* video_out, float* audio_out, void* workspace,
                        size_t workspace_bytes, void* stream) {
  const int st = check_forward(h, mc, w, in, video_out, audio_out, workspace, workspace_bytes);
  if (st != H3BLK_OK) return st;
  return run_forward(h, mc, w, in, video_out, audio_out, workspace, reinterpret_cast<cudaStream_t>(stream));
}

int h3blk_model_check(const void* workspace, void* stream, int* status) {
  if (!workspace || !status) return H3BLK_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return H3BLK_ERR_CUDA;
  int bits = 0;
  if (cudaMemcpy(&bits, workspace, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return H3BLK_ERR_CUDA;
  if (bits & (h3::kErrTimeoutGemm | h3::kErrTimeoutAttn | h3::kErrTimeoutStream))
    *status = H3BLK_ERR_TIMEOUT;
  else if (bits & (h3::kErrBadIndex | h3::kErrBadRowIndex))
    *status = H3BLK_ERR_BAD_INDEX;
  else
    *status = H3BLK_OK;
  return H3BLK_OK;
}

int h3blk_model_graph_create(h3blk_handle h, const h3blk_model_config* mc, const h3blk_model_weights* w,
                             const h3blk_model_inputs* in, float* video_out, float* audio_out, void* workspace,
                             size_t workspace_bytes, h3blk_graph* out) {
  if (!out) return H3BLK_ERR_INVALID_ARG;
  *out = nullptr;
  int st = check_forward(h, mc, w, in, video_out, audio_out, workspace, workspace_bytes);
  if (st != H3BLK_OK) return st;
  // resolve the device info and kernel attributes before capture
  int sms = 0;
  PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
  st = h3api::device_info(&sms, &enc);
  if (st != H3BLK_OK) return st;
  cudaStream_t cs = nullptr;
  if (cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking) != cudaSuccess) return H3BLK_ERR_CUDA;
  cudaGraph_t graph = nullptr;
  if (cudaStreamBeginCapture(cs, cudaStreamCaptureModeThreadLocal) != cudaSuccess) {
    cudaStreamDestroy(cs);
    return H3BLK_ERR_CUDA;
  }
  st = run_forward(h, mc, w, in, video_out, audio_out, workspace, cs);
  const cudaError_t e_end = cudaStreamEndCapture(cs, &graph);
  cudaStreamDestroy(cs);
  if (st != H3BLK_OK || e_end != cudaSuccess || !graph) {
    if (graph) cudaGraphDestroy(graph);
    cudaGetLastError();
    return st != H3BLK_OK ? st : H3BLK_ERR_CUDA;
  }
  // node census: kernel launches vs memsets and the like
  int kernels = 0, others = 0;
  size_t n_nodes = 0;
  if (cudaGraphGetNodes(graph, nullptr, &n_nodes) == cudaSuccess && n_nodes > 0) {
    cudaGraphNode_t* nodes = new (std::nothrow) cudaGraphNode_t[n_nodes];
    if (nodes && cudaGraphGetNodes(graph, nodes, &n_nodes) == cudaSuccess) {
      for (size_t i = 0; i < n_nodes; ++i) {
        cudaGraphNodeType t;
        if (cudaGraphNodeGetType(nodes[i], &t) != cudaSuccess) continue;
        if (t == cudaGraphNodeTypeKernel)
          ++kernels;
        else
          ++others;
      }
    }
    delete[] nodes;
  }
  cudaGraphExec_t exec = nullptr;
  const cudaError_t e_inst = cudaGraphInstantiate(&exec, graph, 0);
  cudaGraphDestroy(graph);
  if (e_inst != cudaSuccess) return H3BLK_ERR_CUDA;
  h3blk_graph g = new (std::nothrow) h3blk_graph_s;
  if (!g) {
    cudaGraphExecDestroy(exec);
    return H3BLK_ERR_INVALID_ARG;
  }
  g->exec = exec;
  g->kernel_nodes = kernels;
  g->other_nodes = others;
  *out = g;
  return H3BLK_OK;
}

int h3blk_graph_launch(h3blk_graph g, void* stream) {
  if (!g) return H3BLK_ERR_INVALID_ARG;
  return h3api::cuda_status(cudaGraphLaunch(g->exec, reinterpret_cast<cudaStream_t>(stream)));
}

int h3blk_graph_info(h3blk_graph g, int* kernel_nodes, int* other_nodes) {
  if (!g || !kernel_nodes || !other_nodes) return H3BLK_ERR_INVALID_ARG;
  *kernel_nodes = g->kernel_nodes;
  *other_nodes = g->other_nodes;
  return H3BLK_OK;
}

void h3blk_graph_destroy(h3blk_graph g) {
  if (!g) return;
  cudaGraphExecDestroy(g->exec);
  delete g;
}

}  // extern "C"
