/*
 * h3blk — forward of one MiniMax-H3 transformer block on a B200 (sm_100a).
 *
 * The block runs over ONE packed 1-D sequence of N rows (text, conditioning
 * image/video, audio and target-video rows, plus optional padding rows) with
 * full self-attention, per-row AdaLN modulation selected by a modality tag and
 * a timestep index, per-head QK RMSNorm, 3D (t, h, w) rotary embedding and a
 * SwiGLU feed-forward:
 *
 *   m      = table[tag[r]][tidx[r]]            (6 vectors; zeros for tag -1)
 *   h1     = rmsnorm(x) * (1 + scale1) + shift1
 *   q,k,v  = h1 Wqkv^T;  q = rope(rmsnorm_D(q) g_q),  k = rope(rmsnorm_D(k) g_k)
 *   o      = softmax(q k^T / sqrt(D) + docmask) v      (doc(r) = tag[r] == -1)
 *   x1     = x  + gate1 * (o Wo^T)
 *   h2     = rmsnorm(x1) * (1 + scale2) + shift2
 *   out    = x1 + gate2 * ((silu(h2 W1^T) * (h2 W3^T)) W2^T)
 *
 * Sources (page title, section):
 *   "MiniMaxH3Transformer3DModel" (diffusers API page)
 *     - introduction: one packed sequence, full self-attention, no
 *       cross-attention, no per-modality block weights; the per-row modality
 *       tag selects the AdaLN modulation; padding rows (tag -1) form their own
 *       attention document;
 *     - constructor: hidden_size, num_attention_heads x attention_head_dim
 *       (larger than hidden), ffn_dim (SwiGLU), rope_theta, norm_eps of the
 *       pre-attention / pre-feed-forward norms, qk_norm_eps of the per-head
 *       query/key norms;
 *     - forward: timestep_indices, token_tags, position_ids (seq_len, 3).
 *   "HyperFlow H3 Flash Brings MiniMax H3 Video to One GPU",
 *     "How it got smaller and faster": rotated W8A8 INT8 linears.
 * The block's equations are not printed on the pages; the reading above
 * (sequential AdaLN pre-norm block, gain-free RMSNorm pre-norms, modulation
 * order shift/scale/gate x 2, adjacent-pair RoPE with per-axis frequencies
 * theta^(-i/n)) is the one this library implements.
 *
 * Conventions for every entry point:
 *   - Return value: H3BLK_OK (0) or one of the H3BLK_ERR_* codes below.
 *     h3blk_error_string() gives a message. Nothing is thrown or aborted.
 *   - Device pointers are CUDA global-memory pointers owned by the caller and
 *     must be 16-byte aligned. The library never allocates device memory:
 *     every intermediate lives in the caller's workspace.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream). Calls are asynchronous on it: no host synchronisation, except
 *     in h3blk_check.
 *   - Matrices are row-major; a linear's weight is [out_features, in_features].
 */
#ifndef H3BLK_H
#define H3BLK_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define H3BLK_API __attribute__((visibility("default")))
#else
#define H3BLK_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ------------------------------------------------------------------ status */
#define H3BLK_OK 0
#define H3BLK_ERR_INVALID_ARG 1 /* null / misaligned pointer, bad size, aliasing */
#define H3BLK_ERR_UNSUPPORTED 2 /* a dimension this library does not handle */
#define H3BLK_ERR_CUDA 3        /* a CUDA runtime / driver call failed */
#define H3BLK_ERR_TIMEOUT 4     /* a kernel pipeline wait gave up (reported by h3blk_check) */
#define H3BLK_ERR_BAD_INDEX 5   /* a tag / timestep index outside the table (h3blk_check) */

/* ------------------------------------------------------------------ config */
typedef struct {
  int hidden;       /* C: channels of the residual stream (multiple of 128)          */
  int heads;        /* H                                                               */
  int head_dim;     /* D: 64 or 128                                                    */
  int ffn;          /* F: SwiGLU inner dimension (multiple of 128)                     */
  int n_tags;       /* modality tags 0..n_tags-1 (tag -1 = padding)                    */
  int n_t;          /* distinct timestep indices 0..n_t-1                              */
  int rope_pairs_t; /* rotary pairs driven by the t / h / w coordinate, in this order; */
  int rope_pairs_h; /* their sum is <= head_dim/2 and the remaining pairs pass through */
  int rope_pairs_w;
  float rope_theta; /* frequency of pair i of an axis with n pairs: theta^(-i/n)       */
  float norm_eps;   /* eps of the two AdaLN pre-norms                                  */
  float qk_norm_eps;/* eps of the per-head q / k RMSNorm                               */
  int quant;        /* 0: bf16 linears; 1: rotated W8A8 INT8 linears                   */
} h3blk_config;

typedef struct h3blk_ctx* h3blk_handle;

/* Weights of one block (device pointers, caller-owned, each 16-byte aligned:
 * the GEMM epilogues read gains and scales 16 bytes at a time; a misaligned
 * pointer is INVALID_ARG).
 * quant == 0: all matrices bf16; s_* unused (may be NULL).
 * quant == 1: matrices int8 as written by h3blk_prepare_int8_weights (input
 *             channels rotated by the block-128 Hadamard transform), s_* the
 *             fp32 per-output-channel scales. q_gain / k_gain stay bf16.
 *   wqkv [3*H*D, C]  rows: q of heads 0..H-1, then k, then v
 *   q_gain, k_gain [D]
 *   wo   [C, H*D]
 *   w13  [2F, C]     rows 0..F-1 = W1 (gate, through silu), F..2F-1 = W3 (up)
 *   w2   [C, F]                                                              */
typedef struct {
  const void* wqkv;
  const void* q_gain;
  const void* k_gain;
  const void* wo;
  const void* w13;
  const void* w2;
  const float* s_qkv; /* [3*H*D] */
  const float* s_o;   /* [C]     */
  const float* s_13;  /* [2F]    */
  const float* s_2;   /* [C]     */
} h3blk_weights;

/* Creates a handle from a configuration. Host-only: touches no GPU.
 * INVALID_ARG for null pointers or non-positive sizes; UNSUPPORTED when
 * hidden or ffn is not a multiple of 128, head_dim is not 64 or 128, heads *
 * head_dim is not a multiple of 128, or the rotary pairs exceed head_dim/2.
 * The handle owns only host memory; release it with h3blk_destroy. */
H3BLK_API int h3blk_create(const h3blk_config* cfg, h3blk_handle* out);

/* Releases a handle (NULL is ignored). */
H3BLK_API void h3blk_destroy(h3blk_handle h);

/* Workspace bytes h3blk_forward needs for n_rows rows (n_rows >= 1). */
H3BLK_API int h3blk_workspace_bytes(h3blk_handle h, int64_t n_rows, size_t* bytes);

/* Stage buffers inside the workspace, readable after h3blk_forward (for
 * stage-by-stage checks). Layout of each stage, all row-major:
 *   H3BLK_STAGE_H1, _H2        bf16 [N, C]      pre-norm outputs (bf16 path only)
 *   H3BLK_STAGE_X1             bf16 [N, C]      residual after the attention branch
 *   H3BLK_STAGE_QKV            bf16 [N, 3*H*D]  q | k | v after QK-norm + RoPE
 *   H3BLK_STAGE_O              bf16 [N, H*D]    attention output
 *   H3BLK_STAGE_A              bf16 [N, F]      SwiGLU output
 *   H3BLK_STAGE_*_Q8           int8 [N, K]      rotated, quantised linear input (W8A8)
 *   H3BLK_STAGE_*_SCALE        fp32 [N]         its per-row scale            (W8A8)
 *   H3BLK_STAGE_ERROR          int32 [1]        device error bits of the last forward
 *   H3BLK_STAGE_KV_LIST        int32 [ceil(N/256)][H][1 + ceil(N/128)]  block-sparse mode
 *                              only: per 256-query block and head, the count of
 *                              kept 128-key tiles, then the tiles ascending */
enum {
  H3BLK_STAGE_H1 = 0,
  H3BLK_STAGE_QKV = 1,
  H3BLK_STAGE_O = 2,
  H3BLK_STAGE_X1 = 3,
  H3BLK_STAGE_H2 = 4,
  H3BLK_STAGE_A = 5,
  H3BLK_STAGE_H1_Q8 = 6,
  H3BLK_STAGE_H1_SCALE = 7,
  H3BLK_STAGE_O_Q8 = 8,
  H3BLK_STAGE_O_SCALE = 9,
  H3BLK_STAGE_H2_Q8 = 10,
  H3BLK_STAGE_H2_SCALE = 11,
  H3BLK_STAGE_A_Q8 = 12,
  H3BLK_STAGE_A_SCALE = 13,
  H3BLK_STAGE_ERROR = 14,
  H3BLK_STAGE_KV_LIST = 15,
  H3BLK_STAGE_COUNT = 16
};
H3BLK_API int h3blk_stage_view(h3blk_handle h, int64_t n_rows, int stage, size_t* offset, size_t* bytes);

/* One block forward over n_rows packed rows.
 *   x         bf16 [N, C]            input rows
 *   tag       int32 [N]              modality tag in [0, n_tags), -1 = padding
 *   tidx      int32 [N]              timestep index in [0, n_t) (ignored for padding)
 *   pos       int32 [N, 3]           (t, h, w) rotary coordinates
 *   mod_table fp32 [n_tags][n_t][6][C]: shift1, scale1, gate1, shift2, scale2, gate2
 *   w         weights (see h3blk_weights)
 *   out       bf16 [N, C]            must not overlap x or the workspace
 *   workspace >= h3blk_workspace_bytes(h, N) bytes of device memory
 * Padding rows leave the block unchanged (out = x) and never influence other
 * rows. Indices outside the table are not read: such rows get zero modulation
 * and the error is reported by h3blk_check. */
H3BLK_API int h3blk_forward(h3blk_handle h, int64_t n_rows, const void* x, const int32_t* tag, const int32_t* tidx,
                  const int32_t* pos, const float* mod_table, const h3blk_weights* w, void* out,
                  void* workspace, size_t workspace_bytes, void* stream);

/* Synchronises `stream` and reads the device error word of the last forward
 * that used `workspace`: *status = H3BLK_OK, H3BLK_ERR_BAD_INDEX or
 * H3BLK_ERR_TIMEOUT. */
H3BLK_API int h3blk_check(h3blk_handle h, int64_t n_rows, const void* workspace, void* stream, int* status);

/* Block-sparse attention for later forwards on this handle (the optional
 * sparse backend of "HyperFlow for MiniMax-H3", model card: summary table and
 * Performance; its method is not described there, so this is this library's
 * reading). density = 1 (the default) is dense attention. For 0 < density < 1,
 * every 256-query block keeps, per head, k = max(1, ceil(n * m / 1024)) of the
 * n 128-key tiles that hold a valid row, m = round(1024 * density): those
 * whose mean key has the largest dot product with the block's mean query
 * (means over valid rows; ties toward the lower tile). Valid rows then attend
 * only to the valid keys of the kept tiles; padding rows' attention output is
 * undefined (the block's zero gates discard it). The workspace grows
 * (h3blk_workspace_bytes follows the setting). INVALID_ARG unless
 * 0 < density <= 1; UNSUPPORTED for the sequence-parallel calls. */
H3BLK_API int h3blk_set_attention_density(h3blk_handle h, float density);

/* Per-kernel timing. When set, every later h3blk_forward on this handle
 * records the caller's CUDA events (cudaEvent_t passed as void*) on its stream
 * at H3BLK_TIMING_POINTS points: before each of the forward's kernel groups
 * and after the last one. Interval i (events[i] -> events[i+1]) covers:
 *   0 prep (error word reset + tile summary), 1 pre-attention norm (+ int8
 *   quant), 2 QKV GEMM, 3 attention, 4 int8 quant of the attention output
 *   (empty on the bf16 path), 5 out-projection GEMM, 6 pre-FFN norm, 7 FFN-up
 *   GEMM + SwiGLU, 8 int8 quant of the SwiGLU output (empty on the bf16
 *   path), 9 FFN-down GEMM.
 * The events stay owned by the caller; n_events = 0 (or events = NULL)
 * switches recording off. INVALID_ARG unless n_events is 0 or
 * H3BLK_TIMING_POINTS. */
#define H3BLK_TIMING_POINTS 11
H3BLK_API int h3blk_set_kernel_events(h3blk_handle h, void* const* events, int n_events);

/* Test-only, W8A8 handles: when gemm is 0 (QKV), 1 (out-projection), 2 (FFN
 * up, W1 | W3) or 3 (FFN down), every later h3blk_forward on this handle also
 * writes that int8 GEMM's raw int32 accumulators, as its epilogue reads them
 * from tensor memory before dequantisation, to `buf` as int32
 * [n_rows, weight rows] row-major (weight rows: 3*heads*head_dim, hidden,
 * 2*ffn, hidden). The integer product of the rotated W8A8 linears ("HyperFlow
 * H3 Flash ...", "How it got smaller and faster") can then be checked bit for
 * bit against the GPU's own int8 operands. `buf` is caller-owned device
 * memory (16-byte aligned) of `bytes`; a forward whose rows need more returns
 * INVALID_ARG before launching the GEMM. gemm = -1 switches it off.
 * UNSUPPORTED on a bf16 handle; INVALID_ARG for other values. */
H3BLK_API int h3blk_set_debug_accumulators(h3blk_handle h, int gemm, void* buf, size_t bytes);

/* --------------------------------------------------------------- W8A8 */
/* Bytes of the int8 weight blob for this configuration. */
H3BLK_API int h3blk_int8_weights_bytes(h3blk_handle h, size_t* bytes);

/* Rotates (block-128 Hadamard on input channels, W' = W H / sqrt(128)) and
 * quantises (per output channel, symmetric, s = amax/127) the bf16 weights in
 * `bf16_in` into `blob` (>= h3blk_int8_weights_bytes). Fills *int8_out with
 * pointers into the blob (q/k gains are copied there too). */
H3BLK_API int h3blk_prepare_int8_weights(h3blk_handle h, const h3blk_weights* bf16_in, void* blob, size_t blob_bytes,
                               h3blk_weights* int8_out, void* stream);

/* ------------------------------------------------------- kernel-level calls */
/* The block's building blocks, exposed for tests and for callers composing
 * their own pipelines. All device pointers, all asynchronous on `stream`. */

/* Block-128 Hadamard rotation of each row of a bf16 [rows, K] matrix (K a
 * multiple of 128, <= 16384), then symmetric per-row int8 quantisation:
 * q = clamp(rint(v / s), -127, 127), s = amax / 127 (s = 0, q = 0 for a zero row). */
H3BLK_API int h3blk_rotate_quantize(int64_t rows, int K, const void* in_bf16, int8_t* out_q, float* out_scale, void* stream);

/* Exact int8 GEMM: C[M, N] = A[M, K] B[N, K]^T with int32 accumulation and
 * no rounding (K a multiple of 128, N a multiple of 128). */
H3BLK_API int h3blk_gemm_s8_s32(int64_t M, int N, int K, const int8_t* A, const int8_t* B, int32_t* C, void* stream);

/* bf16 GEMM: C[M, N] = A[M, K] B[N, K]^T, fp32 accumulation, bf16 output
 * (K a multiple of 64, N a multiple of 128). */
H3BLK_API int h3blk_gemm_bf16(int64_t M, int N, int K, const void* A, const void* B, void* C, void* stream);

/* ------------------------------------------------- modulation-table producer */
/* The step before the block: turns the distinct timesteps of a forward into the
 * AdaLN table h3blk_forward reads.
 *   e_k   = [cos(t_k w_i), sin(t_k w_i)], w_i = 10000^(-i / (freq_dim / 2)),
 *           timesteps unscaled in [0, 1]
 *   E_k   = (1 - g) (W2 silu(W1 e(t_now_k) + b1) + b2)
 *           + g (W2r silu(W1r e(t_end_k) + b1r) + b2r)          (two-time blend)
 *   table[tag][k] = A_tag silu(E_k) + a_tag  -> fp32 [n_tags][n_t][6][hidden]
 * Sources: "MiniMaxH3Transformer3DModel" (diffusers API page), constructor
 * (freq_dim, time_embed_hidden_dim, time_embed_dim) and introduction (the
 * modality tag selects the AdaLN parameters; the timestep MLP is fp32);
 * HyperFlow model card, "How it works" (second time embedder for the step
 * endpoint, fixed blend gate; conditioning rows keep r = t). The embedding's
 * channel order, the SiLU placements and the blend formula are readings. */
typedef struct {
  int freq_dim;     /* multiple of 16, <= 1024 (256 for the model) */
  int time_hidden;  /* multiple of 8 (5376) */
  int time_dim;     /* multiple of 8 (2688) */
  const float *w1, *b1;      /* fp32 [time_hidden, freq_dim], [time_hidden]  */
  const float *w2, *b2;      /* fp32 [time_dim, time_hidden], [time_dim]     */
  const float *w1_r, *b1_r;  /* second-time copies; may be NULL when gate == 0 */
  const float *w2_r, *b2_r;
  const void* adaln_w;       /* bf16 [n_tags][6 * hidden][time_dim] */
  const float* adaln_b;      /* fp32 [n_tags][6 * hidden]           */
} h3blk_mod_weights;

/* Scratch bytes h3blk_modulation_table needs (n_t * (time_hidden + time_dim) floats). */
H3BLK_API int h3blk_modulation_scratch_bytes(h3blk_handle h, const h3blk_mod_weights* w, size_t* bytes);

/* Writes the handle's n_t x n_tags table. t_now and t_end are HOST arrays of
 * n_t timesteps (t_end may be NULL when gate == 0); n_t <= 8. Device pointers
 * for weights, table and scratch. UNSUPPORTED when the sizes break the limits
 * above or the inputs of one product exceed 200 KB of shared memory. */
H3BLK_API int h3blk_modulation_table(h3blk_handle h, const h3blk_mod_weights* w, const float* t_now,
                                     const float* t_end, float gate, float* table, void* scratch,
                                     size_t scratch_bytes, void* stream);

/* ------------------------------------------------------------ model shell */
/* The whole transformer forward around the block ("MiniMaxH3Transformer3DModel",
 * diffusers API page: introduction, constructor and forward parameters):
 *
 *   x[video_idx] = proj_in(video)            fp32 W [hidden, video_in] + b
 *   x[audio_idx] = audio_proj_in(audio)      fp32 W [hidden, audio_in] + b
 *   r = context_embedder(text)               bf16 W [hidden, text_dim] + fp32 b
 *   r = refiner layers over the text rows alone (the same block, each row with
 *       its packed tag / tidx / position), then rmsnorm(r, final_eps) * gain
 *   x[text_idx] = r; every other row (padding) = 0
 *   x = layer_{L-1}( ... layer_0(x))         h3blk_forward per layer
 *   h = rmsnorm(x, final_eps) (1 + scale_o) + shift_o     (norm_out)
 *   video_out = proj_out(h[video_idx]);  audio_out = audio_proj_out(h[audio_idx])
 *
 * Every layer (stack and refiner) owns its AdaLN projection; all of them and
 * norm_out's read the one time embedding of the forward's timestep sets
 * (h3blk_modulation_table's first half). The refiner always runs the bf16
 * block; the stack runs the handle's mode (bf16 or W8A8). The affine form of
 * the projections, the refiner's block structure and output norm, and the
 * AdaLN form of norm_out are readings: the pages name the modules only. */
typedef struct {
  int n_layers;        /* blocks of the stack (50; 47 in the pruned variant) */
  int n_refiner;       /* token-refiner blocks (2) */
  int video_in;        /* in_channels * prod(patch_size) (96); multiple of 4, <= 128 */
  int audio_in;        /* audio_in_channels (32); multiple of 4, <= 128 */
  int text_dim;        /* text_dim (5120); multiple of 64 */
  float final_norm_eps;
} h3blk_model_config;

typedef struct {
  h3blk_weights w;     /* the block's linears (bf16, or the int8 blob's pointers for the W8A8 stack) */
  const void* adaln_w; /* bf16 [n_tags][6 * hidden][time_dim] */
  const float* adaln_b; /* fp32 [n_tags][6 * hidden] */
} h3blk_layer_weights;

typedef struct {
  h3blk_mod_weights time;            /* time MLP (+ r copy); its adaln_w / adaln_b are not read */
  const h3blk_layer_weights* layers;  /* HOST array of n_layers entries */
  const h3blk_layer_weights* refiner; /* HOST array of n_refiner entries (bf16 weights) */
  const void* refiner_gain;          /* bf16 [hidden] */
  const void* out_adaln_w;           /* bf16 [n_tags][2 * hidden][time_dim]: shift, scale */
  const float* out_adaln_b;          /* fp32 [n_tags][2 * hidden] */
  const float *proj_in_w, *proj_in_b;     /* fp32 [hidden][video_in], [hidden] */
  const float *audio_in_w, *audio_in_b;   /* fp32 [hidden][audio_in], [hidden] */
  const void* ctx_w;                      /* bf16 [hidden][text_dim] */
  const float* ctx_b;                     /* fp32 [hidden] */
  const float *proj_out_w, *proj_out_b;   /* fp32 [video_in][hidden], [video_in] */
  const float *audio_out_w, *audio_out_b; /* fp32 [audio_in][hidden], [audio_in] */
} h3blk_model_weights;

/* One packed sequence. Every pointer is device memory. The three index
 * tensors address distinct rows of [0, n_rows); rows none of them addresses
 * must carry tag -1 (padding). An index outside [0, n_rows) is skipped and
 * reported by h3blk_model_check as H3BLK_ERR_BAD_INDEX; rows addressed twice
 * get one of the writers (unspecified which). Counts may be 0. */
typedef struct {
  int64_t n_rows, n_video, n_audio, n_text;
  const int32_t *tag, *tidx, *pos;          /* [n_rows], [n_rows], [n_rows][3] */
  const int32_t *video_idx, *audio_idx, *text_idx;
  const float* video;   /* fp32 [n_video][video_in] patchified latent rows */
  const float* audio;   /* fp32 [n_audio][audio_in] */
  const void* text;     /* bf16 [n_text][text_dim] text-encoder states */
  const float* t_now;   /* fp32 [n_t] per modulation set, in [0, 1] */
  const float* t_end;   /* fp32 [n_t]; may be NULL when gate == 0 */
  float gate;           /* two-time blend weight, in [0, 1] */
} h3blk_model_inputs;

/* Workspace bytes of a model forward over n_rows packed rows of which n_text
 * are text rows. */
H3BLK_API int h3blk_model_workspace_bytes(h3blk_handle h, const h3blk_model_config* mc, const h3blk_mod_weights* time,
                                          int64_t n_rows, int64_t n_text, size_t* bytes);

/* The forward, asynchronous on `stream`: video_out fp32 [n_video][video_in],
 * audio_out fp32 [n_audio][audio_in]. Host-side checks only; device-side
 * errors (bad indices, timeouts) are read by h3blk_model_check. */
H3BLK_API int h3blk_model_forward(h3blk_handle h, const h3blk_model_config* mc, const h3blk_model_weights* w,
                                  const h3blk_model_inputs* in, float* video_out, float* audio_out, void* workspace,
                                  size_t workspace_bytes, void* stream);

/* Synchronises `stream`, then reads the error word a model forward (sticky
 * over all its layers) or a sequence-parallel phase left in `workspace`. */
H3BLK_API int h3blk_model_check(const void* workspace, void* stream, int* status);

/* CUDA graph of one model forward: the same launches as h3blk_model_forward,
 * captured once on a private stream (no work runs during capture) and
 * instantiated. Every pointer of `w`, `in` and the outputs is baked into the
 * graph: to run another step, write the new latents, text states and
 * timesteps into the same device buffers and launch the graph again. The
 * caller keeps all of those buffers alive until h3blk_graph_destroy. */
typedef struct h3blk_graph_s* h3blk_graph;
H3BLK_API int h3blk_model_graph_create(h3blk_handle h, const h3blk_model_config* mc, const h3blk_model_weights* w,
                                       const h3blk_model_inputs* in, float* video_out, float* audio_out,
                                       void* workspace, size_t workspace_bytes, h3blk_graph* out);
H3BLK_API int h3blk_graph_launch(h3blk_graph g, void* stream);
/* Node census of the captured forward: kernel launches (every one of them a
 * kernel of this library) and other nodes (memsets). */
H3BLK_API int h3blk_graph_info(h3blk_graph g, int* kernel_nodes, int* other_nodes);
H3BLK_API void h3blk_graph_destroy(h3blk_graph g);

/* ------------------------------------------- sequence parallelism (Ulysses) */
/* One block forward split over a group of `world` ranks ("HyperFlow for
 * MiniMax-H3" model card: summary table, Usage and Performance, Ulysses
 * context parallelism over up to four GPUs). Rank r holds the contiguous rows
 * [r * N/world, (r+1) * N/world) of the packed sequence; attention, the one
 * step that needs every row, runs head-parallel: rank r computes heads
 * [r * H/world, (r+1) * H/world) over all N rows.
 *
 * The row -> head-group exchange is fused into the QKV projection (each head's
 * q / k / v is stored straight into qkv[owner of its head group]) and the
 * head-group -> row exchange into the attention epilogue (each output row is
 * stored straight into o[owner of the row]). The pointers are peer memory
 * (another GPU's buffer mapped into this process) or, for a collective-based
 * exchange, this rank's own send buffers.
 *
 * Three calls per block, ordered across the group by the caller: every rank's
 * h3blk_ulysses_qkv before any rank's h3blk_ulysses_attention, and every
 * rank's attention before any rank's h3blk_ulysses_out (one stream on one
 * device, or a group barrier between the phases). Per rank:
 *   qkv  bf16 [N][3 * H/world * head_dim]  (q heads | k heads | v heads of its group)
 *   o    bf16 [N/world][H * head_dim]
 * tag, tidx, pos cover the whole sequence ([N], [N], [N][3]); x, out, and
 * the workspace are the rank's own. UNSUPPORTED unless world divides both H
 * and N; world <= H3BLK_MAX_RANKS. Errors are read with h3blk_model_check
 * on the workspace. */
#define H3BLK_MAX_RANKS 8
typedef struct {
  int world;
  int rank;
  void* qkv[H3BLK_MAX_RANKS];  /* every rank's head-group buffer */
  void* o[H3BLK_MAX_RANKS];    /* every rank's attention-output buffer */
} h3blk_ulysses;
H3BLK_API int h3blk_ulysses_buffer_bytes(h3blk_handle h, int64_t n_rows, int world, size_t* qkv_bytes,
                                         size_t* o_bytes);
H3BLK_API int h3blk_ulysses_workspace_bytes(h3blk_handle h, int64_t n_rows, int world, size_t* bytes);
H3BLK_API int h3blk_ulysses_qkv(h3blk_handle h, int64_t n_rows, const h3blk_ulysses* u, const void* x_local,
                                const int32_t* tag, const int32_t* tidx, const int32_t* pos, const float* mod_table,
                                const h3blk_weights* w, void* workspace, size_t workspace_bytes, void* stream);
H3BLK_API int h3blk_ulysses_attention(h3blk_handle h, int64_t n_rows, const h3blk_ulysses* u, const int32_t* tag,
                                      void* workspace, size_t workspace_bytes, void* stream);
H3BLK_API int h3blk_ulysses_out(h3blk_handle h, int64_t n_rows, const h3blk_ulysses* u, const void* x_local,
                                const int32_t* tag, const int32_t* tidx, const float* mod_table,
                                const h3blk_weights* w, void* out_local, void* workspace, size_t workspace_bytes,
                                void* stream);

/* Document-masked attention of the block (the same kernels as the attention
 * step of h3blk_forward) for callers that cannot allocate device memory at run
 * time, such as a plugin inside a host application whose memory pool owns the
 * GPU's memory, or a latency-critical loop that cannot afford the device-wide
 * synchronisation of cudaMalloc / cudaFree. It needs no workspace: its scratch
 * (tile summary and error word) is a fixed ~128 KiB array in the library's
 * own device memory, held by every GPU that loads the library until exit.
 * The pages have no counterpart of this entry point.
 *   qkv  bf16 [N, 3*heads*head_dim]  (the layout of H3BLK_STAGE_QKV)
 *   tag, tidx int32 [N]              (as for h3blk_forward; tidx only validated)
 *   o    bf16 [N, heads*head_dim]    output
 * UNSUPPORTED when n_rows > 524,288 (the fixed scratch's limit), head_dim is
 * not 64 / 128, or heads*head_dim > 16384. It calls no allocator. All calls
 * share the one scratch array, which keeps the last call's contents: calls
 * that overlap on the GPU race, so serialise them. The first call on each
 * device looks up the array's device address and keeps it for the life of
 * the process (it assumes the device's primary context is never reset); make
 * that first call before any stream capture. Errors the kernels find (a tag
 * or timestep index outside the table, a pipeline wait that ran out) are not
 * in the return value, which only covers the launch: read them with
 * h3blk_attention_noalloc_check. */
H3BLK_API int h3blk_attention_noalloc(int64_t n_rows, int heads, int head_dim, int n_tags, int n_t,
                                      const void* qkv, const int32_t* tag, const int32_t* tidx, void* o,
                                      void* stream);

/* Status of the last h3blk_attention_noalloc call on the current device:
 * synchronises `stream`, reads the error word of the fixed scratch array (a
 * copy into host memory, no allocation) and sets *status to H3BLK_OK,
 * H3BLK_ERR_BAD_INDEX (a tag or timestep index outside the table) or
 * H3BLK_ERR_TIMEOUT (a pipeline wait ran out; the output is incomplete).
 * Every call resets the word, so the status covers the latest call only.
 * INVALID_ARG for a null status. The pages have no counterpart either. */
H3BLK_API int h3blk_attention_noalloc_check(void* stream, int* status);

/* Test-only: runs, on `stream`, one bounded wait of the kind every pipeline
 * wait of this library is (an mbarrier phase polled against a time limit), on
 * a barrier whose phase completes first (complete != 0) or never completes
 * (complete == 0), with a limit of limit_ms milliseconds (1..2000). It then
 * synchronises `stream` and sets *status to what h3blk_check reports for the
 * outcome: H3BLK_OK, or H3BLK_ERR_TIMEOUT when the wait ran out. The kernel
 * returns normally either way, so the CUDA context stays usable. `word` is a
 * caller-owned device int32 (4-byte aligned) used as the error word; it is
 * reset by the call. INVALID_ARG for a null pointer or a limit out of range. */
H3BLK_API int h3blk_selftest_wait(int complete, int limit_ms, void* word, void* stream, int* status);

/* Message for a status code (static storage). */
H3BLK_API const char* h3blk_error_string(int status);

/* Library version: major * 10000 + minor * 100 + patch. */
H3BLK_API int h3blk_version(void);

#ifdef __cplusplus
}
#endif
#endif /* H3BLK_H */
