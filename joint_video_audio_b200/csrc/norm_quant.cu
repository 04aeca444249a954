// Bandwidth-bound kernels of the block:
//   * tile_info: validates per-row tags / timestep indices and summarises the
//     padding document of every 128-row tile for the attention kernel;
//   * modnorm (K1): tag-gathered AdaLN modulation + RMSNorm, bf16 out, or
//     fused with the W8A8 input rotation and per-token int8 quantisation;
//   * rotate_quant (K4): block-128 Hadamard rotation + per-row int8 quantisation
//     of a bf16 matrix (attention output, SwiGLU output, weights).
//
// Sources: "MiniMaxH3Transformer3DModel" (diffusers API page) introduction
// (modality tag selects the AdaLN modulation; padding rows are their own
// attention document) and constructor (norm_eps of the pre-attention and
// pre-feed-forward norms); "HyperFlow H3 Flash Brings MiniMax H3 Video to One
// GPU", "How it got smaller and faster" (rotated W8A8 INT8 linears).
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include "kernels.cuh"
#include "ptx.cuh"

namespace h3 {

// ============================================================== tile info
__global__ void tile_info_kernel(const int32_t* __restrict__ tag, const int32_t* __restrict__ tidx, int64_t n,
                                 int n_tags, int n_t, TileInfo* __restrict__ info, int* __restrict__ err) {
  const int64_t row = (int64_t)blockIdx.x * 128 + threadIdx.x;
  const bool present = row < n;
  int tg = present ? tag[row] : 0;
  const int ti = present ? tidx[row] : 0;
  const bool pad = present && tg == -1;
  if (present && !pad && (tg < 0 || tg >= n_tags || ti < 0 || ti >= n_t)) atomicOr(err, kErrBadIndex);
  const uint32_t bits = __ballot_sync(0xffffffffu, pad);
  const uint32_t pres = __ballot_sync(0xffffffffu, present);
  __shared__ uint32_t s_bits[4], s_pres[4];
  if ((threadIdx.x & 31) == 0) {
    s_bits[threadIdx.x >> 5] = bits;
    s_pres[threadIdx.x >> 5] = pres;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    TileInfo t;
    t.rows = 0;
    t.npad = 0;
    for (int w = 0; w < 4; ++w) {
      t.padbits[w] = s_bits[w];
      t.rows += __popc(s_pres[w]);
      t.npad += __popc(s_bits[w]);
    }
    t._unused[0] = t._unused[1] = 0;
    info[blockIdx.x] = t;
  }
}

cudaError_t launch_tile_info(const int32_t* tag, const int32_t* tidx, int64_t n, int n_tags, int n_t,
                             TileInfo* info, int* err, cudaStream_t s) {
  const int64_t tiles = (n + 127) / 128;
  tile_info_kernel<<<(unsigned)tiles, 128, 0, s>>>(tag, tidx, n, n_tags, n_t, info, err);
  return cudaGetLastError();
}

// ============================================================== helpers
__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4& v, float (&f)[8]) {
  float2 a = unpack_bf16x2(v.x), b = unpack_bf16x2(v.y), c = unpack_bf16x2(v.z), d = unpack_bf16x2(v.w);
  f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y; f[4] = c.x; f[5] = c.y; f[6] = d.x; f[7] = d.y;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int m = 16; m; m >>= 1) v += __shfl_xor_sync(0xffffffffu, v, m);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int m = 16; m; m >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, m));
  return v;
}

// Modulation row of a sequence row, or nullptr for padding / invalid indices
// (those rows get zero shift and scale).
__device__ __forceinline__ const float* mod_row(const float* table, const int32_t* tag, const int32_t* tidx,
                                                int64_t row, int n_tags, int n_t, int C) {
  const int tg = tag[row], ti = tidx[row];
  if (tg < 0 || tg >= n_tags || ti < 0 || ti >= n_t) return nullptr;
  return table + ((int64_t)tg * n_t + ti) * 6 * C;
}

// ============================================================== rotation + quant
// One CTA per row at a time; thread t owns chunks t, t + THREADS, ... of 8
// channels (THREADS a multiple of 16). A 128-channel Hadamard block is 16
// consecutive chunks, i.e. one half-warp, so the transform is 3 in-register
// butterfly stages followed by 4 shuffle stages.

__device__ __forceinline__ void fwht128_chunk(float (&h)[8], int lane) {
#pragma unroll
  for (int b = 1; b < 8; b <<= 1) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      if (!(e & b)) {
        const float u = h[e], w = h[e | b];
        h[e] = u + w;
        h[e | b] = u - w;
      }
    }
  }
#pragma unroll
  for (int m = 1; m < 16; m <<= 1) {
    // lower lane: h + other; upper lane: other - h (one FMA with a sign)
    const float sgn = (lane & m) ? -1.f : 1.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float other = __shfl_xor_sync(0xffffffffu, h[e], m);
      h[e] = fmaf(sgn, h[e], other);
    }
  }
  const float inv_sqrt128 = 0.08838834764831845f;
#pragma unroll
  for (int e = 0; e < 8; ++e) h[e] *= inv_sqrt128;
}

__device__ __forceinline__ float block_reduce(float v, bool is_max, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = is_max ? warp_max(v) : warp_sum(v);
  __syncthreads();  // red[] may still be read by a previous reduction
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float r = red[0];
  for (int w = 1; w < (int)(blockDim.x >> 5); ++w) r = is_max ? fmaxf(r, red[w]) : r + red[w];
  return r;
}

// q = clamp(rint(v * inv_s), -127, 127), inv_s = 127 / amax: one multiply per
// value instead of a division (the two can round a value lying within an ulp
// of a half-integer differently, the int8 operand tolerance of the tests).
__device__ __forceinline__ void quant_store(const float (&h)[8], float inv_s, bool zero, int8_t* dst) {
  uint32_t w[2];
#pragma unroll
  for (int g = 0; g < 2; ++g) {
    int q[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      // round to nearest even, then clamp (|h| <= amax keeps it within 127)
      const int v = zero ? 0 : __float2int_rn(h[4 * g + e] * inv_s);
      q[e] = max(-127, min(127, v));
    }
    // bytes 0..3 from the low bytes of q[0..3]
    const uint32_t lo = __byte_perm((uint32_t)q[0], (uint32_t)q[1], 0x0040);
    const uint32_t hi = __byte_perm((uint32_t)q[2], (uint32_t)q[3], 0x0040);
    w[g] = __byte_perm(lo, hi, 0x5410);
  }
  *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
}

// MODNORM = true: the row is x, modulated and normalised first (K1 fused).
// One CTA per row.
template <int CPT, int THREADS, bool MODNORM>
__global__ void __launch_bounds__(THREADS) rotate_quant_kernel(const __nv_bfloat16* __restrict__ in, int64_t rows,
                                                               int K, int8_t* __restrict__ out_q,
                                                               float* __restrict__ out_scale, ModNormArgs a) {
  __shared__ float red[THREADS / 32];
  const int lane = threadIdx.x & 31;
  const int nchunk = K >> 3;
  const int64_t row = blockIdx.x;
  if (row >= rows) return;
  {
    const uint4* src = reinterpret_cast<const uint4*>(in + row * (int64_t)K);
    float h[CPT][8];
#pragma unroll
    for (int i = 0; i < CPT; ++i) {
      const int c = threadIdx.x + THREADS * i;
      if (c < nchunk) {
        bf16x8_to_f32(ld_nc_v4(src + c), h[i]);
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) h[i][e] = 0.f;
      }
    }
    if (MODNORM) {
      float ss = 0.f;
#pragma unroll
      for (int i = 0; i < CPT; ++i)
#pragma unroll
        for (int e = 0; e < 8; ++e) ss = fmaf(h[i][e], h[i][e], ss);
      ss = block_reduce(ss, false, red);
      const float rstd = rsqrtf(ss / (float)K + a.eps);
      const float* m = mod_row(a.table, a.tag, a.tidx, row, a.n_tags, a.n_t, K);
#pragma unroll
      for (int i = 0; i < CPT; ++i) {
        const int c = threadIdx.x + THREADS * i;
        float sh[8], sc[8];
        if (m && c < nchunk) {
          const float4* s4 = reinterpret_cast<const float4*>(m + (int64_t)a.shift_idx * K + c * 8);
          const float4* k4 = reinterpret_cast<const float4*>(m + (int64_t)a.scale_idx * K + c * 8);
          const float4 s0 = __ldg(s4), s1 = __ldg(s4 + 1), k0 = __ldg(k4), k1 = __ldg(k4 + 1);
          sh[0] = s0.x; sh[1] = s0.y; sh[2] = s0.z; sh[3] = s0.w; sh[4] = s1.x; sh[5] = s1.y; sh[6] = s1.z; sh[7] = s1.w;
          sc[0] = k0.x; sc[1] = k0.y; sc[2] = k0.z; sc[3] = k0.w; sc[4] = k1.x; sc[5] = k1.y; sc[6] = k1.z; sc[7] = k1.w;
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) sh[e] = sc[e] = 0.f;
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) h[i][e] = fmaf(h[i][e] * rstd, 1.f + sc[e], sh[e]);
      }
    }
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < CPT; ++i) {
      // all 32 lanes take part in the shuffles; out-of-range chunks hold zeros
      fwht128_chunk(h[i], lane);
#pragma unroll
      for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(h[i][e]));
    }
    amax = block_reduce(amax, true, red);
    const float s = amax / 127.f;
    const bool zero = !(amax > 0.f);
    const float inv_s = zero ? 0.f : 127.f / amax;
    if (threadIdx.x == 0) out_scale[row] = s;
    int8_t* dst = out_q + row * (int64_t)K;
#pragma unroll
    for (int i = 0; i < CPT; ++i) {
      const int c = threadIdx.x + THREADS * i;
      if (c < nchunk) quant_store(h[i], inv_s, zero, dst + c * 8);
    }
  }
}

template <int CPT, int THREADS, bool MODNORM>
static cudaError_t launch_rq_t(const __nv_bfloat16* in, int64_t rows, int K, int8_t* q, float* sc,
                               const ModNormArgs& a, cudaStream_t s) {
  // one CTA per row (measured faster here than a persistent grid that
  // prefetches the next row)
  rotate_quant_kernel<CPT, THREADS, MODNORM><<<(unsigned)rows, THREADS, 0, s>>>(in, rows, K, q, sc, a);
  return cudaGetLastError();
}

// Thread count and chunks per thread for a row of K channels: exact fits for
// the block's widths, otherwise 256 threads with enough chunks each.
template <bool MODNORM>
static cudaError_t launch_rq(const __nv_bfloat16* in, int64_t rows, int K, int8_t* q, float* sc,
                             const ModNormArgs& a, cudaStream_t s) {
  const int nchunk = K / 8;
  if (nchunk == 672) return launch_rq_t<3, 224, MODNORM>(in, rows, K, q, sc, a, s);   // 5376 channels
  if (nchunk == 896) return launch_rq_t<4, 224, MODNORM>(in, rows, K, q, sc, a, s);   // 7168
  if (nchunk == 1792) return launch_rq_t<7, 256, MODNORM>(in, rows, K, q, sc, a, s);  // 14336
  if (nchunk <= 32) return launch_rq_t<1, 32, MODNORM>(in, rows, K, q, sc, a, s);
  if (nchunk <= 128) return launch_rq_t<1, 128, MODNORM>(in, rows, K, q, sc, a, s);
  switch ((nchunk + 255) / 256) {
#define H3_RQ_CASE(N) \
  case N: return launch_rq_t<N, 256, MODNORM>(in, rows, K, q, sc, a, s);
    H3_RQ_CASE(1) H3_RQ_CASE(2) H3_RQ_CASE(3) H3_RQ_CASE(4) H3_RQ_CASE(5) H3_RQ_CASE(6) H3_RQ_CASE(7)
    H3_RQ_CASE(8)
#undef H3_RQ_CASE
    default:
      return cudaErrorInvalidValue;
  }
}

// ============================================================== K1 (bf16), row streaming
// h = rmsnorm(x)(1 + scale) + shift, stored as bf16: a pass bound by moving
// each row in and out once. Persistent CTAs walk the rows (row = blockIdx.x +
// k * gridDim.x); each row reaches shared memory by one bulk copy (TMA
// engine), issued `stages` rows ahead into a ring, so every CTA keeps several
// rows in flight while its threads work on one. Thread t owns the 16-byte
// chunks t, t + THREADS, ... of the row (8 channels each).
constexpr int kMaxStages = 8;
constexpr int kStageBudget = 48 * 1024;  // shared-memory bytes of one CTA's ring

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// Modulation vectors of one chunk (zero without a table row).
__device__ __forceinline__ void mod_chunk(const float* m, const ModNormArgs& a, int K, int c, float (&sh)[8],
                                          float (&sc)[8]) {
  if (m) {
    const float4* s4 = reinterpret_cast<const float4*>(m + (int64_t)a.shift_idx * K + c * 8);
    const float4* k4 = reinterpret_cast<const float4*>(m + (int64_t)a.scale_idx * K + c * 8);
    const float4 s0 = __ldg(s4), s1 = __ldg(s4 + 1), k0 = __ldg(k4), k1 = __ldg(k4 + 1);
    sh[0] = s0.x; sh[1] = s0.y; sh[2] = s0.z; sh[3] = s0.w; sh[4] = s1.x; sh[5] = s1.y; sh[6] = s1.z; sh[7] = s1.w;
    sc[0] = k0.x; sc[1] = k0.y; sc[2] = k0.z; sc[3] = k0.w; sc[4] = k1.x; sc[5] = k1.y; sc[6] = k1.z; sc[7] = k1.w;
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) sh[e] = sc[e] = 0.f;
  }
}

template <int CPT, int THREADS>
__global__ void __launch_bounds__(THREADS) modnorm_stream_kernel(const __nv_bfloat16* __restrict__ in, int64_t rows,
                                                                 int K, int stages, __nv_bfloat16* __restrict__ out_h,
                                                                 ModNormArgs a, int* err) {
  extern __shared__ __align__(128) uint8_t ring[];
  __shared__ uint64_t full[kMaxStages];
  __shared__ float red[THREADS / 32];
  const int nchunk = K >> 3;
  const uint32_t row_bytes = (uint32_t)K * 2u;
  const int64_t step = gridDim.x;
  if (threadIdx.x == 0) {
    for (int i = 0; i < stages; ++i) mbar_init(&full[i], 1);
    fence_mbar_init();
  }
  __syncthreads();
  // load k of this CTA (row blockIdx.x + k * step) goes to stage k % stages
  auto issue = [&](int64_t k) {
    const int64_t row = blockIdx.x + k * step;
    if (row >= rows) return;
    const int st = (int)(k % stages);
    mbar_expect_tx(&full[st], row_bytes);
    bulk_load(ring + (size_t)st * row_bytes, in + row * (int64_t)K, row_bytes, &full[st]);
  };
  if (threadIdx.x == 0)
    for (int k = 0; k < stages; ++k) issue(k);
  for (int64_t k = 0;; ++k) {
    const int64_t row = blockIdx.x + k * step;
    if (row >= rows) break;
    const int st = (int)(k % stages);
    const bool ok = mbar_wait(&full[st], (uint32_t)((k / stages) & 1), nullptr);
    float h[CPT][8];
    const uint4* src = reinterpret_cast<const uint4*>(ring + (size_t)st * row_bytes);
#pragma unroll
    for (int i = 0; i < CPT; ++i) {
      const int c = threadIdx.x + THREADS * i;
      if (ok && c < nchunk) {
        bf16x8_to_f32(src[c], h[i]);
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) h[i][e] = 0.f;
      }
    }
    // every thread has its chunks in registers: the stage is refilled with
    // the row `stages` steps ahead (or the CTA stops if a load never landed)
    if (__syncthreads_or(!ok)) {
      if (threadIdx.x == 0) {
        if (err) atomicOr(err, kErrTimeoutStream);
        // loads still in flight must land before the CTA's shared memory goes
        for (int64_t kk = k; kk < k + stages && blockIdx.x + kk * step < rows; ++kk)
          mbar_wait(&full[kk % stages], (uint32_t)((kk / stages) & 1), nullptr);
      }
      return;
    }
    if (threadIdx.x == 0) {
      fence_proxy_async_smem();
      issue(k + stages);
    }
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < CPT; ++i)
#pragma unroll
      for (int e = 0; e < 8; ++e) ss = fmaf(h[i][e], h[i][e], ss);
    ss = block_reduce(ss, false, red);
    const float rstd = rsqrtf(ss / (float)K + a.eps);
    const float* m = mod_row(a.table, a.tag, a.tidx, row, a.n_tags, a.n_t, K);
    uint4* dst = reinterpret_cast<uint4*>(out_h + row * (int64_t)K);
#pragma unroll
    for (int i = 0; i < CPT; ++i) {
      const int c = threadIdx.x + THREADS * i;
      if (c < nchunk) {
        float sh[8], sc[8];
        mod_chunk(m, a, K, c, sh, sc);
#pragma unroll
        for (int e = 0; e < 8; ++e) h[i][e] = fmaf(h[i][e] * rstd, 1.f + sc[e], sh[e]);
        uint4 o;
        o.x = pack_bf16x2(h[i][0], h[i][1]);
        o.y = pack_bf16x2(h[i][2], h[i][3]);
        o.z = pack_bf16x2(h[i][4], h[i][5]);
        o.w = pack_bf16x2(h[i][6], h[i][7]);
        dst[c] = o;
      }
    }
  }
}

template <int CPT, int THREADS>
static cudaError_t launch_rows_t(const __nv_bfloat16* in, int64_t rows, int K, __nv_bfloat16* out_h,
                                 const ModNormArgs& a, int* err, cudaStream_t s) {
  auto kern = modnorm_stream_kernel<CPT, THREADS>;
  const size_t row_bytes = (size_t)K * 2;
  int stages = (int)(kStageBudget / row_bytes);
  stages = stages < 2 ? 2 : (stages > kMaxStages ? kMaxStages : stages);
  const size_t smem = (size_t)stages * row_bytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0, per_sm = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, THREADS, smem)) != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  const int64_t grid = rows < (int64_t)sms * per_sm ? rows : (int64_t)sms * per_sm;
  kern<<<(unsigned)grid, THREADS, smem, s>>>(in, rows, K, stages, out_h, a, err);
  return cudaGetLastError();
}

// Thread count and chunks per thread for a row of K channels: exact fits for
// the block's widths, otherwise 256 threads with enough chunks each.
static cudaError_t launch_rows(const __nv_bfloat16* in, int64_t rows, int K, __nv_bfloat16* out_h, const ModNormArgs& a,
                               int* err, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  if (K <= 0 || K % 128 != 0) return cudaErrorInvalidValue;  // 16-byte rows, whole chunks per thread
  const int nchunk = K / 8;
#define H3_ROWS(CPT, T) return launch_rows_t<CPT, T>(in, rows, K, out_h, a, err, s)
  if (nchunk == 672) H3_ROWS(3, 224);   // 5376 channels
  if (nchunk == 896) H3_ROWS(4, 224);   // 7168
  if (nchunk == 1792) H3_ROWS(7, 256);  // 14336
  if (nchunk <= 32) H3_ROWS(1, 32);
  if (nchunk <= 128) H3_ROWS(1, 128);
  switch ((nchunk + 255) / 256) {
    case 1: H3_ROWS(1, 256);
    case 2: H3_ROWS(2, 256);
    case 3: H3_ROWS(3, 256);
    case 4: H3_ROWS(4, 256);
    case 5: H3_ROWS(5, 256);
    case 6: H3_ROWS(6, 256);
    case 7: H3_ROWS(7, 256);
    case 8: H3_ROWS(8, 256);
    default:
      return cudaErrorInvalidValue;
  }
#undef H3_ROWS
}

cudaError_t launch_rotate_quant(const __nv_bfloat16* in, int64_t rows, int K, int8_t* out_q, float* out_scale,
                                int* /*err: this pass has no waits*/, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  ModNormArgs none{};
  return launch_rq<false>(in, rows, K, out_q, out_scale, none, s);
}

cudaError_t launch_modnorm(const ModNormArgs& a, cudaStream_t s) {
  if (a.n <= 0) return cudaSuccess;
  if (a.out_q) return launch_rq<true>(a.x, a.n, a.C, a.out_q, a.out_scale, a, s);
  return launch_rows(a.x, a.n, a.C, a.out_bf16, a, a.err, s);
}

}  // namespace h3
