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

// ============================================================== K1 (bf16)
// One warp per row; lane l owns the 16-byte chunks l, l+32, l+64, ...
constexpr int kModNormMaxChunksPerLane = 24;  // hidden <= 6144

__global__ void __launch_bounds__(256) modnorm_bf16_kernel(ModNormArgs a) {
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= a.n) return;
  const int lane = threadIdx.x & 31;
  const int nchunk = a.C >> 3;
  const uint4* xr = reinterpret_cast<const uint4*>(a.x + row * a.C);
  uint4 v[kModNormMaxChunksPerLane];
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < kModNormMaxChunksPerLane; ++i) {
    const int c = lane + 32 * i;
    if (c < nchunk) {
      v[i] = ld_nc_v4(xr + c);
      float f[8];
      bf16x8_to_f32(v[i], f);
#pragma unroll
      for (int e = 0; e < 8; ++e) ss = fmaf(f[e], f[e], ss);
    }
  }
  ss = warp_sum(ss);
  const float rstd = rsqrtf(ss / (float)a.C + a.eps);
  const float* m = mod_row(a.table, a.tag, a.tidx, row, a.n_tags, a.n_t, a.C);
  const float* shift = m ? m + (int64_t)a.shift_idx * a.C : nullptr;
  const float* scale = m ? m + (int64_t)a.scale_idx * a.C : nullptr;
  uint4* outr = reinterpret_cast<uint4*>(a.out_bf16 + row * a.C);
#pragma unroll
  for (int i = 0; i < kModNormMaxChunksPerLane; ++i) {
    const int c = lane + 32 * i;
    if (c < nchunk) {
      float f[8];
      bf16x8_to_f32(v[i], f);
      float sh[8], sc[8];
      if (m) {
        const float4* s4 = reinterpret_cast<const float4*>(shift + c * 8);
        const float4* k4 = reinterpret_cast<const float4*>(scale + c * 8);
        float4 s0 = __ldg(s4), s1 = __ldg(s4 + 1), k0 = __ldg(k4), k1 = __ldg(k4 + 1);
        sh[0] = s0.x; sh[1] = s0.y; sh[2] = s0.z; sh[3] = s0.w; sh[4] = s1.x; sh[5] = s1.y; sh[6] = s1.z; sh[7] = s1.w;
        sc[0] = k0.x; sc[1] = k0.y; sc[2] = k0.z; sc[3] = k0.w; sc[4] = k1.x; sc[5] = k1.y; sc[6] = k1.z; sc[7] = k1.w;
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) sh[e] = sc[e] = 0.f;
      }
      float h[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) h[e] = fmaf(f[e] * rstd, 1.f + sc[e], sh[e]);
      uint4 o;
      o.x = pack_bf16x2(h[0], h[1]);
      o.y = pack_bf16x2(h[2], h[3]);
      o.z = pack_bf16x2(h[4], h[5]);
      o.w = pack_bf16x2(h[6], h[7]);
      outr[c] = o;
    }
  }
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

cudaError_t launch_rotate_quant(const __nv_bfloat16* in, int64_t rows, int K, int8_t* out_q, float* out_scale,
                                cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  ModNormArgs none{};
  return launch_rq<false>(in, rows, K, out_q, out_scale, none, s);
}

cudaError_t launch_modnorm(const ModNormArgs& a, cudaStream_t s) {
  if (a.n <= 0) return cudaSuccess;
  if (a.out_q) return launch_rq<true>(a.x, a.n, a.C, a.out_q, a.out_scale, a, s);
  if (a.C / 8 > 32 * kModNormMaxChunksPerLane) return cudaErrorInvalidValue;
  const int warps = 8;
  const unsigned blocks = (unsigned)((a.n + warps - 1) / warps);
  modnorm_bf16_kernel<<<blocks, warps * 32, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace h3
