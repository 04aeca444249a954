// Kernels of the model shell around the block stack ("MiniMaxH3Transformer3DModel",
// diffusers API page: introduction and constructor): the fp32 input patch
// projections scattered into the packed sequence, the token refiner's output
// norm, norm_out fused with the two fp32 heads, and the gather of the text
// rows' tags / timestep indices / positions.
//
// None of these is on the block's critical path (together well under 1 % of
// one layer at the real sizes). The projections are small-K / small-N fp32
// products, so they run on the FP32 pipes with register tiles: a CTA computes
// a 64-row tile, each thread 8 rows x 4 (or NC) columns, with the operands
// staged in shared memory transposed so the inner loop reads them as
// broadcasts and conflict-free vectors.
#include <cuda_bf16.h>

#include "kernels.cuh"
#include "ptx.cuh"

namespace h3 {
namespace {

constexpr int kTM = 64;      // rows per CTA
constexpr int kTK = 32;      // K per shared-memory stage
constexpr int kThr = 256;    // 8 warps: warp w owns rows 8w .. 8w+7 of the tile

__device__ __forceinline__ void flag(int* err, int bit) {
  if (err) atomicOr(err, bit);
}

// out[idx[m]][n] = bf16(sum_k x[m][k] W[n][k] + b[n]); a 64 x 128 tile per CTA.
__global__ void __launch_bounds__(kThr) embed_rows_kernel(const float* __restrict__ x, int64_t M, int K,
                                                          const float* __restrict__ W, const float* __restrict__ b,
                                                          int C, const int32_t* __restrict__ idx, int64_t n_rows,
                                                          __nv_bfloat16* __restrict__ out, int* err) {
  constexpr int BN = 128;
  __shared__ __align__(16) float xs[kTK][kTM];
  __shared__ __align__(16) float ws[kTK][BN];
  const int64_t m0 = (int64_t)blockIdx.x * kTM;
  const int n0 = blockIdx.y * BN;
  const int tid = threadIdx.x, tn = tid & 31, tm = tid >> 5;
  float acc[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  for (int k0 = 0; k0 < K; k0 += kTK) {
    // x tile: thread -> (row r, 4 consecutive k); a warp covers 32 rows, so the
    // transposed shared-memory writes hit 32 different banks
    for (int i = tid; i < kTM * (kTK / 4); i += kThr) {
      const int r = i % kTM, kq = i / kTM;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (m0 + r < M && k0 + 4 * kq < K) v = __ldg(reinterpret_cast<const float4*>(x + (m0 + r) * K + k0 + 4 * kq));
      xs[4 * kq][r] = v.x;
      xs[4 * kq + 1][r] = v.y;
      xs[4 * kq + 2][r] = v.z;
      xs[4 * kq + 3][r] = v.w;
    }
    for (int i = tid; i < BN * (kTK / 4); i += kThr) {
      const int n = i % BN, kq = i / BN;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (k0 + 4 * kq < K) v = __ldg(reinterpret_cast<const float4*>(W + (int64_t)(n0 + n) * K + k0 + 4 * kq));
      ws[4 * kq][n] = v.x;
      ws[4 * kq + 1][n] = v.y;
      ws[4 * kq + 2][n] = v.z;
      ws[4 * kq + 3][n] = v.w;
    }
    __syncthreads();
#pragma unroll 8
    for (int k = 0; k < kTK; ++k) {
      const float4 a0 = *reinterpret_cast<const float4*>(&xs[k][tm * 8]);
      const float4 a1 = *reinterpret_cast<const float4*>(&xs[k][tm * 8 + 4]);
      const float4 w4 = *reinterpret_cast<const float4*>(&ws[k][tn * 4]);
      const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float w[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], w[j], acc[i][j]);
    }
    __syncthreads();
  }
  const float4 bb = __ldg(reinterpret_cast<const float4*>(b + n0 + tn * 4));
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t m = m0 + tm * 8 + i;
    if (m >= M) break;
    const int64_t r = __ldg(idx + m);
    if (r < 0 || r >= n_rows) {
      if (tn == 0) flag(err, kErrBadRowIndex);
      continue;
    }
    uint2 pk;
    pk.x = pack_bf16x2(acc[i][0] + bb.x, acc[i][1] + bb.y);
    pk.y = pack_bf16x2(acc[i][2] + bb.z, acc[i][3] + bb.w);
    *reinterpret_cast<uint2*>(out + r * C + n0 + tn * 4) = pk;
  }
}

// out[idx[m]] = bf16(r[m] / sqrt(mean(r[m]^2) + eps) * gain), one warp per row
__global__ void __launch_bounds__(kThr) norm_scatter_kernel(const __nv_bfloat16* __restrict__ rin, int64_t M, int C,
                                                            const __nv_bfloat16* __restrict__ gain, float eps,
                                                            const int32_t* __restrict__ idx, int64_t n_rows,
                                                            __nv_bfloat16* __restrict__ out, int* err) {
  const int lane = threadIdx.x & 31;
  const int64_t m = (int64_t)blockIdx.x * (kThr / 32) + (threadIdx.x >> 5);
  if (m >= M) return;
  const int64_t r = __ldg(idx + m);
  if (r < 0 || r >= n_rows) {
    if (lane == 0) flag(err, kErrBadRowIndex);
    return;
  }
  const uint4* src = reinterpret_cast<const uint4*>(rin + m * C);
  const int chunks = C / 8;
  float ss = 0.f;
  for (int c = lane; c < chunks; c += 32) {
    const uint4 q = __ldg(src + c);
    const uint32_t u[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const float2 f = unpack_bf16x2(u[h]);
      ss = fmaf(f.x, f.x, ss);
      ss = fmaf(f.y, f.y, ss);
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float rs = rsqrtf(ss / (float)C + eps);
  uint4* dst = reinterpret_cast<uint4*>(out + r * C);
  const uint4* gp = reinterpret_cast<const uint4*>(gain);
  for (int c = lane; c < chunks; c += 32) {
    const uint4 q = __ldg(src + c), g = __ldg(gp + c);
    const uint32_t u[4] = {q.x, q.y, q.z, q.w}, gu[4] = {g.x, g.y, g.z, g.w};
    uint32_t o[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const float2 f = unpack_bf16x2(u[h]), gg = unpack_bf16x2(gu[h]);
      o[h] = pack_bf16x2(f.x * rs * gg.x, f.y * rs * gg.y);
    }
    dst[c] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// y[m][n] = sum_k W[n][k] (x[idx[m]][k] rstd_m (1 + scale_m[k]) + shift_m[k]) + b[n]
// for n < n_out <= 32 NC; thread = 8 rows x NC columns (n = lane + 32 j).
template <int NC>
__global__ void __launch_bounds__(kThr) head_kernel(HeadArgs p) {
  constexpr int BN = 32 * NC;
  __shared__ __align__(16) float xs[kTK][kTM];
  __shared__ __align__(16) float ws[kTK][BN];
  __shared__ float rstd[kTM];
  __shared__ const float* mod[kTM];
  __shared__ int64_t src[kTM];
  const int64_t m0 = (int64_t)blockIdx.x * kTM;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int C = p.C;
  // row statistics: warp w takes rows 8w .. 8w+7
  for (int i = 0; i < 8; ++i) {
    const int rr = warp * 8 + i;
    const int64_t m = m0 + rr;
    int64_t r = -1;
    if (m < p.M) {
      r = __ldg(p.idx + m);
      if (r < 0 || r >= p.n_rows) {
        if (lane == 0) flag(p.err, kErrBadRowIndex);
        r = -1;
      }
    }
    float ss = 0.f;
    if (r >= 0) {
      const uint4* s4 = reinterpret_cast<const uint4*>(p.x + r * C);
      for (int c = lane; c < C / 8; c += 32) {
        const uint4 q = __ldg(s4 + c);
        const uint32_t u[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const float2 f = unpack_bf16x2(u[h]);
          ss = fmaf(f.x, f.x, ss);
          ss = fmaf(f.y, f.y, ss);
        }
      }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (lane == 0) {
      src[rr] = r;
      rstd[rr] = r >= 0 ? rsqrtf(ss / (float)C + p.eps) : 0.f;
      const float* mp = nullptr;
      if (r >= 0) {
        const int tg = __ldg(p.tag + r), ti = __ldg(p.tidx + r);
        if (tg >= 0 && tg < p.n_tags && ti >= 0 && ti < p.n_t)
          mp = p.table + ((int64_t)tg * p.n_t + ti) * 2 * C;
        else if (tg != -1)
          flag(p.err, kErrBadIndex);
      }
      mod[rr] = mp;
    }
  }
  __syncthreads();
  float acc[8][NC];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < NC; ++j) acc[i][j] = 0.f;
  for (int k0 = 0; k0 < C; k0 += kTK) {
    // normalised, modulated x tile: thread -> (row, 4 consecutive k)
    for (int i = tid; i < kTM * (kTK / 4); i += kThr) {
      const int rr = i % kTM, kq = i / kTM;
      const int k = k0 + 4 * kq;
      float v[4] = {0.f, 0.f, 0.f, 0.f};
      const int64_t r = src[rr];
      if (r >= 0) {
        const uint2 q = __ldg(reinterpret_cast<const uint2*>(p.x + r * C + k));
        const float2 f0 = unpack_bf16x2(q.x), f1 = unpack_bf16x2(q.y);
        const float rs = rstd[rr];
        v[0] = f0.x * rs;
        v[1] = f0.y * rs;
        v[2] = f1.x * rs;
        v[3] = f1.y * rs;
        const float* mp = mod[rr];
        if (mp) {
          const float4 sh = __ldg(reinterpret_cast<const float4*>(mp + k));
          const float4 sc = __ldg(reinterpret_cast<const float4*>(mp + C + k));
          v[0] = fmaf(v[0], 1.f + sc.x, sh.x);
          v[1] = fmaf(v[1], 1.f + sc.y, sh.y);
          v[2] = fmaf(v[2], 1.f + sc.z, sh.z);
          v[3] = fmaf(v[3], 1.f + sc.w, sh.w);
        }
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) xs[4 * kq + e][rr] = v[e];
    }
    for (int i = tid; i < BN * (kTK / 4); i += kThr) {
      const int n = i % BN, kq = i / BN;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (n < p.n_out) v = __ldg(reinterpret_cast<const float4*>(p.W + (int64_t)n * C + k0 + 4 * kq));
      ws[4 * kq][n] = v.x;
      ws[4 * kq + 1][n] = v.y;
      ws[4 * kq + 2][n] = v.z;
      ws[4 * kq + 3][n] = v.w;
    }
    __syncthreads();
#pragma unroll 8
    for (int k = 0; k < kTK; ++k) {
      const float4 a0 = *reinterpret_cast<const float4*>(&xs[k][warp * 8]);
      const float4 a1 = *reinterpret_cast<const float4*>(&xs[k][warp * 8 + 4]);
      const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      float w[NC];
#pragma unroll
      for (int j = 0; j < NC; ++j) w[j] = ws[k][lane + 32 * j];
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < NC; ++j) acc[i][j] = fmaf(a[i], w[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t m = m0 + warp * 8 + i;
    if (m >= p.M) break;
#pragma unroll
    for (int j = 0; j < NC; ++j) {
      const int n = lane + 32 * j;
      if (n < p.n_out) p.y[m * p.n_out + n] = acc[i][j] + __ldg(p.b + n);
    }
  }
}

__global__ void gather_meta_kernel(const int32_t* __restrict__ idx, int64_t M, int64_t n_rows,
                                   const int32_t* __restrict__ tag, const int32_t* __restrict__ tidx,
                                   const int32_t* __restrict__ pos, int32_t* out_tag, int32_t* out_tidx,
                                   int32_t* out_pos, int* err) {
  const int64_t m = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (m >= M) return;
  const int64_t r = idx[m];
  if (r < 0 || r >= n_rows) {
    // an out-of-range text row becomes a padding row of the refiner's sequence
    flag(err, kErrBadRowIndex);
    out_tag[m] = -1;
    out_tidx[m] = 0;
    out_pos[3 * m] = out_pos[3 * m + 1] = out_pos[3 * m + 2] = 0;
    return;
  }
  out_tag[m] = tag[r];
  out_tidx[m] = tidx[r];
  out_pos[3 * m] = pos[3 * r];
  out_pos[3 * m + 1] = pos[3 * r + 1];
  out_pos[3 * m + 2] = pos[3 * r + 2];
}

}  // namespace

cudaError_t launch_embed_rows(const float* x, int64_t M, int K, const float* W, const float* b, int C,
                              const int32_t* idx, int64_t n_rows, __nv_bfloat16* out, int* err, cudaStream_t s) {
  if (M <= 0) return cudaSuccess;
  if (K % 4 || C % 128) return cudaErrorInvalidValue;
  const dim3 grid((unsigned)((M + kTM - 1) / kTM), (unsigned)(C / 128));
  embed_rows_kernel<<<grid, kThr, 0, s>>>(x, M, K, W, b, C, idx, n_rows, out, err);
  return cudaGetLastError();
}

cudaError_t launch_norm_scatter(const __nv_bfloat16* r, int64_t M, int C, const __nv_bfloat16* gain, float eps,
                                const int32_t* idx, int64_t n_rows, __nv_bfloat16* out, int* err, cudaStream_t s) {
  if (M <= 0) return cudaSuccess;
  if (C % 8) return cudaErrorInvalidValue;
  const int rows_per_block = kThr / 32;
  norm_scatter_kernel<<<(unsigned)((M + rows_per_block - 1) / rows_per_block), kThr, 0, s>>>(r, M, C, gain, eps, idx,
                                                                                              n_rows, out, err);
  return cudaGetLastError();
}

cudaError_t launch_head(const HeadArgs& a, int num_sms, cudaStream_t s) {
  (void)num_sms;
  if (a.M <= 0) return cudaSuccess;
  if (a.C % kTK || a.n_out <= 0 || a.n_out > 128) return cudaErrorInvalidValue;
  const unsigned blocks = (unsigned)((a.M + kTM - 1) / kTM);
  switch ((a.n_out + 31) / 32) {
    case 1: head_kernel<1><<<blocks, kThr, 0, s>>>(a); break;
    case 2: head_kernel<2><<<blocks, kThr, 0, s>>>(a); break;
    case 3: head_kernel<3><<<blocks, kThr, 0, s>>>(a); break;
    default: head_kernel<4><<<blocks, kThr, 0, s>>>(a); break;
  }
  return cudaGetLastError();
}

cudaError_t launch_gather_meta(const int32_t* idx, int64_t M, int64_t n_rows, const int32_t* tag,
                               const int32_t* tidx, const int32_t* pos, int32_t* out_tag, int32_t* out_tidx,
                               int32_t* out_pos, int* err, cudaStream_t s) {
  if (M <= 0) return cudaSuccess;
  gather_meta_kernel<<<(unsigned)((M + 255) / 256), 256, 0, s>>>(idx, M, n_rows, tag, tidx, pos, out_tag, out_tidx,
                                                                  out_pos, err);
  return cudaGetLastError();
}

}  // namespace h3
