// Modulation-table producer: the step that feeds the block its AdaLN table.
//
//   e_k   = [cos(t_k w), sin(t_k w)],  w_i = 10000^(-i / (freq_dim / 2))
//   E_k   = (1 - g) (W2 silu(W1 e(t_k) + b1) + b2) + g (W2r silu(W1r e(r_k) + b1r) + b2r)
//   table[tag][k] = A_tag silu(E_k) + a_tag        (n_vec * hidden outputs: 6 for a
//                                                 block, 2 for the output norm)
//
// Sources: "MiniMaxH3Transformer3DModel" (diffusers API page), constructor
// (freq_dim of the sinusoidal embedding, timesteps unscaled in [0, 1]; the
// timestep MLP's inner and output sizes; its output feeds every AdaLN
// projection) and introduction (the per-row modality tag selects the AdaLN
// parameters; the timestep MLP is float32); HyperFlow model card, "How it
// works" (a second time embedder for the step endpoint r, blended with a fixed
// gate). The channel order of the embedding, the SiLU placements and the
// blend formula are this library's reading of those passages.
//
// Every step is a matrix-vector product over a handful of timestep sets, so
// the work is bound by streaming the weights from HBM once: each warp takes
// four output rows at a time with 16-byte loads along them, and all sets'
// inputs sit in shared memory.
#include <cuda_bf16.h>

#include "kernels.cuh"
#include "ptx.cuh"

namespace h3 {
namespace {

constexpr int kGemvThreads = 256;
constexpr int kRows = 4;  // output rows per warp pass

__device__ __forceinline__ float silu_f(float v) { return v / (1.f + __expf(-v)); }

// 8 consecutive weights as floats
__device__ __forceinline__ void load8(const float* w, float (&f)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(w));
  const float4 b = __ldg(reinterpret_cast<const float4*>(w) + 1);
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}
__device__ __forceinline__ void load8(const __nv_bfloat16* w, float (&f)[8]) {
  const uint4 v = __ldg(reinterpret_cast<const uint4*>(w));
  const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 p = unpack_bf16x2(u[i]);
    f[2 * i] = p.x;
    f[2 * i + 1] = p.y;
  }
}

// y[z][v][o] = alpha * (W_z[o] . act(x[v]) + b_z[o]) + (accumulate ? y[z][v][o] : 0)
// for v < V sets; z = blockIdx.y selects one of several weight sets (the
// modality tags). x is [V][I] fp32 in global memory (act = SiLU when
// silu_in), or, when embed_t != nullptr, the sinusoidal embedding of
// embed_t[v] computed here; silu_out applies SiLU to the result.
template <typename WT, int V>
__global__ void __launch_bounds__(kGemvThreads) gemv_sets_kernel(const WT* __restrict__ W, const float* __restrict__ b,
                                                                 int64_t w_stride_z, int64_t b_stride_z, int O, int I,
                                                                 const float* __restrict__ x,
                                                                 ModTimes embed_t, bool silu_in, bool silu_out,
                                                                 float alpha, bool accumulate, float* __restrict__ y,
                                                                 int64_t y_stride_z, int64_t y_stride_v) {
  extern __shared__ float xs[];  // [V][I]
  const int z = blockIdx.y;
  if (embed_t.count > 0) {
    const int h = I / 2;
    for (int idx = threadIdx.x; idx < V * h; idx += blockDim.x) {
      const int v = idx / h, i = idx - v * h;
      const float w = exp2f(-(float)i / (float)h * 13.287712379549449f);  // 10000^(-i/h)
      float sn, cs;
      const float tv = embed_t.dev ? embed_t.dev[v] : embed_t.t[v];
      sincosf(tv * w, &sn, &cs);
      xs[v * I + i] = cs;
      xs[v * I + h + i] = sn;
    }
  } else {
    for (int idx = threadIdx.x; idx < V * I; idx += blockDim.x) {
      const float v = x[idx];
      xs[idx] = silu_in ? silu_f(v) : v;
    }
  }
  __syncthreads();
  const WT* Wz = W + z * w_stride_z;
  const float* bz = b + z * b_stride_z;
  float* yz = y + z * y_stride_z;
  const int lane = threadIdx.x & 31;
  const int warps = gridDim.x * (kGemvThreads / 32);
  // each warp takes kRows output rows at a time, so every input value read
  // from shared memory serves kRows weight rows
  for (int o0 = (blockIdx.x * (kGemvThreads / 32) + (threadIdx.x >> 5)) * kRows; o0 < O; o0 += warps * kRows) {
    float acc[kRows][V];
#pragma unroll
    for (int r = 0; r < kRows; ++r)
#pragma unroll
      for (int v = 0; v < V; ++v) acc[r][v] = 0.f;
#pragma unroll 2
    for (int c = lane * 8; c < I; c += 256) {
      float f[kRows][8];
#pragma unroll
      for (int r = 0; r < kRows; ++r) {
        if (o0 + r < O) {
          load8(Wz + (int64_t)(o0 + r) * I + c, f[r]);
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) f[r][e] = 0.f;
        }
      }
#pragma unroll
      for (int v = 0; v < V; ++v) {
        const float4 x0 = *reinterpret_cast<const float4*>(xs + v * I + c);
        const float4 x1 = *reinterpret_cast<const float4*>(xs + v * I + c + 4);
        const float xv[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
        for (int r = 0; r < kRows; ++r)
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[r][v] = fmaf(f[r][e], xv[e], acc[r][v]);
      }
    }
#pragma unroll
    for (int r = 0; r < kRows; ++r)
#pragma unroll
      for (int v = 0; v < V; ++v)
#pragma unroll
        for (int m = 16; m; m >>= 1) acc[r][v] += __shfl_xor_sync(0xffffffffu, acc[r][v], m);
    if (lane < kRows && o0 + lane < O) {
      const int o = o0 + lane;
      const float bo = bz[o];
#pragma unroll
      for (int r = 0; r < kRows; ++r) {
        if (r != lane) continue;
#pragma unroll
        for (int v = 0; v < V; ++v) {
          float res = acc[r][v] + bo;
          if (silu_out) res = silu_f(res);
          float* dst = yz + v * y_stride_v + o;
          *dst = alpha * res + (accumulate ? *dst : 0.f);
        }
      }
    }
  }
}

template <typename WT, int V>
cudaError_t gemv_v(const WT* W, const float* b, int64_t wz, int64_t bz, int Z, int O, int I, const float* x,
                   const ModTimes& t, bool silu_in, bool silu_out, float alpha, bool acc, float* y, int64_t yz,
                   int64_t yv, int num_sms, cudaStream_t s) {
  const size_t smem = (size_t)V * I * sizeof(float);
  auto k = gemv_sets_kernel<WT, V>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int rows_per_block = (kGemvThreads / 32) * kRows;
  int blocks = (O + rows_per_block - 1) / rows_per_block;
  int per_sm = 1;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, kGemvThreads, smem) != cudaSuccess || per_sm < 1)
    per_sm = 1;
  const int cap = per_sm * num_sms;  // one resident wave; each block stages its inputs once
  if (blocks > cap) blocks = cap;
  k<<<dim3((unsigned)blocks, (unsigned)Z), kGemvThreads, smem, s>>>(W, b, wz, bz, O, I, x, t, silu_in, silu_out, alpha,
                                                                    acc, y, yz, yv);
  return cudaGetLastError();
}

// the number of timestep sets is a template argument so each set's
// accumulators stay in registers
template <typename WT>
cudaError_t gemv(const WT* W, const float* b, int64_t wz, int64_t bz, int Z, int O, int I, int V, const float* x,
                 const ModTimes& t, bool silu_in, bool silu_out, float alpha, bool acc, float* y, int64_t yz, int64_t yv,
                 int num_sms, cudaStream_t s) {
  switch (V) {
#define H3_GEMV_CASE(N) \
  case N: return gemv_v<WT, N>(W, b, wz, bz, Z, O, I, x, t, silu_in, silu_out, alpha, acc, y, yz, yv, num_sms, s);
    H3_GEMV_CASE(1) H3_GEMV_CASE(2) H3_GEMV_CASE(3) H3_GEMV_CASE(4) H3_GEMV_CASE(5) H3_GEMV_CASE(6)
    H3_GEMV_CASE(7) H3_GEMV_CASE(8)
#undef H3_GEMV_CASE
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_time_embedding(const ModTableArgs& a, int num_sms, cudaStream_t s) {
  const int V = a.n_sets, F0 = a.freq_dim, Hh = a.time_hidden, Td = a.time_dim;
  float* hid = a.scratch;                      // [V][Hh]
  float* E = a.scratch + (size_t)V * Hh;       // [V][Td]
  const ModTimes none{};
  const float g = a.gate;
  cudaError_t e;
  // hidden = silu(W1 e(t_now) + b1); E = (1 - g) (W2 hidden + b2)
  e = gemv<float>(a.w1, a.b1, 0, 0, 1, Hh, F0, V, nullptr, a.t_now, false, true, 1.f, false, hid, 0, Hh, num_sms, s);
  if (e != cudaSuccess) return e;
  e = gemv<float>(a.w2, a.b2, 0, 0, 1, Td, Hh, V, hid, none, false, false, 1.f - g, false, E, 0, Td, num_sms, s);
  if (e != cudaSuccess) return e;
  if (g != 0.f) {
    // E += g (W2r silu(W1r e(t_end) + b1r) + b2r)
    e = gemv<float>(a.w1_r, a.b1_r, 0, 0, 1, Hh, F0, V, nullptr, a.t_end, false, true, 1.f, false, hid, 0, Hh, num_sms,
                    s);
    if (e != cudaSuccess) return e;
    e = gemv<float>(a.w2_r, a.b2_r, 0, 0, 1, Td, Hh, V, hid, none, false, false, g, true, E, 0, Td, num_sms, s);
  }
  return e;
}

cudaError_t launch_adaln_projection(const ModTableArgs& a, int num_sms, cudaStream_t s) {
  const int V = a.n_sets, Td = a.time_dim, O = a.n_vec * a.hidden;
  const float* E = a.scratch + (size_t)V * a.time_hidden;
  const ModTimes none{};
  // table[tag][k] = A_tag silu(E_k) + a_tag
  return gemv<__nv_bfloat16>(a.adaln_w, a.adaln_b, (int64_t)O * Td, O, a.n_tags, O, Td, V, E, none, true, false, 1.f,
                             false, a.table, (int64_t)V * O, O, num_sms, s);
}

cudaError_t launch_modulation_table(const ModTableArgs& a, int num_sms, cudaStream_t s) {
  const cudaError_t e = launch_time_embedding(a, num_sms, s);
  return e != cudaSuccess ? e : launch_adaln_projection(a, num_sms, s);
}

}  // namespace h3
