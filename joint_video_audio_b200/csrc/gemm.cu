// Persistent, warp-specialised tcgen05 GEMM  C[M, N] = A[M, K] * B[N, K]^T
// with the block's fused epilogues (K2a/K2b/K2c/K2d, and the int8 K5).
//
//   warp 0      TMA producer: A tile 128 x 128 B and B tile 256 x 128 B per stage
//   warp 1      TMEM allocator + tcgen05.mma issuer (the whole warp runs the
//               loop, lane 0 issues)
//   warps 2..9  epilogue: tcgen05.ld of the fp32 / s32 accumulator (thread =
//               output row; the two warps of a lane quadrant take one half of
//               the tile's columns each), fused math, 16-byte global stores
//
// Accumulators are double-buffered in tensor memory (2 x 256 columns) so the
// epilogue of tile i overlaps the main loop of tile i+1. Operands are staged by
// TMA with the 128-byte swizzle the UMMA descriptors expect.
//
// Two kernels share these roles and epilogues: gemm_pair_kernel (used on
// B200) runs on clusters of two CTAs with 256 x 256 cluster tiles and
// products of M = 256 spanning both SMs (each SM stages its own 128 rows of A
// and half of B's rows: a third less shared-memory operand traffic per SM,
// six stages); gemm_kernel is the single-CTA form.
//
// Fused epilogues (sources: "MiniMaxH3Transformer3DModel", diffusers API
// page, constructor: qk_norm_eps of the per-head query/key norms, rope_theta;
// introduction: AdaLN modulation per modality tag; ffn_dim of the SwiGLU):
//   kEpiQKV    q, k: per-head RMSNorm (fp32) * gain, then 3D RoPE on adjacent
//              pairs, the (sin, cos) of each row's angles read from a table
//              made once per forward (rope_table_kernel); v: stored as is. Output [M, 3*H*D] bf16, or, routed by
//              head group for sequence parallelism, each head's q / k / v to
//              its group owner's [rows, 3*Hg*D] buffer (peer memory or a send
//              buffer).
//   kEpiResid  out = resid + gate[tag][tidx] * acc (padding rows: out = resid).
//   kEpiSwiGLU B holds W1 rows then W3 rows; tile j loads W1 rows j*128.. and W3
//              rows j*128.. into its two 128-column halves: out = silu(g) * u.
//   kEpiStoreBf16 out = acc (+ an fp32 bias per column when given).
//   kEpiStoreS32  raw int32 accumulators (exactness tests of the int8 path).
// int8 mode ("HyperFlow H3 Flash ...", "How it got smaller and faster":
// rotated W8A8): kind::i8, s32 accumulators, value = acc * s_a[row] * s_b[col].
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include "kernels.cuh"
#include "ptx.cuh"

namespace h3 {
namespace {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int kRowBytes = 128;  // one K-block per stage: 64 bf16 or 128 int8
constexpr int kStages = 4;
constexpr int kAStage = BM * kRowBytes;  // 16 KB
constexpr int kBStage = BN * kRowBytes;  // 32 KB
constexpr int kEpiWarps = 8;  // two per TMEM lane quadrant, each on one half of the tile's columns
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int kTmemCols = 512;  // two 256-column fp32 accumulators
constexpr int kGroupN = 8;      // tile raster: 8 N-tiles share each pass over M
constexpr int kGroupNPair = 12; // the CTA-pair kernel's raster (measured best of 4, 8, 12, 16)
constexpr size_t kSmemBytes = 1024 + (size_t)kStages * (kAStage + kBStage) + 256;

struct Smem {
  uint8_t* a;
  uint8_t* b;
  uint64_t* full;
  uint64_t* empty;
  uint64_t* tfull;
  uint64_t* tempty;
  uint64_t* drain;
  uint32_t* tmem_base;
  int* abort;
};

__device__ __forceinline__ Smem carve(uint8_t* raw) {
  const uint32_t base = smem_u32(raw);
  const uint32_t pad = ((base + 1023u) & ~1023u) - base;
  uint8_t* p = raw + pad;
  Smem s;
  s.a = p;
  s.b = p + kStages * kAStage;
  uint64_t* bars = reinterpret_cast<uint64_t*>(p + kStages * (kAStage + kBStage));
  s.full = bars;
  s.empty = bars + kStages;
  s.tfull = bars + 2 * kStages;
  s.tempty = bars + 2 * kStages + 2;
  s.drain = bars + 2 * kStages + 4;
  s.tmem_base = reinterpret_cast<uint32_t*>(bars + 2 * kStages + 5);
  s.abort = reinterpret_cast<int*>(bars + 2 * kStages + 6);
  return s;
}

struct TileCoord {
  int m, n;
};

template <int GROUP = kGroupN>
__device__ __forceinline__ TileCoord tile_coord(int t, int tiles_m, int tiles_n) {
  const int group = t / (GROUP * tiles_m);
  const int first_n = group * GROUP;
  const int gn = min(GROUP, tiles_n - first_n);
  const int idx = t - group * GROUP * tiles_m;
  return {idx / gn, first_n + idx % gn};
}

__device__ __forceinline__ void fail(const Smem& s, int* err) {
  if (err) atomicOr(err, kErrTimeoutGemm);
  *reinterpret_cast<volatile int*>(s.abort) = 1;
}

__device__ __forceinline__ void store_bf16x32(__nv_bfloat16* dst, const float (&v)[32]) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint4 o;
    o.x = pack_bf16x2(v[8 * i + 0], v[8 * i + 1]);
    o.y = pack_bf16x2(v[8 * i + 2], v[8 * i + 3]);
    o.z = pack_bf16x2(v[8 * i + 4], v[8 * i + 5]);
    o.w = pack_bf16x2(v[8 * i + 6], v[8 * i + 7]);
    d[i] = o;
  }
}

template <bool INT8>
__device__ __forceinline__ void load_chunk(uint32_t taddr, float sa, const float* sb, int col, float (&v)[32],
                                           int32_t* dump = nullptr) {
  uint32_t r[32];
  tmem_ld32(taddr, r);
  if (INT8 && dump) {
    uint4* d = reinterpret_cast<uint4*>(dump + col);
#pragma unroll
    for (int i = 0; i < 8; ++i) d[i] = make_uint4(r[4 * i], r[4 * i + 1], r[4 * i + 2], r[4 * i + 3]);
  }
  if (INT8) {
    // the chunk's 32 column scales, 16 bytes at a time (col is a multiple of
    // 32 and the scale vectors are 16-byte aligned)
    const float4* sb4 = reinterpret_cast<const float4*>(sb + col);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float4 b = __ldg(sb4 + i);
      v[4 * i + 0] = (float)(int)r[4 * i + 0] * sa * b.x;
      v[4 * i + 1] = (float)(int)r[4 * i + 1] * sa * b.y;
      v[4 * i + 2] = (float)(int)r[4 * i + 2] * sa * b.z;
      v[4 * i + 3] = (float)(int)r[4 * i + 3] * sa * b.w;
    }
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
  }
}

// cos and sin of a rotary angle: the angle is reduced to [-pi, pi] by a
// two-constant Cody-Waite step (Cody and Waite, "Software Manual for the
// Elementary Functions", 1980: 2 pi split into its nearest float and the
// remainder, each product taken exactly inside an FMA), then the hardware
// sine / cosine, accurate to about 2^-21 on that interval. The angles are
// position x frequency with positions of a few thousand at most.
__device__ __forceinline__ void rope_sincos(float x, float& sn, float& cs) {
  constexpr float kTwoPiHi = 6.28318548202514648f;   // float(2 pi)
  constexpr float kTwoPiLo = -1.74845553146951e-07f;  // 2 pi - float(2 pi)
  constexpr float kInvTwoPi = 0.159154943091895336f;
  const float k = rintf(x * kInvTwoPi);
  float r = fmaf(-k, kTwoPiHi, x);
  r = fmaf(-k, kTwoPiLo, r);
  __sincosf(r, &sn, &cs);
}

// One thread per (row, pair): the table the QKV epilogue reads.
__global__ void rope_table_kernel(const int32_t* __restrict__ pos, int64_t n, const RopeTable rope, int pairs,
                                  float2* __restrict__ tab) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n * pairs) return;
  const int64_t row = i / pairs;
  const int pair = (int)(i - row * pairs);
  const int ax = rope.axis[pair];
  float sn = 0.f, cs = 1.f;
  if (ax < 3) rope_sincos((float)__ldg(pos + row * 3 + ax) * rope.freq[pair], sn, cs);
  tab[i] = make_float2(sn, cs);
}

// ------------------------------------------------------------------ epilogue
template <int EPI, bool INT8>
__device__ __forceinline__ void epilogue_tile(const GemmArgs& p, uint32_t tacc, int64_t row, bool row_ok, int n_tile,
                                              int half) {
  const float sa = (INT8 && row_ok) ? __ldg(p.s_a + row) : 0.f;
  int32_t* dump = (INT8 && p.acc_dump && row_ok) ? p.acc_dump + row * p.ld_dump : nullptr;
  if (EPI == kEpiSwiGLU) {
    const int col0 = n_tile * 128;
#pragma unroll 1
    for (int c = 2 * half; c < 2 * half + 2; ++c) {
      float g[32], u[32];
      load_chunk<INT8>(tacc + c * 32, sa, p.s_b, col0 + c * 32, g, dump);
      load_chunk<INT8>(tacc + 128 + c * 32, sa, p.s_b, p.N + col0 + c * 32, u, dump);
#pragma unroll
      for (int j = 0; j < 32; ++j) g[j] = g[j] / (1.f + __expf(-g[j])) * u[j];
      if (row_ok) store_bf16x32(reinterpret_cast<__nv_bfloat16*>(p.out) + row * p.ld_out + col0 + c * 32, g);
    }
    return;
  }
  const int n0 = n_tile * BN;
  constexpr int kHalfChunks = BN / 64;  // 32-column chunks in one half of the tile
  if (EPI == kEpiStoreS32) {
#pragma unroll 1
    for (int c = half * kHalfChunks; c < (half + 1) * kHalfChunks; ++c) {
      if (n0 + c * 32 >= p.N) break;
      uint32_t r[32];
      tmem_ld32(tacc + c * 32, r);
      if (row_ok) {
        uint4* d = reinterpret_cast<uint4*>(reinterpret_cast<int32_t*>(p.out) + row * p.ld_out + n0 + c * 32);
#pragma unroll
        for (int i = 0; i < 8; ++i) d[i] = make_uint4(r[4 * i], r[4 * i + 1], r[4 * i + 2], r[4 * i + 3]);
      }
    }
    return;
  }
  if (EPI == kEpiStoreBf16 || EPI == kEpiResid) {
    const float* gate = nullptr;
    if (EPI == kEpiResid && row_ok) {
      const int tg = p.tag[row], ti = p.tidx[row];
      if (tg >= 0 && tg < p.n_tags && ti >= 0 && ti < p.n_t)
        gate = p.table + (((int64_t)tg * p.n_t + ti) * 6 + p.gate_idx) * p.N;
    }
#pragma unroll 1
    for (int c = half * kHalfChunks; c < (half + 1) * kHalfChunks; ++c) {
      const int col = n0 + c * 32;
      if (col >= p.N) break;
      float v[32];
      load_chunk<INT8>(tacc + c * 32, sa, p.s_b, col, v, dump);
      if (!row_ok) continue;
      __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.out) + row * p.ld_out + col;
      if (EPI == kEpiStoreBf16 && p.bias) {
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
          const float4 b4 = __ldg(reinterpret_cast<const float4*>(p.bias + col + j));
          v[j] += b4.x;
          v[j + 1] += b4.y;
          v[j + 2] += b4.z;
          v[j + 3] += b4.w;
        }
      }
      if (EPI == kEpiResid) {
        const uint4* rs = reinterpret_cast<const uint4*>(p.resid + row * (int64_t)p.N + col);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint4 q = __ldg(rs + i);
          const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const float2 x2 = unpack_bf16x2(w[h]);
            const int j = 8 * i + 2 * h;
            if (gate) {
              const float2 g2 = __ldg(reinterpret_cast<const float2*>(gate + col + j));
              v[j] = fmaf(g2.x, v[j], x2.x);
              v[j + 1] = fmaf(g2.y, v[j + 1], x2.y);
            } else {
              v[j] = x2.x;
              v[j + 1] = x2.y;
            }
          }
        }
      }
      store_bf16x32(dst, v);
    }
    return;
  }
  if (EPI == kEpiQKV) {
    const int D = p.head_dim;
    const int heads_per_half = (BN / 2) / D;
#pragma unroll 1
    for (int hh = half * heads_per_half; hh < (half + 1) * heads_per_half; ++hh) {
      const int col0 = n0 + hh * D;
      if (col0 >= p.N) break;
      const int region = col0 / p.hd;  // 0 q, 1 k, 2 v
      const uint32_t th = tacc + hh * D;
      __nv_bfloat16* dst;
      if (p.route_ranks > 0) {
        // sequence parallelism: the head's group owner holds q / k / v of
        // every row for its heads
        const int hi = (col0 - region * p.hd) / D;
        const int hg = p.route_hg;
        dst = reinterpret_cast<__nv_bfloat16*>(p.route_dst[hi / hg]) +
              (p.route_row0 + row) * (int64_t)(3 * hg * D) + (region * hg + hi % hg) * D;
      } else {
        dst = reinterpret_cast<__nv_bfloat16*>(p.out) + row * p.ld_out + col0;
      }
      if (region == 2) {
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          float v[32];
          load_chunk<INT8>(th + c * 32, sa, p.s_b, col0 + c * 32, v, dump);
          if (row_ok) store_bf16x32(dst + c * 32, v);
        }
        continue;
      }
      float ss = 0.f;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        float v[32];
        load_chunk<INT8>(th + c * 32, sa, p.s_b, col0 + c * 32, v, dump);
#pragma unroll
        for (int j = 0; j < 32; ++j) ss = fmaf(v[j], v[j], ss);
      }
      const float rstd = rsqrtf(ss / (float)D + p.qk_eps);
      const __nv_bfloat16* gain = region == 0 ? p.q_gain : p.k_gain;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        // this chunk's 16 (sin, cos) pairs, requested before the accumulators
        float4 sc[8];
        if (row_ok) {
          const float4* t4 = reinterpret_cast<const float4*>(p.rope_tab + row * (D / 2) + c * 16);
#pragma unroll
          for (int i = 0; i < 8; ++i) sc[i] = __ldg(t4 + i);
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i) sc[i] = make_float4(0.f, 1.f, 0.f, 1.f);
        }
        float v[32];
        load_chunk<INT8>(th + c * 32, sa, p.s_b, col0 + c * 32, v, dump);
        // the chunk's 32 gains, 16 bytes (8 bf16) at a time
        const uint4* g4 = reinterpret_cast<const uint4*>(gain + c * 32);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint4 gw = __ldg(g4 + i);
          const uint32_t gq[4] = {gw.x, gw.y, gw.z, gw.w};
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const float2 g2 = unpack_bf16x2(gq[h]);
            const int j = 8 * i + 2 * h;
            v[j] = v[j] * rstd * g2.x;
            v[j + 1] = v[j + 1] * rstd * g2.y;
          }
        }
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          if (p.rope.axis[c * 16 + q] < 3) {
            const float sn = (q & 1) ? sc[q >> 1].z : sc[q >> 1].x;
            const float cs = (q & 1) ? sc[q >> 1].w : sc[q >> 1].y;
            const float a = v[2 * q], b = v[2 * q + 1];
            v[2 * q] = a * cs - b * sn;
            v[2 * q + 1] = a * sn + b * cs;
          }
        }
        if (row_ok) store_bf16x32(dst + c * 32, v);
      }
    }
  }
}

// ------------------------------------------------------------------ kernel
template <int EPI, bool INT8>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, const GemmArgs p) {
  extern __shared__ uint8_t smem_raw[];
  const Smem s = carve(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles_m = (int)((p.M + BM - 1) / BM);
  const int tiles_n = EPI == kEpiSwiGLU ? p.N / 128 : (p.N + BN - 1) / BN;
  const int num_tiles = tiles_m * tiles_n;
  const int num_kb = p.K / (INT8 ? 128 : 64);
  volatile int* abort = s.abort;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.tfull[i], 1);
      mbar_init(&s.tempty[i], kEpiWarps);  // one arrival per epilogue warp
    }
    mbar_init(s.drain, 1);
    *s.abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(s.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s.tmem_base;

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      long issued = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        const TileCoord tc = tile_coord(t, tiles_m, tiles_n);
        const int ya = tc.m * BM;
        int yb0, yb1;
        bool second = true;
        if (EPI == kEpiSwiGLU) {
          yb0 = tc.n * 128;
          yb1 = p.N + tc.n * 128;
        } else {
          yb0 = tc.n * BN;
          yb1 = yb0 + 128;
          second = yb1 < p.Nb;
        }
        const uint32_t bytes = kAStage + (second ? kBStage : kBStage / 2);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&s.empty[stage], phase ^ 1, abort)) {
            fail(s, p.err);
            ok = false;
            break;
          }
          const int x = kb * (INT8 ? 128 : 64);
          mbar_expect_tx(&s.full[stage], bytes);
          tma_load_2d(s.a + stage * kAStage, &tmA, &s.full[stage], x, ya);
          tma_load_2d(s.b + stage * kBStage, &tmB, &s.full[stage], x, yb0);
          if (second) tma_load_2d(s.b + stage * kBStage + kBStage / 2, &tmB, &s.full[stage], x, yb1);
          ++issued;
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // Drain: the last loads issued must have landed before the CTA exits.
      const long outstanding = issued < kStages ? issued : kStages;
      for (long i = 0; i < outstanding; ++i) {
        if (--stage < 0) {
          stage = kStages - 1;
          phase ^= 1;
        }
        mbar_wait(&s.full[stage], phase, nullptr);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    // the whole warp runs the loop (warp-uniform descriptors); lane 0 issues
    // every product and commit
    {
      const uint32_t idesc = INT8 ? make_idesc(2, 1, BM, BN, false) : make_idesc(1, 1, BM, BN, false);
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x, ++local) {
        const int buf = local & 1;
        const uint32_t use = (uint32_t)(local >> 1);
        if (!mbar_wait_warp(&s.tempty[buf], (use & 1) ^ 1, abort)) {
          if (lane == 0) fail(s, p.err);
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + buf * BN;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait_warp(&s.full[stage], phase, abort)) {
            if (lane == 0) fail(s, p.err);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(s.a + stage * kAStage);
          const uint32_t b0 = smem_u32(s.b + stage * kBStage);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint64_t ad = sw128_desc(a0 + k * 32, 16);
            const uint64_t bd = sw128_desc(b0 + k * 32, 16);
            if (INT8)
              mma_s8_ss_w(d, ad, bd, idesc, (kb | k) != 0);
            else
              mma_bf16_ss_w(d, ad, bd, idesc, (kb | k) != 0);
          }
          mma_commit_w(&s.empty[stage]);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (ok) mma_commit_w(&s.tfull[buf]);
      }
      // every MMA issued by lane 0 has completed once `drain` flips
      mma_commit_w(s.drain);
      mbar_wait(s.drain, 0, nullptr);
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int quad = warp & 3;
    const int half = (warp - 2) >> 2;
    int local = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++local) {
      const TileCoord tc = tile_coord(t, tiles_m, tiles_n);
      const int buf = local & 1;
      const uint32_t use = (uint32_t)(local >> 1);
      if (!mbar_wait(&s.tfull[buf], use & 1, abort)) {
        if (lane == 0) fail(s, p.err);
        break;
      }
      tc_fence_after();
      const int64_t row = (int64_t)tc.m * BM + quad * 32 + lane;
      const uint32_t tacc = tmem_base + ((uint32_t)(quad * 32) << 16) + buf * BN;
      epilogue_tile<EPI, INT8>(p, tacc, row, row < p.M, tc.n, half);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.tempty[buf]);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, kTmemCols);
}

// ------------------------------------------------------------------ CTA-pair kernel
// The same GEMM on clusters of two CTAs (one per SM of a pair): a cluster
// tile is 256 x 256; each CTA stages its 128 rows of A and its 128 rows of B
// (the weight rows of one half of the tile's columns), and the pair's first
// CTA issues products of M = 256, N = 256 that read A and B from both SMs'
// shared memory and leave each SM's 128 rows of the accumulator in its own
// tensor memory. Per SM that is the single-CTA kernel's 128 x 256 tile with
// two thirds of its shared-memory operand traffic (B is split, not
// duplicated), so more stages fit. Both CTAs' loads signal the first CTA's
// "full" barrier; the issuer's commits arrive on the "empty", "accumulator
// full" and final barriers of both CTAs; the second CTA's epilogue warps
// release an accumulator buffer on the first CTA's barrier.
constexpr int kStagesPair = 6;
constexpr int kBHalfStage = 128 * kRowBytes;  // 16 KB
constexpr size_t kSmemBytesPair = 1024 + (size_t)kStagesPair * (kAStage + kBHalfStage) + 256;

struct SmemPair {
  uint8_t* a;
  uint8_t* b;
  uint64_t* full;
  uint64_t* empty;
  uint64_t* tfull;
  uint64_t* tempty;
  uint64_t* drain;
  uint32_t* tmem_base;
  int* abort;
};

__device__ __forceinline__ SmemPair carve_pair(uint8_t* raw) {
  const uint32_t base = smem_u32(raw);
  const uint32_t pad = ((base + 1023u) & ~1023u) - base;
  uint8_t* p = raw + pad;
  SmemPair s;
  s.a = p;
  s.b = p + kStagesPair * kAStage;
  uint64_t* bars = reinterpret_cast<uint64_t*>(p + kStagesPair * (kAStage + kBHalfStage));
  s.full = bars;
  s.empty = bars + kStagesPair;
  s.tfull = bars + 2 * kStagesPair;
  s.tempty = bars + 2 * kStagesPair + 2;
  s.drain = bars + 2 * kStagesPair + 4;
  s.tmem_base = reinterpret_cast<uint32_t*>(bars + 2 * kStagesPair + 5);
  s.abort = reinterpret_cast<int*>(bars + 2 * kStagesPair + 6);
  return s;
}

__device__ __forceinline__ void fail_pair(const SmemPair& s, int* err) {
  if (err) atomicOr(err, kErrTimeoutGemm);
  *reinterpret_cast<volatile int*>(s.abort) = 1;
}

template <int EPI, bool INT8>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const GemmArgs p) {
  extern __shared__ uint8_t smem_raw[];
  const SmemPair s = carve_pair(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int cluster = blockIdx.x >> 1, n_clusters = gridDim.x >> 1;
  const int tiles_m = (int)((p.M + 2 * BM - 1) / (2 * BM));
  const int tiles_n = EPI == kEpiSwiGLU ? p.N / 128 : (p.N + BN - 1) / BN;
  const int num_tiles = tiles_m * tiles_n;
  const int num_kb = p.K / (INT8 ? 128 : 64);
  volatile int* abort = s.abort;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStagesPair; ++i) {
      mbar_init(&s.full[i], 1);   // the first CTA's producer arrives; both CTAs' bytes complete it
      mbar_init(&s.empty[i], 1);  // one commit of the issuer
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.tfull[i], 1);
      mbar_init(&s.tempty[i], 2 * kEpiWarps);  // every epilogue warp of both CTAs
    }
    mbar_init(s.drain, 1);
    *s.abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc_pair(s.tmem_base, kTmemCols);
    tmem_relinquish_pair();
  }
  // both CTAs' barriers are initialised and their tensor memory allocated
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *s.tmem_base;

  if (warp == 0) {
    // ---------------------------------------------------------------- producer (both CTAs)
    if (lane == 0) {
      const uint32_t full0 = mapa_shared(smem_u32(s.full), 0);  // the first CTA's full barriers
      int stage = 0;
      uint32_t phase = 0;
      long issued = 0;
      bool ok = true;
      for (int t = cluster; t < num_tiles && ok; t += n_clusters) {
        const TileCoord tc = tile_coord<kGroupNPair>(t, tiles_m, tiles_n);
        const int ya = tc.m * 2 * BM + (int)rank * BM;
        const int yb = EPI == kEpiSwiGLU ? (rank == 0 ? tc.n * 128 : p.N + tc.n * 128) : tc.n * BN + (int)rank * 128;
        // A box wholly past the last row (the second CTA's rows of a short
        // last M tile) or a B box wholly past the last weight row (the second
        // half of a last N tile) is not loaded: the accumulator rows / columns
        // it would feed are never stored. The first CTA's boxes always hold
        // data, and it expects the bytes of every box the pair loads.
        const bool a1 = tc.m * 2 * BM + BM < p.M;
        const bool b1 = EPI == kEpiSwiGLU || tc.n * BN + 128 < p.Nb;
        const bool load_a = rank == 0 || a1, load_b = rank == 0 || b1;
        const uint32_t bytes = kAStage + kBHalfStage + (a1 ? kAStage : 0) + (b1 ? kBHalfStage : 0);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&s.empty[stage], phase ^ 1, abort)) {
            fail_pair(s, p.err);
            ok = false;
            break;
          }
          const int x = kb * (INT8 ? 128 : 64);
          if (rank == 0) mbar_expect_tx(&s.full[stage], bytes);
          if (load_a) tma_load_2d_pair(s.a + stage * kAStage, &tmA, full0 + 8u * stage, x, ya);
          if (load_b) tma_load_2d_pair(s.b + stage * kBHalfStage, &tmB, full0 + 8u * stage, x, yb);
          ++issued;
          if (++stage == kStagesPair) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // Drain (first CTA; its full barriers count both CTAs' bytes): the last
      // loads issued must have landed before either CTA exits.
      if (rank == 0) {
        const long outstanding = issued < kStagesPair ? issued : kStagesPair;
        for (long i = 0; i < outstanding; ++i) {
          if (--stage < 0) {
            stage = kStagesPair - 1;
            phase ^= 1;
          }
          mbar_wait(&s.full[stage], phase, nullptr);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer (first CTA)
    // the whole warp runs the loop (warp-uniform descriptors); lane 0 issues
    // every product and commit
    if (rank == 0) {
      const uint32_t idesc = INT8 ? make_idesc(2, 1, 2 * BM, BN, false) : make_idesc(1, 1, 2 * BM, BN, false);
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      for (int t = cluster; t < num_tiles && ok; t += n_clusters, ++local) {
        const int buf = local & 1;
        const uint32_t use = (uint32_t)(local >> 1);
        if (!mbar_wait_warp(&s.tempty[buf], (use & 1) ^ 1, abort)) {
          if (lane == 0) fail_pair(s, p.err);
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + buf * BN;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait_warp(&s.full[stage], phase, abort)) {
            if (lane == 0) fail_pair(s, p.err);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(s.a + stage * kAStage);
          const uint32_t b0 = smem_u32(s.b + stage * kBHalfStage);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint64_t ad = sw128_desc(a0 + k * 32, 16);
            const uint64_t bd = sw128_desc(b0 + k * 32, 16);
            if (INT8)
              mma_s8_ss_pair_w(d, ad, bd, idesc, (kb | k) != 0);
            else
              mma_bf16_ss_pair_w(d, ad, bd, idesc, (kb | k) != 0);
          }
          mma_commit_pair_w(&s.empty[stage], 0x3);
          if (++stage == kStagesPair) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (ok) mma_commit_pair_w(&s.tfull[buf], 0x3);
      }
      // every product issued has completed once `drain` flips (in both CTAs)
      mma_commit_pair_w(s.drain, 0x3);
      mbar_wait(s.drain, 0, nullptr);
    } else if (lane == 0) {
      // second CTA: its shared memory and tensor memory serve the pair's
      // products until the last one completes
      mbar_wait(s.drain, 0, nullptr);
    }
  } else {
    // ---------------------------------------------------------------- epilogue (both CTAs)
    const int quad = warp & 3;
    const int half = (warp - 2) >> 2;
    const uint32_t tempty0 = mapa_shared(smem_u32(s.tempty), 0);
    int local = 0;
    for (int t = cluster; t < num_tiles; t += n_clusters, ++local) {
      const TileCoord tc = tile_coord<kGroupNPair>(t, tiles_m, tiles_n);
      const int buf = local & 1;
      const uint32_t use = (uint32_t)(local >> 1);
      if (!mbar_wait(&s.tfull[buf], use & 1, abort)) {
        if (lane == 0) fail_pair(s, p.err);
        break;
      }
      tc_fence_after();
      const int64_t row = (int64_t)tc.m * 2 * BM + (int64_t)rank * BM + quad * 32 + lane;
      const uint32_t tacc = tmem_base + ((uint32_t)(quad * 32) << 16) + buf * BN;
      epilogue_tile<EPI, INT8>(p, tacc, row, row < p.M, tc.n, half);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty0 + 8u * buf);
    }
  }

  // neither CTA leaves while the other may still signal its barriers or read
  // its memory
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, kTmemCols);
}

CUresult make_map(PFN_cuTensorMapEncodeTiled_v12000 encode, CUtensorMap* m, const void* ptr, uint64_t rows,
                  uint64_t cols, bool int8) {
  const CUtensorMapDataType dt = int8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const uint64_t esz = int8 ? 1 : 2;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * esz};
  cuuint32_t box[2] = {(cuuint32_t)(kRowBytes / esz), 128};
  cuuint32_t estr[2] = {1, 1};
  return encode(m, dt, 2, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

template <int EPI, bool INT8>
cudaError_t launch_t(const GemmArgs& a, const CUtensorMap& ta, const CUtensorMap& tb, int num_sms, cudaStream_t s) {
  auto k = gemm_kernel<EPI, INT8>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  const int tiles_m = (int)((a.M + BM - 1) / BM);
  const int tiles_n = EPI == kEpiSwiGLU ? a.N / 128 : (a.N + BN - 1) / BN;
  const long tiles = (long)tiles_m * tiles_n;
  const int grid = (int)(tiles < num_sms ? tiles : num_sms);
  k<<<grid, kThreads, kSmemBytes, s>>>(ta, tb, a);
  return cudaGetLastError();
}

template <int EPI, bool INT8>
cudaError_t launch_pair_t(const GemmArgs& a, const CUtensorMap& ta, const CUtensorMap& tb, int num_sms,
                          cudaStream_t s) {
  auto k = gemm_pair_kernel<EPI, INT8>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytesPair);
  if (e != cudaSuccess) return e;
  const int tiles_m = (int)((a.M + 2 * BM - 1) / (2 * BM));
  const int tiles_n = EPI == kEpiSwiGLU ? a.N / 128 : (a.N + BN - 1) / BN;
  const long tiles = (long)tiles_m * tiles_n;
  const int max_clusters = num_sms / 2;
  const int clusters = (int)(tiles < max_clusters ? tiles : max_clusters);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * clusters);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytesPair;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k, ta, tb, a);
}

}  // namespace

cudaError_t launch_rope_table(const int32_t* pos, int64_t n, const RopeTable& rope, int pairs, float2* tab,
                              cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  if (pairs < 1 || pairs > kMaxRopePairs || pos == nullptr || tab == nullptr) return cudaErrorInvalidValue;
  const int64_t total = n * pairs;
  rope_table_kernel<<<(unsigned)((total + 255) / 256), 256, 0, s>>>(pos, n, rope, pairs, tab);
  return cudaGetLastError();
}

cudaError_t launch_gemm(const GemmArgs& a, PFN_cuTensorMapEncodeTiled_v12000 encode, int num_sms, cudaStream_t s) {
  if (a.M <= 0) return cudaSuccess;
  const int kb = a.int8 ? 128 : 64;
  if (a.K % kb != 0 || a.N % 128 != 0 || a.Nb % 128 != 0) return cudaErrorInvalidValue;
  if (a.epi == kEpiQKV && (a.head_dim % 32 != 0 || (BN / 2) % a.head_dim != 0 || a.hd % a.head_dim != 0 ||
                           a.rope_tab == nullptr || (reinterpret_cast<uintptr_t>(a.rope_tab) & 15) != 0))
    return cudaErrorInvalidValue;
  CUtensorMap ta, tb;
  if (make_map(encode, &ta, a.A, (uint64_t)a.M, (uint64_t)a.K, a.int8) != CUDA_SUCCESS) return cudaErrorInvalidValue;
  if (make_map(encode, &tb, a.B, (uint64_t)a.Nb, (uint64_t)a.K, a.int8) != CUDA_SUCCESS) return cudaErrorInvalidValue;
#ifndef H3_GEMM_PAIR
#define H3_GEMM_PAIR 1
#endif
  if (H3_GEMM_PAIR && num_sms >= 2) {
    if (a.int8) {
      switch (a.epi) {
        case kEpiStoreBf16: return launch_pair_t<kEpiStoreBf16, true>(a, ta, tb, num_sms, s);
        case kEpiQKV: return launch_pair_t<kEpiQKV, true>(a, ta, tb, num_sms, s);
        case kEpiResid: return launch_pair_t<kEpiResid, true>(a, ta, tb, num_sms, s);
        case kEpiSwiGLU: return launch_pair_t<kEpiSwiGLU, true>(a, ta, tb, num_sms, s);
        case kEpiStoreS32: return launch_pair_t<kEpiStoreS32, true>(a, ta, tb, num_sms, s);
      }
    } else {
      switch (a.epi) {
        case kEpiStoreBf16: return launch_pair_t<kEpiStoreBf16, false>(a, ta, tb, num_sms, s);
        case kEpiQKV: return launch_pair_t<kEpiQKV, false>(a, ta, tb, num_sms, s);
        case kEpiResid: return launch_pair_t<kEpiResid, false>(a, ta, tb, num_sms, s);
        case kEpiSwiGLU: return launch_pair_t<kEpiSwiGLU, false>(a, ta, tb, num_sms, s);
      }
    }
    return cudaErrorInvalidValue;
  }
  if (a.int8) {
    switch (a.epi) {
      case kEpiStoreBf16: return launch_t<kEpiStoreBf16, true>(a, ta, tb, num_sms, s);
      case kEpiQKV: return launch_t<kEpiQKV, true>(a, ta, tb, num_sms, s);
      case kEpiResid: return launch_t<kEpiResid, true>(a, ta, tb, num_sms, s);
      case kEpiSwiGLU: return launch_t<kEpiSwiGLU, true>(a, ta, tb, num_sms, s);
      case kEpiStoreS32: return launch_t<kEpiStoreS32, true>(a, ta, tb, num_sms, s);
    }
  } else {
    switch (a.epi) {
      case kEpiStoreBf16: return launch_t<kEpiStoreBf16, false>(a, ta, tb, num_sms, s);
      case kEpiQKV: return launch_t<kEpiQKV, false>(a, ta, tb, num_sms, s);
      case kEpiResid: return launch_t<kEpiResid, false>(a, ta, tb, num_sms, s);
      case kEpiSwiGLU: return launch_t<kEpiSwiGLU, false>(a, ta, tb, num_sms, s);
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace h3
