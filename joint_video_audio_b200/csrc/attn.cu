// Document-masked flash attention on tcgen05 / TMEM (K3).
//
// Source: "MiniMaxH3Transformer3DModel" (diffusers API page), introduction:
// full self-attention over the packed sequence; padding rows (tag -1) are kept
// in their own attention document by a boolean mask. The attention scale is
// 1/sqrt(head_dim).
//
// One CTA per (128-query tile, head). Roles:
//   warp 0      TMA: Q once; lane 0 streams K tiles, lane 1 streams V tiles
//               (two stages each, so K loads never wait on a P*V product)
//   warp 1      TMEM allocator + single-thread MMA issuer:
//                 S[j%2] = Q K_j^T            (M=128, N=128, K=head_dim)
//                 O     += P_{j-1} V_{j-1}    (M=128, N=head_dim, K=128)
//   warps 2..5  softmax, one thread per query row: S row from TMEM, mask,
//               online max / sum in the exp2 domain, P (bf16) into shared
//               memory in the swizzled K-major layout the MMA reads, and the
//               rescale of O in TMEM when the running max grows by more than
//               2^8 (otherwise the stale max is kept: values stay below 256).
// KV tiles whose rows all lie in the other document are skipped; tiles that
// mix documents, or run past the end of the sequence, are masked per element.
#include <cuda_bf16.h>
#include <cudaTypedefs.h>
#include <math_constants.h>

#include "kernels.cuh"
#include "ptx.cuh"

namespace h3 {
namespace {

constexpr int kThreads = 192;
constexpr int kTile = 128;
constexpr uint32_t kTmemCols = 512;  // S0 | S1 | O
constexpr float kRescaleThreshold = 8.0f;

template <int D>
struct AttnSmem {
  static constexpr int kQBytes = kTile * D * 2;
  static constexpr int kKVBytes = kTile * D * 2;
  static constexpr int kPBytes = kTile * kTile * 2;
  static constexpr int kRegion = kTile * 128;  // one 128-row x 128-byte swizzle region
  static constexpr size_t kBytes = 1024 + kQBytes + 4 * (size_t)kKVBytes + kPBytes + 256;
  uint8_t *q, *k[2], *v[2], *p;
  uint64_t *q_full, *k_full, *k_empty, *v_full, *v_empty, *s_full, *s_free, *p_full, *o_ready, *o_final;
  uint32_t* tmem_base;
  int* abort;

  __device__ explicit AttnSmem(uint8_t* raw) {
    const uint32_t base = smem_u32(raw);
    uint8_t* x = raw + (((base + 1023u) & ~1023u) - base);
    q = x;
    x += kQBytes;
    for (int i = 0; i < 2; ++i) {
      k[i] = x;
      x += kKVBytes;
    }
    for (int i = 0; i < 2; ++i) {
      v[i] = x;
      x += kKVBytes;
    }
    p = x;
    x += kPBytes;
    uint64_t* b = reinterpret_cast<uint64_t*>(x);
    q_full = b;
    k_full = b + 1;
    k_empty = b + 3;
    v_full = b + 5;
    v_empty = b + 7;
    s_full = b + 9;
    s_free = b + 11;
    p_full = b + 13;
    o_ready = b + 14;
    o_final = b + 15;
    tmem_base = reinterpret_cast<uint32_t*>(b + 16);
    abort = reinterpret_cast<int*>(b + 17);
  }
};

// 0: no padding rows, 1: only padding rows, 2: both
__device__ __forceinline__ int tile_kind(const TileInfo& t) {
  return t.npad == 0 ? 0 : (t.npad == t.rows ? 1 : 2);
}

// Advances `kt` to the next KV tile that the query tile must visit.
__device__ __forceinline__ int next_kv_tile(const TileInfo* tiles, int n_tiles, int qkind, int kt) {
  for (; kt < n_tiles; ++kt) {
    const int kk = tile_kind(tiles[kt]);
    if ((qkind == 0 && kk == 1) || (qkind == 1 && kk == 0)) continue;
    return kt;
  }
  return n_tiles;
}

__device__ __forceinline__ void fail(int* err, volatile int* abort) {
  if (err) atomicOr(err, kErrTimeoutAttn);
  *abort = 1;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1) attn_kernel(const __grid_constant__ CUtensorMap tm, const AttnArgs p) {
  extern __shared__ uint8_t smem_raw[];
  AttnSmem<D> s(smem_raw);
  using SM = AttnSmem<D>;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = blockIdx.x, head = blockIdx.y;
  const int n_tiles = (int)((p.n + kTile - 1) / kTile);
  const int HD = p.heads * D;
  const int qkind = tile_kind(p.tiles[qt]);
  volatile int* abort = s.abort;
  constexpr int kRegions = D / 64;  // 64-column swizzle regions of a Q/K/V tile

  if (threadIdx.x == 0) {
    mbar_init(s.q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.k_full[i], 1);
      mbar_init(&s.k_empty[i], 1);
      mbar_init(&s.v_full[i], 1);
      mbar_init(&s.v_empty[i], 1);
      mbar_init(&s.s_full[i], 1);
      mbar_init(&s.s_free[i], 4);
    }
    mbar_init(s.p_full, 4);
    mbar_init(s.o_ready, 1);
    mbar_init(s.o_final, 1);
    *s.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(s.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s.tmem_base;
  const uint32_t t_s = tmem, t_o = tmem + 256;

  if (warp == 0) {
    // ------------------------------------------------------------ loads
    if (lane == 0) {
      tma_prefetch_desc(&tm);
      mbar_expect_tx(s.q_full, SM::kQBytes);
      for (int r = 0; r < kRegions; ++r)
        tma_load_2d(s.q + r * SM::kRegion, &tm, s.q_full, head * D + r * 64, qt * kTile);
    }
    if (lane == 0 || lane == 1) {
      const bool is_k = lane == 0;
      uint64_t* full = is_k ? s.k_full : s.v_full;
      uint64_t* empty = is_k ? s.k_empty : s.v_empty;
      const int col = (is_k ? HD : 2 * HD) + head * D;
      int j = 0;
      for (int kt = next_kv_tile(p.tiles, n_tiles, qkind, 0); kt < n_tiles;
           kt = next_kv_tile(p.tiles, n_tiles, qkind, kt + 1), ++j) {
        const int st = j & 1;
        if (!mbar_wait(&empty[st], ((j >> 1) & 1) ^ 1, abort)) {
          fail(p.err, abort);
          break;
        }
        uint8_t* dst = is_k ? s.k[st] : s.v[st];
        mbar_expect_tx(&full[st], SM::kKVBytes);
        for (int r = 0; r < kRegions; ++r) tma_load_2d(dst + r * SM::kRegion, &tm, &full[st], col + r * 64, kt * kTile);
      }
      // drain the last (up to two) loads before the CTA may exit
      for (int i = 0; i < 2 && j - 1 - i >= 0; ++i) {
        const int jj = j - 1 - i;
        mbar_wait(&full[jj & 1], (jj >> 1) & 1, nullptr);
      }
    }
    if (lane == 0) mbar_wait(s.q_full, 0, nullptr);
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA
    if (lane == 0) {
      constexpr uint32_t idesc_qk = make_idesc(1, 1, kTile, kTile, false);
      constexpr uint32_t idesc_pv = make_idesc(1, 1, kTile, D, true);
      const uint32_t q0 = smem_u32(s.q), p0 = smem_u32(s.p);
      bool ok = mbar_wait(s.q_full, 0, abort);
      int j = 0;
      auto issue_pv = [&](int i) -> bool {
        const int st = i & 1;
        if (!mbar_wait(s.p_full, i & 1, abort)) return false;
        if (!mbar_wait(&s.v_full[st], (i >> 1) & 1, abort)) return false;
        tc_fence_after();
        const uint32_t v0 = smem_u32(s.v[st]);
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk) {
          const uint64_t ad = sw128_desc(p0 + (kk >> 2) * SM::kRegion + (kk & 3) * 32, 16);
          const uint64_t bd = sw128_desc(v0 + kk * 16 * 128, SM::kRegion);
          mma_bf16_ss(t_o, ad, bd, idesc_pv, (i > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&s.v_empty[st]);
        mma_commit(s.o_ready);
        return true;
      };
      if (ok) {
        for (int kt = next_kv_tile(p.tiles, n_tiles, qkind, 0); kt < n_tiles;
             kt = next_kv_tile(p.tiles, n_tiles, qkind, kt + 1), ++j) {
          const int st = j & 1;
          if (!mbar_wait(&s.k_full[st], (j >> 1) & 1, abort) ||
              !mbar_wait(&s.s_free[st], ((j >> 1) & 1) ^ 1, abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t k0 = smem_u32(s.k[st]);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * SM::kRegion + (kk & 3) * 32;
            mma_bf16_ss(t_s + st * kTile, sw128_desc(q0 + off, 16), sw128_desc(k0 + off, 16), idesc_qk,
                        kk > 0 ? 1u : 0u);
          }
          mma_commit(&s.k_empty[st]);
          mma_commit(&s.s_full[st]);
          if (j > 0 && !issue_pv(j - 1)) {
            ok = false;
            break;
          }
        }
        if (ok && j > 0) ok = issue_pv(j - 1);
      }
      if (!ok) fail(p.err, abort);
      mma_commit(s.o_final);
      mbar_wait(s.o_final, 0, nullptr);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int quad = warp & 3;
    const int r = quad * 32 + lane;  // row within the tile = TMEM lane
    const int64_t row = (int64_t)qt * kTile + r;
    const bool row_ok = row < p.n;
    const uint32_t my_pad = (row_ok && p.tag[row] == -1) ? 1u : 0u;
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    const float scale_log2 = 1.4426950408889634f * rsqrtf((float)D);
    float m_run = -CUDART_INF_F, l_run = 0.f;
    uint8_t* prow = s.p + r * 128;
    bool ok = true;
    int j = 0;
    for (int kt = next_kv_tile(p.tiles, n_tiles, qkind, 0); kt < n_tiles;
         kt = next_kv_tile(p.tiles, n_tiles, qkind, kt + 1), ++j) {
      const int sb = j & 1;
      if (!mbar_wait(&s.s_full[sb], (j >> 1) & 1, abort)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float sv[kTile];
#pragma unroll
      for (int c = 0; c < kTile / 32; ++c) {
        uint32_t u[32];
        tmem_ld32(t_s + lane_base + sb * kTile + c * 32, u);
#pragma unroll
        for (int i = 0; i < 32; ++i) sv[c * 32 + i] = __uint_as_float(u[i]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.s_free[sb]);

      const TileInfo ti = p.tiles[kt];
      const bool masked = !(tile_kind(ti) == qkind && qkind != 2) || ti.rows < kTile;
      if (masked) {
#pragma unroll
        for (int c = 0; c < kTile; ++c) {
          const uint32_t pad = (ti.padbits[c >> 5] >> (c & 31)) & 1u;
          if (c >= ti.rows || pad != my_pad) sv[c] = -CUDART_INF_F;
        }
      }
      float mx = -CUDART_INF_F;
#pragma unroll
      for (int c = 0; c < kTile; ++c) mx = fmaxf(mx, sv[c]);
      mx *= scale_log2;
      const float m_new = fmaxf(m_run, mx);
      const bool grow = m_new > m_run + kRescaleThreshold || (m_run == -CUDART_INF_F && m_new != -CUDART_INF_F);
      const float m_use = grow ? m_new : m_run;
      const float m_sub = m_use == -CUDART_INF_F ? 0.f : m_use;
      const float alpha = grow ? ex2_approx(m_run - m_use) : 1.f;
      float rs = 0.f;
#pragma unroll
      for (int c = 0; c < kTile; ++c) {
        sv[c] = ex2_approx(fmaf(sv[c], scale_log2, -m_sub));
        rs += sv[c];
      }
      // P_{j-1} V_{j-1} must be complete: the P buffer is reused and O may be rescaled
      if (j > 0 && !mbar_wait(s.o_ready, (j - 1) & 1, abort)) {
        ok = false;
        break;
      }
      if (j > 0 && __any_sync(0xffffffffu, grow)) {
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t u[32];
          tmem_ld32(t_o + lane_base + c * 32, u);
#pragma unroll
          for (int i = 0; i < 32; ++i) u[i] = __float_as_uint(__uint_as_float(u[i]) * alpha);
          tmem_st32(t_o + lane_base + c * 32, u);
        }
        tmem_wait_st();
      }
      l_run = l_run * alpha + rs;
      m_run = m_use;
      // P row -> shared memory, 128-byte swizzle, two 64-column regions
#pragma unroll
      for (int c = 0; c < kTile / 8; ++c) {
        uint4 w;
        w.x = pack_bf16x2(sv[8 * c + 0], sv[8 * c + 1]);
        w.y = pack_bf16x2(sv[8 * c + 2], sv[8 * c + 3]);
        w.z = pack_bf16x2(sv[8 * c + 4], sv[8 * c + 5]);
        w.w = pack_bf16x2(sv[8 * c + 6], sv[8 * c + 7]);
        const int region = c >> 3, cc = c & 7;
        *reinterpret_cast<uint4*>(prow + region * SM::kRegion + ((cc ^ (r & 7)) << 4)) = w;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s.p_full);
    }
    if (!ok) {
      if (lane == 0) fail(p.err, abort);
    } else if (mbar_wait(s.o_final, 0, abort)) {
      tc_fence_after();
      const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
      __nv_bfloat16* dst = p.o + row * (int64_t)HD + head * D;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t u[32];
        tmem_ld32(t_o + lane_base + c * 32, u);
        if (row_ok) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(u[8 * i + 0]) * inv_l, __uint_as_float(u[8 * i + 1]) * inv_l);
            w.y = pack_bf16x2(__uint_as_float(u[8 * i + 2]) * inv_l, __uint_as_float(u[8 * i + 3]) * inv_l);
            w.z = pack_bf16x2(__uint_as_float(u[8 * i + 4]) * inv_l, __uint_as_float(u[8 * i + 5]) * inv_l);
            w.w = pack_bf16x2(__uint_as_float(u[8 * i + 6]) * inv_l, __uint_as_float(u[8 * i + 7]) * inv_l);
            d4[i] = w;
          }
        }
      }
    } else if (lane == 0) {
      fail(p.err, abort);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

template <int D>
cudaError_t launch_d(const AttnArgs& a, const CUtensorMap& tm, cudaStream_t s) {
  auto k = attn_kernel<D>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)AttnSmem<D>::kBytes);
  if (e != cudaSuccess) return e;
  const dim3 grid((unsigned)((a.n + kTile - 1) / kTile), (unsigned)a.heads);
  k<<<grid, kThreads, AttnSmem<D>::kBytes, s>>>(tm, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention(const AttnArgs& a, PFN_cuTensorMapEncodeTiled_v12000 encode, cudaStream_t s) {
  if (a.n <= 0) return cudaSuccess;
  if (a.head_dim != 64 && a.head_dim != 128) return cudaErrorInvalidValue;
  const uint64_t cols = 3ull * a.heads * a.head_dim;
  CUtensorMap tm;
  cuuint64_t dims[2] = {cols, (cuuint64_t)a.n};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t estr[2] = {1, 1};
  if (encode(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<__nv_bfloat16*>(a.qkv), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  return a.head_dim == 128 ? launch_d<128>(a, tm, s) : launch_d<64>(a, tm, s);
}

}  // namespace h3
