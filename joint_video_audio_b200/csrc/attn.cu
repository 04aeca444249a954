// Document-masked flash attention on tcgen05 / TMEM (K3).
//
// Source: "MiniMaxH3Transformer3DModel" (diffusers API page), introduction:
// full self-attention over the packed sequence; padding rows (tag -1) are kept
// in their own attention document by a boolean mask. The attention scale is
// 1/sqrt(head_dim).
//
// One CTA per (pair of 128-query tiles, head). The two query tiles ping-pong:
// while the softmax warps of one tile work, the tensor core runs the other
// tile's products, so the exponentials overlap the MMAs.
//
//   warp 0      TMA: both Q tiles once, then K_0, V_0, K_1, V_1, ... through a
//               ring of shared-memory slots
//   warp 1      TMEM allocator + single-thread MMA issuer, in the order
//                 S0_0 S1_0 | PV0_0 S0_1 PV1_0 S1_1 | PV0_1 S0_2 PV1_1 S1_2 | ...
//               with Sq_j = Qq K_j^T (M=128, N=128, K=head_dim; both operands in
//               shared memory) and PVq_j: Oq += Pq_j V_j (M=128, N=head_dim,
//               K=128; P in tensor memory, V in shared memory read MN-major)
//   warps 2..5  softmax of query tile 0, warps 6..9 of query tile 1; one
//               thread per query row: S row from TMEM, mask, online max / sum
//               in the exp2 domain, P packed to bf16 pairs and stored back
//               into the first 64 columns of its own S in TMEM (each half of
//               P announced on its own barrier, so P V starts on keys 0..63
//               while keys 64..127 are exponentiated), and the rescale of O
//               in TMEM when the running max grows by more than 2^8
//               (otherwise the stale max is kept, so P stays below 256).
// The P V product reads P straight from tensor memory (A operand in TMEM, V
// from shared memory), so P never touches shared memory: the shared-memory
// port only feeds Q, K and V, and a five-slot K/V ring fits next to the two
// query tiles. Ordering needs no extra barriers: the tensor core runs one
// CTA's MMAs in issue order, so S_t of tile j completing implies P_t V of
// tile j-1 completed (O_t is stable and P_t's columns are free), and S_t of
// tile j+1 is issued only after P_t V of tile j.
// Tensor memory: S0/P0 | S1/P1 | O0 | O1 (128 columns each).
// KV tiles whose rows all lie in the other document are skipped when neither
// query tile needs them; tiles that mix documents, run past the end of the
// sequence, or belong to the other document of one of the two query tiles are
// masked per element. In block-sparse mode the CTA visits only the tiles of its
// list (chosen in sparse.cu), with the same per-element masks.
#include <cuda_bf16.h>
#include <cudaTypedefs.h>
#include <math_constants.h>

#include "kernels.cuh"
#include "ptx.cuh"

namespace h3 {
namespace {

// 64 consecutive 32-bit columns of the warp's 32 lanes, without the wait:
// the registers are valid only after tcgen05.wait::ld.
__device__ __forceinline__ void tmem_ld64_nowait(uint32_t taddr, uint32_t (&r)[64]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,"
      "%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
      "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]),
        "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]),
        "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]),
        "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]),
        "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

constexpr int kTile = 128;
constexpr int kSoftmaxWarps = 8;
constexpr int kThreads = 32 * (2 + kSoftmaxWarps);
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;

template <int D>
struct AttnSmem {
  static constexpr int kSlots = D == 128 ? 5 : 10;
  static constexpr int kQBytes = kTile * D * 2;     // one query tile
  static constexpr int kKVBytes = kTile * D * 2;    // one K or V tile
  static constexpr int kRegion = kTile * 128;       // 128 rows x 128 bytes (one swizzle region)
  static constexpr size_t kBytes = 1024 + 2 * (size_t)kQBytes + kSlots * (size_t)kKVBytes + 512;
  uint8_t *q0, *slot0;  // query tile t at q0 + t * kQBytes, ring slot i at slot0 + i * kKVBytes
  uint64_t *q_full, *ring_full, *ring_empty, *s_full, *p_lo, *p_hi, *o_final;
  uint32_t* tmem_base;
  int* abort;

  __device__ explicit AttnSmem(uint8_t* raw) {
    const uint32_t base = smem_u32(raw);
    uint8_t* x = raw + (((base + 1023u) & ~1023u) - base);
    q0 = x;
    x += 2 * kQBytes;
    slot0 = x;
    x += kSlots * kKVBytes;
    uint64_t* b = reinterpret_cast<uint64_t*>(x);
    q_full = b;
    ring_full = b + 1;
    ring_empty = b + 1 + kSlots;
    s_full = b + 1 + 2 * kSlots;
    p_lo = s_full + 2;
    p_hi = s_full + 4;
    o_final = s_full + 6;
    tmem_base = reinterpret_cast<uint32_t*>(s_full + 7);
    abort = reinterpret_cast<int*>(s_full + 8);
  }
};

// 0: no padding rows, 1: only padding rows, 2: both
__device__ __forceinline__ int tile_kind(const TileInfo& t) {
  return t.npad == 0 ? 0 : (t.npad == t.rows ? 1 : 2);
}

__device__ __forceinline__ bool skips(int qkind, int kkind) {
  return (qkind == 0 && kkind == 1) || (qkind == 1 && kkind == 0);
}

// Next KV tile at or after kt that at least one of the two query tiles needs.
__device__ __forceinline__ int next_kv_tile(const TileInfo* tiles, int n_tiles, int qk0, int qk1, int kt) {
  for (; kt < n_tiles; ++kt) {
    const int kk = tile_kind(tiles[kt]);
    if (!(skips(qk0, kk) && skips(qk1, kk))) return kt;
  }
  return n_tiles;
}

__device__ __forceinline__ int count_kv_tiles(const TileInfo* tiles, int n_tiles, int qk0, int qk1) {
  int n = 0;
  for (int kt = next_kv_tile(tiles, n_tiles, qk0, qk1, 0); kt < n_tiles;
       kt = next_kv_tile(tiles, n_tiles, qk0, qk1, kt + 1))
    ++n;
  return n;
}

// The KV tiles one CTA visits, in order: every tile one of its two query
// tiles needs (dense), or the tiles its block keeps (block-sparse list).
struct KvSeq {
  const TileInfo* tiles;
  int n_tiles, qk0, qk1;
  const int32_t* list;  // [count, tile, tile, ...] or nullptr
  __device__ int count() const { return list ? list[0] : count_kv_tiles(tiles, n_tiles, qk0, qk1); }
  // the tile of step j, given the tile of step j - 1 (-1 before the first)
  __device__ int at(int j, int prev) const {
    if (list) return j < list[0] ? list[1 + j] : n_tiles;
    return next_kv_tile(tiles, n_tiles, qk0, qk1, prev + 1);
  }
};

// Non-blocking look at a barrier phase: true if the phase of parity
// `parity` has completed. Several can be in flight at once, so the issuer
// pays one barrier latency for a batch of checks instead of one per check.
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ void fail(int* err, volatile int* abort) {
  if (err) atomicOr(err, kErrTimeoutAttn);
  *abort = 1;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1) attn_kernel(const __grid_constant__ CUtensorMap tm, const AttnArgs p) {
  extern __shared__ uint8_t smem_raw[];
  using SM = AttnSmem<D>;
  SM s(smem_raw);
  constexpr int kSlots = SM::kSlots;
  constexpr int kRegions = D / 64;  // 64-column swizzle regions of a Q/K/V tile
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pair = blockIdx.x, head = blockIdx.y;
  const int n_tiles = (int)((p.n + kTile - 1) / kTile);
  const int qt0 = 2 * pair;
  const int HD = p.heads * D;
  // a missing second tile (odd tile count) behaves like an all-valid tile
  const int qk0 = tile_kind(p.tiles[qt0]);
  const int qk1 = qt0 + 1 < n_tiles ? tile_kind(p.tiles[qt0 + 1]) : 0;
  volatile int* abort = s.abort;

  if (threadIdx.x == 0) {
    mbar_init(s.q_full, 1);
    for (int i = 0; i < kSlots; ++i) {
      mbar_init(&s.ring_full[i], 1);
      mbar_init(&s.ring_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.s_full[i], 1);
      mbar_init(&s.p_lo[i], 4);
      mbar_init(&s.p_hi[i], 4);
    }
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
  const KvSeq seq{p.tiles, n_tiles, qk0, qk1,
                  p.kv_list ? p.kv_list + ((int64_t)pair * p.heads + head) * p.kv_list_stride : nullptr};
  const int n_kv = seq.count();

  if (warp == 0) {
    // ------------------------------------------------------------ loads
    if (lane == 0) {
      tma_prefetch_desc(&tm);
      // a second query tile past the end of the sequence is not loaded: its
      // rows are never stored
      const int nq = qt0 + 1 < n_tiles ? 2 : 1;
      mbar_expect_tx(s.q_full, nq * SM::kQBytes);
      for (int t = 0; t < nq; ++t)
        for (int r = 0; r < kRegions; ++r)
          tma_load_2d(s.q0 + t * SM::kQBytes + r * SM::kRegion, &tm, s.q_full, head * D + r * 64, (qt0 + t) * kTile);
      int u = 0;
      for (int jj = 0, kt = seq.at(0, -1); kt < n_tiles; ++jj, kt = seq.at(jj, kt)) {
        bool ok = true;
        for (int kv = 0; kv < 2; ++kv, ++u) {  // K_j then V_j
          const int sl = u % kSlots;
          if (!mbar_wait_relaxed(&s.ring_empty[sl], ((u / kSlots) & 1) ^ 1, abort)) {
            fail(p.err, abort);
            ok = false;
            break;
          }
          mbar_expect_tx(&s.ring_full[sl], SM::kKVBytes);
          const int col = (kv == 0 ? HD : 2 * HD) + head * D;
          for (int r = 0; r < kRegions; ++r)
            tma_load_2d(s.slot0 + sl * SM::kKVBytes + r * SM::kRegion, &tm, &s.ring_full[sl], col + r * 64, kt * kTile);
        }
        if (!ok) break;
      }
      // drain: the last loads must land before the CTA may exit
      for (int i = 0; i < kSlots && u - 1 - i >= 0; ++i) {
        const int uu = u - 1 - i;
        mbar_wait(&s.ring_full[uu % kSlots], (uu / kSlots) & 1, nullptr);
      }
      mbar_wait(s.q_full, 0, nullptr);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA
    if (lane == 0) {
      constexpr uint32_t idesc_qk = make_idesc(1, 1, kTile, kTile, false);
      constexpr uint32_t idesc_pv = make_idesc(1, 1, kTile, D, true);
      const uint32_t q0 = smem_u32(s.q0), ring0 = smem_u32(s.slot0);
      // ring position of load u = 2 j (K_j) or 2 j + 1 (V_j): slot u % kSlots,
      // phase (u / kSlots) & 1, tracked incrementally (no division per step)
      struct RingPos {
        int slot;
        uint32_t phase;
        __device__ void advance(int by) {
          slot += by;
          while (slot >= kSlots) {
            slot -= kSlots;
            phase ^= 1u;
          }
        }
      };
      auto wait_ring = [&](const RingPos& r) { return mbar_wait(&s.ring_full[r.slot], r.phase, abort); };
      // S_t = Q_t K_j^T into TMEM columns [t*128, t*128+128)
      // Shared-memory descriptors: the start-address field (bits 0..13, in
      // 16-byte units) never carries out of its 14 bits inside shared memory,
      // so a K step's descriptor is the tile's base descriptor plus a constant.
      const uint64_t qdesc0 = sw128_desc(q0, 16);
      const uint64_t ring_desc0 = sw128_desc(ring0, 16);
      const uint64_t vdesc0 = sw128_desc(ring0, SM::kRegion);
      auto issue_s = [&](int t, int kslot) -> bool {
        tc_fence_after();
        const uint64_t qd = qdesc0 + (uint64_t)((t * SM::kQBytes) >> 4);
        const uint64_t kd = ring_desc0 + (uint64_t)((kslot * SM::kKVBytes) >> 4);
        const uint32_t dtm = tmem + t * kTile;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = (uint64_t)(((kk >> 2) * SM::kRegion + (kk & 3) * 32) >> 4);
          mma_bf16_ss(dtm, qd + off, kd + off, idesc_qk, kk > 0 ? 1u : 0u);
        }
        mma_commit(&s.s_full[t]);
        return true;
      };
      // O_t += P_t V_j into TMEM columns [256 + t*128, ...); P_t is read from
      // TMEM columns [t*128, t*128 + 64), 8 columns per K = 16 step
      // Each half of P (keys 0..63, 64..127) has its own ready barrier, so the
      // first four K steps run while the softmax still works on the second half.
      auto issue_pv = [&](int t, int j, int vslot, bool lo_seen) -> bool {
        const uint64_t vd = vdesc0 + (uint64_t)((vslot * SM::kKVBytes) >> 4);
        const uint32_t dtm = tmem + 256 + t * kTile, atm = tmem + t * kTile;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          if (!(half == 0 && lo_seen) && !mbar_wait(half == 0 ? &s.p_lo[t] : &s.p_hi[t], j & 1, abort)) return false;
          tc_fence_after();
#pragma unroll
          for (int kk = 4 * half; kk < 4 * half + 4; ++kk)
            mma_bf16_ts(dtm, atm + kk * 8, vd + (uint64_t)((kk * 16 * 128) >> 4), idesc_pv,
                        (j > 0 || kk > 0) ? 1u : 0u);
        }
        return true;
      };
      bool ok = mbar_wait(s.q_full, 0, abort);
      if (ok && n_kv > 0) {
        const RingPos k0{0, 0u};
        ok = wait_ring(k0) && issue_s(0, 0) && issue_s(1, 0);
        if (ok) mma_commit(&s.ring_empty[0]);
        RingPos vpos{1, 0u}, kpos{2 % kSlots, 2 >= kSlots ? 1u : 0u};  // V_j and K_{j+1}
        for (int j = 0; ok && j < n_kv; ++j) {
          // The tensor pipe queues only two or three products, so every
          // barrier latency this thread sits through while the queue is empty
          // is tensor idle time: the ring slots of V_j and K_{j+1} and the
          // first half of P_0 are looked at in one batch (the latencies
          // overlap), with a blocking wait only for what is not complete yet;
          // the look at P_1 is answered while S_0 issues.
          const bool more = j + 1 < n_kv;
          const bool tv = mbar_test(&s.ring_full[vpos.slot], vpos.phase);
          const bool tk = !more || mbar_test(&s.ring_full[kpos.slot], kpos.phase);
          const bool tp0 = mbar_test(&s.p_lo[0], j & 1);
          ok = (tv || wait_ring(vpos)) && (tk || wait_ring(kpos)) && issue_pv(0, j, vpos.slot, tp0);
          if (!ok) break;
          const bool tp1 = mbar_test(&s.p_lo[1], j & 1);  // answered while S0 issues
          if (more) ok = issue_s(0, kpos.slot);
          if (!ok) break;
          ok = issue_pv(1, j, vpos.slot, tp1);
          if (!ok) break;
          mma_commit(&s.ring_empty[vpos.slot]);
          if (more) {
            ok = issue_s(1, kpos.slot);
            if (!ok) break;
            mma_commit(&s.ring_empty[kpos.slot]);
          }
          vpos.advance(2);
          kpos.advance(2);
        }
      }
      if (!ok) fail(p.err, abort);
      mma_commit(s.o_final);
      mbar_wait(s.o_final, 0, nullptr);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int t = (warp - 2) >> 2;  // query tile of this warpgroup
    const int quad = warp & 3;
    const int r = quad * 32 + lane;  // row within the tile = TMEM lane
    const int qt = qt0 + t;
    const int64_t row = (int64_t)qt * kTile + r;
    const bool row_ok = row < p.n;
    const uint32_t my_pad = (row_ok && p.tag[row] == -1) ? 1u : 0u;
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    const uint32_t t_s = tmem + lane_base + t * kTile;
    const uint32_t t_o = tmem + lane_base + 256 + t * kTile;
    const float scale_log2 = 1.4426950408889634f * rsqrtf((float)D);
    const int myk = t == 0 ? qk0 : qk1;
    float m_run = -CUDART_INF_F, l_run = 0.f;
    bool ok = true;
    int j = 0;
    int kt = seq.at(0, -1);
    for (; kt < n_tiles; ++j) {
      // the tile summary is fetched before waiting for S, so its global-memory
      // latency hides behind the wait
      const int4 tiw0 = __ldg(reinterpret_cast<const int4*>(p.tiles + kt));
      const int2 tiw1 = __ldg(reinterpret_cast<const int2*>(p.tiles + kt) + 2);
      const int kt_next = seq.at(j + 1, kt);
      if (!mbar_wait(&s.s_full[t], j & 1, abort)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // S is read from tensor memory in 64-column halves, twice (once for the
      // row max, once for the exponentials), so only 64 S values are live in
      // registers at a time.
      TileInfo ti;
      ti.rows = tiw0.x;
      ti.npad = tiw0.y;
      ti.padbits[0] = (uint32_t)tiw0.z;
      ti.padbits[1] = (uint32_t)tiw0.w;
      ti.padbits[2] = (uint32_t)tiw1.x;
      ti.padbits[3] = (uint32_t)tiw1.y;
      const int kk_kind = tile_kind(ti);
      const bool need_mask = !(kk_kind == myk && myk != 2) || ti.rows < kTile;
      auto mask_half = [&](float* sv, int h) {
        if (!need_mask) return;
#pragma unroll
        for (int ww = 0; ww < 2; ++ww) {
          const int w = 2 * h + ww;
          const uint32_t bits = ti.padbits[w] ^ (my_pad ? 0xffffffffu : 0u);  // 1 = other document
#pragma unroll
          for (int c = 0; c < 32; ++c)
            if (((bits >> c) & 1u) || w * 32 + c >= ti.rows) sv[ww * 32 + c] = -CUDART_INF_F;
        }
      };
      // S in two 64-column halves: the second half's load is in flight while
      // the first half's max is taken; both stay in registers for the
      // exponentials (one read of S per tile)
      uint32_t u0[64], u1[64];
      tmem_ld64_nowait(t_s, u0);
      tmem_wait_ld();
      tmem_ld64_nowait(t_s + 64, u1);
      float mc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mc[i] = -CUDART_INF_F;
      {
        float* sv = reinterpret_cast<float*>(u0);
        mask_half(sv, 0);
#pragma unroll
        for (int c = 0; c < 64; c += 16)
#pragma unroll
          for (int i = 0; i < 8; ++i) mc[i] = max3f(mc[i], sv[c + 2 * i], sv[c + 2 * i + 1]);
      }
      tmem_wait_ld();
      {
        float* sv = reinterpret_cast<float*>(u1);
        mask_half(sv, 1);
#pragma unroll
        for (int c = 0; c < 64; c += 16)
#pragma unroll
          for (int i = 0; i < 8; ++i) mc[i] = max3f(mc[i], sv[c + 2 * i], sv[c + 2 * i + 1]);
      }
      const float m8 = fmaxf(max3f(mc[0], mc[1], mc[2]), max3f(mc[3], mc[4], max3f(mc[5], mc[6], mc[7])));
      const float m_new = fmaxf(m_run, m8 * scale_log2);
      const bool grow = m_new > m_run + kRescaleThreshold || (m_run == -CUDART_INF_F && m_new != -CUDART_INF_F);
      const float m_use = grow ? m_new : m_run;
      const float m_sub = m_use == -CUDART_INF_F ? 0.f : m_use;
      const float alpha = grow ? ex2_approx(m_run - m_use) : 1.f;
      // exponentials on pairs: x = s * scale - m with one packed FMA, then
      // the MUFU's 2^x (measured: the exponentials are not on this kernel's
      // critical path, so none are moved to the FMA pipe). Each half of P
      // (keys 0..63, then 64..127) is packed to bf16 pairs, stored over the
      // first 64 columns of this tile's S and announced on its own barrier, so
      // the P V product starts on the first half while the second is
      // computed. The row sum runs in two packed accumulators.
      const uint64_t sc2 = f2_pack(scale_log2, scale_log2), nm2 = f2_pack(-m_sub, -m_sub);
      uint64_t acc0 = f2_pack(0.f, 0.f), acc1 = acc0;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t* u = h == 0 ? u0 : u1;
        float* sv = reinterpret_cast<float*>(u);
#pragma unroll
        for (int c = 0; c < 64; c += 2) {
          const int cg = 64 * h + c;  // column within the tile
          float x0, x1;
          f2_unpack(f2_fma(f2_pack(sv[c], sv[c + 1]), sc2, nm2), x0, x1);
          const uint64_t e = f2_pack(ex2_approx(x0), ex2_approx(x1));
          if ((cg >> 1) & 1)
            acc1 = f2_add(acc1, e);
          else
            acc0 = f2_add(acc0, e);
          float e0, e1;
          f2_unpack(e, e0, e1);
          u[c >> 1] = pack_bf16x2(e0, e1);
        }
        tmem_st32(t_s + 32 * h, *reinterpret_cast<const uint32_t(*)[32]>(u));
        if (h == 0 && j > 0 && __any_sync(0xffffffffu, grow)) {
          // O must be rescaled before the first P V step of this tile adds to
          // it; S_t of this tile completing implied the previous P V completed
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(t_o + c * 32, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(t_o + c * 32, o);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(h == 0 ? &s.p_lo[t] : &s.p_hi[t]);
      }
      float rs0, rs1;
      f2_unpack(f2_add(acc0, acc1), rs0, rs1);
      l_run = l_run * alpha + (rs0 + rs1);
      m_run = m_use;
      kt = kt_next;
    }
    if (!ok) {
      if (lane == 0) fail(p.err, abort);
    } else if (mbar_wait(s.o_final, 0, abort)) {
      tc_fence_after();
      const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
      __nv_bfloat16* dst;
      if (p.route_ranks > 0) {
        // sequence parallelism: the row's owner gathers every head group's output
        const int64_t d = row / p.route_rows;
        dst = p.route_dst[row_ok ? d : 0] + (row - d * p.route_rows) * p.route_ld + (int64_t)(p.route_head0 + head) * D;
      } else {
        dst = p.o + row * (int64_t)HD + head * D;
      }
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(t_o + c * 32, o);
        if (row_ok) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(o[8 * i + 0]) * inv_l, __uint_as_float(o[8 * i + 1]) * inv_l);
            w.y = pack_bf16x2(__uint_as_float(o[8 * i + 2]) * inv_l, __uint_as_float(o[8 * i + 3]) * inv_l);
            w.z = pack_bf16x2(__uint_as_float(o[8 * i + 4]) * inv_l, __uint_as_float(o[8 * i + 5]) * inv_l);
            w.w = pack_bf16x2(__uint_as_float(o[8 * i + 6]) * inv_l, __uint_as_float(o[8 * i + 7]) * inv_l);
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
  const int n_tiles = (int)((a.n + kTile - 1) / kTile);
  const dim3 grid((unsigned)((n_tiles + 1) / 2), (unsigned)a.heads);
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
