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
// One CTA per row; thread t owns the 64 consecutive channels [64 t, 64 t + 64),
// the lower (t even) or upper (t odd) half of Hadamard block t / 2, all in
// registers. The 128-point transform is six butterfly stages inside the
// thread (channel bits 0..5) and one across the lane pair (bit 6), so each
// value crosses lanes once. The 1/sqrt(128) normalisation is folded into the
// quantisation scale. Arithmetic is on fp32 pairs (sm_100 f32x2 ops) wherever
// the two lanes of a pair do the same thing.

__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {  // a - b
  return f2_fma(b, f2_pack(-1.f, -1.f), a);
}

// Sum (IS_MAX = false) or max of non-negative values (IS_MAX = true) over the
// CTA; `red` holds one slot per warp. Every call is a barrier of the CTA.
template <int WARPS, bool IS_MAX>
__device__ __forceinline__ float cta_reduce(float v, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (IS_MAX) {
    // non-negative floats order like their bit patterns
    v = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(v)));
  } else {
#pragma unroll
    for (int m = 16; m; m >>= 1) v += __shfl_xor_sync(0xffffffffu, v, m);
  }
  if (WARPS == 1) {
    __syncwarp();  // callers rely on the reduction being a barrier
    return v;
  }
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float r = red[0];
#pragma unroll
  for (int w = 1; w < WARPS; ++w) r = IS_MAX ? fmaxf(r, red[w]) : r + red[w];
  return r;
}

// int8 codes of 8 values: q = round-half-even(v * inv), taken from the low
// byte of v * inv + 1.5 * 2^23 computed in one FMA (|v * inv| <= 127, so the
// sum stays in the binade where the float spacing is 1 and its low mantissa
// byte is q in two's complement).
__device__ __forceinline__ uint2 quant8(const float* v, uint64_t inv2) {
  const uint64_t magic = f2_pack(12582912.f, 12582912.f);
  uint32_t b[8];
#pragma unroll
  for (int e = 0; e < 8; e += 2) {
    const uint64_t r = f2_fma(f2_pack(v[e], v[e + 1]), inv2, magic);
    asm("mov.b64 {%0, %1}, %2;" : "=r"(b[e]), "=r"(b[e + 1]) : "l"(r));
  }
  const uint32_t lo = __byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040), 0x5410);
  const uint32_t hi = __byte_perm(__byte_perm(b[4], b[5], 0x0040), __byte_perm(b[6], b[7], 0x0040), 0x5410);
  return make_uint2(lo, hi);
}

// Rotation + int8 row passes of the W8A8 path, one kernel (rowring_kernel):
//   kRowQuant      K4: block-128 Hadamard rotation + per-row int8 of a bf16
//                  matrix (attention and SwiGLU outputs, weights)
//   kRowNormQuant  K1 fused with K4 (W8A8 pre-norms): AdaLN RMSNorm of x,
//                  then the rotation and int8 quantisation
// Each persistent CTA takes a contiguous slice of the rows (visited grouped
// by modulation key, sorted in shared memory, so the shift / scale vectors it
// reads stay in L1). Rows arrive by bulk copies (TMA engine) into a
// shared-memory ring issued several rows ahead and leave, as int8 codes, by
// bulk stores from a double-buffered slot, so the load/store path carries
// only the threads' conflict-free shared-memory accesses. Thread t of a row
// owns channels [32 t, 32 t + 32); the 128-point transform is three
// butterfly stages inside each 8-channel slot, two across the thread's
// slots and two across the four lanes of a block (fwht128_slots), its
// 1/sqrt(128) folded into the quantisation scale. Arithmetic is on fp32
// pairs (sm_100 f32x2 ops) wherever the two lanes of a pair do the same
// thing.
enum RowMode : int { kRowQuant = 0, kRowNormQuant = 1 };
constexpr int kRowChans = 32;              // channels per thread
constexpr int kRowRingBudget = 32 * 1024;  // shared-memory bytes of one CTA's input ring
constexpr int kRowMaxStages = 8;
constexpr int kRowSortChunk = 512;         // rows sorted by key at a time

__device__ __forceinline__ void bulk_store(void* gdst, const void* ssrc, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(reinterpret_cast<uint64_t>(gdst)),
               "r"(smem_u32(ssrc)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// every committed bulk store but the newest N has finished reading shared memory
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
// every committed bulk store has completed
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void bulk_load_row(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// ---- row ring: shared-memory layout of a thread's channels
// Thread t owns channels [32 t, 32 t + 32) as four 8-channel chunks. Its
// register slot j holds chunk j ^ r, r = ((t >> 1) ^ (t >> 3)) & 3: the
// 16-byte shared-memory accesses of a warp to a bf16 row (slot j at byte
// 64 t + 16 (j ^ r)) fall on distinct bank groups within every 8-thread
// phase, and so do the 8-byte stores of int8 codes (slot j at byte
// 32 t + 8 (j ^ r)) within every 16-thread phase. Lanes t and t ^ 1 share r;
// lane t ^ 2 has r ^ 1.
__device__ __forceinline__ int slot_perm(int t) { return ((t >> 1) ^ (t >> 3)) & 3; }

// Unnormalised 128-point Walsh-Hadamard transform of a block held by four
// consecutive lanes in permuted slots (see slot_perm): channel bits 0..2 in a
// slot, bits 3..4 across slots (the butterfly's lower element is the one whose
// chunk bit is clear, so the thread's permutation sets a sign), bits 5..6
// across lanes (lane bit 1 pairs slot j with the partner's slot j ^ 1).
__device__ __forceinline__ void fwht128_slots(float (&h)[32], int lane) {
  const int r = slot_perm(lane);
  // bits 0..2: inside each 8-channel slot
#pragma unroll
  for (int e = 0; e < 32; e += 2) {
    const float u = h[e], w = h[e + 1];
    h[e] = u + w;
    h[e + 1] = u - w;
  }
#pragma unroll
  for (int b = 2; b < 8; b <<= 1) {
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
      if (!(e & b)) {
        const uint64_t u = f2_pack(h[e], h[e + 1]), w = f2_pack(h[e + b], h[e + b + 1]);
        f2_unpack(f2_add(u, w), h[e], h[e + 1]);
        f2_unpack(f2_sub(u, w), h[e + b], h[e + b + 1]);
      }
    }
  }
  // bits 3, 4: slot j against slot j ^ s (s = 1, 2); the slot holding the
  // chunk with the bit clear takes a + b, the other a - b
#pragma unroll
  for (int sb = 1; sb <= 2; sb <<= 1) {
    const float sg = (r & sb) ? -1.f : 1.f;
    const uint64_t sg2 = f2_pack(sg, sg), nsg2 = f2_pack(-sg, -sg);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (j & sb) continue;
#pragma unroll
      for (int e = 0; e < 8; e += 2) {
        const int x = 8 * j + e, y = 8 * (j ^ sb) + e;
        const uint64_t a = f2_pack(h[x], h[x + 1]), bb = f2_pack(h[y], h[y + 1]);
        f2_unpack(f2_fma(sg2, a, bb), h[x], h[x + 1]);    // sg a + b
        f2_unpack(f2_fma(nsg2, bb, a), h[y], h[y + 1]);   // a - sg b
      }
    }
  }
  // bits 5, 6: across lanes; the lower partner takes h + other, the upper
  // other - h
  {
    const float sg = (lane & 1) ? -1.f : 1.f;
    const uint64_t sg2 = f2_pack(sg, sg);
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
      const float o0 = __shfl_xor_sync(0xffffffffu, h[e], 1);
      const float o1 = __shfl_xor_sync(0xffffffffu, h[e + 1], 1);
      f2_unpack(f2_fma(sg2, f2_pack(h[e], h[e + 1]), f2_pack(o0, o1)), h[e], h[e + 1]);
    }
  }
  {
    const float sg = (lane & 2) ? -1.f : 1.f;
    const uint64_t sg2 = f2_pack(sg, sg);
    float o[32];
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int e = 0; e < 8; ++e) o[8 * j + e] = __shfl_xor_sync(0xffffffffu, h[8 * (j ^ 1) + e], 2);
#pragma unroll
    for (int e = 0; e < 32; e += 2)
      f2_unpack(f2_fma(sg2, f2_pack(h[e], h[e + 1]), f2_pack(o[e], o[e + 1])), h[e], h[e + 1]);
  }
}

// Modulation vectors rearranged for rowring_kernel: float4 (((key * 4 + v) * 8
// + 2 j + hf) * nact + t) holds channels 32 t + 8 (j ^ r(t)) + 4 hf .. + 3 of
// vector v (0 shift1, 1: 1 + scale1, 2 shift2, 3: 1 + scale2) of table row
// key = tag * n_t + tidx, so a warp's reads of one slot are contiguous.
__global__ void modt_kernel(const float* __restrict__ table, int n_keys, int K, float4* __restrict__ modt) {
  const int nact = K / kRowChans;
  const int64_t total = (int64_t)n_keys * 4 * 8 * nact;
  const int vidx[4] = {0, 1, 3, 4};
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const int t = (int)(i % nact);
    const int sj = (int)((i / nact) % 8);
    const int v = (int)((i / ((int64_t)nact * 8)) % 4);
    const int64_t key = i / ((int64_t)nact * 32);
    const int ch = kRowChans * t + 8 * ((sj >> 1) ^ slot_perm(t)) + 4 * (sj & 1);
    float4 x = *reinterpret_cast<const float4*>(table + (key * 6 + vidx[v]) * K + ch);
    if (v & 1) x = make_float4(1.f + x.x, 1.f + x.y, 1.f + x.z, 1.f + x.w);
    modt[i] = x;
  }
}

// MODE: kRowQuant (K4) or kRowNormQuant (K1 + K4).
template <int WARPS, int MODE>
__global__ void __launch_bounds__(WARPS * 32) rowring_kernel(const __nv_bfloat16* __restrict__ in, int64_t rows,
                                                             int K, int stages, int8_t* __restrict__ out_q,
                                                             float* __restrict__ out_scale,
                                                             ModNormArgs a,
                                                             int* err) {
  constexpr bool NORM = MODE != kRowQuant;
  extern __shared__ __align__(128) uint8_t rsm[];
  __shared__ uint64_t full[kRowMaxStages];
  __shared__ float red[4][WARPS];
  __shared__ int fail[2];
  __shared__ int32_t ord[kRowSortChunk];
  __shared__ int32_t keys[kRowSortChunk];
  const int lane = threadIdx.x & 31;
  const int nact = K / kRowChans;
  const bool act = threadIdx.x < nact;
  const int c0 = kRowChans * threadIdx.x;
  const int r = slot_perm(threadIdx.x);
  const uint32_t row_bytes = (uint32_t)K * 2u, out_bytes = (uint32_t)K;  // bf16 in, int8 out
  uint8_t* ring = rsm;
  uint8_t* outb = rsm + (size_t)stages * row_bytes;  // two output slots
  // this CTA's slice of the rows, taken in chunks of up to kRowSortChunk rows
  const int64_t per = (rows + gridDim.x - 1) / gridDim.x;
  const int64_t s0 = (int64_t)blockIdx.x * per;
  const int64_t s1 = s0 + per < rows ? s0 + per : rows;
  if (s0 >= s1) return;
  if (threadIdx.x == 0) {
    for (int i = 0; i < stages; ++i) mbar_init(&full[i], 1);
    fail[0] = fail[1] = 0;
    fence_mbar_init();
  }
  int64_t k = 0;  // rows visited so far: ring slot k % stages, output slot k & 1
  for (int64_t c = s0; c < s1; c += kRowSortChunk) {
    const int n = (int)(s1 - c < kRowSortChunk ? s1 - c : kRowSortChunk);
    __syncthreads();  // the previous chunk's order is no longer read
    if (NORM) {
      // visit the chunk's rows grouped by modulation key (rank = rows with a
      // smaller key, or the same key and a smaller index)
      for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const int tg = a.tag[c + i], ti = a.tidx[c + i];
        keys[i] = (tg >= 0 && tg < a.n_tags && ti >= 0 && ti < a.n_t) ? tg * a.n_t + ti : -1;
      }
      __syncthreads();
      for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const int ki = keys[i];
        int rank = 0;
        for (int j = 0; j < n; ++j) {
          const int kj = keys[j];
          rank += (kj < ki) || (kj == ki && j < i);
        }
        ord[rank] = i;
      }
    } else {
      for (int i = threadIdx.x; i < n; i += blockDim.x) ord[i] = i;
    }
    __syncthreads();
    const int64_t kbase = k;
    auto row_of = [&](int64_t kk) -> int64_t { return c + ord[kk - kbase]; };
    const int64_t kend = k + n;  // visit index one past this chunk
    auto issue = [&](int64_t kk) {
      if (kk >= kend) return;
      const int st = (int)(kk % stages);
      mbar_expect_tx(&full[st], row_bytes);
      bulk_load_row(ring + (size_t)st * row_bytes, in + row_of(kk) * (int64_t)K, row_bytes, &full[st]);
    };
    if (threadIdx.x == 0) {
      fence_proxy_async_smem();  // the slots' last generic reads come before these copies
      for (int64_t kk = k; kk < k + stages; ++kk) issue(kk);
    }
    for (; k < kend; ++k) {
      const int64_t row = row_of(k);
      const int st = (int)(k % stages);
      const bool ok = mbar_wait(&full[st], (uint32_t)((k / stages) & 1), nullptr);
      float h[kRowChans];
      if (ok && act) {
        const uint8_t* src = ring + (size_t)st * row_bytes + 2 * c0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint4 v = *reinterpret_cast<const uint4*>(src + 16 * (j ^ r));
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            h[8 * j + 2 * q] = __uint_as_float(w[q] << 16);
            h[8 * j + 2 * q + 1] = __uint_as_float(w[q] & 0xffff0000u);
          }
        }
      } else {
#pragma unroll
        for (int e = 0; e < kRowChans; ++e) h[e] = 0.f;
      }
      if (!ok) fail[k & 1] = 1;
      // the output slot of this row was last read by the bulk store of row k-2
      if (threadIdx.x == 0) bulk_wait_read<1>();
      float* rd = red[2 * (k & 1)];
      // after the first reduction (a barrier) every thread has read its ring
      // slot and set its failure flag: check it, then refill the slot
      auto after_first_barrier = [&]() -> bool {
        if (fail[k & 1]) {
          if (threadIdx.x == 0) {
            if (err) atomicOr(err, kErrTimeoutStream);
            // loads still in flight must land before the CTA's shared memory goes
            for (int64_t kk = k; kk < k + stages && kk < kend; ++kk)
              mbar_wait(&full[kk % stages], (uint32_t)((kk / stages) & 1), nullptr);
            bulk_wait_all();
          }
          return false;
        }
        if (threadIdx.x == 0) {
          fail[(k + 1) & 1] = 0;  // every thread passed the last row's check of that flag
          fence_proxy_async_smem();
          issue(k + stages);
        }
        return true;
      };
      if (NORM) {
        uint64_t ss2 = f2_pack(0.f, 0.f);
#pragma unroll
        for (int e = 0; e < kRowChans; e += 2) {
          const uint64_t x2 = f2_pack(h[e], h[e + 1]);
          ss2 = f2_fma(x2, x2, ss2);
        }
        float s0f, s1f;
        f2_unpack(ss2, s0f, s1f);
        const float ss = cta_reduce<WARPS, false>(s0f + s1f, rd);
        if (!after_first_barrier()) return;
        const float rstd = rsqrtf(ss / (float)K + a.eps);
        const uint64_t r2 = f2_pack(rstd, rstd);
        const int tg = a.tag[row], ti = a.tidx[row];
        if (act && tg >= 0 && tg < a.n_tags && ti >= 0 && ti < a.n_t) {
          // h * rstd * (1 + scale) + shift; the rows of a key are visited
          // together, so these reads hit L1
          const float4* sh4 = a.modt + ((int64_t)(tg * a.n_t + ti) * 4 + a.modt_v0) * 8 * nact + threadIdx.x;
          const float4* g4 = sh4 + 8 * nact;
#pragma unroll
          for (int sj = 0; sj < 8; ++sj) {
            const float4 sh = __ldg(sh4 + sj * nact), g = __ldg(g4 + sj * nact);
            const int e = 4 * sj;
            f2_unpack(f2_fma(f2_pack(h[e], h[e + 1]), f2_fma(r2, f2_pack(g.x, g.y), f2_pack(0.f, 0.f)),
                             f2_pack(sh.x, sh.y)), h[e], h[e + 1]);
            f2_unpack(f2_fma(f2_pack(h[e + 2], h[e + 3]), f2_fma(r2, f2_pack(g.z, g.w), f2_pack(0.f, 0.f)),
                             f2_pack(sh.z, sh.w)), h[e + 2], h[e + 3]);
          }
        } else {
          // padding rows (and indices outside the table) get no modulation
#pragma unroll
          for (int e = 0; e < kRowChans; e += 2)
            f2_unpack(f2_fma(f2_pack(h[e], h[e + 1]), r2, f2_pack(0.f, 0.f)), h[e], h[e + 1]);
        }
      }
      uint8_t* ob = outb + (size_t)(k & 1) * out_bytes;
      {
        fwht128_slots(h, lane);
        float mx[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int e = 0; e < kRowChans; e += 8)
#pragma unroll
          for (int q = 0; q < 4; ++q) mx[q] = max3f(mx[q], fabsf(h[e + 2 * q]), fabsf(h[e + 2 * q + 1]));
        const float amax = cta_reduce<WARPS, true>(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])), rd + WARPS);
        if (!NORM && !after_first_barrier()) return;
        // the transform above is unnormalised: the rotated values are h / sqrt(128)
        const float inv = amax > 0.f ? 127.f / amax : 0.f;
        if (threadIdx.x == 0) out_scale[row] = amax * (0.08838834764831845f / 127.f);
        if (act) {
          const uint64_t inv2 = f2_pack(inv, inv);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            *reinterpret_cast<uint2*>(ob + c0 + 8 * (j ^ r)) = quant8(h + 8 * j, inv2);
        }
      }
      // the row leaves by one bulk store once every thread's part is in place
      fence_proxy_async_smem();
      __syncthreads();
      if (threadIdx.x == 0) {
        bulk_store(out_q + row * (int64_t)K, ob, out_bytes);
        bulk_commit();
      }
    }
  }
  if (threadIdx.x == 0) bulk_wait_all();
}

template <typename Kern>
static cudaError_t persistent_grid(Kern kern, int threads, size_t smem, int64_t rows, int64_t* grid) {
  cudaError_t e;
  if (smem > 48 * 1024 &&
      (e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
    return e;
  int dev = 0, sms = 0, per_sm = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem)) != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  *grid = rows < (int64_t)sms * per_sm ? rows : (int64_t)sms * per_sm;
  return cudaSuccess;
}

template <int WARPS, int MODE>
static cudaError_t launch_rowring_t(const __nv_bfloat16* in, int64_t rows, int K, int8_t* q, float* sc,
                                    const ModNormArgs& a, int* err, cudaStream_t s) {
  const size_t row_bytes = (size_t)K * 2, out_bytes = (size_t)K;
  int stages = (int)(kRowRingBudget / row_bytes);
  stages = stages < 2 ? 2 : (stages > kRowMaxStages ? kRowMaxStages : stages);
  const size_t smem = (size_t)stages * row_bytes + 2 * out_bytes;
  int64_t grid = 0;
  cudaError_t e = persistent_grid(rowring_kernel<WARPS, MODE>, WARPS * 32, smem, rows, &grid);
  if (e != cudaSuccess) return e;
  rowring_kernel<WARPS, MODE><<<(unsigned)grid, WARPS * 32, smem, s>>>(in, rows, K, stages, q, sc, a, err);
  return cudaGetLastError();
}

// One thread per 32 channels, rounded up to whole warps (K <= 16384).
#define H3_ROW_WARPS(MACRO)                                                                                  \
  switch ((K / kRowChans + 31) / 32) {                                                                       \
    MACRO(1) MACRO(2) MACRO(3) MACRO(4) MACRO(5) MACRO(6) MACRO(7) MACRO(8) MACRO(9) MACRO(10) MACRO(11)     \
    MACRO(12) MACRO(13) MACRO(14) MACRO(15) MACRO(16)                                                        \
    default: return cudaErrorInvalidValue;                                                                   \
  }

template <int MODE>
static cudaError_t launch_rowring(const __nv_bfloat16* in, int64_t rows, int K, int8_t* q, float* sc,
                                  const ModNormArgs& a, int* err, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  if (K <= 0 || K % 128 != 0 || K > 16384) return cudaErrorInvalidValue;
#define H3_RR_CASE(W) \
  case W: return launch_rowring_t<W, MODE>(in, rows, K, q, sc, a, err, s);
  H3_ROW_WARPS(H3_RR_CASE)
#undef H3_RR_CASE
}
#undef H3_ROW_WARPS

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
                                int* err, cudaStream_t s) {
  ModNormArgs none{};
  return launch_rowring<kRowQuant>(in, rows, K, out_q, out_scale, none, err, s);
}

cudaError_t launch_modt(const float* table, int n_tags, int n_t, int K, float4* modt, cudaStream_t s) {
  if (K % 128 != 0 || K > 16384) return cudaErrorInvalidValue;
  const int64_t total = (int64_t)n_tags * n_t * 4 * 8 * (K / kRowChans);
  if (total == 0) return cudaSuccess;
  const int64_t blocks = (total + 255) / 256 < 1184 ? (total + 255) / 256 : 1184;
  modt_kernel<<<(unsigned)blocks, 256, 0, s>>>(table, n_tags * n_t, K, modt);
  return cudaGetLastError();
}

cudaError_t launch_modnorm(const ModNormArgs& a, cudaStream_t s) {
  if (a.n <= 0) return cudaSuccess;
  if (a.out_q) {
    if (!a.modt) return cudaErrorInvalidValue;
    return launch_rowring<kRowNormQuant>(a.x, a.n, a.C, a.out_q, a.out_scale, a, a.err, s);
  }
  return launch_rows(a.x, a.n, a.C, a.out_bf16, a, a.err, s);
}

}  // namespace h3
