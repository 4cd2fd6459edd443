// Backward pass of the ring/striped attention (sm_100a): dQ, dK, dV.
//
// The pages give no backward algorithm; this is the derivative of
// Softmax(Q K^T * scale + C) V (Striped review, 核心公式) with the forward's
// saved lse:
//     P  = exp(S - lse)        D = rowsum(dO o O)       dS = P o (dO V^T - D)
//     dV = P^T dO              dK = dS^T Q * scale       dQ = dS K * scale
// over the same virtual shards, GetMask blocks and skipped tiles as the
// forward (ra_tiles.cuh).
//
// Three kernels, no atomics:
//   bwd_rowdot   D[row] = sum_i dO[row, i] O[row, i]               (fp32)
//   bwd_dkdv     one CTA per key tile: loops over the query tiles that can
//                see it, S^T = K Q^T and dP^T = V dO^T on the tensor cores,
//                P^T and dS^T in TMEM (bf16), dV += P^T dO, dK += dS^T Q
//   bwd_dq       one CTA per query tile: loops over the key tiles it sees,
//                S = Q K^T, dP = dO V^T, dS in TMEM, dQ += dS K
// Both tile kernels are warp-specialised like the forward: a TMA producer
// warp (a three-slot ring for the tile of the score MMA, a two-slot ring for
// the other streamed tile), an MMA warp, and two element-wise warpgroups
// (thread = TMEM lane, each warpgroup one half of the 128 columns).  The MMA
// order overlaps the next tile's score MMA with the exponentials of the
// current one.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "ra_internal.h"
#include "ra_bwd.h"
#include "ra_ptx.cuh"
#include "ra_tiles.cuh"

namespace ra {

struct BwdParams {
  const __nv_bfloat16* o;
  const __nv_bfloat16* dout;
  const float* lse;
  float* dvec;            // D, [BH, N] fp32 (workspace)
  __nv_bfloat16* dq;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  int BH, N, c, P, T, striped, zigzag, causal;
  int tok;                // all tensors in token order (the layout applied in
                          // the TMA coordinates and the row indices)
  float c2;               // scale * log2(e)
  float scale;
  unsigned long long timeout_ns;
  unsigned int* fault;    // the library's device fault word
};

// ------------------------------------------------------------------ D
template <int D>
__global__ void bwd_rowdot_kernel(const __nv_bfloat16* __restrict__ o,
                                  const __nv_bfloat16* __restrict__ dout, float* __restrict__ dvec,
                                  long long rows) {
  const int lane = threadIdx.x & 31;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long r = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows;
       r += warps) {
    float acc = 0.f;
    for (int i = lane * 2; i < D; i += 64) {
      const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(o + r * D + i));
      const float2 b =
          __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(dout + r * D + i));
      acc = fmaf(a.x, b.x, fmaf(a.y, b.y, acc));
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) dvec[r] = acc;
  }
}

// ------------------------------------------------------------ helpers
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float bex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Packed fp32 pairs (f32x2 arithmetic of sm_100).
__device__ __forceinline__ uint64_t pk2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void unpk2(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t sub2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

// Shared memory of both tile kernels (no slack: the dynamic shared memory
// base must be 1024-byte aligned, which the kernels check):
//   F0, F1   the fixed tile pair of the CTA
//   ring A   3 slots of the tile that feeds the score MMA (Q, resp. K)
//   ring B   2 slots of the other streamed tile (dO, resp. V)
//   vectors  per ring-B slot: {lse2, D} x 128 fp32 (dK/dV kernel only)
template <int D>
struct BwdCfg {
  static constexpr int kTile = kBM * D * 2;   // bytes of a 128 x D bf16 tile
  static constexpr int kSlotsA = 3, kSlotsB = 2;
  static constexpr int kFixed0 = 0, kFixed1 = kTile;
  static constexpr int kRingA = 2 * kTile;
  static constexpr int kRingB = kRingA + kSlotsA * kTile;
  static constexpr int kVec = kRingB + kSlotsB * kTile;
  static constexpr int kBar = kVec + kSlotsB * 2 * kBM * 4;
  static constexpr int kSmem = kBar + 256;
  static constexpr int kThreads = 320;   // 8 element-wise warps, producer, MMA
};

// Barrier offsets from BwdCfg::kBar (8 bytes each); tmem slot and abort flag
// after them.
enum : uint32_t {
  kBarFixed = 0, kBarFullA = 8, kBarEmptyA = 32, kBarFullB = 56, kBarEmptyB = 72, kBarS = 88,
  kBarDP = 96, kBarP = 104, kBarDS = 112, kBarAcc = 120, kBarDrain = 128, kTmemSlot = 136,
  kAbort = 140
};

// TMA: one 128 x D tile of shard `shard` starting at local row row0.  In
// layout order the map is [BH, P, c, D] and the coordinates (row0, shard);
// in token order the striped map is [BH, c, P, D] read as (shard, row0)
// (shard j's rows are tokens x*P + j), the zigzag map [BH, 2P, c/2, D]
// read as (row in chunk, chunk), and contiguous token order is layout order.
template <bool ZZ>
__device__ __forceinline__ void tile_coord(const BwdParams& p, int shard, int row0, int& c1,
                                           int& c2) {
  c1 = row0;
  c2 = shard;
  if (!p.tok) return;
  if (p.striped) {
    c1 = shard;
    c2 = row0;
  } else if (ZZ) {
    const int h = p.c >> 1;
    if (row0 >= h) {
      c1 = row0 - h;
      c2 = 2 * p.P - 1 - shard;
    }
  }
}

template <int D, bool ZZ>
__device__ __forceinline__ void load_tile(const BwdParams& p, uint32_t dst, const CUtensorMap* tm,
                                          uint32_t bar, int row0, int shard, int bh) {
  int c1, c2;
  tile_coord<ZZ>(p, shard, row0, c1, c2);
#pragma unroll
  for (int ch = 0; ch < D / 64; ++ch) tma_load_4d(dst + ch * 16384, tm, bar, ch * 64, c1, c2, bh);
}

// Row (in the tensors' order) of local row x of shard j.
template <bool ZZ>
__device__ __forceinline__ size_t bwd_row(const BwdParams& p, int bh, int j, int x) {
  size_t t = (size_t)j * p.c + x;
  if (p.tok) {
    if (p.striped) {
      t = (size_t)x * p.P + j;
    } else if (ZZ) {
      const int h = p.c >> 1;
      t = x < h ? (size_t)j * h + x : (size_t)(2 * p.P - 1 - j) * h + (x - h);
    }
  }
  return (size_t)bh * p.N + t;
}

// Whole-warp bounded wait (same result in every lane).
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort,
                                          uint64_t limit) {
  const bool ok = mbar_wait(bar, parity, abort, limit);
  return __all_sync(0xffffffffu, ok) != 0;
}

// S (TMEM, 128 x 128) = A (smem 128 x D, K-major) x B (smem 128 x D, K-major)^T
template <int D>
__device__ __forceinline__ void bwd_mma_ss(uint32_t d_tmem, uint32_t a, uint32_t b) {
  constexpr uint32_t idesc = idesc_bf16_f32(kBM, kBN, 0, 0);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = (kk / 4) * 16384 + (kk % 4) * 32;
    mma_ss_w(d_tmem, smem_desc_sw128(a + off, 16, 1024), smem_desc_sw128(b + off, 16, 1024), idesc,
             kk > 0);
  }
}

// D (TMEM, 128 x D) (+)= A (TMEM, bf16 128 x 128) x B (smem tile [128 x D],
// D contiguous, read as MN-major K x N).  A is kept as two halves written by
// the two element-wise warpgroups: K columns 0-63 packed at a_tmem + 0..31,
// K columns 64-127 packed at a_tmem + 64..95.
template <int D>
__device__ __forceinline__ void bwd_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint32_t b,
                                           uint32_t acc) {
  constexpr uint32_t idesc = idesc_bf16_f32(kBM, D, 0, 1);
#pragma unroll
  for (int kk = 0; kk < kBN / 16; ++kk)
    mma_ts_w(d_tmem, a_tmem + (kk / 4) * 64 + (kk % 4) * 8,
             smem_desc_sw128(b + kk * 2048, 16384, 1024), idesc, (acc | (uint32_t)kk) != 0);
}

// Store 32 fp32 TMEM values (one row chunk) as bf16, times `mul`.
__device__ __forceinline__ void store_row32(__nv_bfloat16* dst, const uint32_t (&r)[32],
                                            float mul) {
  uint32_t w[16];
#pragma unroll
  for (int i = 0; i < 16; ++i)
    w[i] = pack2(__uint_as_float(r[2 * i]) * mul, __uint_as_float(r[2 * i + 1]) * mul);
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int i = 0; i < 4; ++i) d4[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
}

// Common set-up of both kernels: barriers, TMEM (512 columns), descriptor
// prefetch.  Returns the TMEM base.
template <int D>
__device__ __forceinline__ uint32_t bwd_setup(uint8_t* smem, int warp, int lane,
                                              uint32_t fullb_count, const CUtensorMap* m0,
                                              const CUtensorMap* m1, const CUtensorMap* m2,
                                              const CUtensorMap* m3) {
  using C = BwdCfg<D>;
  const uint32_t bar = smem_u32(smem) + C::kBar;
  if (threadIdx.x == 0) {
    mbar_init(bar + kBarFixed, 1);
    for (int s = 0; s < C::kSlotsA; ++s) {
      mbar_init(bar + kBarFullA + 8 * s, 1);
      mbar_init(bar + kBarEmptyA + 8 * s, 1);
    }
    for (int s = 0; s < C::kSlotsB; ++s) {
      mbar_init(bar + kBarFullB + 8 * s, fullb_count);
      mbar_init(bar + kBarEmptyB + 8 * s, 1);
    }
    mbar_init(bar + kBarS, 1);
    mbar_init(bar + kBarDP, 1);
    mbar_init(bar + kBarP, 8);     // one arrival per element-wise warp
    mbar_init(bar + kBarDS, 8);
    mbar_init(bar + kBarAcc, 1);
    mbar_init(bar + kBarDrain, 1);
    *reinterpret_cast<volatile int*>(smem + C::kBar + kAbort) = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(smem + C::kBar + kTmemSlot), 512);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    tma_prefetch_desc(m0);
    tma_prefetch_desc(m1);
    tma_prefetch_desc(m2);
    tma_prefetch_desc(m3);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  return *reinterpret_cast<volatile uint32_t*>(smem + C::kBar + kTmemSlot);
}

// Common tear-down: every role has finished; record an abort, free TMEM.
template <int D>
__device__ __forceinline__ void bwd_teardown(uint8_t* smem, uint32_t tmem, int warp,
                                             const BwdParams& p, unsigned int code) {
  using C = BwdCfg<D>;
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && *reinterpret_cast<volatile int*>(smem + C::kBar + kAbort) && p.fault)
    atomicOr(p.fault, code);
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// The tile layouts need a 1024-byte aligned shared memory base; the launch
// leaves no slack to align it by hand.  A misaligned base (not expected) is
// reported as fault code 16 and the CTA does nothing.
__device__ __forceinline__ bool smem_base_ok(const uint8_t* smem, const BwdParams& p) {
  if ((smem_u32(smem) & 1023u) == 0) return true;
  if (threadIdx.x == 0 && p.fault) atomicOr(p.fault, 16u);
  return false;
}

// ------------------------------------------------------------- dK, dV
// Work item: key tile kt of block kb of (b, h).  Query tiles visiting it:
// every (query shard j, tile qt) whose tile against this key tile is not
// skipped; shards in ascending order, so that the CTAs running at the same
// time stream the same query tiles through L2 (the gradient is a sum, its
// order is free).  On a diagonal block, query tiles before kt - 1 cannot see
// key tile kt (a query tile qt reaches keys up to (qt + 1) * 128 - 1 + e),
// so the walk starts there.
template <bool ZZ>
struct QCursor {
  int j, qt, P, T, c, kb, striped, causal, y0;
  BlockMask m;
  int qh, xo, yo;           // zigzag: query chunk half, chunk offsets (query, key)
  int ktl;                  // key tile index inside its chunk (zigzag) or block
  // Mask coordinates of the current tile: query row x and key row y of the
  // shards are x - xo and y - yo in a block (or chunk pair) of length mc().
  __device__ __forceinline__ int mc() const { return ZZ ? (c >> 1) : c; }
  __device__ void init(const BwdParams& p, int kb_, int y0_) {
    j = 0; qt = -1; P = p.P; T = p.T; c = p.c; kb = kb_; striped = p.striped; causal = p.causal;
    y0 = y0_;
    qh = 0; xo = 0;
    const int h = c >> 1;
    yo = (ZZ && y0 >= h) ? h : 0;
    ktl = (y0 - yo) / kBN;
  }
  __device__ bool next(int& oj, int& oqt) {
    const int Tq = ZZ ? (T >> 1) : T;         // query tiles per (chunk or block)
    while (j < P) {
      if (qt < 0) {
        if (ZZ) {
          const int h = c >> 1;
          m = chunk_mask(qh ? 2 * P - 1 - j : j, zz_chunk(kb, y0, h, P), causal);
          xo = qh * h;
        } else {
          m = block_mask(j, kb, striped, causal);
        }
        if (m.all_hidden) {
          qt = -1;
          if (!ZZ || qh == 1) { qh = 0; ++j; } else { qh = 1; }
          continue;
        }
        qt = (m.use_diag && ktl > 0) ? ktl - 1 : 0;
      }
      if (qt >= Tq) {
        qt = -1;
        if (!ZZ || qh == 1) { qh = 0; ++j; } else { qh = 1; }
        continue;
      }
      const int k = tile_kind(m, qt * kBM, y0 - yo, mc());
      ++qt;
      if (k != TILE_SKIP) { oj = j; oqt = (ZZ ? qh * Tq : 0) + qt - 1; return true; }
    }
    return false;
  }
};

// Item order: longest first.  Causal striped / non-causal: key tile kt is
// seen by about T - kt query tiles of every shard, so kt ascending; causal
// contiguous: block kb is seen by shards kb..P-1, so kb ascending.  Heads
// vary slowest, so the CTAs of one wave share one head's tiles in L2.
__device__ __forceinline__ void dkdv_item(const BwdParams& p, int idx, int& bh, int& kb, int& kt) {
  const int per_head = p.P * p.T;
  bh = idx / per_head;
  const int r = idx % per_head;
  if (p.causal && !p.striped) { kb = r / p.T; kt = r % p.T; }
  else { kt = r / p.P; kb = r % p.P; }
}

template <int D, bool ZZ>
__global__ void __launch_bounds__(320, 1)
bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                const BwdParams p) {
  using C = BwdCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  if (!smem_base_ok(smem, p)) return;
  const uint32_t sb = smem_u32(smem), bar = sb + C::kBar;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kBar + kAbort);
  float* vec = reinterpret_cast<float*>(smem + C::kVec);   // [ring-B slot][lse2 | D][128]
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  int bh, kb, kt;
  dkdv_item(p, blockIdx.x, bh, kb, kt);
  const int y0 = kt * kBN;

  // ring B (dO + vectors): the 32 producer lanes arrive after their writes
  const uint32_t tmem = bwd_setup<D>(smem, warp, lane, 32, &tmQ, &tmK, &tmV, &tmdO);
  const uint32_t tS = tmem, tdP = tmem + 128, tdV = tmem + 256, tdK = tmem + 256 + D;
  const uint32_t ringA = sb + C::kRingA, ringB = sb + C::kRingB;

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      mbar_arrive_expect_tx(bar + kBarFixed, 2 * C::kTile);
      load_tile<D, ZZ>(p, sb + C::kFixed0, &tmK, bar + kBarFixed, y0, kb, bh);
      load_tile<D, ZZ>(p, sb + C::kFixed1, &tmV, bar + kBarFixed, y0, kb, bh);
    }
    QCursor<ZZ> cur;
    cur.init(p, kb, y0);
    uint32_t na = 0, nb = 0;   // tiles issued into ring A / ring B
    int j, qt;
    while (cur.next(j, qt)) {
      // per-column lse (log2 units) and D of this query tile, loaded before
      // the waits so that their latency is hidden
      float lv[4], dv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int x = qt * kBM + lane + 32 * u;
        const bool valid = x < p.c;
        const size_t row = bwd_row<ZZ>(p, bh, j, valid ? x : 0);
        lv[u] = valid ? p.lse[row] * 1.4426950408889634f : INFINITY;
        dv[u] = valid ? p.dvec[row] : 0.f;
      }
      const uint32_t a = na % C::kSlotsA;
      if (na >= C::kSlotsA &&
          !warp_wait(bar + kBarEmptyA + 8 * a, (na / C::kSlotsA - 1) & 1, abort_flag, p.timeout_ns))
        break;
      if (lane == 0) {
        mbar_arrive_expect_tx(bar + kBarFullA + 8 * a, C::kTile);
        load_tile<D, ZZ>(p, ringA + a * C::kTile, &tmQ, bar + kBarFullA + 8 * a, qt * kBM, j, bh);
      }
      ++na;
      const uint32_t b = nb & 1;
      if (nb >= 2 && !warp_wait(bar + kBarEmptyB + 8 * b, ((nb >> 1) - 1) & 1, abort_flag, p.timeout_ns))
        break;
      float* v = vec + b * 2 * kBM;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        v[lane + 32 * u] = lv[u];
        v[kBM + lane + 32 * u] = dv[u];
      }
      if (lane == 0) {
        mbar_arrive_expect_tx(bar + kBarFullB + 8 * b, C::kTile);
        load_tile<D, ZZ>(p, ringB + b * C::kTile, &tmdO, bar + kBarFullB + 8 * b, qt * kBM, j, bh);
      } else {
        mbar_arrive(bar + kBarFullB + 8 * b);
      }
      ++nb;
    }
    // every issued load must have landed before the CTA exits
    if (lane == 0) {
      volatile int no_abort = 0;
      mbar_wait(bar + kBarFixed, 0, &no_abort, p.timeout_ns);
      for (uint32_t m = na > (uint32_t)C::kSlotsA ? na - C::kSlotsA : 0; m < na; ++m)
        mbar_wait(bar + kBarFullA + 8 * (m % C::kSlotsA), (m / C::kSlotsA) & 1, &no_abort,
                  p.timeout_ns);
      for (uint32_t m = nb > 2u ? nb - 2 : 0; m < nb; ++m)
        mbar_wait(bar + kBarFullB + 8 * (m & 1), (m >> 1) & 1, &no_abort, p.timeout_ns);
    }
    __syncwarp();
  } else if (warp == 9) {
    // ---------------------------------------------------------- MMA issuer
    // Order per query tile i:  dV += P_i^T dO_i, S_{i+1} = K Q_{i+1}^T,
    // dK += dS_i^T Q_i, dP_{i+1} = V dO_{i+1}^T.  S_{i+1} reuses the columns
    // of P_i right after the MMA that reads them (tcgen05 MMAs of one CTA
    // run in issue order), so the tensor core computes the next scores while
    // the element-wise warps finish dS_i and start on P_{i+1}.
    QCursor<ZZ> cur;
    cur.init(p, kb, y0);
    int j, qt;
    bool ok = warp_wait(bar + kBarFixed, 0, abort_flag, p.timeout_ns);
    bool have = cur.next(j, qt);
    uint32_t i = 0;
    if (ok && have) {
      ok = warp_wait(bar + kBarFullA, 0, abort_flag, p.timeout_ns);
      if (ok) {
        tc_fence_after();
        bwd_mma_ss<D>(tS, sb + C::kFixed0, ringA);
        mma_commit_w(bar + kBarS);
        ok = warp_wait(bar + kBarFullB, 0, abort_flag, p.timeout_ns);
      }
      if (ok) {
        tc_fence_after();
        bwd_mma_ss<D>(tdP, sb + C::kFixed1, ringB);
        mma_commit_w(bar + kBarDP);
      }
    }
    while (ok && have) {
      const uint32_t a = i % C::kSlotsA, b = i & 1;
      const uint32_t an = (i + 1) % C::kSlotsA, bn = b ^ 1;
      const bool more = cur.next(j, qt);
      if (!warp_wait(bar + kBarP, i & 1, abort_flag, p.timeout_ns)) { ok = false; break; }
      tc_fence_after();
      bwd_mma_ts<D>(tdV, tS, ringB + b * C::kTile, i > 0);
      if (more) {
        if (!warp_wait(bar + kBarFullA + 8 * an, ((i + 1) / C::kSlotsA) & 1, abort_flag,
                       p.timeout_ns)) {
          ok = false; break;
        }
        tc_fence_after();
        bwd_mma_ss<D>(tS, sb + C::kFixed0, ringA + an * C::kTile);
        mma_commit_w(bar + kBarS);
      }
      if (!warp_wait(bar + kBarDS, i & 1, abort_flag, p.timeout_ns)) { ok = false; break; }
      tc_fence_after();
      bwd_mma_ts<D>(tdK, tdP, ringA + a * C::kTile, i > 0);
      mma_commit_w(bar + kBarEmptyA + 8 * a);
      mma_commit_w(bar + kBarEmptyB + 8 * b);
      if (more) {
        if (!warp_wait(bar + kBarFullB + 8 * bn, ((i + 1) >> 1) & 1, abort_flag, p.timeout_ns)) {
          ok = false; break;
        }
        tc_fence_after();
        bwd_mma_ss<D>(tdP, sb + C::kFixed1, ringB + bn * C::kTile);
        mma_commit_w(bar + kBarDP);
      }
      ++i;
      have = more;
    }
    if (ok) mma_commit_w(bar + kBarAcc);
    // all MMAs must be complete before TMEM is freed
    mma_commit_w(bar + kBarDrain);
    volatile int no_abort = 0;
    warp_wait(bar + kBarDrain, 0, &no_abort, p.timeout_ns);
  } else {
    // ------------------------------------------------- element-wise warps
    // Thread = key row y (TMEM lane); warpgroup wg takes query columns
    // [64 wg, 64 wg + 64) of every tile.
    const int wg = warp / 4, wq = warp % 4;
    const int y = y0 + wq * 32 + lane;
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t myS = tS + lane_off + 64 * wg, mydP = tdP + lane_off + 64 * wg;
    const uint64_t c2x2 = pk2(p.c2, p.c2);
    QCursor<ZZ> cur;
    cur.init(p, kb, y0);
    int j, qt;
    uint32_t i = 0;
    bool ok = true;
    while (cur.next(j, qt)) {
      const uint32_t b = i & 1;
      // visible query columns [lo, hi), in the block's (chunk pair's) rows
      const int qx0 = qt * kBM - cur.xo, yl = y - cur.yo;
      int lo = 0, hi = cur.mc() - qx0;
      if (cur.m.use_diag) {
        const int l2 = yl + 1 - cur.m.e - qx0;   // query x sees key y iff y < x + e
        lo = l2 > 0 ? l2 : 0;
      }
      if (y >= p.c) hi = 0;
      lo -= 64 * wg;
      hi -= 64 * wg;
      const bool all_vis = __all_sync(0xffffffffu, lo <= 0 && hi >= 64) != 0;
      if (!warp_wait(bar + kBarS, i & 1, abort_flag, p.timeout_ns) ||
          !warp_wait(bar + kBarFullB + 8 * b, (i >> 1) & 1, abort_flag, p.timeout_ns)) {
        ok = false; break;
      }
      tc_fence_after();
      uint32_t a[2][32];
      tmem_ld32(myS, a[0]);
      tmem_ld32(myS + 32, a[1]);
      tmem_wait_ld();
      const float4* lse2 = reinterpret_cast<const float4*>(vec + b * 2 * kBM + 64 * wg);
      const float4* dcol = lse2 + kBM / 4;
      float pr[64];
      uint32_t pkd[32];
      // P = exp2(S * c2 - lse2), packed pairs
#pragma unroll
      for (int q4 = 0; q4 < 16; ++q4) {
        const float4 l4 = lse2[q4];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int q = 4 * q4 + 2 * h;
          const uint64_t nl = pk2(-(h ? l4.z : l4.x), -(h ? l4.w : l4.y));
          const uint64_t t = fma2(pk2(__uint_as_float(a[q / 32][q % 32]),
                                      __uint_as_float(a[q / 32][q % 32 + 1])), c2x2, nl);
          float t0, t1;
          unpk2(t, t0, t1);
          pr[q] = bex2(t0);
          pr[q + 1] = bex2(t1);
        }
      }
      if (!all_vis) {
#pragma unroll
        for (int q = 0; q < 64; ++q)
          if (q < lo || q >= hi) pr[q] = 0.f;
      }
#pragma unroll
      for (int q = 0; q < 32; ++q) pkd[q] = pack2(pr[2 * q], pr[2 * q + 1]);
      tmem_st32(myS, pkd);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar + kBarP);
      if (!warp_wait(bar + kBarDP, i & 1, abort_flag, p.timeout_ns)) { ok = false; break; }
      tc_fence_after();
      tmem_ld32(mydP, a[0]);
      tmem_ld32(mydP + 32, a[1]);
      tmem_wait_ld();
      // dS = P (dP - D), packed pairs
#pragma unroll
      for (int q4 = 0; q4 < 16; ++q4) {
        const float4 d4 = dcol[q4];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int q = 4 * q4 + 2 * h;
          const uint64_t dp = pk2(__uint_as_float(a[q / 32][q % 32]),
                                  __uint_as_float(a[q / 32][q % 32 + 1]));
          const uint64_t ds =
              mul2(pk2(pr[q], pr[q + 1]), sub2(dp, pk2(h ? d4.z : d4.x, h ? d4.w : d4.y)));
          float d0, d1;
          unpk2(ds, d0, d1);
          pkd[q / 2] = pack2(d0, d1);
        }
      }
      tmem_st32(mydP, pkd);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar + kBarDS);
      ++i;
    }
    // Epilogue: dK (times scale) and dV rows of this key tile, columns
    // [wg D/2, (wg+1) D/2).  TMEM loads are warp-collective; only the stores
    // are guarded per row.
    if (ok && (i == 0 || warp_wait(bar + kBarAcc, 0, abort_flag, p.timeout_ns))) {
      tc_fence_after();
      const bool valid = y < p.c;
      const size_t row = bwd_row<ZZ>(p, bh, kb, valid ? y : 0);
#pragma unroll 1
      for (int q = 0; q < D / 64; ++q) {
        const int col = wg * (D / 2) + q * 32;
        uint32_t r[32];
        if (i) {
          tmem_ld32(tdK + lane_off + col, r);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int u = 0; u < 32; ++u) r[u] = 0u;
        }
        if (valid) store_row32(p.dk + row * D + col, r, p.scale);
        if (i) {
          tmem_ld32(tdV + lane_off + col, r);
          tmem_wait_ld();
        }
        if (valid) store_row32(p.dv + row * D + col, r, 1.f);
      }
    }
  }
  bwd_teardown<D>(smem, tmem, warp, p, 4u);
}

// ----------------------------------------------------------------- dQ
// Work item: query tile qt of shard j of (b, h); key tiles of every block
// that is not hidden, blocks in ascending order (the same order in every
// CTA, for L2 reuse; the gradient is a sum), skipped tiles left out.
template <bool ZZ>
struct KCursor {
  int kb, kt, kend, P, c, j, striped, causal, x0;
  BlockMask bm;
  TileSpan sp;
  int r, xo, yo, kt_off;    // zigzag: sub-round, chunk offsets, key tile offset
  __device__ __forceinline__ int mc() const { return ZZ ? (c >> 1) : c; }
  __device__ void init(const BwdParams& p, int j_, int x0_) {
    kb = -1; kt = 0; kend = 0; P = p.P; c = p.c; j = j_; striped = p.striped; causal = p.causal;
    x0 = x0_;
    r = -1; xo = 0; yo = 0; kt_off = 0;
  }
  __device__ bool next(int& okb, int& oy0, int& kind, BlockMask& m) {
    while (kt >= kend) {
      if (ZZ) {
        // sub-round r = 2 * block + chunk half of the key block
        if (++r >= 2 * P) return false;
        kb = r >> 1;
        const int h = c >> 1, hk = r & 1;
        xo = x0 < h ? 0 : h;
        yo = hk * h;
        bm = chunk_mask(zz_chunk(j, x0, h, P), hk ? 2 * P - 1 - kb : kb, causal);
        sp = tile_span(bm, x0 - xo, h);
        kt_off = hk * (h / kBN);
      } else {
        if (++kb >= P) return false;
        bm = block_mask(j, kb, striped, causal);
        sp = tile_span(bm, x0, c);
      }
      kend = sp.part_end;
      kt = 0;
    }
    okb = kb;
    oy0 = ((ZZ ? kt_off : 0) + kt) * kBN;
    kind = tile_kind_at(sp, kt);
    m = bm;
    ++kt;
    return true;
  }
};

// Longest first: causal striped, the last query tiles of a shard see the
// most keys (qt descending); causal contiguous, shard j sees blocks 0..j
// (j descending, then qt descending).  Heads vary slowest.
__device__ __forceinline__ void dq_item(const BwdParams& p, int idx, int& bh, int& j, int& qt) {
  const int per_head = p.P * p.T;
  bh = idx / per_head;
  const int r = idx % per_head;
  if (p.causal && !p.striped) { j = p.P - 1 - r / p.T; qt = p.T - 1 - r % p.T; }
  else { qt = p.T - 1 - r / p.P; j = r % p.P; }
}

template <int D, bool ZZ>
__global__ void __launch_bounds__(320, 1)
bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
              const BwdParams p) {
  using C = BwdCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  if (!smem_base_ok(smem, p)) return;
  const uint32_t sb = smem_u32(smem), bar = sb + C::kBar;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kBar + kAbort);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  int bh, j, qt;
  dq_item(p, blockIdx.x, bh, j, qt);
  const int x0 = qt * kBM;

  const uint32_t tmem = bwd_setup<D>(smem, warp, lane, 1, &tmQ, &tmK, &tmV, &tmdO);
  const uint32_t tS = tmem, tdP = tmem + 128, tdQ = tmem + 256;
  const uint32_t ringA = sb + C::kRingA, ringB = sb + C::kRingB;

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      mbar_arrive_expect_tx(bar + kBarFixed, 2 * C::kTile);
      load_tile<D, ZZ>(p, sb + C::kFixed0, &tmQ, bar + kBarFixed, x0, j, bh);
      load_tile<D, ZZ>(p, sb + C::kFixed1, &tmdO, bar + kBarFixed, x0, j, bh);
      KCursor<ZZ> cur;
      cur.init(p, j, x0);
      uint32_t na = 0, nb = 0;
      int kb, y0, kind;
      BlockMask bm;
      while (cur.next(kb, y0, kind, bm)) {
        const uint32_t a = na % C::kSlotsA;
        if (na >= C::kSlotsA &&
            !mbar_wait(bar + kBarEmptyA + 8 * a, (na / C::kSlotsA - 1) & 1, abort_flag, p.timeout_ns))
          break;
        mbar_arrive_expect_tx(bar + kBarFullA + 8 * a, C::kTile);
        load_tile<D, ZZ>(p, ringA + a * C::kTile, &tmK, bar + kBarFullA + 8 * a, y0, kb, bh);
        ++na;
        const uint32_t b = nb & 1;
        if (nb >= 2 && !mbar_wait(bar + kBarEmptyB + 8 * b, ((nb >> 1) - 1) & 1, abort_flag, p.timeout_ns))
          break;
        mbar_arrive_expect_tx(bar + kBarFullB + 8 * b, C::kTile);
        load_tile<D, ZZ>(p, ringB + b * C::kTile, &tmV, bar + kBarFullB + 8 * b, y0, kb, bh);
        ++nb;
      }
      volatile int no_abort = 0;
      mbar_wait(bar + kBarFixed, 0, &no_abort, p.timeout_ns);
      for (uint32_t m = na > (uint32_t)C::kSlotsA ? na - C::kSlotsA : 0; m < na; ++m)
        mbar_wait(bar + kBarFullA + 8 * (m % C::kSlotsA), (m / C::kSlotsA) & 1, &no_abort,
                  p.timeout_ns);
      for (uint32_t m = nb > 2u ? nb - 2 : 0; m < nb; ++m)
        mbar_wait(bar + kBarFullB + 8 * (m & 1), (m >> 1) & 1, &no_abort, p.timeout_ns);
    }
    __syncwarp();
  } else if (warp == 9) {
    // ---------------------------------------------------------- MMA issuer
    // Order per key tile i: S_{i+1} = Q K_{i+1}^T as soon as the element-wise
    // warps have read S_i; dQ += dS_i K_i; dP_{i+1} = dO V_{i+1}^T into the
    // columns of dS_i right after the MMA that reads them.
    KCursor<ZZ> cur;
    cur.init(p, j, x0);
    int kb, y0, kind;
    BlockMask bm;
    bool ok = warp_wait(bar + kBarFixed, 0, abort_flag, p.timeout_ns);
    bool have = cur.next(kb, y0, kind, bm);
    uint32_t i = 0;
    if (ok && have) {
      ok = warp_wait(bar + kBarFullA, 0, abort_flag, p.timeout_ns);
      if (ok) {
        tc_fence_after();
        bwd_mma_ss<D>(tS, sb + C::kFixed0, ringA);
        mma_commit_w(bar + kBarS);
        ok = warp_wait(bar + kBarFullB, 0, abort_flag, p.timeout_ns);
      }
      if (ok) {
        tc_fence_after();
        bwd_mma_ss<D>(tdP, sb + C::kFixed1, ringB);
        mma_commit_w(bar + kBarDP);
      }
    }
    while (ok && have) {
      const uint32_t a = i % C::kSlotsA, b = i & 1;
      const uint32_t an = (i + 1) % C::kSlotsA, bn = b ^ 1;
      const bool more = cur.next(kb, y0, kind, bm);
      if (more) {
        // kBarP: the element-wise warps have read S_i
        if (!warp_wait(bar + kBarP, i & 1, abort_flag, p.timeout_ns) ||
            !warp_wait(bar + kBarFullA + 8 * an, ((i + 1) / C::kSlotsA) & 1, abort_flag,
                       p.timeout_ns)) {
          ok = false; break;
        }
        tc_fence_after();
        bwd_mma_ss<D>(tS, sb + C::kFixed0, ringA + an * C::kTile);
        mma_commit_w(bar + kBarS);
      }
      if (!warp_wait(bar + kBarDS, i & 1, abort_flag, p.timeout_ns)) { ok = false; break; }
      tc_fence_after();
      bwd_mma_ts<D>(tdQ, tdP, ringA + a * C::kTile, i > 0);
      mma_commit_w(bar + kBarEmptyA + 8 * a);
      mma_commit_w(bar + kBarEmptyB + 8 * b);
      if (more) {
        if (!warp_wait(bar + kBarFullB + 8 * bn, ((i + 1) >> 1) & 1, abort_flag, p.timeout_ns)) {
          ok = false; break;
        }
        tc_fence_after();
        bwd_mma_ss<D>(tdP, sb + C::kFixed1, ringB + bn * C::kTile);
        mma_commit_w(bar + kBarDP);
      }
      ++i;
      have = more;
    }
    if (ok) mma_commit_w(bar + kBarAcc);
    mma_commit_w(bar + kBarDrain);
    volatile int no_abort = 0;
    warp_wait(bar + kBarDrain, 0, &no_abort, p.timeout_ns);
  } else {
    // ------------------------------------------------- element-wise warps
    // Thread = query row x (TMEM lane); warpgroup wg takes key columns
    // [64 wg, 64 wg + 64) of every tile.
    const int wg = warp / 4, wq = warp % 4;
    const int x = x0 + wq * 32 + lane;
    const bool xvalid = x < p.c;
    const size_t xrow = bwd_row<ZZ>(p, bh, j, xvalid ? x : 0);
    const float lse2 = xvalid ? p.lse[xrow] * 1.4426950408889634f : INFINITY;
    const float drow = xvalid ? p.dvec[xrow] : 0.f;
    const uint64_t c2x2 = pk2(p.c2, p.c2), nl2 = pk2(-lse2, -lse2), d2 = pk2(drow, drow);
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t myS = tS + lane_off + 64 * wg, mydP = tdP + lane_off + 64 * wg;
    KCursor<ZZ> cur;
    cur.init(p, j, x0);
    int kb, y0, kind;
    BlockMask bm;
    uint32_t i = 0;
    bool ok = true;
    while (cur.next(kb, y0, kind, bm)) {
      const int lim =
          (xvalid ? ((kind == TILE_PARTIAL) ? row_limit(bm, x - cur.xo, y0 - cur.yo, cur.mc()) : kBN)
                  : 0) - 64 * wg;
      const bool all_vis = __all_sync(0xffffffffu, lim >= 64) != 0;
      if (!warp_wait(bar + kBarS, i & 1, abort_flag, p.timeout_ns)) { ok = false; break; }
      tc_fence_after();
      uint32_t a[2][32];
      tmem_ld32(myS, a[0]);
      tmem_ld32(myS + 32, a[1]);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar + kBarP);   // S_i read: its columns may be reused
      float pr[64];
#pragma unroll
      for (int q = 0; q < 64; q += 2) {
        const uint64_t t = fma2(pk2(__uint_as_float(a[q / 32][q % 32]),
                                    __uint_as_float(a[q / 32][q % 32 + 1])), c2x2, nl2);
        float t0, t1;
        unpk2(t, t0, t1);
        pr[q] = bex2(t0);
        pr[q + 1] = bex2(t1);
      }
      if (!all_vis) {
#pragma unroll
        for (int q = 0; q < 64; ++q)
          if (q >= lim) pr[q] = 0.f;
      }
      if (!warp_wait(bar + kBarDP, i & 1, abort_flag, p.timeout_ns)) { ok = false; break; }
      tc_fence_after();
      tmem_ld32(mydP, a[0]);
      tmem_ld32(mydP + 32, a[1]);
      tmem_wait_ld();
      uint32_t pkd[32];
#pragma unroll
      for (int q = 0; q < 64; q += 2) {
        const uint64_t dp = pk2(__uint_as_float(a[q / 32][q % 32]),
                                __uint_as_float(a[q / 32][q % 32 + 1]));
        const uint64_t ds = mul2(pk2(pr[q], pr[q + 1]), sub2(dp, d2));
        float d0, d1;
        unpk2(ds, d0, d1);
        pkd[q / 2] = pack2(d0, d1);
      }
      tmem_st32(mydP, pkd);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar + kBarDS);
      ++i;
    }
    if (ok && (i == 0 || warp_wait(bar + kBarAcc, 0, abort_flag, p.timeout_ns))) {
      tc_fence_after();
      __nv_bfloat16* dst = p.dq + xrow * D;
#pragma unroll 1
      for (int q = 0; q < D / 64; ++q) {
        const int col = wg * (D / 2) + q * 32;
        uint32_t r[32];
        if (i) {
          tmem_ld32(tdQ + lane_off + col, r);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int u = 0; u < 32; ++u) r[u] = 0u;
        }
        if (xvalid) store_row32(dst + col, r, p.scale);
      }
    }
  }
  bwd_teardown<D>(smem, tmem, warp, p, 8u);
}

// ------------------------------------------------------------------ host
// mode 0: [BH, P, c, d]; 1: striped token order [BH, c, P, d] (box over c);
// 2: zigzag token order [BH, 2P, c/2, d].
static bool encode_map(CUtensorMap* map, const void* base, int64_t BH, int64_t N, int64_t c, int P,
                       int d, int mode) {
  PFN_encodeTiled enc = get_encode_tiled();
  if (!enc) return false;
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)c, (cuuint64_t)P, (cuuint64_t)BH};
  cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)c * d * 2, (cuuint64_t)N * d * 2};
  cuuint32_t box[4] = {64, (cuuint32_t)kBM, 1, 1};
  if (mode == 1) {
    dims[1] = (cuuint64_t)P;
    dims[2] = (cuuint64_t)c;
    strides[1] = (cuuint64_t)P * d * 2;
    box[1] = 1;
    box[2] = (cuuint32_t)kBM;
  } else if (mode == 2) {
    dims[1] = (cuuint64_t)(c / 2);
    dims[2] = (cuuint64_t)(2 * P);
    strides[1] = (cuuint64_t)(c / 2) * d * 2;
  }
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, bool ZZ>
static ra_status launch_bwd(const BwdLaunch& a) {
  using C = BwdCfg<D>;
  const int64_t c = a.N / a.P;
  CUtensorMap tq, tk, tv, tdo;
  const int mode = !a.tok ? 0 : a.striped ? 1 : a.zigzag ? 2 : 0;
  if (!encode_map(&tq, a.q, a.BH, a.N, c, a.P, D, mode) ||
      !encode_map(&tk, a.k, a.BH, a.N, c, a.P, D, mode) ||
      !encode_map(&tv, a.v, a.BH, a.N, c, a.P, D, mode) ||
      !encode_map(&tdo, a.dout, a.BH, a.N, c, a.P, D, mode))
    return RA_ERR_CUDA;
  // once per device (setting the attribute again is harmless; the flag only
  // saves the calls)
  static std::atomic<int> attr_set[64];
  if (a.device < 64 && !attr_set[a.device].load(std::memory_order_acquire)) {
    if (cudaFuncSetAttribute(bwd_dkdv_kernel<D, ZZ>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::kSmem) != cudaSuccess ||
        cudaFuncSetAttribute(bwd_dq_kernel<D, ZZ>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::kSmem) != cudaSuccess)
      return RA_ERR_CUDA;
    attr_set[a.device].store(1, std::memory_order_release);
  }
  BwdParams p;
  p.o = reinterpret_cast<const __nv_bfloat16*>(a.o);
  p.dout = reinterpret_cast<const __nv_bfloat16*>(a.dout);
  p.lse = a.lse;
  p.dvec = a.workspace;
  p.dq = reinterpret_cast<__nv_bfloat16*>(a.dq);
  p.dk = reinterpret_cast<__nv_bfloat16*>(a.dk);
  p.dv = reinterpret_cast<__nv_bfloat16*>(a.dv);
  p.BH = (int)a.BH;
  p.N = (int)a.N;
  p.c = (int)c;
  p.P = a.P;
  p.T = (int)((c + kBM - 1) / kBM);
  p.striped = a.striped;
  p.zigzag = a.zigzag;
  p.tok = a.tok;
  p.causal = a.causal;
  p.c2 = (float)((double)a.scale * 1.4426950408889634074);
  p.scale = a.scale;
  p.timeout_ns = 2000000000ull;
  p.fault = device_fault_word();
  if (!p.fault) return RA_ERR_CUDA;
  cudaStream_t st = (cudaStream_t)a.stream;
  const long long rows = a.BH * a.N;
  long long blocks = (rows + 7) / 8;
  if (blocks > (long long)a.num_sms * 16) blocks = (long long)a.num_sms * 16;
  bwd_rowdot_kernel<D><<<(int)blocks, 256, 0, st>>>(p.o, p.dout, p.dvec, rows);
  const long long items = (long long)p.BH * p.P * p.T;
  bwd_dkdv_kernel<D, ZZ><<<(unsigned)items, C::kThreads, C::kSmem, st>>>(tq, tk, tv, tdo, p);
  bwd_dq_kernel<D, ZZ><<<(unsigned)items, C::kThreads, C::kSmem, st>>>(tq, tk, tv, tdo, p);
  return cudaGetLastError() == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

ra_status attn_bwd_launch(const BwdLaunch& a) {
  if (a.zigzag) {
    if (a.d == 128) return launch_bwd<128, true>(a);
    if (a.d == 64) return launch_bwd<64, true>(a);
  } else {
    if (a.d == 128) return launch_bwd<128, false>(a);
    if (a.d == 64) return launch_bwd<64, false>(a);
  }
  return RA_ERR_HEADDIM;
}

// ------------------------------------------- backward without allocation
// For callers that must not allocate device memory themselves: the scratch
// row vector D of the backward lives in this fixed device array instead of a
// caller workspace.  Every GPU that loads the library reserves it until the
// process exits.  All calls on one device share that device's copy: two
// calls whose kernels overlap on the same GPU (another stream, or another
// host thread) race on it; calls on different devices use separate copies.
// D is fully rewritten by every call, so nothing has to be cleared.
static __device__ __align__(256) float g_bwd_scratch[kNoAllocScratchFloats];

ra_status attn_bwd_noalloc_launch(BwdLaunch a) {
  if (a.BH * a.N > kNoAllocScratchFloats) return RA_ERR_SCRATCH;
  // In host code `g_bwd_scratch` names a host-side stand-in; the kernels need
  // the device address, looked up once per device with that device current.
  static float* addr[64] = {nullptr};
  static std::mutex mu;
  if (a.device < 0 || a.device >= 64) return RA_ERR_DEVICE;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[a.device]) {
      void* ptr = nullptr;
      if (cudaGetSymbolAddress(&ptr, g_bwd_scratch) != cudaSuccess || !ptr) return RA_ERR_CUDA;
      addr[a.device] = reinterpret_cast<float*>(ptr);
    }
    a.workspace = addr[a.device];
  }
  return attn_bwd_launch(a);
}

}  // namespace ra
