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
//   bwd_dq       one CTA per query tile: loops over key tiles in ring order,
//                S = Q K^T, dP = dO V^T, dS in TMEM, dQ += dS K
// Each CTA is one warpgroup (thread i owns TMEM lane i); one elected thread
// issues TMA loads and MMAs; the next query (resp. key/value) tile is loaded
// into a second shared-memory buffer while the current one is computed.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "ra_internal.h"
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
  int BH, N, c, P, T, striped, causal;
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

// Wait by the whole CTA; gives up (and flags the CTA) after the time limit.
__device__ __forceinline__ bool cta_wait(uint32_t bar, uint32_t parity, volatile int* abort,
                                         uint64_t limit) {
  const bool ok = mbar_wait(bar, parity, abort, limit);
  return __syncthreads_and(ok) != 0;
}

// S (TMEM) = A (smem, 128 x D, K-major) x B (smem, 128 x D, K-major)^T
template <int D>
__device__ __forceinline__ void bwd_mma_ss(uint32_t d_tmem, uint32_t a, uint32_t b) {
  constexpr uint32_t idesc = idesc_bf16_f32(kBM, kBN, 0, 0);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = (kk / 4) * 16384 + (kk % 4) * 32;
    mma_ss(d_tmem, smem_desc_sw128(a + off, 16, 1024), smem_desc_sw128(b + off, 16, 1024), idesc,
           kk > 0);
  }
}

// D (TMEM, 128 x D) (+)= A (TMEM, bf16 128 x 128) x B (smem tile [128 x D],
// D contiguous, read as MN-major K x N).
template <int D>
__device__ __forceinline__ void bwd_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint32_t b,
                                           uint32_t acc) {
  constexpr uint32_t idesc = idesc_bf16_f32(kBM, D, 0, 1);
#pragma unroll
  for (int kk = 0; kk < kBN / 16; ++kk)
    mma_ts(d_tmem, a_tmem + kk * 8, smem_desc_sw128(b + kk * 2048, 16384, 1024), idesc,
           (acc | (uint32_t)kk) != 0);
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

template <int D>
struct BwdCfg {
  static constexpr int kTile = kBM * D * 2;   // bytes of a 128 x D bf16 tile
  static constexpr int kChunks = D / 64;
  // smem: fixed tile pair (A0, A1), two buffers of the streamed tile pair,
  // per-column vectors (2 buffers x {lse2, D} x 128 fp32), barriers
  static constexpr int kFixed0 = 0, kFixed1 = kTile;
  static constexpr int kStream = 2 * kTile;            // + buf * 2 * kTile
  static constexpr int kVec = 6 * kTile;
  static constexpr int kBar = kVec + 2 * 2 * kBM * 4;
  static constexpr int kSmem = kBar + 64 + 1024;
};

// TMA: one 128 x D tile of a [BH, P, c, D] tensor at (shard, row0, bh).
template <int D>
__device__ __forceinline__ void load_tile(uint32_t dst, const CUtensorMap* tm, uint32_t bar,
                                          int row0, int shard, int bh) {
#pragma unroll
  for (int ch = 0; ch < D / 64; ++ch) tma_load_4d(dst + ch * 16384, tm, bar, ch * 64, row0, shard, bh);
}

// ------------------------------------------------------------- dK, dV
// Work item: key tile kt of block kb of (b, h).  Query tiles visiting it:
// every (query shard j, tile qt) whose tile against this key tile is not
// skipped, shards in the order kb, kb+1, ... (the reverse ring).
template <int D>
__global__ void __launch_bounds__(128, 1)
bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                const BwdParams p) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const uint32_t bar_fixed = sb + C::kBar, bar_ld0 = bar_fixed + 8, bar_mma = bar_fixed + 24;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + C::kBar + 40);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kBar + 44);
  float* vec = reinterpret_cast<float*>(smem + C::kVec);   // [buf][lse2|D][128]
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;

  const int T = p.T;
  const int kt = blockIdx.x % T;
  const int kb = (blockIdx.x / T) % p.P;
  const int bh = blockIdx.x / (T * p.P);
  const int y0 = kt * kBN;
  const int y = y0 + tid;                       // this thread's key (local in block kb)

  if (tid == 0) {
    mbar_init(bar_fixed, 1);
    mbar_init(bar_ld0, 1);
    mbar_init(bar_ld0 + 8, 1);
    mbar_init(bar_mma, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tslot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  const uint32_t tS = tmem, tdP = tmem + 128, tdV = tmem + 256, tdK = tmem + 256 + D;
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;

  // The query tiles of this key tile, in order; one cursor for loads (one
  // ahead) and one for compute.
  struct Cursor {
    int j, qt, P, T, c, kb, striped, causal, y0, done;
    __device__ bool next(int& oj, int& oqt, int& kind) {
      while (!done) {
        if (qt >= T) {
          qt = 0;
          if (++j >= P) { done = 1; return false; }
        }
        const int jj = (kb + j) % P;
        const BlockMask m = block_mask(jj, kb, striped, causal);
        const int k = tile_kind(m, qt * kBM, y0, c);
        ++qt;
        if (k != TILE_SKIP) { oj = jj; oqt = qt - 1; kind = k; return true; }
      }
      return false;
    }
  };
  Cursor ld{0, 0, p.P, T, p.c, kb, p.striped, p.causal, y0, 0};
  Cursor cm = ld;

  bool ok = true;
  uint32_t issued[2] = {0, 0}, consumed[2] = {0, 0};
  if (tid == 0) {
    mbar_arrive_expect_tx(bar_fixed, 2 * C::kTile);
    load_tile<D>(sb + C::kFixed0, &tmK, bar_fixed, y0, kb, bh);
    load_tile<D>(sb + C::kFixed1, &tmV, bar_fixed, y0, kb, bh);
  }
  // Query tile loads run one ahead of the compute cursor, alternating buffers.
  int lj, lqt, lkind;
  auto issue_load = [&](int buf, int j, int qt) {
    const uint32_t dst = sb + C::kStream + buf * 2 * C::kTile;
    if (tid == 0) {
      mbar_arrive_expect_tx(bar_ld0 + 8 * buf, 2 * C::kTile);
      load_tile<D>(dst, &tmQ, bar_ld0 + 8 * buf, qt * kBM, j, bh);
      load_tile<D>(dst + C::kTile, &tmdO, bar_ld0 + 8 * buf, qt * kBM, j, bh);
    }
    ++issued[buf];
    // per-column lse (log2 units) and D of this query tile
    const int x = qt * kBM + tid;
    float* v = vec + buf * 2 * kBM;
    const size_t row = (size_t)bh * p.N + (size_t)j * p.c + (size_t)(x < p.c ? x : 0);
    v[tid] = (x < p.c) ? p.lse[row] * 1.4426950408889634f : INFINITY;
    v[kBM + tid] = (x < p.c) ? p.dvec[row] : 0.f;
  };
  if (ld.next(lj, lqt, lkind)) issue_load(0, lj, lqt);
  bool fixed_done = cta_wait(bar_fixed, 0, abort_flag, p.timeout_ns);
  if (!fixed_done) ok = false;
  tc_fence_after();

  uint32_t n = 0, mma_ph = 0, accum = 0;
  int cj, cqt, ckind;
  while (ok && cm.next(cj, cqt, ckind)) {
    const int buf = n & 1;
    // Next query tile into the other buffer; the MMAs that read it last
    // completed at the end of the previous iteration.
    __syncthreads();
    if (ld.next(lj, lqt, lkind)) issue_load(buf ^ 1, lj, lqt);
    if (!cta_wait(bar_ld0 + 8 * buf, consumed[buf] & 1, abort_flag, p.timeout_ns)) {
      ok = false;
      break;
    }
    ++consumed[buf];
    tc_fence_after();
    const uint32_t sq = sb + C::kStream + buf * 2 * C::kTile, sdo = sq + C::kTile;
    if (warp == 0 && lane == 0) {
      bwd_mma_ss<D>(tS, sb + C::kFixed0, sq);     // S^T = K Q^T
      bwd_mma_ss<D>(tdP, sb + C::kFixed1, sdo);   // dP^T = V dO^T
      mma_commit(bar_mma);
    }
    __syncwarp();
    if (!cta_wait(bar_mma, mma_ph, abort_flag, p.timeout_ns)) { ok = false; break; }
    mma_ph ^= 1;
    tc_fence_after();
    // P^T and dS^T for this thread's key row; column q = query qt*128 + q
    const float* lse2 = vec + buf * 2 * kBM;
    const float* dcol = lse2 + kBM;
    const BlockMask bm = block_mask(cj, kb, p.striped, p.causal);
    int lo = 0, hi = p.c - cqt * kBM;             // visible query columns [lo, hi)
    if (bm.use_diag) {
      const int l2 = y + 1 - bm.e - cqt * kBM;    // query x sees key y iff y < x + e
      lo = l2 > 0 ? l2 : 0;
    }
    if (y >= p.c) hi = 0;
#pragma unroll 1
    for (int ch = 0; ch < 4; ++ch) {
      uint32_t sv[32], dv[32];
      tmem_ld32(tS + lane_off + ch * 32, sv);
      tmem_ld32(tdP + lane_off + ch * 32, dv);
      tmem_wait_ld();
      uint32_t pk[16], dk[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        float pr[2], ds[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int q = ch * 32 + 2 * i + u;
          const bool vis = (q >= lo) && (q < hi);
          const float pv = vis ? bex2(fmaf(__uint_as_float(sv[2 * i + u]), p.c2, -lse2[q])) : 0.f;
          pr[u] = pv;
          ds[u] = pv * (__uint_as_float(dv[2 * i + u]) - dcol[q]);
        }
        pk[i] = pack2(pr[0], pr[1]);
        dk[i] = pack2(ds[0], ds[1]);
      }
      tmem_st16(tS + lane_off + ch * 16, pk);
      tmem_st16(tdP + lane_off + ch * 16, dk);
    }
    tmem_wait_st();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0 && lane == 0) {
      bwd_mma_ts<D>(tdV, tS, sdo, accum);   // dV += P^T dO
      bwd_mma_ts<D>(tdK, tdP, sq, accum);   // dK += dS^T Q
      mma_commit(bar_mma);
    }
    __syncwarp();
    accum = 1;
    if (!cta_wait(bar_mma, mma_ph, abort_flag, p.timeout_ns)) { ok = false; break; }
    mma_ph ^= 1;
    tc_fence_after();
    ++n;
  }
  // Epilogue: dK (times scale) and dV rows of this key tile.  TMEM loads are
  // warp-collective; only the stores are guarded per row.
  if (ok) {
    const bool valid = y < p.c;
    const size_t row = (size_t)bh * p.N + (size_t)kb * p.c + (size_t)(valid ? y : 0);
#pragma unroll 1
    for (int q = 0; q < D / 32; ++q) {
      uint32_t r[32];
      if (accum) {
        tmem_ld32(tdK + lane_off + q * 32, r);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) r[i] = 0u;
      }
      if (valid) store_row32(p.dk + row * D + q * 32, r, p.scale);
      if (accum) {
        tmem_ld32(tdV + lane_off + q * 32, r);
        tmem_wait_ld();
      }
      if (valid) store_row32(p.dv + row * D + q * 32, r, 1.f);
    }
  }
  // Drain: every issued load and MMA must have completed before exit.
  if (tid == 0) {
    volatile int no_abort = 0;
    mma_commit(bar_mma);
    mbar_wait(bar_mma, mma_ph, &no_abort, p.timeout_ns);
    if (!fixed_done) mbar_wait(bar_fixed, 0, &no_abort, p.timeout_ns);
    for (int b2 = 0; b2 < 2; ++b2)
      if (issued[b2] > consumed[b2])
        mbar_wait(bar_ld0 + 8 * b2, (issued[b2] - 1) & 1, &no_abort, p.timeout_ns);
  }
  tc_fence_before();
  __syncthreads();
  if (tid == 0 && *abort_flag && p.fault) atomicOr(p.fault, 4u);
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ----------------------------------------------------------------- dQ
// Work item: query tile qt of shard j of (b, h); key tiles in ring order
// (block (j - r) mod P in round r), skipped tiles left out.
template <int D>
__global__ void __launch_bounds__(128, 1)
bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
              const BwdParams p) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const uint32_t bar_fixed = sb + C::kBar, bar_ld0 = bar_fixed + 8, bar_mma = bar_fixed + 24;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + C::kBar + 40);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kBar + 44);
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;

  const int T = p.T;
  const int qt = blockIdx.x % T;
  const int j = (blockIdx.x / T) % p.P;
  const int bh = blockIdx.x / (T * p.P);
  const int x0 = qt * kBM;
  const int x = x0 + tid;                       // this thread's query (local in shard j)
  const bool xvalid = x < p.c;
  const size_t xrow = (size_t)bh * p.N + (size_t)j * p.c + (size_t)(xvalid ? x : 0);
  const float lse2 = xvalid ? p.lse[xrow] * 1.4426950408889634f : INFINITY;
  const float drow = xvalid ? p.dvec[xrow] : 0.f;

  if (tid == 0) {
    mbar_init(bar_fixed, 1);
    mbar_init(bar_ld0, 1);
    mbar_init(bar_ld0 + 8, 1);
    mbar_init(bar_mma, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tslot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  const uint32_t tS = tmem, tdP = tmem + 128, tdQ = tmem + 256;
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;

  struct Cursor {
    int r, kt, kend, P, c, j, striped, causal, x0;
    BlockMask bm;
    TileSpan sp;
    int kb;
    __device__ bool next(int& okb, int& oy0, int& kind, BlockMask& m) {
      while (kt >= kend) {
        if (++r >= P) return false;
        kb = key_block(j, r, P);
        bm = block_mask(j, kb, striped, causal);
        sp = tile_span(bm, x0, c);
        kend = sp.part_end;
        kt = 0;
      }
      okb = kb;
      oy0 = kt * kBN;
      kind = tile_kind_at(sp, kt);
      m = bm;
      ++kt;
      return true;
    }
  };
  Cursor ld;
  ld.r = -1; ld.kt = 0; ld.kend = 0; ld.P = p.P; ld.c = p.c; ld.j = j; ld.striped = p.striped;
  ld.causal = p.causal; ld.x0 = x0; ld.kb = 0;
  Cursor cm = ld;

  bool ok = true;
  uint32_t issued[2] = {0, 0}, consumed[2] = {0, 0};
  if (tid == 0) {
    mbar_arrive_expect_tx(bar_fixed, 2 * C::kTile);
    load_tile<D>(sb + C::kFixed0, &tmQ, bar_fixed, x0, j, bh);
    load_tile<D>(sb + C::kFixed1, &tmdO, bar_fixed, x0, j, bh);
  }
  int lkb, ly0, lkind;
  BlockMask lbm;
  auto issue_load = [&](int buf, int kb, int y0) {
    if (tid == 0) {
      const uint32_t dst = sb + C::kStream + buf * 2 * C::kTile;
      mbar_arrive_expect_tx(bar_ld0 + 8 * buf, 2 * C::kTile);
      load_tile<D>(dst, &tmK, bar_ld0 + 8 * buf, y0, kb, bh);
      load_tile<D>(dst + C::kTile, &tmV, bar_ld0 + 8 * buf, y0, kb, bh);
    }
    ++issued[buf];
  };
  if (ld.next(lkb, ly0, lkind, lbm)) issue_load(0, lkb, ly0);
  bool fixed_done = cta_wait(bar_fixed, 0, abort_flag, p.timeout_ns);
  if (!fixed_done) ok = false;
  tc_fence_after();

  uint32_t n = 0, mma_ph = 0, accum = 0;
  int ckb, cy0, ckind;
  BlockMask cbm;
  while (ok && cm.next(ckb, cy0, ckind, cbm)) {
    const int buf = n & 1;
    __syncthreads();
    if (ld.next(lkb, ly0, lkind, lbm)) issue_load(buf ^ 1, lkb, ly0);
    if (!cta_wait(bar_ld0 + 8 * buf, consumed[buf] & 1, abort_flag, p.timeout_ns)) {
      ok = false;
      break;
    }
    ++consumed[buf];
    tc_fence_after();
    const uint32_t sk = sb + C::kStream + buf * 2 * C::kTile, sv = sk + C::kTile;
    if (warp == 0 && lane == 0) {
      bwd_mma_ss<D>(tS, sb + C::kFixed0, sk);     // S = Q K^T
      bwd_mma_ss<D>(tdP, sb + C::kFixed1, sv);    // dP = dO V^T
      mma_commit(bar_mma);
    }
    __syncwarp();
    if (!cta_wait(bar_mma, mma_ph, abort_flag, p.timeout_ns)) { ok = false; break; }
    mma_ph ^= 1;
    tc_fence_after();
    const int lim = xvalid ? ((ckind == TILE_PARTIAL) ? row_limit(cbm, x, cy0, p.c) : kBN) : 0;
#pragma unroll 1
    for (int ch = 0; ch < 4; ++ch) {
      uint32_t s32[32], d32[32];
      tmem_ld32(tS + lane_off + ch * 32, s32);
      tmem_ld32(tdP + lane_off + ch * 32, d32);
      tmem_wait_ld();
      uint32_t dk[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        float ds[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int col = ch * 32 + 2 * i + u;
          const float pv = (col < lim) ? bex2(fmaf(__uint_as_float(s32[2 * i + u]), p.c2, -lse2)) : 0.f;
          ds[u] = pv * (__uint_as_float(d32[2 * i + u]) - drow);
        }
        dk[i] = pack2(ds[0], ds[1]);
      }
      tmem_st16(tS + lane_off + ch * 16, dk);
    }
    tmem_wait_st();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0 && lane == 0) {
      bwd_mma_ts<D>(tdQ, tS, sk, accum);    // dQ += dS K
      mma_commit(bar_mma);
    }
    __syncwarp();
    accum = 1;
    if (!cta_wait(bar_mma, mma_ph, abort_flag, p.timeout_ns)) { ok = false; break; }
    mma_ph ^= 1;
    tc_fence_after();
    ++n;
  }
  if (ok) {
    __nv_bfloat16* dst = p.dq + xrow * D;
#pragma unroll 1
    for (int q = 0; q < D / 32; ++q) {
      uint32_t r[32];
      if (accum) {
        tmem_ld32(tdQ + lane_off + q * 32, r);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) r[i] = 0u;
      }
      if (xvalid) store_row32(dst + q * 32, r, p.scale);
    }
  }
  if (tid == 0) {
    volatile int no_abort = 0;
    mma_commit(bar_mma);
    mbar_wait(bar_mma, mma_ph, &no_abort, p.timeout_ns);
    if (!fixed_done) mbar_wait(bar_fixed, 0, &no_abort, p.timeout_ns);
    for (int b2 = 0; b2 < 2; ++b2)
      if (issued[b2] > consumed[b2])
        mbar_wait(bar_ld0 + 8 * b2, (issued[b2] - 1) & 1, &no_abort, p.timeout_ns);
  }
  tc_fence_before();
  __syncthreads();
  if (tid == 0 && *abort_flag && p.fault) atomicOr(p.fault, 8u);
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ host
static bool encode_map(CUtensorMap* map, const void* base, int64_t BH, int64_t N, int64_t c, int P,
                       int d) {
  PFN_encodeTiled enc = get_encode_tiled();
  if (!enc) return false;
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)c, (cuuint64_t)P, (cuuint64_t)BH};
  cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)c * d * 2, (cuuint64_t)N * d * 2};
  cuuint32_t box[4] = {64, (cuuint32_t)kBM, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
static ra_status launch_bwd(const BwdLaunch& a) {
  using C = BwdCfg<D>;
  const int64_t c = a.N / a.P;
  CUtensorMap tq, tk, tv, tdo;
  if (!encode_map(&tq, a.q, a.BH, a.N, c, a.P, D) || !encode_map(&tk, a.k, a.BH, a.N, c, a.P, D) ||
      !encode_map(&tv, a.v, a.BH, a.N, c, a.P, D) || !encode_map(&tdo, a.dout, a.BH, a.N, c, a.P, D))
    return RA_ERR_CUDA;
  static int attr_set[64] = {0};
  if (a.device < 64 && !attr_set[a.device]) {
    if (cudaFuncSetAttribute(bwd_dkdv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::kSmem) != cudaSuccess ||
        cudaFuncSetAttribute(bwd_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::kSmem) != cudaSuccess)
      return RA_ERR_CUDA;
    attr_set[a.device] = 1;
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
  bwd_dkdv_kernel<D><<<(unsigned)items, 128, C::kSmem, st>>>(tq, tk, tv, tdo, p);
  bwd_dq_kernel<D><<<(unsigned)items, 128, C::kSmem, st>>>(tq, tk, tv, tdo, p);
  return cudaGetLastError() == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

ra_status attn_bwd_launch(const BwdLaunch& a) {
  if (a.d == 128) return launch_bwd<128>(a);
  if (a.d == 64) return launch_bwd<64>(a);
  return RA_ERR_HEADDIM;
}

// ------------------------------------------- backward without allocation
// For callers that must not allocate device memory themselves: the scratch
// row vector D of the backward lives in this fixed device array instead of a
// caller workspace.  Every GPU that loads the library reserves it until the
// process exits.  All calls share it: two calls whose kernels overlap on the
// GPU (different streams, or devices sharing nothing but this library) race
// on it.  D is fully rewritten by every call, so nothing has to be cleared.
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
  }
  a.workspace = addr[a.device];
  return attn_bwd_launch(a);
}

}  // namespace ra
