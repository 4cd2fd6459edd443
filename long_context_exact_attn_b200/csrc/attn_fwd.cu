// Exact blockwise ring/striped attention forward for sm_100a (B200).
//
// What is computed (Ring Attention explainer "ICLR 2024論文解説: Ring
// Attention", ステップ2/ステップ3 and 実装例; Striped Attention review,
// 核心公式 / GetMask 函数 / 分块与分瓦片): for each virtual shard j, its query
// tiles stay resident while the key/value blocks arrive in ring order
// (round r brings block (j - r) mod P); each key tile is folded into the
// running row max m, row sum l and unnormalised output O by online softmax,
// and O is divided by l once at the end.  Tiles that the block's causal
// mask hides completely are never loaded or computed.
//
// Kernel organisation (one persistent CTA per SM, 384 threads):
//   warps 0-3  softmax warpgroup for query tile 0 of the CTA's tile pair
//   warps 4-7  softmax warpgroup for query tile 1
//   warp  8    TMA producer: Q tile pair once per work item, then K and V
//              tiles into a ring of shared-memory slots
//   warp  9    tcgen05 issuer (warp-uniform, one elected lane issues) and
//              TMEM owner
//   warps 10-11 idle: with warps 8-9 they form the warpgroup that hands
//              registers to the softmax warpgroups (setmaxnreg)
// Variants of the same kernel: the zigzag layout (template parameter ZZ:
// each key block walked as its two chunks), token-order addressing (the
// layout's permutation applied in the TMA coordinates and the epilogue's
// rows), float32 output, and a single-block mode (one query shard against
// one key block, the per-round step of a physical ring).
// Tensor memory (512 columns x 128 lanes x 32 bit):
//   [0,128)  S0 = Q0 K^T (fp32), later overwritten in place by P0 (bf16x2,
//            columns [0,64)) which is the A operand of P0 V
//   [128,256) S1 / P1
//   [256,256+D) O0 accumulator (fp32),  [256+D, 256+2D) O1
// With the 32x32b TMEM access pattern thread i of a softmax warpgroup owns
// query row i: the row max and row sum are plain per-thread reductions.
//
// The two query tiles are ping-ponged on the tensor core: while warpgroup 0
// turns S0 into P0, the tensor core runs P1 V and the next Q1 K^T, and vice
// versa.  Every wait is bounded (see mbar_wait); on a timeout the kernel
// raises an abort flag, drains its own MMAs and TMA loads, frees TMEM and
// returns, recording the fault in the library's device fault word.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <atomic>
#include <cstring>
#include <map>
#include <memory>
#include <mutex>
#include <type_traits>
#include <vector>

#include "exp2_poly.h"
#include "ra_internal.h"
#include "ra_ptx.cuh"
#include "ra_tiles.cuh"

namespace ra {

__device__ unsigned int g_device_fault = 0;

// Phase profile (profiling build only: RA_PROFILE=1, a library of its own).
// Each softmax warp (slots 0-7) and the MMA warp (slot 8) of the first
// kProfCtas CTAs accumulate clock64 cycles per phase of their loop; the
// counters are read and cleared through ra_fwd_phase_profile.  Without
// RA_PROFILE every marker below compiles to nothing.
#ifndef RA_PROFILE
#define RA_PROFILE 0
#endif
#if RA_PROFILE
__device__ unsigned long long g_fwd_profile[kProfCtas * kProfSlots * kProfPhases];
// 32-bit counts per launch and warp (a warp's launch is far below 2^32
// cycles), added into the 64-bit counters at the end: fewer registers.
struct PhaseClock {
  uint32_t acc[kProfPhases];
  uint32_t last;
  __device__ __forceinline__ void start() {
#pragma unroll
    for (int i = 0; i < kProfPhases; ++i) acc[i] = 0;
    last = (uint32_t)clock64();
  }
  __device__ __forceinline__ void mark(int i) {
    const uint32_t t = (uint32_t)clock64();
    acc[i] += t - last;
    last = t;
  }
  __device__ __forceinline__ void count() { acc[kProfPhases - 1] += 1; }
  __device__ __forceinline__ void store(int slot) {
    if ((threadIdx.x % 32) == 0 && blockIdx.x < kProfCtas)
#pragma unroll
      for (int i = 0; i < kProfPhases; ++i)
        atomicAdd(&g_fwd_profile[(blockIdx.x * kProfSlots + slot) * kProfPhases + i],
                  (unsigned long long)acc[i]);
  }
};
#define RA_PHASE_START(c) (c).start()
#define RA_PHASE(c, i) (c).mark(i)
#define RA_PHASE_COUNT(c) (c).count()
#define RA_PHASE_STORE(c, slot) (c).store(slot)
#else
struct PhaseClock {};
#define RA_PHASE_START(c) ((void)0)
#define RA_PHASE(c, i) ((void)0)
#define RA_PHASE_COUNT(c) ((void)0)
#define RA_PHASE_STORE(c, slot) ((void)0)
#endif

// Work lists for small problems (see WorkLists): capacity, and the largest
// problem (items of all heads and shards) that uses them.  At N = 8192
// (512 items) the whole K/V fits in L2 and the lists only rebalance work;
// at N = 131072 (4096 items) they would break the head-major order that
// keeps the running CTAs in one head's K/V (measured 13 % slower).
constexpr int kMaxListItems = 1024;
constexpr int kMaxListCtas = 160;
constexpr int kListItemsUsed = 1024;

struct AttnParams {
  __nv_bfloat16* o;
  float* lse;
  int o_f32;          // O written as float32 (o then points to float rows)
  int o_v8;           // o is 32-byte aligned: O rows written in 32-byte stores
  int tok;            // q, k, v, o, lse in token order: the layout's permutation
                      // is applied in the TMA coordinates and the epilogue
  int BH;             // B * H
  int N;              // sequence length
  int c;              // shard length N / P
  int P;              // shards
  int npairs;         // query-tile pairs per shard = ceil(ceil(c/128) / 2)
  int striped;        // layout: striped
  int zigzag;         // layout: zigzag (c a multiple of 512)
  int causal;
  int groups;         // shard groups (owner schedule) or 1 (free schedule)
  int ctas_per_group;
  int helpers;        // owner schedule: CTAs on the SMs left over by the groups
  int ceded;          // items at the end of every group's list that the helpers take
  float c2;           // scale * log2(e)
  unsigned long long timeout_ns;        // limit of every main-loop wait
  unsigned long long drain_timeout_ns;  // limit of the waits that drain the CTA's own
                                        // MMAs and TMA loads before it exits
  int withhold_first_s;                 // self-test: the first S-ready signal of every
                                        // CTA is never sent (the waits must give up)
  // Single-block mode (blk_kb >= 0): Q is one query shard, K/V one key
  // block (both stored as shard 0 of a P = 1 tensor); the mask is the
  // GetMask of the real pair (blk_j, blk_kb).
  int blk_j, blk_kb;
};

// Per-CTA work lists of the owner schedule (the kernel instance that takes
// them): CTA b processes the items item[start[b] .. start[b+1]) of its
// group, in that order.  The other instances take NoLists and deal a
// group's items to its CTAs in snake order.
struct WorkLists {
  uint16_t start[kMaxListCtas + 1];
  uint16_t item[kMaxListItems];
};
struct NoLists {};

template <int D>
struct Cfg {
  static constexpr int kTileBytes = kBM * D * 2;           // one Q, K or V tile
  static constexpr int kChunks = D / 64;                   // 128-byte swizzle chunks per row
  static constexpr int kSlots = (D == 128) ? 5 : 10;       // K/V ring slots
  static constexpr int kQOff = 0;
  static constexpr int kRingOff = 2 * kTileBytes;
  static constexpr int kBarOff = kRingOff + kSlots * kTileBytes;
  // barriers: q_full, q_empty, full[kSlots], empty[kSlots], s_full[2],
  // p_full[2] (first part of P ready), p_full2[2] (the rest),
  // o_full[2], o_free[2], drain
  static constexpr int kNumBars = 2 + 2 * kSlots + 10 + 1;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kSmemBytes = kMiscOff + 16 + 1024;  // + alignment slack
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO0 = 256, kColO1 = 256 + D;
  static constexpr int kThreads = 384;
  // Register split (setmaxnreg, per warpgroup): the CTA is launched with
  // 384 x kRegsLaunch registers; the warpgroup of producer, MMA and two idle
  // warps gives some back (down to kRegsLow) and the two softmax warpgroups
  // take them (up to kRegsHigh).  The split may not need more than the launch
  // holds, or the softmax warpgroups' request would wait forever; the host
  // checks the built kernel's register count before the first launch.
  static constexpr int kRegsLaunch = 168, kRegsLow = 112, kRegsHigh = 192;
  static_assert(256 * kRegsHigh + 128 * kRegsLow <= kThreads * kRegsLaunch,
                "register split must fit in the launched registers");
};

// ------------------------------------------------------------ work items
struct Item {
  int bh, j, pair;
};

// Items of a shard group.  Head-major, so that the CTAs running at the same
// time share one head's K/V blocks in L2; inside a head, work is
// non-increasing (causal striped and non-causal work grows with the pair's
// local index, causal contiguous work with the shard index first), so each
// head's list ends with its lightest items.
__device__ __forceinline__ bool item_at(const AttnParams& p, int g, int u, Item& it) {
  const int n_sh = (p.P - g + p.groups - 1) / p.groups;   // shards g, g+groups, ...
  const int per_head = p.npairs * n_sh;
  if (u >= per_head * p.BH) return false;
  it.bh = u / per_head;
  const int rem = u - it.bh * per_head;
  if (p.causal && !p.striped) {
    const int sh_rank = rem / p.npairs;
    it.j = g + (n_sh - 1 - sh_rank) * p.groups;
    it.pair = p.npairs - 1 - (rem - sh_rank * p.npairs);
  } else {
    const int pr = rem / n_sh;
    it.pair = p.npairs - 1 - pr;
    it.j = g + (rem - pr * n_sh) * p.groups;
  }
  return true;
}

// Items of group g.
__device__ __forceinline__ int group_items(const AttnParams& p, int g) {
  return p.npairs * ((p.P - g + p.groups - 1) / p.groups) * p.BH;
}

// k-th item of this CTA: snake order over the group's members, except the
// group's last `ceded` items (its lightest), which go to the helper CTAs.
// Helper h takes them from groups h, h + helpers, h + 2 helpers, ...
__device__ __forceinline__ bool cta_item(const AttnParams& p, const NoLists&, int k, Item& it) {
  const int G = p.ctas_per_group;
  const int base = p.groups * G;
  if ((int)blockIdx.x >= base) {
    if (p.ceded == 0) return false;
    const int gi = k / p.ceded;
    const int g = (int)blockIdx.x - base + gi * p.helpers;
    if (g >= p.groups) return false;
    return item_at(p, g, group_items(p, g) - p.ceded + (k - gi * p.ceded), it);
  }
  const int g = blockIdx.x / G;
  const int m = blockIdx.x % G;
  const int u = k * G + ((k & 1) ? (G - 1 - m) : m);
  if (u >= group_items(p, g) - p.ceded) return false;
  return item_at(p, g, u, it);
}

// k-th item of this CTA from its work list.
__device__ __forceinline__ bool cta_item(const AttnParams& p, const WorkLists& wl, int k,
                                         Item& it) {
  const int g = blockIdx.x / p.ctas_per_group;
  if (g >= p.groups) return false;
  const int idx = wl.start[blockIdx.x] + k;
  if (idx >= wl.start[blockIdx.x + 1]) return false;
  return item_at(p, g, wl.item[idx], it);
}

// The key tiles met by a query-tile pair, in ring order.  Per block the two
// query tiles' FULL / PARTIAL / SKIP thresholds are computed once; per tile
// the classification is two compares each.  In the zigzag layout (ZZ) every
// block is walked as its two chunks (the thresholds are per chunk pair, in
// chunk-local rows); mxo() / myo() / mc() give the partial-tile mask its
// coordinates: query x and key y0 of the shard are x - mxo() and y0 - myo()
// in a block of length mc().
template <bool ZZ>
struct TileSeq {
  int j, P, c, striped, causal, blk_j, blk_kb;
  int x0;                   // first row of query tile 0
  int r, kt, kend;
  TileSpan s0, s1;
  BlockMask bm;
  int kb;
  int zx, zy, kt_off;       // zigzag: chunk offsets of the current chunk pair

  __device__ __forceinline__ int mxo() const { return ZZ ? zx : 0; }
  __device__ __forceinline__ int myo() const { return ZZ ? zy : 0; }
  __device__ __forceinline__ int mc() const { return ZZ ? (c >> 1) : c; }

  __device__ __forceinline__ void init(const AttnParams& p, const Item& it) {
    j = it.j; P = p.P; c = p.c; striped = p.striped; causal = p.causal;
    blk_j = p.blk_j; blk_kb = p.blk_kb;
    x0 = it.pair * 2 * kBM;
    r = -1; kt = 0; kend = 0;
    zx = 0; zy = 0; kt_off = 0;
  }
  // Next tile; false at the end.  Fills block index, key start and the kind
  // of the tile for each of the two query tiles.
  __device__ __forceinline__ bool next(int& kb_out, int& y0, int& k0, int& k1, BlockMask& m) {
    while (kt >= kend) {
      if (ZZ) {
        // sub-round r = 2 * round + chunk half of the key block
        if (++r >= 2 * P) return false;
        kb = key_block(j, r >> 1, P);
        const int h = c >> 1, hk = r & 1;
        zx = x0 < h ? 0 : h;
        zy = hk * h;
        bm = chunk_mask(zz_chunk(j, x0, h, P), hk ? 2 * P - 1 - kb : kb, causal);
        s0 = tile_span(bm, x0 - zx, h);
        s1 = tile_span(bm, x0 - zx + kBM, h);
        kt_off = hk * (h / kBN);
      } else {
        if (++r >= P) return false;
        if (blk_kb >= 0) {
          kb = 0;
          bm = block_mask(blk_j, blk_kb, striped, causal);
        } else {
          kb = key_block(j, r, P);
          bm = block_mask(j, kb, striped, causal);
        }
        s0 = tile_span(bm, x0, c);
        s1 = tile_span(bm, x0 + kBM, c);
      }
      kend = s0.part_end > s1.part_end ? s0.part_end : s1.part_end;
      kt = 0;
    }
    kb_out = kb;
    y0 = ((ZZ ? kt_off : 0) + kt) * kBN;
    k0 = tile_kind_at(s0, kt);
    k1 = tile_kind_at(s1, kt);
    m = bm;
    ++kt;
    return true;
  }
};

// mbar_wait for a whole warp: the result is the same in every lane (a lane
// that gave up makes the warp give up).
__device__ __forceinline__ bool wmbar_wait(uint32_t bar, uint32_t parity, volatile int* abort,
                                           uint64_t limit_ns) {
  const bool ok = mbar_wait(bar, parity, abort, limit_ns);
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Max of 128 scores: eight independent chains of 3-input max.
__device__ __forceinline__ float row_max128(const float (&s)[128]) {
  float mx8[8];
#pragma unroll
  for (int a = 0; a < 8; ++a) {
    float acc = fmax3(s[a], s[a + 8], s[a + 16]);
#pragma unroll
    for (int kq = 3; kq < 15; kq += 2) acc = fmax3(acc, s[a + 8 * kq], s[a + 8 * kq + 8]);
    mx8[a] = fmaxf(acc, s[a + 120]);
  }
  return fmaxf(fmax3(mx8[0], mx8[1], mx8[2]),
               fmaxf(fmax3(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
}

// Packed pairs of fp32 (sm_100 f32x2 arithmetic: one instruction, two lanes).
__device__ __forceinline__ uint64_t f2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void unf2(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

// r[i] *= alpha for 32 fp32 values held as raw bits (packed f32x2 multiplies).
__device__ __forceinline__ void scale_row32(uint32_t (&r)[32], uint64_t a2) {
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    uint64_t v = f2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
    asm("mul.rn.f32x2 %0, %0, %1;" : "+l"(v) : "l"(a2));
    float lo, hi;
    unf2(v, lo, hi);
    r[2 * i] = __float_as_uint(lo);
    r[2 * i + 1] = __float_as_uint(hi);
  }
}

// 2^x for a pair of fp32 values on the FMA/ALU pipes instead of the MUFU:
// x = j + f with j = round(x) (added to the exponent field) and f in
// [-1/2, 1/2] (minimax polynomial of exp2_poly.h).  x is clamped below at
// -125 so that the exponent field stays normal; 2^-125 in place of 0 for a
// masked score changes no sum at fp32 resolution.
__device__ __forceinline__ void exp2_poly2(uint64_t x2, float& r0, float& r1) {
  float x0, x1;
  unf2(x2, x0, x1);
  x0 = fmaxf(x0, -125.f);
  x1 = fmaxf(x1, -125.f);
  const uint64_t magic = f2(12582912.f, 12582912.f);        // 1.5 * 2^23
  const uint64_t t = fadd2(f2(x0, x1), magic);               // round to nearest integer
  const uint64_t j = fadd2(t, f2(-12582912.f, -12582912.f));
  float j0, j1;
  unf2(j, j0, j1);
  const uint64_t fr = fadd2(f2(x0, x1), f2(-j0, -j1));
  uint64_t p = ffma2(fr, f2(RA_EXP2_C3, RA_EXP2_C3), f2(RA_EXP2_C2, RA_EXP2_C2));
  p = ffma2(p, fr, f2(RA_EXP2_C1, RA_EXP2_C1));
  p = ffma2(p, fr, f2(1.f, 1.f));
  float p0, p1, t0, t1;
  unf2(p, p0, p1);
  unf2(t, t0, t1);
  r0 = __int_as_float(__float_as_int(p0) + (__float_as_int(t0) << 23));
  r1 = __int_as_float(__float_as_int(p1) + (__float_as_int(t1) << 23));
}

// S (TMEM, fp32 128 x 128) = Q tile (smem) x K tile (smem)^T; both K-major
// with 128-byte swizzle, d/16 MMAs of K = 16.
template <int D>
__device__ __forceinline__ void mma_qk(uint32_t s_tmem, uint32_t qa, uint32_t ka) {
  constexpr uint32_t idesc = idesc_bf16_f32(kBM, kBN, 0, 0);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = (kk / 4) * 16384 + (kk % 4) * 32;
    mma_ss_w(s_tmem, smem_desc_sw128(qa + off, 16, 1024), smem_desc_sw128(ka + off, 16, 1024),
             idesc, kk > 0);
  }
}

// O (TMEM, fp32 128 x D) (+)= P (TMEM, bf16 128 x 128) x V tile (smem, 128
// keys x D, D contiguous = MN-major, 128-byte swizzle): 8 MMAs of K = 16 keys.
template <int D, int KK0 = 0, int KK1 = kBN / 16>
__device__ __forceinline__ void mma_pv(uint32_t o_tmem, uint32_t p_tmem, uint32_t va,
                                       uint32_t acc) {
  constexpr uint32_t idesc = idesc_bf16_f32(kBM, D, 0, 1);
#pragma unroll
  for (int kk = KK0; kk < KK1; ++kk)
    mma_ts_w(o_tmem, p_tmem + kk * 8, smem_desc_sw128(va + kk * 2048, 16384, 1024), idesc,
             (acc | (uint32_t)kk) != 0);
}

// One pair in kPolyEvery of each row's exps goes to the FMA-pipe polynomial
// (0: all on the MUFU).
#ifndef RA_POLY_EVERY
#define RA_POLY_EVERY 0
#endif
constexpr int kPolyEvery = RA_POLY_EVERY;

// TMA coordinates (second, third) of the 128-row tile of shard `shard`
// starting at local row x0.  Layout order: (x0, shard) of a [BH, P, c, d]
// map.  Token order: striped rows are token x*P + shard, read through a
// [BH, c, P, d] map as (shard, x0); zigzag rows lie in chunk shard or
// 2P-1-shard of a [BH, 2P, h, d] map; contiguous token order is layout order.
template <bool ZZ>
__device__ __forceinline__ void tile_coord(const AttnParams& p, int shard, int x0, int& c1,
                                           int& c2) {
  c1 = x0;
  c2 = shard;
  if (!p.tok) return;
  if (p.striped) {
    c1 = shard;
    c2 = x0;
  } else if (ZZ) {
    const int h = p.c >> 1;
    if (x0 >= h) {
      c1 = x0 - h;
      c2 = 2 * p.P - 1 - shard;
    }
  }
}

// Row of (shard j, local row x) in the output tensors' order.
template <bool ZZ>
__device__ __forceinline__ size_t out_row(const AttnParams& p, int bh, int j, int x) {
  size_t t;
  if (!p.tok) {
    t = (size_t)j * p.c + x;
  } else if (p.striped) {
    t = (size_t)x * p.P + j;
  } else if (ZZ) {
    const int h = p.c >> 1;
    t = x < h ? (size_t)j * h + x : (size_t)(2 * p.P - 1 - j) * h + (x - h);
  } else {
    t = (size_t)j * p.c + x;
  }
  return (size_t)bh * p.N + t;
}

// 32 bytes (8 words) to global memory in one store; dst 32-byte aligned.
__device__ __forceinline__ void st_global_v8(void* dst, const uint32_t* w) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(dst), "r"(w[0]),
               "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
               : "memory");
}

// Per-warpgroup register budget (setmaxnreg; every warp of the warpgroup
// executes the same instruction).
template <int N>
__device__ __forceinline__ void reg_alloc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void reg_dealloc() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

template <int D, bool ZZ, class Lists>
__global__ void __launch_bounds__(384, 1)
attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const AttnParams p,
                const __grid_constant__ Lists wl) {
  using C = Cfg<D>;
  // P is published in two parts: keys [0, 32 kPub) and the rest; P V runs
  // in the same two parts (2 kPub and 8 - 2 kPub k-steps of 16 keys).  The
  // work-list instance (small striped problems: short rows, where the O
  // rescale before the first part is frequent) publishes after 96 keys, the
  // other instances after 64 (measured: +1.3 % and -0.5 % respectively with
  // 96 at N = 8192 and N = 262144).
  constexpr int kPub = std::is_same<Lists, WorkLists>::value ? 3 : 2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + C::kQOff;
  const uint32_t sRing = sbase + C::kRingOff;
  const uint32_t bars = sbase + C::kBarOff;
  const uint32_t bar_q_full = bars + 0 * 8;
  const uint32_t bar_q_empty = bars + 1 * 8;
  auto bar_full = [&](int s) { return bars + (2 + s) * 8; };
  auto bar_empty = [&](int s) { return bars + (2 + C::kSlots + s) * 8; };
  const uint32_t bar_s_full = bars + (2 + 2 * C::kSlots) * 8;   // [2]
  const uint32_t bar_p_full = bar_s_full + 16;                  // [2]
  const uint32_t bar_p_full2 = bar_p_full + 16;                 // [2]
  const uint32_t bar_o_full = bar_p_full2 + 16;                 // [2]
  const uint32_t bar_o_free = bar_o_full + 16;                  // [2]
  const uint32_t bar_drain = bar_o_free + 16;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 4);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    mbar_init(bar_q_full, 1);
    mbar_init(bar_q_empty, 1);
    for (int s = 0; s < C::kSlots; ++s) {
      mbar_init(bar_full(s), 1);
      mbar_init(bar_empty(s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar_s_full + 8 * t, 1);
      mbar_init(bar_p_full + 8 * t, 4);     // one arrival per softmax warp
      mbar_init(bar_p_full2 + 8 * t, 4);
      mbar_init(bar_o_full + 8 * t, 1);
      mbar_init(bar_o_free + 8 * t, 4);
    }
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // Register budgets: each warpgroup executes one setmaxnreg, all its warps
  // at the same instruction, at the top of the branch that holds all of its
  // code (so that the compiler allocates every branch within its budget).
  // Warps 10 and 11 only complete the third warpgroup.
  if (warp >= 8) {
  reg_dealloc<C::kRegsLow>();
  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t n_loads = 0;
      Item it;
      bool ok = true;
      for (int k = 0; ok && cta_item(p, wl, k, it); ++k) {
        if (!mbar_wait(bar_q_empty, (k & 1) ^ 1, abort_flag, p.timeout_ns)) { ok = false; break; }
        mbar_arrive_expect_tx(bar_q_full, 2 * C::kTileBytes);
        const int x0 = it.pair * 2 * kBM;
        for (int t = 0; t < 2; ++t) {
          int c1, c2;
          tile_coord<ZZ>(p, it.j, x0 + t * kBM, c1, c2);
          for (int ch = 0; ch < C::kChunks; ++ch)
            tma_load_4d(sQ + t * C::kTileBytes + ch * 16384, &tmQ, bar_q_full, ch * 64, c1, c2,
                        it.bh);
        }
        TileSeq<ZZ> seq;
        seq.init(p, it);
        int kb, y0, k0, k1;
        BlockMask bm;
        while (seq.next(kb, y0, k0, k1, bm)) {
          for (int kv = 0; kv < 2; ++kv) {
            const int s = n_loads % C::kSlots;
            const uint32_t ph = (n_loads / C::kSlots) & 1;
            if (!mbar_wait(bar_empty(s), ph ^ 1, abort_flag, p.timeout_ns)) { ok = false; break; }
            mbar_arrive_expect_tx(bar_full(s), C::kTileBytes);
            const CUtensorMap* tm = kv ? &tmV : &tmK;
            int c1, c2;
            tile_coord<ZZ>(p, kb, y0, c1, c2);
            for (int ch = 0; ch < C::kChunks; ++ch)
              tma_load_4d(sRing + s * C::kTileBytes + ch * 16384, tm, bar_full(s), ch * 64, c1,
                          c2, it.bh);
            ++n_loads;
          }
          if (!ok) break;
        }
      }
      // Every load this thread issued must have landed before the CTA exits.
      volatile int no_abort = 0;
      const uint32_t first = n_loads > (uint32_t)C::kSlots ? n_loads - C::kSlots : 0;
      for (uint32_t n = first; n < n_loads; ++n)
        mbar_wait(bar_full(n % C::kSlots), (n / C::kSlots) & 1, &no_abort, p.drain_timeout_ns);
    }
    __syncwarp();
  } else if (warp == 9) {
    // ---------------------------------------------------------- MMA issuer
    // The whole warp runs this loop with identical values (warp-uniform, so
    // addresses and descriptors stay in uniform registers); each MMA and
    // commit is issued by one elected lane.  The issue rate of this warp is
    // on the tensor core's critical path.
    {
      const uint32_t tS0 = tmem + C::kColS0, tS1 = tmem + C::kColS1;
      const uint32_t tO0 = tmem + C::kColO0, tO1 = tmem + C::kColO1;
      const uint32_t sQ0 = sQ, sQ1 = sQ + C::kTileBytes;
      const uint32_t s_full0 = bar_s_full, s_full1 = bar_s_full + 8;
      const uint32_t p_full0 = bar_p_full, p_full1 = bar_p_full + 8;
      const uint32_t p_full2_0 = bar_p_full2, p_full2_1 = bar_p_full2 + 8;
      bool withhold = p.withhold_first_s != 0;
      const uint32_t o_free0 = bar_o_free, o_free1 = bar_o_free + 8;
      const uint32_t full0 = bars + 2 * 8, empty0 = bars + (2 + C::kSlots) * 8;
      uint32_t slot = 0, phase = 0;       // next K/V tile to consume, in producer order
      uint32_t pc0 = 0, pc1 = 0;          // p_full phases consumed per query tile
      // o_free phases consumed per query tile.  The waits catch up one phase
      // at a time: a parity wait is only unambiguous one phase ahead, and a
      // query tile without key tiles in an item skips its lazy wait.
      uint32_t of0 = 0, of1 = 0;
      PhaseClock mc;
      (void)mc;
      RA_PHASE_START(mc);
      Item it;
      bool ok = true;
      for (int k = 0; ok && cta_item(p, wl, k, it); ++k) {
        if (!wmbar_wait(bar_q_full, k & 1, abort_flag, p.timeout_ns)) { ok = false; break; }
        TileSeq<ZZ> seq;
        seq.init(p, it);
        int kb, y0, c0, c1, n0 = TILE_SKIP, n1 = TILE_SKIP;
        BlockMask bm;
        uint32_t acc0 = 0, acc1 = 0;
        bool have = seq.next(kb, y0, c0, c1, bm);
        if (!have) {
          // no visible key tile for either query tile (only possible for a
          // single block): release the item without touching O, once the
          // previous item's epilogue has passed (keeps o_full one phase ahead
          // of the softmax warps at most)
          bool okw = true;
          while (okw && of0 < (uint32_t)k) okw = wmbar_wait(o_free0, of0++ & 1, abort_flag, p.timeout_ns);
          while (okw && of1 < (uint32_t)k) okw = wmbar_wait(o_free1, of1++ & 1, abort_flag, p.timeout_ns);
          if (!okw) { ok = false; break; }
          mma_commit_w(bar_o_full + 0);
          mma_commit_w(bar_o_full + 8);
          mma_commit_w(bar_q_empty);
          continue;
        }
        // prologue: Q K^T of the first tile
        uint32_t kslot = slot;
        if (!wmbar_wait(full0 + 8 * kslot, phase, abort_flag, p.timeout_ns)) { ok = false; break; }
        tc_fence_after();
        const uint32_t ka0 = sRing + kslot * C::kTileBytes;
        if (c0 != TILE_SKIP) {
          mma_qk<D>(tS0, sQ0, ka0);
          if (!withhold) mma_commit_w(s_full0);
          withhold = false;
        }
        if (c1 != TILE_SKIP) { mma_qk<D>(tS1, sQ1, ka0); mma_commit_w(s_full1); }
        mma_commit_w(empty0 + 8 * kslot);
        if (++slot == C::kSlots) { slot = 0; phase ^= 1; }
        while (have) {
          const bool more = seq.next(kb, y0, n0, n1, bm);
          const uint32_t vslot = slot, vph = phase;
          if (++slot == C::kSlots) { slot = 0; phase ^= 1; }
          uint32_t nkslot = 0;
          RA_PHASE(mc, 0);
          if (more) {
            nkslot = slot;
            if (!wmbar_wait(full0 + 8 * nkslot, phase, abort_flag, p.timeout_ns)) { ok = false; break; }
            if (++slot == C::kSlots) { slot = 0; phase ^= 1; }
          }
          RA_PHASE(mc, 1);
          if (!wmbar_wait(full0 + 8 * vslot, vph, abort_flag, p.timeout_ns)) { ok = false; break; }
          RA_PHASE(mc, 2);
          const uint32_t va = sRing + vslot * C::kTileBytes;
          const uint32_t nka = sRing + nkslot * C::kTileBytes;
          // query tile 0: P0 V, then the next Q0 K^T into the freed S0/P0 columns
          if (c0 != TILE_SKIP) {
            bool okw = true;
            RA_PHASE(mc, 0);
            while (okw && of0 < (uint32_t)k) okw = wmbar_wait(o_free0, of0++ & 1, abort_flag, p.timeout_ns);
            if (!okw) { ok = false; break; }
            RA_PHASE(mc, 5);
            // P in two parts: the first 2 kPub k-steps start while the
            // softmax is still producing the rest.
            if (!wmbar_wait(p_full0, pc0 & 1, abort_flag, p.timeout_ns)) { ok = false; break; }
            RA_PHASE(mc, 3);
            tc_fence_after();
            mma_pv<D, 0, 2 * kPub>(tO0, tS0, va, acc0);
            RA_PHASE(mc, 0);
            if (!wmbar_wait(p_full2_0, pc0 & 1, abort_flag, p.timeout_ns)) { ok = false; break; }
            RA_PHASE(mc, 4);
            ++pc0;
            tc_fence_after();
            mma_pv<D, 2 * kPub, 8>(tO0, tS0, va, 1);
            acc0 = 1;
          }
          if (more && n0 != TILE_SKIP) { tc_fence_after(); mma_qk<D>(tS0, sQ0, nka); mma_commit_w(s_full0); }
          // query tile 1
          if (c1 != TILE_SKIP) {
            bool okw = true;
            RA_PHASE(mc, 0);
            while (okw && of1 < (uint32_t)k) okw = wmbar_wait(o_free1, of1++ & 1, abort_flag, p.timeout_ns);
            if (!okw) { ok = false; break; }
            RA_PHASE(mc, 5);
            // P in two parts: the first 2 kPub k-steps start while the
            // softmax is still producing the rest.
            if (!wmbar_wait(p_full1, pc1 & 1, abort_flag, p.timeout_ns)) { ok = false; break; }
            RA_PHASE(mc, 3);
            tc_fence_after();
            mma_pv<D, 0, 2 * kPub>(tO1, tS1, va, acc1);
            RA_PHASE(mc, 0);
            if (!wmbar_wait(p_full2_1, pc1 & 1, abort_flag, p.timeout_ns)) { ok = false; break; }
            RA_PHASE(mc, 4);
            ++pc1;
            tc_fence_after();
            mma_pv<D, 2 * kPub, 8>(tO1, tS1, va, 1);
            acc1 = 1;
          }
          mma_commit_w(empty0 + 8 * vslot);
          if (more && n1 != TILE_SKIP) { tc_fence_after(); mma_qk<D>(tS1, sQ1, nka); mma_commit_w(s_full1); }
          if (more) mma_commit_w(empty0 + 8 * nkslot);
          have = more;
          c0 = n0;
          c1 = n1;
          RA_PHASE(mc, 0);
          RA_PHASE_COUNT(mc);
        }
        if (!ok) break;
        {
          bool okw = true;
          while (okw && of0 < (uint32_t)k) okw = wmbar_wait(o_free0, of0++ & 1, abort_flag, p.timeout_ns);
          while (okw && of1 < (uint32_t)k) okw = wmbar_wait(o_free1, of1++ & 1, abort_flag, p.timeout_ns);
          if (!okw) { ok = false; break; }
        }
        mma_commit_w(bar_o_full + 0);
        mma_commit_w(bar_o_full + 8);
        mma_commit_w(bar_q_empty);
      }
      RA_PHASE(mc, 0);
      RA_PHASE_STORE(mc, 8);
      // All MMAs issued by this thread must be complete before TMEM is freed.
      mma_commit_w(bar_drain);
      volatile int no_abort = 0;
      wmbar_wait(bar_drain, 0, &no_abort, p.drain_timeout_ns);
    }
    __syncwarp();
  }
  } else {
    // ----------------------------------------------------- softmax warpgroups
    reg_alloc<C::kRegsHigh>();
    const int t = warp / 4;                 // query tile of the pair
    const int wq = warp % 4;                // TMEM lane quarter
    const int row = wq * 32 + lane;         // row within the query tile
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t tS = tmem + (t ? C::kColS1 : C::kColS0) + lane_off;
    const uint32_t tO = tmem + (t ? C::kColO1 : C::kColO0) + lane_off;
    const uint32_t my_s_full = bar_s_full + 8 * t;
    const uint32_t my_p_full = bar_p_full + 8 * t;
    const uint32_t my_p_full2 = bar_p_full2 + 8 * t;
    const uint32_t my_o_full = bar_o_full + 8 * t;
    const uint32_t my_o_free = bar_o_free + 8 * t;
    const float c2 = p.c2;
    uint32_t s_cnt = 0;
    PhaseClock pc;
    (void)pc;
    RA_PHASE_START(pc);
    Item it;
    bool ok = true;
    for (int k = 0; ok && cta_item(p, wl, k, it); ++k) {
      TileSeq<ZZ> seq;
      seq.init(p, it);
      const int x = it.pair * 2 * kBM + t * kBM + row;   // local query row in shard
      float m2 = -INFINITY;   // running max, in units of log2 (scores * c2)
      float l = 0.f;    // row sum of the probabilities (fp32)
      bool acc = false;
      int kb, y0, k0, k1;
      BlockMask bm;
      while (seq.next(kb, y0, k0, k1, bm)) {
        const int kind = t ? k1 : k0;
        if (kind == TILE_SKIP) continue;
        // warp-uniform: a lane that gives up makes the whole warp give up, so
        // the warp-collective TMEM accesses and votes below never diverge
        RA_PHASE(pc, 0);
        if (!wmbar_wait(my_s_full, s_cnt & 1, abort_flag, p.timeout_ns)) { ok = false; break; }
        ++s_cnt;
        RA_PHASE(pc, 1);
        tc_fence_after();
        uint32_t sr[4][32];
#pragma unroll
        for (int q = 0; q < 4; ++q) tmem_ld32(tS + q * 32, sr[q]);
        tmem_wait_ld();
        float s[128];
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
          for (int i = 0; i < 32; ++i) s[q * 32 + i] = __uint_as_float(sr[q][i]);
        RA_PHASE(pc, 2);
        if (kind == TILE_PARTIAL) {
          const int lim = row_limit(bm, x - seq.mxo(), y0 - seq.myo(), seq.mc());
#pragma unroll
          for (int i = 0; i < 128; ++i)
            if (i >= lim) s[i] = -INFINITY;
        }
        // Row max: eight independent chains of 3-input max.
        float mx8[8];
#pragma unroll
        for (int a = 0; a < 8; ++a) {
          float acc = fmax3(s[a], s[a + 8], s[a + 16]);
#pragma unroll
          for (int kq = 3; kq < 15; kq += 2) acc = fmax3(acc, s[a + 8 * kq], s[a + 8 * kq + 8]);
          mx8[a] = fmaxf(acc, s[a + 120]);
        }
        const float mx = fmaxf(fmax3(mx8[0], mx8[1], mx8[2]),
                               fmaxf(fmax3(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
        const float m_cand = fmaxf(m2, mx * c2);
        // Rescale whenever the running max grows: the largest probability of
        // the row is then exactly 1, so its bf16 rounding in P V costs
        // nothing (a lazy threshold lets it reach 2^t with an uncovered
        // rounding error of up to 2^-8 of the dominant term).
        const bool need = m_cand > m2;
        // The O rescale itself comes after the exps of the first part of P:
        // it only has to land before this tile's P V, and by then those
        // scores are dead, which leaves the registers for 64 columns of O per
        // round trip.
        const bool rescale = __any_sync(0xffffffffu, need);
        float alpha = 1.f;
        if (rescale) {
          alpha = (m_cand == -INFINITY) ? 1.f : ex2(m2 - m_cand);
          l *= alpha;
          m2 = m_cand;
        }
        const float msub = (m2 == -INFINITY) ? 0.f : m2;
        const uint64_t c2x2 = f2(c2, c2);
        const uint64_t nm2 = f2(-msub, -msub);
        RA_PHASE(pc, 3);
        uint64_t sum_e[4] = {0, 0, 0, 0};   // row sum of the probabilities
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int e = ch * 32 + 2 * i;
            const uint64_t x2 = ffma2(f2(s[e], s[e + 1]), c2x2, nm2);
            float p0, p1;
            if (kPolyEvery > 0 && (i % (kPolyEvery > 0 ? kPolyEvery : 1)) == kPolyEvery - 1) {
              exp2_poly2(x2, p0, p1);          // a share of the exps off the MUFU
            } else {
              float a0, a1;
              unf2(x2, a0, a1);
              p0 = ex2(a0);
              p1 = ex2(a1);
            }
            pk[i] = pack_bf16x2(p0, p1);
            sum_e[i & 3] = fadd2(sum_e[i & 3], f2(p0, p1));

          }
          tmem_st16(tS + ch * 16, pk);
          if (ch == kPub - 1) {
            if (rescale && acc) {
              // O (the previous tiles' P V: complete, since this tile's
              // scores were committed after it) moves to the new max before
              // this tile's P V adds to it; 64 columns per TMEM round trip
              // (one wait for two loads), while the scores of the second
              // part are still held
              const uint64_t a2 = f2(alpha, alpha);
#pragma unroll 1
              for (int q4 = 0; q4 < D / 32; q4 += 2) {
                uint32_t o32[32], o32b[32];
                tmem_ld32(tO + q4 * 32, o32);
                tmem_ld32(tO + q4 * 32 + 32, o32b);
                tmem_wait_ld();
                scale_row32(o32, a2);
                scale_row32(o32b, a2);
                tmem_st32(tO + q4 * 32, o32);
                tmem_st32(tO + q4 * 32 + 32, o32b);
              }
            }
            // the first part of P (and a rescaled O) is in TMEM: let P V start
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(my_p_full);
            RA_PHASE(pc, 4);
          }
        }
        {
          float a, b;
          unf2(fadd2(fadd2(sum_e[0], sum_e[1]), fadd2(sum_e[2], sum_e[3])), a, b);
          l += a + b;
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(my_p_full2);
        RA_PHASE(pc, 5);
        RA_PHASE_COUNT(pc);
        acc = true;
      }
      if (!ok) break;
      // --------------------------------------------------------- epilogue
      if (!wmbar_wait(my_o_full, k & 1, abort_flag, p.timeout_ns)) { ok = false; break; }
      tc_fence_after();
      const bool valid = x < p.c;
      // a row that saw no key (possible only for a single block) gets O = 0
      // and lse = -inf; its O columns in TMEM were never written
      const float inv_l = (acc && l > 0.f) ? 1.f / l : 0.f;
      const size_t grow = out_row<ZZ>(p, it.bh, it.j, valid ? x : 0);
      __nv_bfloat16* orow_g = p.o + grow * D;
#pragma unroll 1
      for (int q = 0; q < D / 32; ++q) {
        uint32_t orow[32];
        tmem_ld32(tO + q * 32, orow);
        tmem_wait_ld();
        if (!acc) {
#pragma unroll
          for (int i = 0; i < 32; ++i) orow[i] = 0u;
        }
        if (valid && p.o_f32) {
          float* dstf = reinterpret_cast<float*>(p.o) + grow * D + q * 32;
          if (p.o_v8) {
            uint32_t w[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) w[i] = __float_as_uint(__uint_as_float(orow[i]) * inv_l);
#pragma unroll
            for (int i = 0; i < 4; ++i) st_global_v8(dstf + 8 * i, w + 8 * i);
          } else {
            float4* dst = reinterpret_cast<float4*>(dstf);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              dst[i] = make_float4(__uint_as_float(orow[4 * i]) * inv_l,
                                   __uint_as_float(orow[4 * i + 1]) * inv_l,
                                   __uint_as_float(orow[4 * i + 2]) * inv_l,
                                   __uint_as_float(orow[4 * i + 3]) * inv_l);
          }
        } else if (valid) {
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            w[i] = pack_bf16x2(__uint_as_float(orow[2 * i]) * inv_l,
                               __uint_as_float(orow[2 * i + 1]) * inv_l);
          if (p.o_v8) {
            // 32-byte stores: every store fills whole 32-byte sectors
            st_global_v8(orow_g + q * 32, w);
            st_global_v8(orow_g + q * 32 + 16, w + 8);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(orow_g + q * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
          }
        }
      }
      if (valid) p.lse[grow] = (acc && l > 0.f) ? (m2 + __log2f(l)) * 0.69314718055994530942f : -INFINITY;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(my_o_free);
    }
    RA_PHASE(pc, 0);
    RA_PHASE_STORE(pc, warp);
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) atomicOr(&g_device_fault, 1u);
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ===================================================== CTA-pair forward
// The same method with the tensor-core work of two SMs fused: a cluster of
// two CTAs issues M = 256 tcgen05 MMAs (cta_group::2).  CTA r of the pair
// holds query tiles 4q+2r and 4q+2r+1 of its item (query tiles 4q..4q+3 of
// one shard), and of every key/value tile only its half: key rows
// [64r, 64r+64) of K and value columns [64r, 64r+64) of V.  Each SM thus
// reads half of the B operand from its shared memory per MMA and loads half
// of every K/V tile, and its ring of half-tile slots looks twice as far
// ahead.  MMA slot t multiplies the pair's tiles 4q+t (rows 0-127, CTA 0)
// and 4q+2+t (rows 128-255, CTA 1); each CTA's softmax warpgroup t handles
// its own 128 rows of slot t in its own tensor memory, exactly as in the
// single-CTA kernel.  CTA 0 issues every MMA; the barriers that gather both
// CTAs' inputs (loaded tiles, published P, released O) live in CTA 0, and
// each of CTA 0's commits is sent to the matching barrier of both CTAs.
template <int D>
struct PairCfg {
  static constexpr int kTileBytes = kBM * D * 2;      // one query tile of this CTA
  static constexpr int kHalfBytes = kTileBytes / 2;   // this CTA's half of a K or V tile
  static constexpr int kChunks = D / 64;
  static constexpr int kSlots = 10;                   // half-tile ring slots
  static constexpr int kQOff = 0;
  static constexpr int kRingOff = 2 * kTileBytes;
  static constexpr int kBarOff = kRingOff + kSlots * kHalfBytes;
  // barriers: q_full, q_empty, full[kSlots], empty[kSlots], s_full[2],
  // p_full[2], p_full2[2], o_full[2], o_free[2], drain
  static constexpr int kNumBars = 2 + 2 * kSlots + 10 + 1;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kSmemBytes = kMiscOff + 16 + 1024;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO0 = 256, kColO1 = 256 + D;
  static constexpr int kThreads = 384;
  static constexpr int kRegsLaunch = 168, kRegsLow = 112, kRegsHigh = 192;
};

// Items of the pair kernel are (b*h, shard, quad of query tiles); the
// schedule is the single-CTA one over clusters (npairs counts quads).
__device__ __forceinline__ bool pair_item(const AttnParams& p, int k, Item& it) {
  const int ci = blockIdx.x >> 1;
  const int G = p.ctas_per_group;
  const int base = p.groups * G;
  if (ci >= base) {
    if (p.ceded == 0) return false;
    const int gi = k / p.ceded;
    const int g = ci - base + gi * p.helpers;
    if (g >= p.groups) return false;
    return item_at(p, g, group_items(p, g) - p.ceded + (k - gi * p.ceded), it);
  }
  const int g = ci / G;
  const int m = ci % G;
  const int u = k * G + ((k & 1) ? (G - 1 - m) : m);
  if (u >= group_items(p, g) - p.ceded) return false;
  return item_at(p, g, u, it);
}

// The key tiles met by a quad of query tiles, in ring order (the union of
// the four tiles' spans); kind[i] is the kind of tile 4q+i.
struct TileSeqQuad {
  int j, P, c, striped, causal;
  int x0;
  int r, kt, kend;
  TileSpan sp[4];
  BlockMask bm;
  int kb;
  __device__ __forceinline__ void init(const AttnParams& p, const Item& it) {
    j = it.j; P = p.P; c = p.c; striped = p.striped; causal = p.causal;
    x0 = it.pair * 4 * kBM;
    r = -1; kt = 0; kend = 0;
  }
  __device__ __forceinline__ bool next(int& kb_out, int& y0, int (&kind)[4], BlockMask& m) {
    while (kt >= kend) {
      if (++r >= P) return false;
      kb = key_block(j, r, P);
      bm = block_mask(j, kb, striped, causal);
      kend = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        sp[i] = tile_span(bm, x0 + i * kBM, c);
        kend = sp[i].part_end > kend ? sp[i].part_end : kend;
      }
      kt = 0;
    }
    kb_out = kb;
    y0 = kt * kBN;
#pragma unroll
    for (int i = 0; i < 4; ++i) kind[i] = tile_kind_at(sp[i], kt);
    m = bm;
    ++kt;
    return true;
  }
};

// Bounded wait against a deadline shared by several waits (drains).
__device__ __forceinline__ bool mbar_wait_until(uint32_t bar, uint32_t parity,
                                                unsigned long long deadline);
__device__ __forceinline__ bool wmbar_wait_until(uint32_t bar, uint32_t parity,
                                                 unsigned long long deadline) {
  return __all_sync(0xffffffffu, mbar_wait_until(bar, parity, deadline));
}
__device__ __forceinline__ bool mbar_wait_until(uint32_t bar, uint32_t parity,
                                                unsigned long long deadline) {
  while (!mbar_try_wait(bar, parity))
    if (global_timer_ns() > deadline) return false;
  return true;
}

template <int D>
__device__ __forceinline__ void pair_mma_qk(uint32_t s_tmem, uint32_t qa, uint32_t ka) {
  constexpr uint32_t idesc = idesc_bf16_f32(2 * kBM, kBN, 0, 0);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk)
    pair::mma_ss_w(s_tmem, smem_desc_sw128(qa + (kk / 4) * 16384 + (kk % 4) * 32, 16, 1024),
                   smem_desc_sw128(ka + (kk / 4) * 8192 + (kk % 4) * 32, 16, 1024), idesc, kk > 0);
}

template <int D, int KK0, int KK1>
__device__ __forceinline__ void pair_mma_pv(uint32_t o_tmem, uint32_t p_tmem, uint32_t va,
                                            uint32_t acc) {
  constexpr uint32_t idesc = idesc_bf16_f32(2 * kBM, D, 0, 1);
#pragma unroll
  for (int kk = KK0; kk < KK1; ++kk)
    pair::mma_ts_w(o_tmem, p_tmem + kk * 8, smem_desc_sw128(va + kk * 2048, 16384, 1024), idesc,
                   (acc | (uint32_t)kk) != 0);
}

template <int D>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(384, 1)
attn_fwd_pair_kernel(const __grid_constant__ CUtensorMap tmQ,
                     const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  using C = PairCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + C::kQOff;
  const uint32_t sRing = sbase + C::kRingOff;
  const uint32_t bars = sbase + C::kBarOff;
  const uint32_t bar_q_full = bars + 0 * 8;
  const uint32_t bar_q_empty = bars + 1 * 8;
  auto bar_full = [&](int s) { return bars + (2 + s) * 8; };
  auto bar_empty = [&](int s) { return bars + (2 + C::kSlots + s) * 8; };
  const uint32_t bar_s_full = bars + (2 + 2 * C::kSlots) * 8;   // [2]
  const uint32_t bar_p_full = bar_s_full + 16;                  // [2]
  const uint32_t bar_p_full2 = bar_p_full + 16;                 // [2]
  const uint32_t bar_o_full = bar_p_full2 + 16;                 // [2]
  const uint32_t bar_o_free = bar_o_full + 16;                  // [2]
  const uint32_t bar_drain = bar_o_free + 16;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 4);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const uint32_t rank = pair::cta_rank();
  const bool leader = rank == 0;
  // the even CTA's copy of a barrier, and the odd CTA's
  auto at0 = [&](uint32_t bar) { return pair::map_to(bar, 0); };
  auto at1 = [&](uint32_t bar) { return pair::map_to(bar, 1); };

  if (threadIdx.x == 0) {
    mbar_init(bar_q_full, 1);
    mbar_init(bar_q_empty, 1);
    for (int s = 0; s < C::kSlots; ++s) {
      mbar_init(bar_full(s), 1);
      mbar_init(bar_empty(s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar_s_full + 8 * t, 1);
      mbar_init(bar_p_full + 8 * t, 8);     // four softmax warps of each CTA
      mbar_init(bar_p_full2 + 8 * t, 8);
      mbar_init(bar_o_full + 8 * t, 1);
      mbar_init(bar_o_free + 8 * t, 8);
    }
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    pair::tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
    pair::tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  tc_fence_before();
  // both CTAs' barriers are initialised and tensor memory is allocated
  // before either CTA touches the other's barriers
  pair::cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= 8) {
  reg_dealloc<C::kRegsLow>();
  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t n_loads = 0;
      Item it;
      bool ok = true;
      for (int k = 0; ok && pair_item(p, k, it); ++k) {
        if (!mbar_wait(bar_q_empty, (k & 1) ^ 1, abort_flag, p.timeout_ns)) { ok = false; break; }
        if (leader) mbar_arrive_expect_tx(bar_q_full, 4 * C::kTileBytes);
        const int x0 = it.pair * 4 * kBM + (int)rank * 2 * kBM;
        for (int t = 0; t < 2; ++t)
          for (int ch = 0; ch < C::kChunks; ++ch)
            pair::tma_load_4d(sQ + t * C::kTileBytes + ch * 16384, &tmQ, at0(bar_q_full), ch * 64,
                              x0 + t * kBM, it.j, it.bh);
        TileSeqQuad seq;
        seq.init(p, it);
        int kb, y0, kind[4];
        BlockMask bm;
        while (seq.next(kb, y0, kind, bm)) {
          for (int kv = 0; kv < 2; ++kv) {
            const int s = n_loads % C::kSlots;
            const uint32_t ph = (n_loads / C::kSlots) & 1;
            if (!mbar_wait(bar_empty(s), ph ^ 1, abort_flag, p.timeout_ns)) { ok = false; break; }
            if (leader) mbar_arrive_expect_tx(bar_full(s), 2 * C::kHalfBytes);
            const uint32_t dst = sRing + s * C::kHalfBytes;
            if (kv == 0) {
              // key rows [64 rank, 64 rank + 64) of the tile, all d
              for (int ch = 0; ch < C::kChunks; ++ch)
                pair::tma_load_4d(dst + ch * (C::kHalfBytes / C::kChunks), &tmK, at0(bar_full(s)),
                                  ch * 64, y0 + (int)rank * (kBN / 2), kb, it.bh);
            } else {
              // value columns [64 rank, 64 rank + 64) of the tile, all keys
              pair::tma_load_4d(dst, &tmV, at0(bar_full(s)), (int)rank * 64, y0, kb, it.bh);
            }
            ++n_loads;
          }
          if (!ok) break;
        }
      }
      if (leader) {
        // Every load issued (by both CTAs) lands on this CTA's barriers;
        // wait for the ones not consumed yet, under one deadline.
        const unsigned long long deadline = global_timer_ns() + p.drain_timeout_ns;
        const uint32_t first = n_loads > (uint32_t)C::kSlots ? n_loads - C::kSlots : 0;
        for (uint32_t n = first; n < n_loads; ++n)
          if (!mbar_wait_until(bar_full(n % C::kSlots), (n / C::kSlots) & 1, deadline)) break;
      } else if (!ok) {
        // after an abort the even CTA may never count these loads: give
        // them time to land before this CTA can exit
        const unsigned long long until = global_timer_ns() + 200000ull;
        while (global_timer_ns() < until) {
        }
      }
    }
    __syncwarp();
  } else if (warp == 9 && leader) {
    // ------------------------------------------------ MMA issuer (CTA 0)
    {
      const uint32_t tS0 = tmem + C::kColS0, tS1 = tmem + C::kColS1;
      const uint32_t tO0 = tmem + C::kColO0, tO1 = tmem + C::kColO1;
      const uint32_t sQ0 = sQ, sQ1 = sQ + C::kTileBytes;
      const uint32_t s_full0 = bar_s_full, s_full1 = bar_s_full + 8;
      const uint32_t p_full0 = bar_p_full, p_full1 = bar_p_full + 8;
      const uint32_t p_full2_0 = bar_p_full2, p_full2_1 = bar_p_full2 + 8;
      const uint32_t o_free0 = bar_o_free, o_free1 = bar_o_free + 8;
      bool withhold = p.withhold_first_s != 0;
      // a commit reaches the barrier of both CTAs
      auto commit2 = [&](uint32_t bar) {
        pair::mma_commit_w(bar);
        pair::mma_commit_w(at1(bar));
      };
      uint32_t slot = 0, phase = 0;
      uint32_t pc0 = 0, pc1 = 0;
      uint32_t of0 = 0, of1 = 0;
      Item it;
      bool ok = true;
      for (int k = 0; ok && pair_item(p, k, it); ++k) {
        if (!pair::wmbar_wait(bar_q_full, k & 1, abort_flag, p.timeout_ns)) { ok = false; break; }
        TileSeqQuad seq;
        seq.init(p, it);
        int kb, y0, kind[4];
        BlockMask bm;
        bool have = seq.next(kb, y0, kind, bm);
        // slot t computes when either CTA's tile of it is visible
        bool c0 = have && (kind[0] != TILE_SKIP || kind[2] != TILE_SKIP);
        bool c1 = have && (kind[1] != TILE_SKIP || kind[3] != TILE_SKIP);
        uint32_t acc0 = 0, acc1 = 0;
        if (!have) {
          bool okw = true;
          while (okw && of0 < (uint32_t)k) okw = pair::wmbar_wait(o_free0, of0++ & 1, abort_flag, p.timeout_ns);
          while (okw && of1 < (uint32_t)k) okw = pair::wmbar_wait(o_free1, of1++ & 1, abort_flag, p.timeout_ns);
          if (!okw) { ok = false; break; }
          commit2(bar_o_full + 0);
          commit2(bar_o_full + 8);
          commit2(bar_q_empty);
          continue;
        }
        uint32_t kslot = slot;
        if (!pair::wmbar_wait(bar_full(kslot), phase, abort_flag, p.timeout_ns)) { ok = false; break; }
        tc_fence_after();
        const uint32_t ka0 = sRing + kslot * C::kHalfBytes;
        if (c0) {
          pair_mma_qk<D>(tS0, sQ0, ka0);
          if (!withhold) commit2(s_full0);
          withhold = false;
        }
        if (c1) { pair_mma_qk<D>(tS1, sQ1, ka0); commit2(s_full1); }
        commit2(bar_empty(kslot));
        if (++slot == C::kSlots) { slot = 0; phase ^= 1; }
        while (have) {
          int nkind[4];
          const bool more = seq.next(kb, y0, nkind, bm);
          const bool n0 = more && (nkind[0] != TILE_SKIP || nkind[2] != TILE_SKIP);
          const bool n1 = more && (nkind[1] != TILE_SKIP || nkind[3] != TILE_SKIP);
          const uint32_t vslot = slot, vph = phase;
          if (++slot == C::kSlots) { slot = 0; phase ^= 1; }
          uint32_t nkslot = 0;
          if (more) {
            nkslot = slot;
            if (!pair::wmbar_wait(bar_full(nkslot), phase, abort_flag, p.timeout_ns)) { ok = false; break; }
            if (++slot == C::kSlots) { slot = 0; phase ^= 1; }
          }
          if (!pair::wmbar_wait(bar_full(vslot), vph, abort_flag, p.timeout_ns)) { ok = false; break; }
          const uint32_t va = sRing + vslot * C::kHalfBytes;
          const uint32_t nka = sRing + nkslot * C::kHalfBytes;
          if (c0) {
            bool okw = true;
            while (okw && of0 < (uint32_t)k) okw = pair::wmbar_wait(o_free0, of0++ & 1, abort_flag, p.timeout_ns);
            if (!okw) { ok = false; break; }
            if (!pair::wmbar_wait(p_full0, pc0 & 1, abort_flag, p.timeout_ns)) { ok = false; break; }
            tc_fence_after();
            pair_mma_pv<D, 0, 4>(tO0, tS0, va, acc0);
            if (!pair::wmbar_wait(p_full2_0, pc0 & 1, abort_flag, p.timeout_ns)) { ok = false; break; }
            ++pc0;
            tc_fence_after();
            pair_mma_pv<D, 4, 8>(tO0, tS0, va, 1);
            acc0 = 1;
          }
          if (n0) { tc_fence_after(); pair_mma_qk<D>(tS0, sQ0, nka); commit2(s_full0); }
          if (c1) {
            bool okw = true;
            while (okw && of1 < (uint32_t)k) okw = pair::wmbar_wait(o_free1, of1++ & 1, abort_flag, p.timeout_ns);
            if (!okw) { ok = false; break; }
            if (!pair::wmbar_wait(p_full1, pc1 & 1, abort_flag, p.timeout_ns)) { ok = false; break; }
            tc_fence_after();
            pair_mma_pv<D, 0, 4>(tO1, tS1, va, acc1);
            if (!pair::wmbar_wait(p_full2_1, pc1 & 1, abort_flag, p.timeout_ns)) { ok = false; break; }
            ++pc1;
            tc_fence_after();
            pair_mma_pv<D, 4, 8>(tO1, tS1, va, 1);
            acc1 = 1;
          }
          commit2(bar_empty(vslot));
          if (n1) { tc_fence_after(); pair_mma_qk<D>(tS1, sQ1, nka); commit2(s_full1); }
          if (more) commit2(bar_empty(nkslot));
          have = more;
          c0 = n0;
          c1 = n1;
        }
        if (!ok) break;
        {
          bool okw = true;
          while (okw && of0 < (uint32_t)k) okw = pair::wmbar_wait(o_free0, of0++ & 1, abort_flag, p.timeout_ns);
          while (okw && of1 < (uint32_t)k) okw = pair::wmbar_wait(o_free1, of1++ & 1, abort_flag, p.timeout_ns);
          if (!okw) { ok = false; break; }
        }
        commit2(bar_o_full + 0);
        commit2(bar_o_full + 8);
        commit2(bar_q_empty);
      }
      // Every pair MMA must be complete before either CTA frees its TMEM.
      pair::mma_commit_w(bar_drain);
      wmbar_wait_until(bar_drain, 0, global_timer_ns() + p.drain_timeout_ns);
    }
    __syncwarp();
  }
  } else {
    // ----------------------------------------------------- softmax warpgroups
    reg_alloc<C::kRegsHigh>();
    const int t = warp / 4;                 // MMA slot; this CTA's tile 2 rank + t of the quad
    const int wq = warp % 4;                // TMEM lane quarter
    const int row = wq * 32 + lane;         // row within the query tile
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t tS = tmem + (t ? C::kColS1 : C::kColS0) + lane_off;
    const uint32_t tO = tmem + (t ? C::kColO1 : C::kColO0) + lane_off;
    const uint32_t my_s_full = bar_s_full + 8 * t;
    const uint32_t their_p_full = at0(bar_p_full + 8 * t);
    const uint32_t their_p_full2 = at0(bar_p_full2 + 8 * t);
    const uint32_t my_o_full = bar_o_full + 8 * t;
    const uint32_t their_o_free = at0(bar_o_free + 8 * t);
    const int mine = 2 * (int)rank + t;     // this warpgroup's tile of the quad
    const float c2 = p.c2;
    uint32_t s_cnt = 0;
    Item it;
    bool ok = true;
    for (int k = 0; ok && pair_item(p, k, it); ++k) {
      TileSeqQuad seq;
      seq.init(p, it);
      const int x = it.pair * 4 * kBM + mine * kBM + row;   // local query row in shard
      float m2 = -INFINITY;
      float l = 0.f;
      bool acc = false;
      int kb, y0, kind[4];
      BlockMask bm;
      while (seq.next(kb, y0, kind, bm)) {
        if (kind[t] == TILE_SKIP && kind[2 + t] == TILE_SKIP) continue;   // slot not computed
        const int my_kind = kind[mine];
        if (!wmbar_wait(my_s_full, s_cnt & 1, abort_flag, p.timeout_ns)) { ok = false; break; }
        ++s_cnt;
        tc_fence_after();
        uint32_t sr[4][32];
#pragma unroll
        for (int q = 0; q < 4; ++q) tmem_ld32(tS + q * 32, sr[q]);
        tmem_wait_ld();
        float s[128];
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
          for (int i = 0; i < 32; ++i) s[q * 32 + i] = __uint_as_float(sr[q][i]);
        if (my_kind != TILE_FULL) {
          // this CTA's tile of the slot is partial, or hidden entirely
          // (the other CTA's tile needed the MMA): mask by the row limit
          const int lim = my_kind == TILE_SKIP ? 0 : row_limit(bm, x, y0, p.c);
#pragma unroll
          for (int i = 0; i < 128; ++i)
            if (i >= lim) s[i] = -INFINITY;
        }
        const float mx = row_max128(s);
        const float m_cand = fmaxf(m2, mx * c2);
        const bool rescale = __any_sync(0xffffffffu, m_cand > m2);
        float alpha = 1.f;
        if (rescale) {
          alpha = (m_cand == -INFINITY) ? 1.f : ex2(m2 - m_cand);
          l *= alpha;
          m2 = m_cand;
        }
        const float msub = (m2 == -INFINITY) ? 0.f : m2;
        const uint64_t c2x2 = f2(c2, c2);
        const uint64_t nm2 = f2(-msub, -msub);
        uint64_t sum_e[4] = {0, 0, 0, 0};
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int e = ch * 32 + 2 * i;
            const uint64_t x2 = ffma2(f2(s[e], s[e + 1]), c2x2, nm2);
            float a0, a1;
            unf2(x2, a0, a1);
            const float p0 = ex2(a0), p1 = ex2(a1);
            pk[i] = pack_bf16x2(p0, p1);
            sum_e[i & 3] = fadd2(sum_e[i & 3], f2(p0, p1));
          }
          tmem_st16(tS + ch * 16, pk);
          if (ch == 1) {
            if (rescale && acc) {
              const uint64_t a2 = f2(alpha, alpha);
#pragma unroll 1
              for (int q4 = 0; q4 < D / 32; ++q4) {
                uint32_t o32[32];
                tmem_ld32(tO + q4 * 32, o32);
                tmem_wait_ld();
                scale_row32(o32, a2);
                tmem_st32(tO + q4 * 32, o32);
              }
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) pair::mbar_arrive_cluster(their_p_full);
          }
        }
        {
          float a, b;
          unf2(fadd2(fadd2(sum_e[0], sum_e[1]), fadd2(sum_e[2], sum_e[3])), a, b);
          l += a + b;
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) pair::mbar_arrive_cluster(their_p_full2);
        acc = true;
      }
      if (!ok) break;
      if (!wmbar_wait(my_o_full, k & 1, abort_flag, p.timeout_ns)) { ok = false; break; }
      tc_fence_after();
      const bool valid = x < p.c;
      const float inv_l = (acc && l > 0.f) ? 1.f / l : 0.f;
      const size_t grow = out_row<false>(p, it.bh, it.j, valid ? x : 0);
      __nv_bfloat16* orow_g = p.o + grow * D;
#pragma unroll 1
      for (int q = 0; q < D / 32; ++q) {
        uint32_t orow[32];
        tmem_ld32(tO + q * 32, orow);
        tmem_wait_ld();
        if (!acc) {
#pragma unroll
          for (int i = 0; i < 32; ++i) orow[i] = 0u;
        }
        if (valid && p.o_f32) {
          float* dstf = reinterpret_cast<float*>(p.o) + grow * D + q * 32;
          if (p.o_v8) {
            uint32_t w[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) w[i] = __float_as_uint(__uint_as_float(orow[i]) * inv_l);
#pragma unroll
            for (int i = 0; i < 4; ++i) st_global_v8(dstf + 8 * i, w + 8 * i);
          } else {
            float4* dst = reinterpret_cast<float4*>(dstf);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              dst[i] = make_float4(__uint_as_float(orow[4 * i]) * inv_l,
                                   __uint_as_float(orow[4 * i + 1]) * inv_l,
                                   __uint_as_float(orow[4 * i + 2]) * inv_l,
                                   __uint_as_float(orow[4 * i + 3]) * inv_l);
          }
        } else if (valid) {
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            w[i] = pack_bf16x2(__uint_as_float(orow[2 * i]) * inv_l,
                               __uint_as_float(orow[2 * i + 1]) * inv_l);
          if (p.o_v8) {
            st_global_v8(orow_g + q * 32, w);
            st_global_v8(orow_g + q * 32 + 16, w + 8);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(orow_g + q * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
          }
        }
      }
      if (valid) p.lse[grow] = (acc && l > 0.f) ? (m2 + __log2f(l)) * 0.69314718055994530942f : -INFINITY;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) pair::mbar_arrive_cluster(their_o_free);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) atomicOr(&g_device_fault, 1u);
  // CTA 0's MMAs (which write both CTAs' tensor memory) are complete: both
  // CTAs may free their columns
  pair::cluster_sync();
  if (warp == 9) {
    tc_fence_after();
    pair::tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ------------------------------------------------------------------ host
// mode 0: [BH, P, c, d] (layout order, or token order of the contiguous
// layout); mode 1: striped token order as [BH, c, P, d] (box over c);
// mode 2: zigzag token order as [BH, 2P, c/2, d].
static bool encode_qkv_map(CUtensorMap* map, const void* base, int64_t BH, int64_t N, int64_t c,
                           int P, int d, int mode = 0, int box_rows = kBM) {
  PFN_encodeTiled enc = get_encode_tiled();
  if (!enc) return false;
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)c, (cuuint64_t)P, (cuuint64_t)BH};
  cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)c * d * 2, (cuuint64_t)N * d * 2};
  cuuint32_t box[4] = {64, (cuuint32_t)box_rows, 1, 1};
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
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Key-tile steps of a work item (the MMA warp's iterations): for each round
// (each chunk pair in the zigzag layout) the larger of the two query tiles'
// PARTIAL/FULL spans.  Mirrors TileSeq::next.
static long long item_steps(const AttnParams& p, int j, int pair, bool zz) {
  const int x0 = pair * 2 * kBM;
  long long steps = 0;
  if (zz) {
    const int h = p.c >> 1;
    for (int r = 0; r < 2 * p.P; ++r) {
      const int kb = key_block(j, r >> 1, p.P);
      const int hk = r & 1;
      const int zx = x0 < h ? 0 : h;
      const BlockMask bm = chunk_mask(zz_chunk(j, x0, h, p.P), hk ? 2 * p.P - 1 - kb : kb,
                                      p.causal);
      const TileSpan s0 = tile_span(bm, x0 - zx, h), s1 = tile_span(bm, x0 - zx + kBM, h);
      steps += s0.part_end > s1.part_end ? s0.part_end : s1.part_end;
    }
  } else {
    for (int r = 0; r < p.P; ++r) {
      const BlockMask bm = block_mask(j, key_block(j, r, p.P), p.striped, p.causal);
      const TileSpan s0 = tile_span(bm, x0, p.c), s1 = tile_span(bm, x0 + kBM, p.c);
      steps += s0.part_end > s1.part_end ? s0.part_end : s1.part_end;
    }
  }
  return steps;
}

// Per-CTA work lists of the owner schedule by longest-processing-time-first
// list scheduling: every item of a group, heaviest first (head order kept
// among equal weights), goes to the group's least-loaded CTA.  Used when the
// items fit the parameter block; a snake deal of the head-major item order
// leaves the CTAs of small problems unevenly loaded (at N = 8192 with 18
// CTAs per group the busiest CTA gets 160 key-tile steps where 142 is the
// mean; the lists bring it to 144).
static bool build_lists(const AttnParams& p, bool zz, WorkLists& wl) {
  const int G = p.ctas_per_group;
  if (p.groups * G > kMaxListCtas) return false;
  const int n_sh_max = (p.P + p.groups - 1) / p.groups;
  const long long per_group_max = (long long)p.npairs * n_sh_max * p.BH;
  if (per_group_max * p.groups > kMaxListItems) return false;
  int pos = 0;
  std::vector<long long> w;
  std::vector<int> ord;
  std::vector<std::vector<int>> lists(G);
  for (int g = 0; g < p.groups; ++g) {
    const int n_sh = (p.P - g + p.groups - 1) / p.groups;
    const int n = p.npairs * n_sh * p.BH;
    w.assign(n, 0);
    for (int u = 0; u < n; ++u) {
      // the same mapping as item_at (head-major)
      const int per_head = p.npairs * n_sh;
      const int rem = u % per_head;
      int j, pair;
      if (p.causal && !p.striped) {
        const int sh_rank = rem / p.npairs;
        j = g + (n_sh - 1 - sh_rank) * p.groups;
        pair = p.npairs - 1 - (rem - sh_rank * p.npairs);
      } else {
        const int pr = rem / n_sh;
        pair = p.npairs - 1 - pr;
        j = g + (rem - pr * n_sh) * p.groups;
      }
      w[u] = item_steps(p, j, pair, zz);
    }
    ord.resize(n);
    for (int u = 0; u < n; ++u) ord[u] = u;
    std::stable_sort(ord.begin(), ord.end(), [&](int x, int y) { return w[x] > w[y]; });
    std::vector<long long> load(G, 0);
    for (auto& l : lists) l.clear();
    for (int u : ord) {
      int best = 0;
      for (int m = 1; m < G; ++m)
        if (load[m] < load[best]) best = m;
      load[best] += w[u];
      lists[best].push_back(u);
    }
    for (int m = 0; m < G; ++m) {
      wl.start[g * G + m] = (uint16_t)pos;
      for (int u : lists[m]) wl.item[pos++] = (uint16_t)u;
    }
  }
  wl.start[p.groups * G] = (uint16_t)pos;
  return true;
}

// The softmax warpgroups' setmaxnreg.inc waits until the other warpgroup's
// .dec has freed enough of the registers the CTA was launched with: a build
// whose register count would leave it waiting is never launched.
template <int D, class K>
static bool register_split_fits(K kernel) {
  using C = Cfg<D>;
  cudaFuncAttributes fa;
  return cudaFuncGetAttributes(&fa, kernel) == cudaSuccess &&
         fa.numRegs * C::kThreads >= 256 * C::kRegsHigh + 128 * C::kRegsLow;
}

static int group_items_host(const AttnParams& p, int g) {
  return p.npairs * ((p.P - g + p.groups - 1) / p.groups) * p.BH;
}

// Items each owner group cedes to the helper CTAs (the SMs left over after
// groups x G): the count that minimises the busiest CTA's key-tile steps,
// with the groups' CTAs dealing the rest of their lists in snake order and
// helper h taking the ceded items of groups h, h + E, ...  The same count
// for every group; 0 when ceding does not help.
static int plan_ceded(const AttnParams& p, bool zz, int E) {
  const int G = p.ctas_per_group;
  if (E <= 0) return 0;
  int n_min = INT32_MAX;
  for (int g = 0; g < p.groups; ++g) {
    const int n_sh = (p.P - g + p.groups - 1) / p.groups;
    n_min = std::min(n_min, p.npairs * n_sh * p.BH);
  }
  const int t_max = n_min / 2;
  if (t_max < 1) return 0;
  // cta[g][m]: load of CTA m of group g with t items ceded; help[h]
  std::vector<std::vector<long long>> cta(p.groups, std::vector<long long>(G, 0));
  std::vector<std::vector<long long>> w(p.groups);
  std::vector<long long> help(E, 0);
  for (int g = 0; g < p.groups; ++g) {
    const int n_sh = (p.P - g + p.groups - 1) / p.groups;
    const int n = p.npairs * n_sh * p.BH;
    const int per_head = p.npairs * n_sh;
    w[g].resize(n);
    for (int u = 0; u < n; ++u) {
      const int rem = u % per_head;
      int j, pair;
      if (p.causal && !p.striped) {
        const int sh_rank = rem / p.npairs;
        j = g + (n_sh - 1 - sh_rank) * p.groups;
        pair = p.npairs - 1 - (rem - sh_rank * p.npairs);
      } else {
        const int pr = rem / n_sh;
        pair = p.npairs - 1 - pr;
        j = g + (rem - pr * n_sh) * p.groups;
      }
      w[g][u] = item_steps(p, j, pair, zz);
      const int k = u / G, r = u % G;
      cta[g][(k & 1) ? (G - 1 - r) : r] += w[g][u];
    }
  }
  auto makespan = [&]() {
    long long mx = 0;
    for (auto& row : cta)
      for (long long v : row) mx = std::max(mx, v);
    for (long long v : help) mx = std::max(mx, v);
    return mx;
  };
  long long best = makespan();
  int best_t = 0;
  for (int t = 1; t <= t_max; ++t) {
    for (int g = 0; g < p.groups; ++g) {
      const int u = (int)w[g].size() - t;   // the item ceded at this step
      const int k = u / G, r = u % G;
      cta[g][(k & 1) ? (G - 1 - r) : r] -= w[g][u];
      help[g % E] += w[g][u];
    }
    const long long ms = makespan();
    if (ms < best) {
      best = ms;
      best_t = t;
    }
  }
  return best_t;
}

template <int D, bool ZZ>
static ra_status launch(const AttnLaunch& a) {
  using C = Cfg<D>;
  CUtensorMap tq, tk, tv;
  const int64_t c = a.N / a.P;
  const int mode = !a.tok ? 0 : a.striped ? 1 : a.zigzag ? 2 : 0;
  if (!encode_qkv_map(&tq, a.q, a.BH, a.N, c, a.P, D, mode) ||
      !encode_qkv_map(&tk, a.k, a.BH, a.N, c, a.P, D, mode) ||
      !encode_qkv_map(&tv, a.v, a.BH, a.N, c, a.P, D, mode))
    return RA_ERR_CUDA;
  // once per device and instance (setting the attribute again is harmless;
  // the flags only save the calls)
  static std::atomic<int> attr_set[64];
  static std::atomic<int> attr_list_set[64];
  if (a.device < 64 && !attr_set[a.device].load(std::memory_order_acquire)) {
    if (cudaFuncSetAttribute(attn_fwd_kernel<D, ZZ, NoLists>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::kSmemBytes) != cudaSuccess ||
        !register_split_fits<D>(attn_fwd_kernel<D, ZZ, NoLists>))
      return RA_ERR_CUDA;
    attr_set[a.device].store(1, std::memory_order_release);
  }
  AttnParams p;
  p.o = reinterpret_cast<__nv_bfloat16*>(a.o);
  p.o_f32 = a.o_f32;
  p.o_v8 = (reinterpret_cast<uintptr_t>(a.o) % 32) == 0;
  p.tok = a.tok;
  p.lse = a.lse;
  p.BH = (int)a.BH;
  p.N = (int)a.N;
  p.c = (int)c;
  p.P = a.P;
  const int T = (int)((c + kBM - 1) / kBM);
  p.npairs = (T + 1) / 2;
  p.striped = a.striped;
  p.zigzag = a.zigzag;
  p.causal = a.causal;
  p.c2 = (float)((double)a.scale * 1.4426950408889634074);
  p.drain_timeout_ns = 2000000000ull;
  p.timeout_ns = a.main_limit_ns > 0 ? (unsigned long long)a.main_limit_ns : p.drain_timeout_ns;
  p.withhold_first_s = a.withhold_first_s;
  p.blk_j = a.blk_j;
  p.blk_kb = a.blk_kb;
  const long long items_total = (long long)p.npairs * a.P * a.BH;
  int grid;
  if (a.sched_free) {
    p.groups = 1;
    grid = (int)(items_total < a.num_sms ? items_total : a.num_sms);
    p.ctas_per_group = grid;
  } else {
    p.groups = a.P < a.num_sms ? a.P : a.num_sms;
    int G = a.num_sms / p.groups;
    const long long per_group =
        (long long)p.npairs * a.BH * ((a.P + p.groups - 1) / p.groups);
    if (per_group < G) G = (int)per_group;
    p.ctas_per_group = G;
    grid = G * p.groups;
  }
  p.helpers = 0;
  p.ceded = 0;
  // Work lists for small causal problems of the striped layout (whose items
  // differ in weight by pair index; measured at N = 8192, H = 16, P = 8:
  // +11 % striped, while the zigzag and contiguous layouts measured equal or
  // slower with them); they depend only on the shape and are built once per
  // shape.
  if (!a.sched_free && a.blk_kb < 0 && a.causal && a.striped && items_total <= kListItemsUsed) {
    static std::mutex mu;
    static std::map<std::vector<long long>, std::shared_ptr<WorkLists>> cache;
    const std::vector<long long> key = {p.BH, p.N, p.P, p.striped, p.zigzag, p.causal,
                                        p.groups, p.ctas_per_group};
    std::shared_ptr<WorkLists> wl;
    {
      std::lock_guard<std::mutex> lock(mu);
      auto found = cache.find(key);
      if (found == cache.end()) {
        auto built = std::make_shared<WorkLists>();
        if (!build_lists(p, ZZ, *built)) built.reset();
        found = cache.emplace(key, built).first;
      }
      wl = found->second;
    }
    if (wl) {
      if (a.device < 64 && !attr_list_set[a.device].load(std::memory_order_acquire)) {
        if (cudaFuncSetAttribute(attn_fwd_kernel<D, ZZ, WorkLists>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 C::kSmemBytes) != cudaSuccess ||
            !register_split_fits<D>(attn_fwd_kernel<D, ZZ, WorkLists>))
          return RA_ERR_CUDA;
        attr_list_set[a.device].store(1, std::memory_order_release);
      }
      attn_fwd_kernel<D, ZZ, WorkLists>
          <<<grid, C::kThreads, C::kSmemBytes, (cudaStream_t)a.stream>>>(tq, tk, tv, p, *wl);
      return cudaGetLastError() == cudaSuccess ? RA_OK : RA_ERR_CUDA;
    }
  }
  // Owner schedule: the SMs left over by the groups become helper CTAs that
  // take the lightest items of every group (planned once per shape).
  if (!a.sched_free && a.blk_kb < 0 && a.num_sms - grid > 0 && p.groups > 1) {
    const int E = std::min(a.num_sms - grid, p.groups);
    static std::mutex mu;
    static std::map<std::vector<long long>, int> cache;
    const std::vector<long long> key = {p.BH, p.N, p.P, p.striped, p.zigzag, p.causal,
                                        p.groups, p.ctas_per_group, E};
    int t;
    {
      std::lock_guard<std::mutex> lock(mu);
      auto found = cache.find(key);
      if (found == cache.end()) found = cache.emplace(key, plan_ceded(p, ZZ, E)).first;
      t = found->second;
    }
    if (t > 0) {
      p.helpers = E;
      p.ceded = t;
      grid += E;
    }
  }
  attn_fwd_kernel<D, ZZ, NoLists>
      <<<grid, C::kThreads, C::kSmemBytes, (cudaStream_t)a.stream>>>(tq, tk, tv, p, NoLists{});
  return cudaGetLastError() == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

// Key-tile steps of a quad of query tiles in the pair kernel (the union of
// the four tiles' spans per round).  Mirrors TileSeqQuad::next.
static long long quad_steps(const AttnParams& p, int j, int quad) {
  long long steps = 0;
  for (int r = 0; r < p.P; ++r) {
    const BlockMask bm = block_mask(j, key_block(j, r, p.P), p.striped, p.causal);
    int kend = 0;
    for (int i = 0; i < 4; ++i) {
      const TileSpan sp = tile_span(bm, quad * 4 * kBM + i * kBM, p.c);
      kend = sp.part_end > kend ? sp.part_end : kend;
    }
    steps += kend;
  }
  return steps;
}

// Helper planning of the pair kernel: as plan_ceded, over clusters and quads.
static int plan_ceded_quads(const AttnParams& p, int E) {
  const int G = p.ctas_per_group;
  if (E <= 0) return 0;
  int n_min = INT32_MAX;
  for (int g = 0; g < p.groups; ++g) n_min = std::min(n_min, group_items_host(p, g));
  const int t_max = n_min / 2;
  if (t_max < 1) return 0;
  std::vector<std::vector<long long>> cta(p.groups, std::vector<long long>(G, 0));
  std::vector<std::vector<long long>> w(p.groups);
  std::vector<long long> help(E, 0);
  for (int g = 0; g < p.groups; ++g) {
    const int n = group_items_host(p, g);
    const int n_sh = (p.P - g + p.groups - 1) / p.groups;
    const int per_head = p.npairs * n_sh;
    w[g].resize(n);
    for (int u = 0; u < n; ++u) {
      const int rem = u % per_head;
      int j, quad;
      if (p.causal && !p.striped) {
        const int sh_rank = rem / p.npairs;
        j = g + (n_sh - 1 - sh_rank) * p.groups;
        quad = p.npairs - 1 - (rem - sh_rank * p.npairs);
      } else {
        const int pr = rem / n_sh;
        quad = p.npairs - 1 - pr;
        j = g + (rem - pr * n_sh) * p.groups;
      }
      w[g][u] = quad_steps(p, j, quad);
      const int k = u / G, r = u % G;
      cta[g][(k & 1) ? (G - 1 - r) : r] += w[g][u];
    }
  }
  auto makespan = [&]() {
    long long mx = 0;
    for (auto& row : cta)
      for (long long v : row) mx = std::max(mx, v);
    for (long long v : help) mx = std::max(mx, v);
    return mx;
  };
  long long best = makespan();
  int best_t = 0;
  for (int t = 1; t <= t_max; ++t) {
    for (int g = 0; g < p.groups; ++g) {
      const int u = (int)w[g].size() - t;
      const int k = u / G, r = u % G;
      cta[g][(k & 1) ? (G - 1 - r) : r] -= w[g][u];
      help[g % E] += w[g][u];
    }
    const long long ms = makespan();
    if (ms < best) {
      best = ms;
      best_t = t;
    }
  }
  return best_t;
}

// The CTA-pair kernel: d = 128, layout order (no token-order addressing),
// not zigzag, not the single-block mode.
static ra_status launch_pair(const AttnLaunch& a) {
  constexpr int D = 128;
  using C = PairCfg<D>;
  CUtensorMap tq, tk, tv;
  const int64_t c = a.N / a.P;
  if (!encode_qkv_map(&tq, a.q, a.BH, a.N, c, a.P, D, 0, kBM) ||
      !encode_qkv_map(&tk, a.k, a.BH, a.N, c, a.P, D, 0, kBN / 2) ||
      !encode_qkv_map(&tv, a.v, a.BH, a.N, c, a.P, D, 0, kBN))
    return RA_ERR_CUDA;
  // Per device, once (under a lock: the cluster count is read by every
  // launch): the shared-memory attribute, the register check, and the number
  // of clusters of two that can be resident at once (one CTA per SM).
  if (a.device < 0 || a.device >= 64) return RA_ERR_DEVICE;
  static std::mutex init_mu;
  static int clusters[64] = {0};
  int n_clusters;
  {
    std::lock_guard<std::mutex> lock(init_mu);
    if (!clusters[a.device]) {
      if (cudaFuncSetAttribute(attn_fwd_pair_kernel<D>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               C::kSmemBytes) != cudaSuccess)
        return RA_ERR_CUDA;
      cudaFuncAttributes fa;
      if (cudaFuncGetAttributes(&fa, attn_fwd_pair_kernel<D>) != cudaSuccess ||
          fa.numRegs * C::kThreads < 256 * C::kRegsHigh + 128 * C::kRegsLow)
        return RA_ERR_CUDA;
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(2 * (a.num_sms / 2), 1, 1);
      cfg.blockDim = dim3(C::kThreads, 1, 1);
      cfg.dynamicSmemBytes = C::kSmemBytes;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, attn_fwd_pair_kernel<D>, &cfg) != cudaSuccess ||
          n < 1)
        return RA_ERR_CUDA;
      clusters[a.device] = n;
    }
    n_clusters = clusters[a.device];
  }
  AttnParams p;
  p.o = reinterpret_cast<__nv_bfloat16*>(a.o);
  p.o_f32 = a.o_f32;
  p.o_v8 = (reinterpret_cast<uintptr_t>(a.o) % 32) == 0;
  p.tok = 0;
  p.lse = a.lse;
  p.BH = (int)a.BH;
  p.N = (int)a.N;
  p.c = (int)c;
  p.P = a.P;
  const int T = (int)((c + kBM - 1) / kBM);
  p.npairs = (T + 3) / 4;                // quads of query tiles
  p.striped = a.striped;
  p.zigzag = 0;
  p.causal = a.causal;
  p.c2 = (float)((double)a.scale * 1.4426950408889634074);
  p.drain_timeout_ns = 2000000000ull;
  p.timeout_ns = a.main_limit_ns > 0 ? (unsigned long long)a.main_limit_ns : p.drain_timeout_ns;
  p.withhold_first_s = a.withhold_first_s;
  p.blk_j = -1;
  p.blk_kb = -1;
  p.helpers = 0;
  p.ceded = 0;
  const long long items_total = (long long)p.npairs * a.P * a.BH;
  int used;
  if (a.sched_free) {
    p.groups = 1;
    used = (int)(items_total < n_clusters ? items_total : n_clusters);
    p.ctas_per_group = used;
  } else {
    p.groups = a.P < n_clusters ? a.P : n_clusters;
    int G = n_clusters / p.groups;
    const long long per_group =
        (long long)p.npairs * a.BH * ((a.P + p.groups - 1) / p.groups);
    if (per_group < G) G = (int)per_group;
    p.ctas_per_group = G;
    used = G * p.groups;
    const int E = std::min(n_clusters - used, p.groups);
    if (E > 0 && p.groups > 1) {
      static std::mutex mu;
      static std::map<std::vector<long long>, int> cache;
      const std::vector<long long> key = {p.BH, p.N, p.P, p.striped, p.causal, p.groups, G, E};
      int t;
      {
        std::lock_guard<std::mutex> lock(mu);
        auto found = cache.find(key);
        if (found == cache.end()) found = cache.emplace(key, plan_ceded_quads(p, E)).first;
        t = found->second;
      }
      if (t > 0) {
        p.helpers = E;
        p.ceded = t;
        used += E;
      }
    }
  }
  attn_fwd_pair_kernel<D><<<2 * used, C::kThreads, C::kSmemBytes, (cudaStream_t)a.stream>>>(
      tq, tk, tv, p);
  return cudaGetLastError() == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

ra_status attn_fwd_launch(const AttnLaunch& a) {
  if (a.pair && a.d == 128 && !a.zigzag && !a.tok && a.blk_kb < 0) return launch_pair(a);
  if (a.zigzag) {
    if (a.d == 128) return launch<128, true>(a);
    if (a.d == 64) return launch<64, true>(a);
  } else {
    if (a.d == 128) return launch<128, false>(a);
    if (a.d == 64) return launch<64, false>(a);
  }
  return RA_ERR_HEADDIM;
}

// Bounded-wait self-test: one warp initialises an mbarrier that nothing ever
// arrives on and waits for it through the same bounded wait the attention
// kernel uses.  The wait gives up after `limit_ns`, the abort path records
// fault code 2 in the device fault word, and the kernel returns normally.
__global__ void wait_selftest_kernel(unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncwarp();
  const bool ok = mbar_wait(smem_u32(&bar), 0, &abort_flag, limit_ns);
  __syncwarp();
  if (threadIdx.x == 0 && (!ok || abort_flag)) atomicOr(&g_device_fault, 2u);
}

ra_status wait_selftest_launch(int64_t limit_ns, void* stream) {
  wait_selftest_kernel<<<1, 32, 0, (cudaStream_t)stream>>>((unsigned long long)limit_ns);
  return cudaGetLastError() == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

// Device address of the fault word on the current device, for kernels of
// other translation units (device symbols are not shared across files
// without relocatable device code).
unsigned int* device_fault_word() {
  static unsigned int* cache[64] = {nullptr};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!cache[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_device_fault) != cudaSuccess) return nullptr;
    cache[dev] = reinterpret_cast<unsigned int*>(ptr);
  }
  return cache[dev];
}

ra_status fwd_profile_read(unsigned long long* host, int64_t capacity) {
#if RA_PROFILE
  const int64_t n = (int64_t)kProfCtas * kProfSlots * kProfPhases;
  if (capacity < n) return RA_ERR_SHAPE;
  if (cudaDeviceSynchronize() != cudaSuccess) return RA_ERR_CUDA;
  if (cudaMemcpyFromSymbol(host, g_fwd_profile, n * sizeof(unsigned long long)) != cudaSuccess)
    return RA_ERR_CUDA;
  static const unsigned long long zeros[kProfCtas * kProfSlots * kProfPhases] = {};
  if (cudaMemcpyToSymbol(g_fwd_profile, zeros, sizeof(zeros)) != cudaSuccess) return RA_ERR_CUDA;
  return RA_OK;
#else
  (void)host;
  (void)capacity;
  return RA_ERR_NOPROFILE;
#endif
}

ra_status read_device_fault(int* code) {
  unsigned int v = 0;
  if (cudaDeviceSynchronize() != cudaSuccess) return RA_ERR_CUDA;
  if (cudaMemcpyFromSymbol(&v, g_device_fault, sizeof(v)) != cudaSuccess) return RA_ERR_CUDA;
  const unsigned int zero = 0;
  if (cudaMemcpyToSymbol(g_device_fault, &zero, sizeof(zero)) != cudaSuccess) return RA_ERR_CUDA;
  *code = (int)v;
  return v ? RA_ERR_DEVICE_FAULT : RA_OK;
}

}  // namespace ra
