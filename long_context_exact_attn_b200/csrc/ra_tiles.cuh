// Tile schedule and causal masks of the virtual-shard ring, shared by the
// attention kernel and the tile-census kernel (host and device).
//
// Geometry.  The sequence of N tokens is stored in LAYOUT order: P shards of
// c = N / P rows each, shard after shard.  Shard j holds
//   contiguous ("Ring"):  tokens j*c + x          (Ring Attention explainer,
//                         ステップ1: シーケンスの分割)
//   striped:              tokens x*P + j          (Striped Attention review,
//                         分区策略对比: token t on device t mod P)
// for local index x in [0, c).
//
// Causal mask over ORIGINAL positions (Striped review, 核心公式, matrix C):
// key (shard kb, local y) is visible to query (shard j, local x) iff its
// token index is <= the query's.  That reduces, per block pair, to
//   contiguous: kb < j all visible; kb > j none; kb == j  y <= x
//   striped:    kb <= j  y <= x;                 kb >  j  y <  x
// i.e. the two GetMask procedures of the Striped review (GetMask 函数), read
// with MASK indexed [key, query].  Both are "y < x + e" with e = 1 or 0, so
// a tile needs one integer limit per query row.
//
// Rounds (Ring Attention explainer, ステップ2): in round r the device that
// owns shard j holds key block kb = (j - r) mod P.
//
// Tiles are BM query rows x BN keys inside one (query shard, key block)
// pair; a ragged last tile of a shard (c not a multiple of the tile) has
// its out-of-shard rows/columns masked.  A tile is SKIP (nothing visible,
// never computed), FULL (everything visible, no per-element mask) or
// PARTIAL (per-element mask) -- the tile skipping of the Striped review,
// 实现细节 / 分块与分瓦片.
#pragma once

#include <stdint.h>

#if defined(__CUDACC__)
#define RA_HD __host__ __device__ __forceinline__
#else
#define RA_HD inline
#endif

namespace ra {

constexpr int kBM = 128;   // query rows per Q tile (one TMEM lane per row)
constexpr int kBN = 128;   // keys per K/V tile

enum TileKind : int { TILE_SKIP = 0, TILE_FULL = 1, TILE_PARTIAL = 2 };

// Per (query shard j, key block kb) mask parameters.
struct BlockMask {
  int all_hidden;   // whole block masked (contiguous causal, kb > j)
  int use_diag;     // causal comparison needed (y < x + e)
  int e;            // 1: key may equal query local index; 0: strictly before
};

RA_HD BlockMask block_mask(int j, int kb, int layout_striped, int causal) {
  BlockMask m{0, 0, 1};
  if (!causal) return m;
  if (layout_striped) {
    m.use_diag = 1;
    m.e = (kb <= j) ? 1 : 0;
  } else {
    if (kb > j) {
      m.all_hidden = 1;
    } else if (kb == j) {
      m.use_diag = 1;
      m.e = 1;
    }
  }
  return m;
}

// Number of valid query rows in the Q tile starting at local row x0.
RA_HD int tile_rows(int x0, int c) {
  int r = c - x0;
  return r < 0 ? 0 : (r > kBM ? kBM : r);
}

// Along the key tiles of one block, the tiles of a query tile are FULL for
// kt < full_end, PARTIAL for full_end <= kt < part_end and SKIP from part_end
// on (visibility y < min(x + e, c) is monotone in y): one pair of thresholds
// per (block, query tile) classifies every tile.
struct TileSpan {
  int full_end, part_end;
};

RA_HD TileSpan tile_span(const BlockMask& m, int x0, int c) {
  const int rows = tile_rows(x0, c);
  const int T = (c + kBN - 1) / kBN;
  TileSpan s{0, 0};
  if (rows == 0 || m.all_hidden) return s;
  int part_end = T, full_lim = c;
  if (m.use_diag) {
    const int v = x0 + rows - 1 + m.e;      // the last row sees keys y < v
    const int pe = (v + kBN - 1) / kBN;
    part_end = pe < T ? pe : T;
    const int f = x0 + m.e;                 // the first row sees keys y < f
    full_lim = f < c ? f : c;
  }
  int full_end = full_lim / kBN;            // tiles entirely below full_lim
  s.full_end = full_end < part_end ? full_end : part_end;
  s.part_end = part_end;
  return s;
}

RA_HD int tile_kind_at(const TileSpan& s, int kt) {
  return kt < s.full_end ? TILE_FULL : (kt < s.part_end ? TILE_PARTIAL : TILE_SKIP);
}

// Classify the tile (query rows [x0, x0+BM), keys [y0, y0+BN)) of block
// pair (j, kb); y0 is a multiple of BN.
RA_HD int tile_kind(const BlockMask& m, int x0, int y0, int c) {
  return tile_kind_at(tile_span(m, x0, c), y0 / kBN);
}

// For a PARTIAL tile: keys with column index col < limit are visible to the
// query at local row x (col = key local index - y0).  Result may be <= 0
// (row sees nothing in this tile) or >= BN (row sees the whole tile).
RA_HD int row_limit(const BlockMask& m, int x, int y0, int c) {
  int lim = c - y0;
  if (m.use_diag) {
    const int d = x + m.e - y0;
    lim = d < lim ? d : lim;
  }
  return lim;
}

// Zigzag layout (a reading: the pages only name it): shard j holds chunk j
// (local rows [0, h)) followed by chunk 2P-1-j (local rows [h, 2h)), with
// h = c / 2.  Within a pair of chunks the causal structure is that of the
// contiguous layout: an earlier key chunk is fully visible, the same chunk
// is the diagonal (key y' visible to query x' iff y' < x' + 1), a later
// chunk is hidden.
RA_HD int zz_chunk(int shard, int local, int h, int P) {
  return local < h ? shard : 2 * P - 1 - shard;
}

RA_HD BlockMask chunk_mask(int query_chunk, int key_chunk, int causal) {
  BlockMask m{0, 0, 1};
  if (!causal) return m;
  if (key_chunk > query_chunk) m.all_hidden = 1;
  else if (key_chunk == query_chunk) m.use_diag = 1;
  return m;
}

RA_HD int key_block(int j, int r, int P) {
  int kb = j - r;
  return kb < 0 ? kb + P : kb;
}

}  // namespace ra
