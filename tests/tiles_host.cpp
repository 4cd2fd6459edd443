// Host build of the attention kernels' tile classifier (csrc/ra_tiles.cuh,
// compiled here as plain C++) for tests/test_tiles_host.py.
//
// usage: tiles_host c P layout causal
//   layout 0 contiguous, 1 striped, 2 zigzag (c even, c/2 a multiple of 128)
// Writes, for every query shard j and round r (key block kb = key_block(j,
// r, P)), in that order:
//   - 3 little-endian int64: SKIP, FULL, PARTIAL tile counts (square 128
//     tiles over the block pair, the count the tile census reports; zigzag:
//     over both chunk pairs of each query chunk),
//   - c*c bytes: visible[x][y] for query local row x and key local row y,
//     derived only from the tile kinds and the per-row limits the kernels
//     use (FULL: all of the tile; PARTIAL: column < row_limit; SKIP: none).
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <vector>

#include "../long_context_exact_attn_b200/csrc/ra_tiles.cuh"

using namespace ra;

namespace {

// One (query rows, key rows) pair of length-n segments with mask m: fills
// vis[(qoff + x) * c + koff + y] and adds the tile counts.
void segment_pair(const BlockMask& m, int n, int qoff, int koff, int c,
                  std::vector<uint8_t>& vis, int64_t cnt[3]) {
  const int T = (n + kBN - 1) / kBN;
  for (int x0 = 0; x0 < n; x0 += kBM) {
    const TileSpan s = tile_span(m, x0, n);
    const int rows = tile_rows(x0, n);
    for (int kt = 0; kt < T; ++kt) {
      const int kind = tile_kind_at(s, kt);
      ++cnt[kind];
      const int y0 = kt * kBN;
      for (int x = x0; x < x0 + rows; ++x) {
        const int lim = kind == TILE_PARTIAL ? row_limit(m, x, y0, n) : 0;
        for (int col = 0; col < kBN && y0 + col < n; ++col) {
          const bool v = kind == TILE_FULL || (kind == TILE_PARTIAL && col < lim);
          vis[(size_t)(qoff + x) * c + koff + y0 + col] = v ? 1 : 0;
        }
      }
    }
  }
}

}  // namespace

int main(int argc, char** argv) {
  if (argc != 5) {
    std::fprintf(stderr, "usage: %s c P layout causal\n", argv[0]);
    return 2;
  }
  const int c = std::atoi(argv[1]), P = std::atoi(argv[2]);
  const int layout = std::atoi(argv[3]), causal = std::atoi(argv[4]);
  if (c < 1 || P < 1 || layout < 0 || layout > 2 || (layout == 2 && c % 2)) return 2;
  std::vector<uint8_t> vis((size_t)c * c);
  for (int j = 0; j < P; ++j) {
    for (int r = 0; r < P; ++r) {
      const int kb = key_block(j, r, P);
      int64_t cnt[3] = {0, 0, 0};
      if (layout == 2) {
        // the zigzag kernel walks each key block as its two chunks, each
        // query chunk against each key chunk with the chunk pair's mask
        const int h = c / 2;
        for (int qh = 0; qh < 2; ++qh)
          for (int kh = 0; kh < 2; ++kh) {
            const BlockMask m = chunk_mask(zz_chunk(j, qh * h, h, P),
                                           kh ? 2 * P - 1 - kb : kb, causal);
            segment_pair(m, h, qh * h, kh * h, c, vis, cnt);
          }
      } else {
        segment_pair(block_mask(j, kb, layout == 1, causal), c, 0, 0, c, vis, cnt);
      }
      std::fwrite(cnt, sizeof(int64_t), 3, stdout);
      std::fwrite(vis.data(), 1, vis.size(), stdout);
    }
  }
  return 0;
}
