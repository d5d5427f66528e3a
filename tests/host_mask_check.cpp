// Host-side check of the kernels' mask and tile-range logic against the oracle's visibility
// predicate.  Test infrastructure: tests/test_mask_tiles_host.py builds it from
//   - "mask_logic.inc": the integer mask helpers cut out of the library's CUDA headers at test
//     time (the MaskSpec region of the common header, and the backward header's tile
//     helpers), compiled here as plain host C++;
//   - oracle_visible() from the oracle's C source;
// and runs it on the configurations read from stdin, one per line:
//   kind Nq Nk window n_sink
// For each configuration it checks, over every query row and key of the (Nq, Nk) problem:
//   1. key_visible(p, j) equals the oracle's predicate (and is false for keys j >= Nk);
//   2. the 128-bit column set that row_cols + row_bits give for each (row, key tile) is exactly
//      the set of the tile's visible keys;
//   3. key_tiles(first row, last row) of each block of 128 query rows (a tile) and of 256 (a
//      forward CTA) lists every key tile holding a visible pair, each once, and no key tile
//      without one, and the TileRange membership test agrees with the listing;
//   4. block_visible() of every block of 128 or 64 query positions by a 128-key tile (the
//      forward and backward calls) is true only when every pair of the block is visible;
//   5. query_tiles() of each key tile lists every query tile holding a visible pair, each
//      once, and pair_index() numbers the listed tiles 0 .. count-1 (and gives -1 elsewhere).
// Prints "ok <configs> <pairs checked>" or one "FAIL ..." line per failed check (at most 20).
#include <cstdint>
#include <cstdio>
#include <set>
#include <vector>

#include "attn.h"

extern "C" int oracle_visible(int64_t p, int64_t j, int mask_kind, int64_t window,
                              int64_t n_sink);

#define __host__
#define __device__
#define __forceinline__ inline

namespace attn {
constexpr int kT = 128;
#include "mask_logic.inc"
}  // namespace attn

using attn::MaskSpec;
using attn::TileRange;

static int g_fail = 0;
#define CHECK(cond, ...)                          \
  do {                                            \
    if (!(cond)) {                                \
      if (g_fail < 20) {                          \
        std::printf("FAIL " __VA_ARGS__);         \
        std::printf("\n");                        \
      }                                           \
      ++g_fail;                                   \
    }                                             \
  } while (0)

static std::vector<int> listed(const TileRange& r) {
  std::vector<int> v;
  for (int j = 0; j < r.count(); ++j) v.push_back(r.tile(j));
  return v;
}

static long long check_config(int kind, int Nq, int Nk, int w, int s) {
  const MaskSpec m{kind, w, s, Nk};
  const int off = Nk - Nq;
  const int nqt = (Nq + 127) / 128, nkt = (Nk + 127) / 128;
  auto vis = [&](long long p, long long j) {
    return j >= 0 && j < Nk && oracle_visible(p, j, kind, w, s) != 0;
  };
  // visible[qt][kt]: the block holds a visible pair
  std::vector<std::vector<char>> any(nqt, std::vector<char>(nkt, 0));
  long long pairs = 0;
  for (int i = 0; i < Nq; ++i) {
    const int p = i + off;
    for (int kt = 0; kt < nkt; ++kt) {
      const int key0 = kt * 128;
      int hi, lo, sk;
      attn::row_cols(m, p, key0, hi, lo, sk);
      for (int wd = 0; wd < 4; ++wd) {
        const uint32_t bits = attn::row_bits(hi, lo, sk, wd);
        for (int b = 0; b < 32; ++b) {
          const int j = key0 + 32 * wd + b;
          const bool want = vis(p, j);
          const bool got = (bits >> b) & 1u;
          CHECK(got == want, "row_bits kind=%d Nq=%d Nk=%d w=%d s=%d p=%d j=%d got=%d", kind, Nq,
                Nk, w, s, p, j, got);
          CHECK(attn::key_visible(m, p, j) == want, "key_visible kind=%d Nq=%d Nk=%d w=%d s=%d p=%d j=%d",
                kind, Nq, Nk, w, s, p, j);
          if (want) any[i / 128][kt] = 1;
          ++pairs;
        }
      }
    }
  }
  // key_tiles over blocks of 128 query rows (one tile) and of 256 (a forward CTA's two tiles)
  for (int rows : {128, 256}) {
    for (int r0 = 0; r0 < Nq; r0 += rows) {
      const int r1 = (r0 + rows < Nq ? r0 + rows : Nq) - 1;
      const TileRange tr = attn::key_tiles(m, r0 + off, r1 + off, 128);
      const std::vector<int> tiles = listed(tr);
      std::set<int> uniq(tiles.begin(), tiles.end());
      CHECK(uniq.size() == tiles.size(),
            "key_tiles repeats a tile kind=%d Nq=%d Nk=%d w=%d s=%d rows=%d r0=%d", kind, Nq, Nk,
            w, s, rows, r0);
      for (int t : tiles)
        CHECK(t >= 0 && t < nkt, "key_tiles out of range kind=%d Nq=%d Nk=%d w=%d s=%d r0=%d t=%d",
              kind, Nq, Nk, w, s, r0, t);
      for (int kt = 0; kt < nkt; ++kt) {
        bool holds = false;
        for (int qt = r0 / 128; qt <= r1 / 128; ++qt) holds = holds || any[qt][kt];
        const bool in = uniq.count(kt) != 0;
        CHECK(in == holds,
              "key_tiles kind=%d Nq=%d Nk=%d w=%d s=%d rows=%d r0=%d kt=%d listed=%d holds_pair=%d",
              kind, Nq, Nk, w, s, rows, r0, kt, in, holds);
        // the forward kernel's membership test on a tile's range
        const bool member = kt < tr.ns || (kt >= tr.lo && kt <= tr.hi);
        CHECK(member == in, "TileRange membership kind=%d Nq=%d Nk=%d w=%d s=%d r0=%d kt=%d", kind,
              Nq, Nk, w, s, r0, kt);
      }
    }
  }
  // block_visible as the kernels call it: 128 key columns, blocks of 128 query positions
  // (forward) and of 64 (backward sub-steps), rows past Nq included
  for (int rows : {128, 64}) {
    for (int r0 = 0; r0 < Nq; r0 += rows) {
      for (int kt = 0; kt < nkt; ++kt) {
        if (!attn::block_visible(m, r0 + off, rows, kt * 128, 128)) continue;
        bool all = kt * 128 + 128 <= Nk;
        for (int i = r0; i < r0 + rows && all; ++i)
          for (int j = kt * 128; j < kt * 128 + 128; ++j)
            if (!oracle_visible(i + off, j, kind, w, s)) {
              all = false;
              break;
            }
        CHECK(all, "block_visible true on a block with a hidden pair kind=%d Nq=%d Nk=%d w=%d s=%d rows=%d r0=%d kt=%d",
              kind, Nq, Nk, w, s, rows, r0, kt);
      }
    }
  }
  for (int kt = 0; kt < nkt; ++kt) {
    const int c0 = kt * 128, c1 = (c0 + 128 < Nk ? c0 + 128 : Nk) - 1;
    const attn::QueryTiles r = attn::query_tiles(m, c0, c1, off, Nq);
    std::vector<int> tiles;
    for (int j = 0; j < r.count(); ++j) tiles.push_back(r.tile(j));
    std::set<int> uniq(tiles.begin(), tiles.end());
    CHECK(uniq.size() == tiles.size(), "query_tiles repeats a tile kind=%d Nq=%d Nk=%d w=%d s=%d kt=%d",
          kind, Nq, Nk, w, s, kt);
    for (int qt = 0; qt < nqt; ++qt) {
      const bool in = uniq.count(qt) != 0;
      CHECK(in == (any[qt][kt] != 0),
            "query_tiles kind=%d Nq=%d Nk=%d w=%d s=%d kt=%d qt=%d listed=%d holds_pair=%d", kind,
            Nq, Nk, w, s, kt, qt, in, any[qt][kt]);
      const int idx = attn::pair_index(r, qt);
      if (in) {
        int want = -1;
        for (size_t u = 0; u < tiles.size(); ++u)
          if (tiles[u] == qt) want = static_cast<int>(u);
        CHECK(idx == want, "pair_index kind=%d Nq=%d Nk=%d w=%d s=%d kt=%d qt=%d idx=%d want=%d",
              kind, Nq, Nk, w, s, kt, qt, idx, want);
      } else {
        CHECK(idx == -1, "pair_index of an unlisted tile kind=%d Nq=%d Nk=%d w=%d s=%d kt=%d qt=%d idx=%d",
              kind, Nq, Nk, w, s, kt, qt, idx);
      }
    }
    for (int t : tiles)
      CHECK(t >= 0 && t < nqt, "query_tiles out of range kind=%d Nq=%d Nk=%d w=%d s=%d kt=%d t=%d",
            kind, Nq, Nk, w, s, kt, t);
  }
  return pairs;
}

int main() {
  int kind, Nq, Nk, w, s, n = 0;
  long long pairs = 0;
  while (std::scanf("%d %d %d %d %d", &kind, &Nq, &Nk, &w, &s) == 5) {
    pairs += check_config(kind, Nq, Nk, w, s);
    ++n;
  }
  if (g_fail) {
    std::printf("failed %d checks\n", g_fail);
    return 1;
  }
  std::printf("ok %d %lld\n", n, pairs);
  return 0;
}
