// Host-side check of the prefill kernels' work units.  Test infrastructure:
// tests/test_unit_schedule_host.py builds it from "unit_logic.inc", which holds, cut out of the
// library's sources at test time and compiled here as plain host C++:
//   - the integer mask helpers of the common header (MaskSpec, TileRange, key_tiles, ...);
//   - the forward header's tile constants, Params, Unit and decode_unit();
//   - the launch code's FwdSchedule and fwd_schedule().
// For dense and packed variable-length problems over every mask kind, group sizes with and
// without head pairs and both work orders, it walks every unit of the launch and checks:
//   1. every (batch row or sequence, query head, query row) is covered by exactly one unit
//      tile, and no tile covers a row past its sequence; a unit decode_unit() accepts has a row,
//      one it rejects has no row of its sequence;
//   2. both tiles of a unit read one kv head (h / G), the unit's K/V row block is that head's,
//      and paired heads are 2i and 2i + 1;
//   3. every key a row of the unit sees lies in a key tile of the unit's range;
//   4. a unit that visits the second tile's extra key tile first (rot) holds no key of that tile
//      visible to a row of the first tile, which skips that step.
// Prints "ok <configs> <rows checked>" or one "FAIL ..." line per failed check (at most 20).
#include <algorithm>
#include <cstdint>
#include <cstdio>
#include <vector>

#include "attn.h"

#define __host__
#define __device__
#define __forceinline__ inline

typedef uint16_t __nv_bfloat16;
template <typename T>
static inline T __ldg(const T* p) {
  return *p;
}

namespace attn {
using std::max;
using std::min;
constexpr int kT = 128;
#include "unit_logic.inc"
}  // namespace attn

using namespace attn;
using attn::fwd::Params;
using attn::fwd::Unit;

static int g_fail = 0;
#define CHECK(cond, ...)                  \
  do {                                    \
    if (!(cond)) {                        \
      if (g_fail < 20) {                  \
        std::printf("FAIL " __VA_ARGS__); \
        std::printf("\n");                \
        std::fflush(stdout);              \
      }                                   \
      ++g_fail;                           \
    }                                     \
  } while (0)

struct Config {
  int B, Hq, Hkv, mask, window, n_sink;
  std::vector<int> lens_q, lens_k;  // packed sequences; empty: dense with Nq, Nk below
  int Nq, Nk;
};

static MaskSpec make_spec(int kind, int w, int s, int nk) { return MaskSpec{kind, w, s, nk}; }

static long long check(const Config& c, int front_heavy) {
  const bool varlen = !c.lens_q.empty();
  const int nseq = varlen ? static_cast<int>(c.lens_q.size()) : c.B;
  std::vector<int> cu_q(nseq + 1, 0), cu_k(nseq + 1, 0);
  int max_q = 0;
  for (int s = 0; s < nseq; ++s) {
    const int lq = varlen ? c.lens_q[s] : c.Nq, lk = varlen ? c.lens_k[s] : c.Nk;
    cu_q[s + 1] = cu_q[s] + lq;
    cu_k[s + 1] = cu_k[s] + lk;
    max_q = std::max(max_q, lq);
  }
  const int total_q = cu_q[nseq], total_k = cu_k[nseq];
  const FwdSchedule sc = fwd_schedule(nseq, c.Hq, c.Hkv, varlen ? max_q : c.Nq);
  Params p{};
  p.B = nseq;
  p.Hq = c.Hq;
  p.Hkv = c.Hkv;
  p.Nq = varlen ? total_q : c.Nq;
  p.Nk = varlen ? total_k : c.Nk;
  p.G = c.Hq / c.Hkv;
  p.mask = make_spec(c.mask, c.window, c.n_sink, p.Nk);
  p.cu_q = varlen ? cu_q.data() : nullptr;
  p.cu_k = varlen ? cu_k.data() : nullptr;
  p.num_qblocks = sc.num_qblocks;
  p.front_heavy = front_heavy;
  p.head_pair = sc.head_pair;
  p.units = static_cast<int>(sc.units);
  CHECK(!sc.head_pair || p.G % 2 == 0, "head pairs with odd G=%d", p.G);

  // coverage[(s * Hq + h) * rows + i]
  const int rows = varlen ? max_q : c.Nq;
  std::vector<int> cover(static_cast<size_t>(nseq) * c.Hq * std::max(rows, 1), 0);
  for (int f = 0; f < p.units; ++f) {
    Unit U{};
    const bool has = varlen ? fwd::decode_unit<true, false>(p, f, U)
                            : fwd::decode_unit<false, false>(p, f, U);
    if (!has) {
      // a rejected unit: its rows lie wholly past its sequence
      const int groups = c.Hq / (sc.head_pair ? 2 : 1), nbh = nseq * groups;
      const int qb = front_heavy ? f / nbh : p.num_qblocks - 1 - f / nbh;
      const int s = (f % nbh) / groups;
      const int r0 = qb * (sc.head_pair ? fwd::kBM : fwd::kRowsPerCta);
      CHECK(r0 >= cu_q[s + 1] - cu_q[s], "unit %d rejected but row %d of sequence %d exists", f, r0, s);
      continue;
    }
    const int s = U.b;
    const int nq = cu_q[s + 1] - cu_q[s];
    CHECK(U.nq == nq, "unit %d: nq %d vs %d", f, U.nq, nq);
    CHECK(U.tiles != 0, "unit %d accepted without a row", f);
    CHECK(U.r0 >= 0, "unit %d starts at row %d", f, U.r0);
    if (U.r0 < 0) continue;
    CHECK(U.bkv == s * c.Hkv + U.h / p.G, "unit %d: K/V row block %d", f, U.bkv);
    if (sc.head_pair) CHECK(U.h % 2 == 0 && U.h + 1 < c.Hq, "unit %d: paired heads start at %d", f, U.h);
    const int nk = cu_k[s + 1] - cu_k[s];
    const MaskSpec m = make_spec(c.mask, c.window, c.n_sink, nk);
    for (int t = 0; t < 2; ++t) {
      const int row0 = sc.head_pair ? U.r0 : U.r0 + t * fwd::kBM;
      const int head = sc.head_pair ? U.h + t : U.h;
      const bool has_rows = row0 < nq;
      CHECK(((U.tiles >> t) & 1) == (has_rows ? 1 : 0), "unit %d tile %d: rows flag", f, t);
      if (!has_rows) continue;
      CHECK(head / p.G == U.h / p.G, "unit %d: tile %d reads kv head %d", f, t, head / p.G);
      for (int i = row0; i < std::min(row0 + fwd::kBM, nq); ++i) {
        ++cover[(static_cast<size_t>(s) * c.Hq + head) * rows + i];
        const int pos = i + U.off;
        for (int kt = 0; kt * fwd::kBN < nk; ++kt) {
          bool any = false;
          for (int j = kt * fwd::kBN; j < std::min((kt + 1) * fwd::kBN, nk); ++j)
            any = any || key_visible(m, pos, j);
          if (any) {
            CHECK(fwd::in_range(U.tr, kt), "unit %d row %d: visible key tile %d outside the range", f, i, kt);
            if (U.rot && t == 0) CHECK(kt != U.tr.hi, "unit %d row %d: tile 0 skips key tile %d it sees", f, i, kt);
          }
        }
      }
    }
  }
  long long checked = 0;
  for (int s = 0; s < nseq; ++s) {
    const int nq = cu_q[s + 1] - cu_q[s];
    for (int h = 0; h < c.Hq; ++h)
      for (int i = 0; i < rows; ++i) {
        const int n = cover[(static_cast<size_t>(s) * c.Hq + h) * rows + i];
        CHECK(n == (i < nq ? 1 : 0), "seq %d head %d row %d covered %d times", s, h, i, n);
        ++checked;
      }
  }
  return checked;
}

int main() {
  std::vector<Config> cfgs;
  const int heads[][2] = {{1, 1}, {4, 2}, {8, 1}, {6, 3}, {8, 8}, {32, 8}, {3, 1}, {4, 4}};
  const int kinds[][3] = {{ATTN_MASK_FULL, 0, 0},      {ATTN_MASK_CAUSAL, 0, 0},
                          {ATTN_MASK_SLIDING, 200, 4}, {ATTN_MASK_SLIDING, 1, 0},
                          {ATTN_MASK_LOCAL_GLOBAL, 100, 3}, {ATTN_MASK_LOCAL_GLOBAL, 0, 130}};
  for (auto& hk : heads)
    for (auto& mk : kinds) {
      for (int nq : {1, 127, 128, 129, 255, 256, 257, 700})
        for (int extra : {0, 100, -1}) {
          const int nk = extra < 0 ? std::max(1, nq / 2) : nq + extra;
          cfgs.push_back(Config{2, hk[0], hk[1], mk[0], mk[1], mk[2], {}, {}, nq, nk});
        }
      cfgs.push_back(Config{0, hk[0], hk[1], mk[0], mk[1], mk[2], {1, 127, 128, 129, 300},
                            {1, 127, 128, 129, 300}, 0, 0});
      cfgs.push_back(Config{0, hk[0], hk[1], mk[0], mk[1], mk[2], {513, 0, 64, 1000, 255},
                            {513, 0, 64, 1000, 255}, 0, 0});
      cfgs.push_back(Config{0, hk[0], hk[1], mk[0], mk[1], mk[2], {200, 700, 33},
                            {500, 700, 90}, 0, 0});
    }
  long long rows = 0;
  int n = 0;
  for (const Config& c : cfgs)
    for (int fh = 0; fh < 2; ++fh) {
      rows += check(c, fh);
      ++n;
    }
  if (g_fail) return 1;
  std::printf("ok %d %lld\n", n, rows);
  return 0;
}
