// Exact attention forward for sm_100a: TMA -> shared memory -> tcgen05.mma (TMEM
// accumulators) -> online softmax in registers -> P back to TMEM -> tcgen05.mma for P V.
// Operands are bf16 (fwd_bf16_sm100_kernel, dense or packed variable-length) or E4M3 codes with
// per-(b, head) scales (fwd_fp8_sm100_kernel); every mask of common.cuh is supported.
//
// The method: "FlashAttention and sparse attention" (grasp.study), section 1 (tiling, kernel
// fusion, online softmax: running max and running sum, earlier partial results rescaled when
// the max grows); "Chapter 3.1 - The Cost of Attention" (llmis.ru), sections 5 and 6 (the score
// matrix never reaches HBM; work partitioned across thread blocks and warps); "Attention
// Research" (learning-materials), section 2 (TMA and warp specialisation as in
// FlashAttention-3, here re-expressed with tcgen05 and tensor memory).
//
// A work unit is two 128-row query tiles Q0, Q1 that share every K/V tile: the same 128 rows of
// two query heads of one kv head when the group size is even (both tiles then see exactly the
// same keys, so every step feeds both), otherwise 256 consecutive rows of one query head.  The
// grid is persistent (one CTA per SM, each walking units in order from a shared counter).
// Warp roles (12 warps = 3 warpgroups, 384 threads):
//   warps 0-3   softmax + epilogue for Q0 (thread t owns row t, TMEM lanes 0-127)
//   warps 4-7   softmax + epilogue for Q1
//   warp 8      TMEM allocation and the single-thread tcgen05.mma issuer
//   warp 9      unit fetch and decode (block-sparse: the unit's step list), TMA producer (Q once
//               per unit, then K_j and V_j through two 2-stage rings)
//   warps 10-11 idle (they complete the third warpgroup)
// Registers: launched at kRegsLaunch per thread; the two softmax warpgroups then raise their
// limit to kRegsSoftmax (a whole 128-column score row lives in registers) and the third
// warpgroup lowers its own to kRegsOther.  Per SM sub-partition (3 warps each) the split sums
// to the launch budget: 2 * kRegsSoftmax + kRegsOther == 3 * kRegsLaunch.
// Tensor memory (512 columns x 128 lanes, fp32): S0 [0,128) S1 [128,256) O0 [256,384)
// O1 [384,512).  P_t (bf16, two per column) overwrites the first 64 columns of S_t.
// MMA issue order per key tile j (ping-pong between the two query tiles):
//   PV0(j), S0(j+1), PV1(j), S1(j+1)
// so the tensor core computes one tile while the other tile's softmax runs; one thread issues
// both tiles' MMAs, so each tile's P V and next S run back to back at full rate (measured:
// two issuing threads interleave the tiles on the tensor core and lengthen both chains).
// tcgen05.mma executes in issue order, so S_t(j+1) never overwrites P_t(j) before PV_t(j)
// has read it, and the commit that signals S_t(j+1) also covers PV_t(j): the softmax may then
// rescale O_t.  A unit visits only the key tiles some of its rows can see; under a block-sparse
// layout each query tile takes only its selected tiles, otherwise both tiles take every step
// (an edge tile one of them cannot see adds exact zeros for it), except that in 256 causal rows
// of one head the second tile's diagonal tile goes first, to that tile alone.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "dev/ptx_f8.cuh"
#include "dev/ptx_store.cuh"

namespace attn {
namespace fwd {

constexpr int kBM = 128;  // query rows per tile
constexpr int kBN = 128;  // keys per tile
constexpr int kD = 128;   // head dimension
constexpr int kRowsPerCta = 2 * kBM;
constexpr int kThreads = 384;
constexpr int kMmaWarp = 8;
constexpr int kLoadWarp = 9;
constexpr uint32_t kRegsLaunch = 168;
constexpr uint32_t kRegsSoftmax = 208;
constexpr uint32_t kRegsOther = 88;
static_assert(2 * kRegsSoftmax + kRegsOther == 3 * kRegsLaunch, "register split must balance");
static_assert(kThreads * kRegsLaunch <= 65536, "launch register budget");
constexpr uint32_t kTileBytes = kBM * kD * 2;  // 32 KB, bf16
constexpr uint32_t kHalfBytes = kBM * 64 * 2;  // one 128-byte-swizzled column half
constexpr float kRescaleThreshold = 8.0f;      // log2 units: rescale O only if the max grows by >8


// E4M3 operands (kFp8): P is scaled by kPScaleF8 before it is rounded to E4M3 and the running
// maximum is refreshed whenever it grows by more than 4 (log2 units), so scaled P stays below
// 2^4 * 16 = 256 <= 448 (the largest E4M3 value) while weights down to 2^-13 of the reference
// keep a code.  (A threshold of 1 with a scale of 128 rescaled O every few steps and ran 10-15%
// slower.)
constexpr float kPScaleF8 = 16.0f;
constexpr float kLog2PScaleF8 = 4.0f;

constexpr float kRescaleThresholdF8 = 4.0f;

struct Params {
  int B, Hq, Hkv, Nq, Nk, G;  // packed variable-length mode: B = number of sequences,
                              // Nq / Nk = total query / key rows of the packed tensors
  MaskSpec mask;              // mask.Nk is replaced per sequence in variable-length mode
  const int* cu_q;            // variable-length mode: sequence s owns query rows
  const int* cu_k;            // [cu_q[s], cu_q[s+1]) and key rows [cu_k[s], cu_k[s+1])
  float c;  // scale * log2(e): scores are handled in log2 units (never 0, see the host code)
  int num_qblocks;
  // query blocks are taken in ascending order (the heaviest come first when the rows that see
  // the most keys are at the front: global query rows, or a block layout's global block row);
  // otherwise descending (causal and sliding masks: later rows see more keys)
  int front_heavy;
  // 1: a CTA takes rows [128 qb, 128 qb + 128) of query heads 2i and 2i + 1 (G even, so both
  // read kv head 2i / G); 0: rows [256 qb, 256 qb + 256) of one query head
  int head_pair;
  int units;                  // work units (query blocks x head groups x batch rows)
  unsigned int* unit_counter; // zero at launch; the CTAs take units from it in order and the
                              // last taker sets it back to zero
  __nv_bfloat16* o;
  float* lse;
  // E4M3 operands only: per (b, head) factors that turn the codes into values
  const float* descale_q;  // [B][Hq]
  const float* descale_k;  // [B][Hkv]
  const float* descale_v;  // [B][Hkv]
  // block-sparse layout (dense tensors only): block_mask[hm][query tile][key tile] != 0
  // selects that 128 x 128 block, hm = h when mask_heads == Hq and 0 when mask_heads == 1
  const uint8_t* block_mask;
  int mask_heads;
  int mask_qtiles, mask_ktiles;  // ceil(Nq / 128), ceil(Nk / 128)
};

// One work unit: the two query tiles of a CTA-sized block and the key tiles they visit.
// Decoded once by the producer warp and handed to the other roles through shared memory.
struct Unit {
  int valid;             // 0: the work is exhausted and the reader leaves
  int b, h;              // batch row (sequence in variable-length mode), first query head
  int bkv;               // row block of K/V in the dense [B * Hkv] layout
  int r0;                // first query row of the block (inside its sequence)
  int q_base, k_base;    // first packed row of the sequence (variable-length mode)
  int nq;                // query rows of the sequence
  int off;               // keys - queries of the sequence (key position of row i = i + off)
  int nk;                // steps: key tiles the unit visits
  int s_total;           // S products of the unit (steps summed over the query tiles)
  int tiles;             // bit t: query tile t has rows (without a block-sparse layout, a tile
                         // with rows takes part in every step of the unit, but see rot)
  int rot;               // 1: step 0 visits the second tile's extra key tile, which the first
                         // tile skips; steps 1.. visit the rest of the range in order
  MaskSpec mask;         // mask.Nk is the sequence's key count in variable-length mode
  TileRange tr, trt[2];  // key tiles of the unit and of each query tile
};

struct __align__(1024) Smem {
  uint8_t q[2][kTileBytes];
  uint8_t k[2][kTileBytes];
  uint8_t v[2][kTileBytes];
  uint64_t bar_q, bar_qempty;
  uint64_t bar_kfull[2], bar_kempty[2], bar_vfull[2], bar_vempty[2];
  uint64_t bar_s[2], bar_p[2], bar_o[2], bar_drain;
  uint64_t bar_unit_full[2], bar_unit_empty[2];
  Unit unit[2];
  uint32_t tmem_base;
  int abort;
};

// Output staging right after Smem: each softmax warp writes its 32 rows of O as boxes of 32
// rows x 32 columns (64-byte swizzle, 2 KB), stored by TMA; two boxes per warp alternate (one for
// block-sparse CTAs, whose step lists take the room).
constexpr uint32_t kOBoxBytes = 32 * 32 * 2;
constexpr int kOBoxesDense = 2, kOBoxesSparse = 1;
constexpr size_t kOStageDense = 8 * kOBoxesDense * kOBoxBytes;
constexpr size_t kOStageSparse = 8 * kOBoxesSparse * kOBoxBytes;

constexpr size_t kSmemBytes = sizeof(Smem) + kOStageDense + 1024;  // + slack to align to 1024 B

// Block-sparse units list the key tiles they visit (selected for one of their two query tiles
// and admitted by the base mask) after the output staging, one list per unit slot: per entry the
// key tile (low 14 bits) and which query tiles take part (bit 14 + t).
constexpr int kMaxSparseTiles = 4096;  // key tiles per row of the layout (Nk <= 524288)
struct SparseList {
  uint16_t e[kMaxSparseTiles];
  int count;
};
__device__ __forceinline__ int sparse_tile(const SparseList& sl, int j) { return sl.e[j] & 0x3fff; }
__device__ __forceinline__ bool sparse_part(const SparseList& sl, int j, int t) {
  return ((sl.e[j] >> (14 + t)) & 1u) != 0u;
}
constexpr size_t kSmemBytesSparse = sizeof(Smem) + kOStageSparse + 2 * sizeof(SparseList) + 1024;
static_assert(kSmemBytes <= 227 * 1024, "shared memory of a prefill CTA");
static_assert(kSmemBytesSparse <= 227 * 1024, "shared memory of a block-sparse CTA");

// The readers of a unit slot: the 8 softmax warps and the MMA thread.
constexpr uint32_t kUnitReaders = 9;

// Is every (row, key) of the 128x128 block of query tile rows [P0, P0+127] x keys of tile kt
// visible?  Conservative (uses all 128 rows even past Nq).
__device__ __forceinline__ bool tile_is_full(const MaskSpec& m, int P0, int kt) {
  return block_visible(m, P0, kBM, kt * kBN, kBN);
}

__device__ __forceinline__ float neg_inf() { return __int_as_float(0xff800000); }
__device__ __forceinline__ float pos_inf() { return __int_as_float(0x7f800000); }

// Work unit `unit` (0 <= unit < units): heaviest query blocks first, the G heads of a kv head
// adjacent.  Returns false for a block wholly past its sequence (variable-length mode).
template <bool kVarlen, bool kSparse>
__device__ __forceinline__ bool decode_unit(const Params& p, int unit, Unit& u) {
  const bool pair = p.head_pair != 0;
  const int heads_cta = pair ? 2 : 1;            // query heads of one unit
  const int rows_cta = pair ? kBM : kRowsPerCta;  // query rows of one unit (per head)
  const int groups = p.Hq / heads_cta;           // units of one query block per batch row
  const int nbh = p.B * groups;
  const int qb = p.front_heavy ? unit / nbh : p.num_qblocks - 1 - unit / nbh;
  u.b = (unit % nbh) / groups;
  u.h = (unit % nbh) % groups * heads_cta;
  u.bkv = u.b * p.Hkv + u.h / p.G;
  u.r0 = qb * rows_cta;
  u.q_base = 0;
  u.k_base = 0;
  u.nq = p.Nq;
  int nkeys = p.Nk;
  u.mask = p.mask;
  if (kVarlen) {
    u.q_base = __ldg(p.cu_q + u.b);
    u.k_base = __ldg(p.cu_k + u.b);
    // rows are clamped to the packed tensors, so inconsistent offsets cannot reach past them
    u.nq = u.q_base < 0 ? 0 : max(0, min(__ldg(p.cu_q + u.b + 1), p.Nq) - u.q_base);
    nkeys = u.k_base < 0 ? 0 : max(0, min(__ldg(p.cu_k + u.b + 1), p.Nk) - u.k_base);
    u.mask.Nk = nkeys;
    if (u.r0 >= u.nq) return false;  // this sequence is shorter
  }
  u.off = nkeys - u.nq;
  const int last_row = min(u.r0 + rows_cta, u.nq) - 1;
  // key tiles of the whole unit (what the producer loads, in this order) ...
  u.tr = key_tiles(u.mask, u.r0 + u.off, last_row + u.off, kBN);
  // ... and of each query tile.  Under a block-sparse layout a query tile visits only its own
  // key tiles.  Otherwise a query tile with rows takes part in every step of the unit: its
  // range differs from the unit's by at most a tile at either end (256 rows of one head under a
  // causal or window mask), whose entries are all masked and add exact zeros, and keeping both
  // tiles on every step lets them end together, so the next unit's products start at once
  // instead of after one tile's extra step.
  u.tiles = 0;
  u.rot = 0;
  for (int t = 0; t < 2; ++t) {
    const int lo_row = pair ? u.r0 : u.r0 + t * kBM, hi_row = min(lo_row + kBM, u.nq) - 1;
    if (hi_row >= lo_row) u.tiles |= 1 << t;
    u.trt[t] = hi_row < lo_row ? TileRange{0, 0, -1}
               : kSparse ? key_tiles(u.mask, lo_row + u.off, hi_row + u.off, kBN) : u.tr;
  }
  u.nk = u.tr.count();
  // 256 causal rows of one head: the second tile sees one key tile (its diagonal) beyond the
  // first tile's range.  That tile goes first, to the second tile alone, while the first tile
  // starts on the next step: both tiles then end on the same step without a masked step.
  if (!kSparse && !pair && u.tiles == 3 && u.mask.kind == ATTN_MASK_CAUSAL && u.tr.ns == 0) {
    const TileRange a = key_tiles(u.mask, u.r0 + u.off, u.r0 + kBM - 1 + u.off, kBN);
    if (a.ns == 0 && a.lo == u.tr.lo && a.hi + 1 == u.tr.hi) u.rot = 1;
  }
  return true;
}

// Key tile of step j of a unit (non-sparse): the range in order, or (rot) its last tile first.
__device__ __forceinline__ int unit_tile(const TileRange& tr, int rot, int j) {
  return rot ? (j == 0 ? tr.hi : tr.lo + (j - 1)) : tr.tile(j);
}

// does a query tile with key-tile range r take part in the step whose key tile is u?
__device__ __forceinline__ bool in_range(const TileRange& r, int u) {
  return u < r.ns || (u >= r.lo && u <= r.hi);
}

// kNeg: the scale is negative, so the largest scaled score comes from the smallest raw score.
// kVarlen: packed variable-length sequences ("What Lost, and Why", the sequence-packing note:
// attention is block diagonal, reset at every sequence boundary given by cu_seqlens); tensors
// are token-major, Q/O [total_q][Hq][d], K/V [total_k][Hkv][d], LSE [total_q][Hq], and each
// sequence is masked on its own (p_i = i + Nk_s - Nq_s).  Otherwise the dense [B][H][N][d] form.
// kFp8: Q, K, V hold E4M3 codes (a 128 x 128 tile is 16 KB, one 128-byte-wide TMA box) and both
// products run as kind::f8f6f4 MMAs, P being rounded to E4M3 (times kPScaleF8) in TMEM.
// kSparse: a block-sparse layout (Params::block_mask) further restricts the key tiles of each
// query tile ("Quadratic Complexity Bottleneck", sparse attention patterns: attention within and
// between selected blocks); dense bf16 tensors only.
//
// The grid is persistent: each CTA takes units from p.unit_counter in unit order (heaviest
// first) until they run out.  Every role walks the same unit sequence; the barrier phases, the
// K/V ring position and the per-tile step counts run on across units, so a step is the same
// whether it opens a unit or not.  The producer publishes each unit in one of two slots
// (bar_unit_full) and reuses a slot once its readers released it (bar_unit_empty); it loads the
// next unit's Q as soon as the MMA thread has issued the current unit's last S (bar_qempty), so
// the next unit's first S products follow the current unit's last P V while the softmax warps
// write the current unit's output.
template <bool kNeg, bool kVarlen, bool kFp8, bool kSparse>
__device__ __forceinline__ void fwd_sm100(const CUtensorMap& tm_q, const CUtensorMap& tm_k,
                                          const CUtensorMap& tm_v, const CUtensorMap& tm_o,
                                          const Params& p) {
  static_assert(!kSparse || (!kVarlen && !kFp8), "block-sparse layouts take dense bf16 tensors");
  constexpr int kHalves = kFp8 ? 1 : 2;                          // TMA boxes per tile
  constexpr uint32_t kTile = kFp8 ? kTileBytes / 2 : kTileBytes;  // bytes of one tile
  constexpr float kThreshold = kFp8 ? kRescaleThresholdF8 : kRescaleThreshold;
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                      ~uintptr_t(1023));
  constexpr int kOBoxes = kSparse ? kOBoxesSparse : kOBoxesDense;
  const uint32_t ostage = dev::smem_u32(&sm) + static_cast<uint32_t>(sizeof(Smem));
  SparseList* lists = reinterpret_cast<SparseList*>(reinterpret_cast<uint8_t*>(&sm) + sizeof(Smem) +
                                                    kOStageSparse);
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const bool pair = p.head_pair != 0;
  // query tile t of unit u: its first row and its query head
  auto tile_row0 = [&](const Unit& u, int t) { return pair ? u.r0 : u.r0 + t * kBM; };
  auto tile_head = [&](const Unit& u, int t) { return pair ? u.h + t : u.h; };
  // key tile of step j, and whether query tile t takes part in it
  auto step_tile = [&](const Unit& u, const SparseList& sl, int j) {
    return kSparse ? sparse_tile(sl, j) : unit_tile(u.tr, u.rot, j);
  };

  // ---- set-up ----
  if (tid == 0) {
    dev::mbar_init(dev::smem_u32(&sm.bar_q), 1);
    dev::mbar_init(dev::smem_u32(&sm.bar_qempty), 1);
    for (int s = 0; s < 2; ++s) {
      dev::mbar_init(dev::smem_u32(&sm.bar_kfull[s]), 1);
      dev::mbar_init(dev::smem_u32(&sm.bar_kempty[s]), 1);
      dev::mbar_init(dev::smem_u32(&sm.bar_vfull[s]), 1);
      dev::mbar_init(dev::smem_u32(&sm.bar_vempty[s]), 1);
      dev::mbar_init(dev::smem_u32(&sm.bar_s[s]), 1);
      dev::mbar_init(dev::smem_u32(&sm.bar_p[s]), kBM);
      dev::mbar_init(dev::smem_u32(&sm.bar_o[s]), 1);
      dev::mbar_init(dev::smem_u32(&sm.bar_unit_full[s]), 1);
      dev::mbar_init(dev::smem_u32(&sm.bar_unit_empty[s]), kUnitReaders);
    }
    dev::mbar_init(dev::smem_u32(&sm.bar_drain), 1);
    sm.abort = 0;
    dev::fence_barrier_init();
  }
  if (warp == kLoadWarp && lane == 0) {
    dev::tma_prefetch_desc(&tm_q);
    dev::tma_prefetch_desc(&tm_k);
    dev::tma_prefetch_desc(&tm_v);
    dev::tma_prefetch_desc(&tm_o);
  }
  if (warp == kMmaWarp) {
    dev::tmem_alloc(dev::smem_u32(&sm.tmem_base), 512);
    dev::tmem_relinquish();
  }
  dev::tc_fence_before();
  __syncthreads();
  dev::tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort = &sm.abort;
  if (warp >= 8) {
    // ========== third warpgroup: TMA producer, MMA issuer, two idle warps ==========
    dev::regs_decrease<kRegsOther>();
  if (warp == kLoadWarp) {
    // ============================ unit fetch + TMA producer ============================
    int published = 0;            // units handed to the other roles
    int q_loads = 0;              // Q copies started (one per unit with steps)
    int k_issued = 0, v_issued = 0;  // K / V copies started (the ring position runs on)
    bool ok = true, exhausted = false;
    while (ok) {
      const int slot = published & 1;
      // the slot's previous unit (two back) has been released by all its readers
      if (published >= 2 &&
          !wait_bounded(dev::smem_u32(&sm.bar_unit_empty[slot]), ((published - 2) >> 1) & 1, abort)) {
        ok = false;
        break;
      }
      // take units until one has rows; the last taker of the counter resets it for the next launch
      Unit u;
      u.valid = 0;
      while (true) {
        int f = 0;
        if (lane == 0) f = static_cast<int>(atomicAdd(p.unit_counter, 1u));
        f = __shfl_sync(0xffffffffu, f, 0);
        if (f >= p.units) {
          if (lane == 0 && f == p.units + static_cast<int>(gridDim.x) - 1) atomicExch(p.unit_counter, 0u);
          exhausted = true;
          break;
        }
        if (decode_unit<kVarlen, kSparse>(p, f, u)) {
          u.valid = 1;
          break;
        }
      }
      if (u.valid) {
        if (kSparse) {
          // the unit's steps: the range's key tiles selected for query tile 0 or 1, compacted in
          // range order by the warp (ballot + prefix count)
          SparseList& sl = lists[slot];
          const uint8_t* row[2];
          for (int t = 0; t < 2; ++t) {
            const int hm = p.mask_heads == 1 ? 0 : tile_head(u, t);
            row[t] = p.block_mask +
                     (static_cast<size_t>(hm) * p.mask_qtiles + tile_row0(u, t) / kBM) * p.mask_ktiles;
          }
          int base = 0, parts = 0;
          for (int j0 = 0; j0 < u.nk; j0 += 32) {
            const int j = j0 + lane;
            uint32_t bits = 0u;
            int kt = 0;
            if (j < u.nk) {
              kt = u.tr.tile(j);
              // a layout row is read only if its query tile has rows
              const bool t0 = in_range(u.trt[0], kt) && __ldg(row[0] + kt) != 0;
              const bool t1 = in_range(u.trt[1], kt) && __ldg(row[1] + kt) != 0;
              bits = (t0 ? 1u : 0u) | (t1 ? 2u : 0u);
            }
            const uint32_t sel = __ballot_sync(0xffffffffu, bits != 0u);
            if (bits != 0u) {
              const int pos = base + __popc(sel & ((1u << lane) - 1u));
              sl.e[pos] = static_cast<uint16_t>(kt | (bits << 14));
            }
            base += __popc(sel);
            parts += __reduce_add_sync(0xffffffffu, static_cast<uint32_t>(__popc(bits)));
          }
          u.nk = base;
          u.s_total = parts;
          if (lane == 0) sl.count = base;
        } else {
          u.s_total = u.nk * __popc(u.tiles) - u.rot;
        }
      }
      if (lane == 0) sm.unit[slot] = u;
      __threadfence_block();
      __syncwarp();
      if (lane == 0) dev::mbar_arrive(dev::smem_u32(&sm.bar_unit_full[slot]));
      if (!u.valid) break;
      ++published;
      if (lane == 0 && u.nk > 0) {
        const SparseList& sl = lists[slot];
        // Q of this unit once the previous unit's last S products have read the Q buffers
        if (q_loads > 0 && !wait_bounded(dev::smem_u32(&sm.bar_qempty), (q_loads - 1) & 1, abort)) {
          ok = false;
        } else {
          const uint32_t bq = dev::smem_u32(&sm.bar_q);
          dev::mbar_arrive_expect_tx(bq, 2 * kTile);
          for (int t = 0; t < 2; ++t)
            for (int half = 0; half < kHalves; ++half)
              if (kVarlen)
                dev::tma_load_3d(dev::smem_u32(sm.q[t]) + half * kHalfBytes, &tm_q, bq, half * 64,
                                 u.q_base + tile_row0(u, t), tile_head(u, t));
              else
                dev::tma_load_3d(dev::smem_u32(sm.q[t]) + half * kHalfBytes, &tm_q, bq, half * 64,
                                 tile_row0(u, t), u.b * p.Hq + tile_head(u, t));
          ++q_loads;
        }
        for (int j = 0; ok && j < u.nk; ++j) {
          const int kt = step_tile(u, sl, j);
          const int g = k_issued;  // ring position of this step
          const int s = g & 1;
          const uint32_t ph = ((g >> 1) & 1) ^ 1;
          if (!wait_bounded(dev::smem_u32(&sm.bar_kempty[s]), ph, abort)) { ok = false; break; }
          const uint32_t bk = dev::smem_u32(&sm.bar_kfull[s]);
          dev::mbar_arrive_expect_tx(bk, kTile);
          for (int half = 0; half < kHalves; ++half)
            if (kVarlen)
              dev::tma_load_3d(dev::smem_u32(sm.k[s]) + half * kHalfBytes, &tm_k, bk, half * 64,
                               u.k_base + kt * kBN, u.h / p.G);
            else
              dev::tma_load_3d(dev::smem_u32(sm.k[s]) + half * kHalfBytes, &tm_k, bk, half * 64,
                               kt * kBN, u.bkv);
          ++k_issued;
          if (!wait_bounded(dev::smem_u32(&sm.bar_vempty[s]), ph, abort)) { ok = false; break; }
          const uint32_t bv = dev::smem_u32(&sm.bar_vfull[s]);
          dev::mbar_arrive_expect_tx(bv, kTile);
          for (int half = 0; half < kHalves; ++half)
            if (kVarlen)
              dev::tma_load_3d(dev::smem_u32(sm.v[s]) + half * kHalfBytes, &tm_v, bv, half * 64,
                               u.k_base + kt * kBN, u.h / p.G);
            else
              dev::tma_load_3d(dev::smem_u32(sm.v[s]) + half * kHalfBytes, &tm_v, bv, half * 64,
                               kt * kBN, u.bkv);
          ++v_issued;
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    }
    if (lane == 0) {
      // a producer that gave up still takes its share of the counter, so that the last taker
      // resets it
      if (!exhausted) {
        while (true) {
          const int f = static_cast<int>(atomicAdd(p.unit_counter, 1u));
          if (f >= p.units) {
            if (f == p.units + static_cast<int>(gridDim.x) - 1) atomicExch(p.unit_counter, 0u);
            break;
          }
        }
      }
      // ---- drain: wait until every copy this thread started has landed ----
      if (q_loads > 0) wait_drain(dev::smem_u32(&sm.bar_q), (q_loads - 1) & 1);
      for (int s = 0; s < 2; ++s) {
        // the last load into stage s among loads 0..n-1 is u = largest u < n with u % 2 == s;
        // it completed phase (u / 2) of that stage's full barrier
        const int uk = (k_issued - 1 - s) >= 0 ? ((k_issued - 1 - s) & ~1) + s : -1;
        if (uk >= 0) wait_drain(dev::smem_u32(&sm.bar_kfull[s]), (uk >> 1) & 1);
        const int uv = (v_issued - 1 - s) >= 0 ? ((v_issued - 1 - s) & ~1) + s : -1;
        if (uv >= 0) wait_drain(dev::smem_u32(&sm.bar_vfull[s]), (uv >> 1) & 1);
      }
    }
  } else if (warp == kMmaWarp) {
    // ============================ tcgen05.mma issuer =============================
    if (lane == 0) {
      // Q, K both K-major; P (TMEM), V MN-major
      constexpr uint32_t idesc_s = kFp8 ? dev::idesc_e4m3_f32(kBM, kBN, 0, 0)
                                        : dev::idesc_bf16_f32(kBM, kBN, 0, 0);
      constexpr uint32_t idesc_o = kFp8 ? dev::idesc_e4m3_f32(kBM, kD, 0, 1)
                                        : dev::idesc_bf16_f32(kBM, kD, 0, 1);
      // Descriptors are built once; the second buffer of a pair and a K-step only move the start
      // address, which is the low field of the descriptor (addresses stay far below its 256 KB
      // range, so adding the offset >> 4 never carries out of the field).
      constexpr uint32_t kBufStep = kTileBytes >> 4;  // q[1] - q[0], k[1] - k[0], v[1] - v[0]
      const uint64_t dq0 = dev::smem_desc(dev::smem_u32(sm.q[0]), 16, 1024, dev::kSwizzle128B);
      const uint64_t dk0 = dev::smem_desc(dev::smem_u32(sm.k[0]), 16, 1024, dev::kSwizzle128B);
      const uint64_t dv0 =
          dev::smem_desc(dev::smem_u32(sm.v[0]), kHalfBytes, 1024, dev::kSwizzle128B);
      auto issue_s = [&](int t, int s) {
        const uint64_t a0 = dq0 + static_cast<uint64_t>(t * kBufStep);
        const uint64_t b0 = dk0 + static_cast<uint64_t>(s * kBufStep);
        const uint32_t d = tmem + t * 128;
        if constexpr (kFp8) {
          // K = 32 one-byte elements (32 bytes) per MMA, all inside one 128-byte swizzle row
#pragma unroll
          for (int ks = 0; ks < kD / 32; ++ks)
            dev::umma_ss_f8(d, a0 + ks * 2, b0 + ks * 2, idesc_s, ks > 0 ? 1u : 0u);
        } else {
#pragma unroll
          for (int ks = 0; ks < kD / 16; ++ks) {
            const uint32_t koff = ((ks >> 2) * kHalfBytes + (ks & 3) * 32) >> 4;
            dev::umma_ss(d, a0 + koff, b0 + koff, idesc_s, ks > 0 ? 1u : 0u);
          }
        }
      };
      auto issue_pv = [&](int t, int s, bool acc) {
        const uint64_t b0 = dv0 + static_cast<uint64_t>(s * kBufStep);
        const uint32_t d = tmem + 256 + t * 128;
        const uint32_t a = tmem + t * 128;
        if constexpr (kFp8) {
          // 32 keys per MMA: 8 TMEM columns of packed E4M3 P, 32 rows (4 KB) of V
#pragma unroll
          for (int ks = 0; ks < kBN / 32; ++ks)
            dev::umma_ts_f8(d, a + ks * 8, b0 + ((ks * 32 * 128) >> 4), idesc_o,
                            (acc || ks > 0) ? 1u : 0u);
        } else {
#pragma unroll
          for (int ks = 0; ks < kBN / 16; ++ks)
            dev::umma_ts(d, a + ks * 8, b0 + ((ks * 16 * 128) >> 4), idesc_o,
                         (acc || ks > 0) ? 1u : 0u);
        }
      };

      bool ok = true;
      int taken = 0;        // units read from the slots
      int q_waits = 0;      // Q copies consumed (units with steps)
      int gbase = 0;        // ring position of the unit's first step
      int ptot[2] = {0, 0}; // P barrier phases completed per tile, over all units
      while (ok) {
        const int slot = taken & 1;
        if (!(ok = wait_bounded(dev::smem_u32(&sm.bar_unit_full[slot]), (taken >> 1) & 1, abort))) break;
        const Unit& us = sm.unit[slot];
        const SparseList& sl = lists[slot];
        ++taken;
        if (!us.valid) break;
        const int nk = us.nk, s_total = us.s_total, tiles = us.tiles, rot = us.rot;
        auto takes = [&](int t, int j) {
          if (kSparse) return sparse_part(sl, j, t);
          return ((tiles >> t) & 1) != 0 && !(rot && t == 0 && j == 0);
        };
        if (nk == 0) {
          dev::mbar_arrive(dev::smem_u32(&sm.bar_unit_empty[slot]));
          continue;
        }
        // K_j lives in k[g & 1] (phase (g >> 1) & 1 of its barriers), g = gbase + j; V likewise
        auto wait_k = [&](int j) {
          const int g = gbase + j;
          return wait_bounded(dev::smem_u32(&sm.bar_kfull[g & 1]), (g >> 1) & 1, abort);
        };
        auto wait_v = [&](int j) {
          const int g = gbase + j;
          return wait_bounded(dev::smem_u32(&sm.bar_vfull[g & 1]), (g >> 1) & 1, abort);
        };
        auto next_step = [&](int t, int j) {
          int q = j + 1;
          while (q < nk && !takes(t, q)) ++q;
          return q;
        };
        // per tile: cur = the step whose S has been issued and whose P V is next; cnt = steps
        // of this unit whose P V has been issued
        int cur0 = next_step(0, -1), cur1 = next_step(1, -1);
        int cnt0 = 0, cnt1 = 0;
        int s_issued = 0;
        // K_j can be waited for at any time up to step j + 2: K_(j+2) reuses the slot of K_j,
        // which is released at the end of step j - 1.  A block-sparse tile may skip many steps
        // (the other tile takes them); the S of a step more than two ahead is then deferred
        // (pend) and issued during the step before it, ahead of that K slot's release.  Without
        // a layout a tile with rows takes every step.
        int pend0 = -1, pend1 = -1;
        auto issue_s_at = [&](int t, int j) {
          if (!wait_k(j)) return false;
          dev::tc_fence_after();
          issue_s(t, (gbase + j) & 1);
          dev::umma_commit(dev::smem_u32(&sm.bar_s[t]));
          // the unit's last S product: once it completes, the producer may refill the Q buffers
          if (++s_issued == s_total) dev::umma_commit(dev::smem_u32(&sm.bar_qempty));
          return true;
        };
        auto first_s = [&](int t, int cur) {
          if (cur >= nk) return true;
          if (kSparse && cur > 1) {
            (t ? pend1 : pend0) = cur;
            return true;
          }
          return issue_s_at(t, cur);
        };
        // one step of tile t at step j: P V, then the S of its next step (or the final commit)
        auto step = [&](int t, int j, int& cur, int& cnt) {
          if (cur != j) return true;
          if (!wait_bounded(dev::smem_u32(&sm.bar_p[t]), ptot[t] & 1, abort)) return false;
          dev::tc_fence_after();
          issue_pv(t, (gbase + j) & 1, cnt > 0);
          ++cnt;
          ++ptot[t];
          const int nxt = next_step(t, j);
          if (nxt < nk) {
            if (kSparse && nxt > j + 2) {
              (t ? pend1 : pend0) = nxt;
            } else if (!issue_s_at(t, nxt)) {
              return false;
            }
          } else {
            dev::umma_commit(dev::smem_u32(&sm.bar_o[t]));
          }
          cur = nxt;
          return true;
        };
        ok = wait_bounded(dev::smem_u32(&sm.bar_q), q_waits & 1, abort);
        ++q_waits;
        // first S of each tile, earlier key tile first (the producer loads in step order)
        if (ok) ok = cur0 <= cur1 ? (first_s(0, cur0) && first_s(1, cur1))
                                  : (first_s(1, cur1) && first_s(0, cur0));
        // K_0 is released once every S that reads it is issued; a slot is always waited for
        // before it is handed back, so a copy still landing is never overwritten
        if (ok) {
          if ((ok = wait_k(0))) dev::umma_commit(dev::smem_u32(&sm.bar_kempty[gbase & 1]));
        }
        for (int j = 0; ok && j < nk; ++j) {
          if (!(ok = wait_v(j))) break;
          if (!(ok = step(0, j, cur0, cnt0) && step(1, j, cur1, cnt1))) break;
          if constexpr (kSparse) {
            // deferred S of step j + 1 (K_(j+1) is released below)
            if (pend0 == j + 1) {
              if (!(ok = issue_s_at(0, j + 1))) break;
              pend0 = -1;
            }
            if (pend1 == j + 1) {
              if (!(ok = issue_s_at(1, j + 1))) break;
              pend1 = -1;
            }
          }
          // every P V reading V_j and every S reading K_(j+1) is issued by now
          dev::umma_commit(dev::smem_u32(&sm.bar_vempty[(gbase + j) & 1]));
          if (j + 1 < nk) {
            if (!(ok = wait_k(j + 1))) break;
            dev::umma_commit(dev::smem_u32(&sm.bar_kempty[(gbase + j + 1) & 1]));
          }
        }
        gbase += nk;
        // every MMA of the unit is issued: the slot may be reused once the softmax warps are done
        dev::mbar_arrive(dev::smem_u32(&sm.bar_unit_empty[slot]));
      }
      // drain: every MMA issued above has completed once this commit arrives
      dev::umma_commit(dev::smem_u32(&sm.bar_drain));
      wait_drain(dev::smem_u32(&sm.bar_drain), 0);
    }
  }
  } else {
    // ====================== softmax + epilogue (one row per thread) ======================
    dev::regs_increase<kRegsSoftmax>();
    const int t = warp >> 2;    // query tile of this warpgroup
    const int row = tid & 127;  // row inside the tile == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t t_s = tmem + lane_off + t * 128;
    const uint32_t t_o = tmem + lane_off + 256 + t * 128;
    const float masked = kNeg ? pos_inf() : neg_inf();
    // O_t *= alpha (per row), in tensor memory; O_t is complete here (the commit for S_t(j)
    // covered PV_t(j-1)) and the next P V has not been issued
    auto rescale_o = [&](float alpha) {
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t o[32];
        dev::tmem_ld32(t_o + cc * 32, o);
        dev::tmem_wait_ld_regs(o);
#pragma unroll
        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
        dev::tmem_st32(t_o + cc * 32, o);
      }
    };
    bool ok = true;
    int taken = 0;  // units read from the slots
    int stot = 0;   // S barrier phases completed for this tile, over all units
    int otot = 0;   // O barrier phases completed for this tile, over all units
    while (ok) {
      const int slot = taken & 1;
      ok = wait_bounded(dev::smem_u32(&sm.bar_unit_full[slot]), (taken >> 1) & 1, abort);
      if (!(ok = __all_sync(0xffffffffu, ok))) break;
      const Unit& us = sm.unit[slot];
      if (!us.valid) break;
      ++taken;
      const SparseList& sl = lists[slot];
      const int nk = us.nk;
      const TileRange utr = us.tr;  // step j -> key tile (dense)
      const int rot = us.rot;
      const bool mine = ((us.tiles >> t) & 1) != 0;  // this tile has rows
      const MaskSpec mask = us.mask;
      const int P0 = tile_row0(us, t) + us.off;  // key position of the tile's first row
      const int prow = P0 + row;                 // key position of this thread's row
      // scores in log2 units: c = scale * log2(e), times the Q and K descale factors for E4M3
      const float c = kFp8 ? p.c * __ldg(p.descale_q + us.b * p.Hq + tile_head(us, t)) *
                                 __ldg(p.descale_k + us.bkv)
                           : p.c;
      float m_ref = neg_inf();  // running max (log2 units) used as the exponent reference
      float l = 0.f;            // running sum of exp2(s*c - m_ref)
      int cnt = 0;              // steps this tile has processed in this unit
      for (int j = 0; j < nk; ++j) {
        const int kt = kSparse ? sparse_tile(sl, j) : unit_tile(utr, rot, j);
        if (kSparse ? !sparse_part(sl, j, t) : (!mine || (rot && t == 0 && j == 0))) continue;
        ok = wait_bounded(dev::smem_u32(&sm.bar_s[t]), stot & 1, abort);
        if (!(ok = __all_sync(0xffffffffu, ok))) break;
        dev::tc_fence_after();
        const int key0 = kt * kBN;

        // the whole 128-column score row of this thread, one wait
        uint32_t r[128];
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) dev::tmem_ld32(t_s + cc * 32, r + cc * 32);
        dev::tmem_wait_ld_regs(r);

        const bool full = tile_is_full(mask, P0, kt);
        if (!full) {
          // visible columns of this row inside the tile: (lo <= col <= hi) or col < sk,
          // as a 128-bit set built with shifts, then one bit test and select per column (no
          // per-column branches, whatever the compiler knows about hi, lo and sk)
          int hi, lo, sk;
          row_cols(mask, prow, key0, hi, lo, sk);
          uint32_t vis[4];
#pragma unroll
          for (int w = 0; w < 4; ++w)
            vis[w] = row_bits(hi, lo, sk, w);
#pragma unroll
          for (int e = 0; e < 128; ++e)
            r[e] = ((vis[e >> 5] >> (e & 31)) & 1u) ? r[e] : __float_as_uint(masked);
        }

        // row max of the raw scores (min when the scale is negative): 3-input max tree
        auto row_max = [&]() {
          float a[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) a[i] = __uint_as_float(r[i]);
#pragma unroll
          for (int e = 8; e < 120; e += 16) {
#pragma unroll
            for (int i = 0; i < 8; ++i)
              a[i] = kNeg ? dev::min3(a[i], __uint_as_float(r[e + i]), __uint_as_float(r[e + 8 + i]))
                          : dev::max3(a[i], __uint_as_float(r[e + i]), __uint_as_float(r[e + 8 + i]));
          }
          // the loop folded columns 8..119 into a[]; fold 120..127, then reduce a[] to one value
#pragma unroll
          for (int i = 0; i < 8; ++i)
            a[i] = kNeg ? fminf(a[i], __uint_as_float(r[120 + i])) : fmaxf(a[i], __uint_as_float(r[120 + i]));
          const float mx =
              kNeg ? dev::min3(dev::min3(a[0], a[1], a[2]), dev::min3(a[3], a[4], a[5]), fminf(a[6], a[7]))
                   : dev::max3(dev::max3(a[0], a[1], a[2]), dev::max3(a[3], a[4], a[5]), fmaxf(a[6], a[7]));
          return (mx == masked) ? neg_inf() : mx * c;  // in log2 units
        };

        // P = exp2(s*c - m_use) -> bf16 pairs over the first 64 columns of S_t (E4M3: four
        // codes of kPScaleF8 * P per column over the first 32); the row sum accumulates in 8
        // independent packed pairs
        float2 acc[4];
        auto weights = [&](float m_ref_now) {
          const float m_use = (m_ref_now == neg_inf()) ? 0.f : m_ref_now;
#pragma unroll
          for (int i = 0; i < 4; ++i) acc[i] = make_float2(0.f, 0.f);
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            if constexpr (kFp8) {
              // the exponent carries log2(kPScaleF8), so the weights come out already scaled
              // for the E4M3 product (the row sum takes the factor back out below)
              const uint64_t c2 = dev::pack2(c, c);
              const uint64_t nm2 = dev::pack2(kLog2PScaleF8 - m_use, kLog2PScaleF8 - m_use);
              uint32_t pk[16];
#pragma unroll
              for (int e = 0; e < 64; e += 4) {
                const int col = half * 64 + e;
                float2 pr[2];
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                  const int cc2 = col + 2 * h2;
                  const float2 xx = dev::unpack2(dev::fma2(
                      dev::pack2(__uint_as_float(r[cc2]), __uint_as_float(r[cc2 + 1])), c2, nm2));
                  pr[h2] = make_float2(dev::ex2_approx(xx.x), dev::ex2_approx(xx.y));
                }
                acc[(e >> 1) & 3] = dev::add2(acc[(e >> 1) & 3], pr[0]);
                acc[((e >> 1) + 1) & 3] = dev::add2(acc[((e >> 1) + 1) & 3], pr[1]);
                pk[e >> 2] = dev::pack_e4m3x4(pr[0].x, pr[0].y, pr[1].x, pr[1].y);
              }
              dev::tmem_st16(t_s + half * 16, pk);
            } else {
              // s * c - m_use two at a time (packed fp32 FMA), 2^x on the multi-function unit
              const uint64_t c2 = dev::pack2(c, c), nm2 = dev::pack2(-m_use, -m_use);
              uint32_t pk[32];
#pragma unroll
              for (int e = 0; e < 64; e += 2) {
                const int col = half * 64 + e;
                const float2 xx = dev::unpack2(dev::fma2(
                    dev::pack2(__uint_as_float(r[col]), __uint_as_float(r[col + 1])), c2, nm2));
                const float2 pr = make_float2(dev::ex2_approx(xx.x), dev::ex2_approx(xx.y));
                acc[(e >> 1) & 3] = dev::add2(acc[(e >> 1) & 3], pr);
                pk[e >> 1] = dev::pack_bf16x2(pr.x, pr.y);
              }
              dev::tmem_st32(t_s + half * 32, pk);
            }
          }
        };

        const float tmax = row_max();
        const float m_new = fmaxf(m_ref, tmax);
        float alpha = 1.f;
        if (m_new > m_ref + kThreshold) {
          alpha = dev::ex2_approx(m_ref - m_new);  // 0 when m_ref = -inf
          m_ref = m_new;
        }
        l *= alpha;
        if (cnt > 0 && __any_sync(0xffffffffu, alpha != 1.f)) rescale_o(alpha);
        weights(m_ref);
        acc[0] = dev::add2(acc[0], acc[1]);
        acc[2] = dev::add2(acc[2], acc[3]);
        acc[0] = dev::add2(acc[0], acc[2]);
        l += kFp8 ? (acc[0].x + acc[0].y) * (1.f / kPScaleF8) : acc[0].x + acc[0].y;
        dev::tmem_wait_st();
        dev::tc_fence_before();
        dev::mbar_arrive(dev::smem_u32(&sm.bar_p[t]));
        ++cnt;
        ++stot;
      }

      // ---- epilogue: O = O / l in bf16, LSE = ln(sum exp(scale * s)) ----
      // O_t leaves TMEM before this warpgroup releases its next P (the next unit's first P V
      // overwrites O_t), so the next unit's first S products may already be running.
      if (ok && cnt > 0) ok = wait_bounded(dev::smem_u32(&sm.bar_o[t]), otot & 1, abort);
      if (cnt > 0) ++otot;
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
        dev::tc_fence_after();
        // the unit's fields again from its slot (kept out of registers during the steps)
        const int hq = tile_head(us, t), bkv = us.bkv;
        const int grow = tile_row0(us, t) + row;
        const bool valid = grow < us.nq;
        // E4M3: undo the scale of P and apply the V descale factor
        const float o_mul = kFp8 ? __ldg(p.descale_v + bkv) / kPScaleF8 : 1.f;
        const float inv_l = l > 0.f ? o_mul / l : 0.f;
        const size_t orow = kVarlen ? static_cast<size_t>(us.q_base + grow) * p.Hq + hq
                                    : static_cast<size_t>(us.b * p.Hq + hq) * p.Nq + grow;
        uint4* dst = reinterpret_cast<uint4*>(p.o + orow * kD);
        // This warp's 32 rows leave as four boxes of 32 rows x 32 columns, staged (64-byte
        // swizzle: 16-byte chunk c of row r at chunk c ^ ((r >> 1) & 3)) in this warp's boxes and
        // stored by TMA; a box is rewritten once the store before last from it has read it.  A
        // box of packed sequences must not reach past its sequence: such rows use plain stores
        // (a dense box is clipped at Nq by the tensor map).
        const int wrow0 = tile_row0(us, t) + (warp & 3) * 32;  // first row of this warp's boxes
        const bool tma_out = wrow0 < us.nq && (!kVarlen || wrow0 + 31 < us.nq);
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t o[32];
          if (cnt > 0) {
            dev::tmem_ld32(t_o + cc * 32, o);
            dev::tmem_wait_ld_regs(o);
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = 0u;
          }
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 32; e += 2)
            pk[e >> 1] = dev::pack_bf16x2(__uint_as_float(o[e]) * inv_l,
                                          __uint_as_float(o[e + 1]) * inv_l);
          if (tma_out) {
            const uint32_t box = ostage + (warp * kOBoxes + (cc % kOBoxes)) * kOBoxBytes;
            if (lane == 0) {
              if (kOBoxes == 2) dev::bulk_wait_group_read1();
              else dev::bulk_wait_group_read0();
            }
            __syncwarp();
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4)
              dev::st_shared_v4(box + lane * 64 + (static_cast<uint32_t>(v4 ^ ((lane >> 1) & 3)) << 4),
                                pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
            dev::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              dev::tma_store_3d(&tm_o, box, cc * 32, kVarlen ? us.q_base + wrow0 : wrow0,
                                kVarlen ? hq : us.b * p.Hq + hq);
              dev::bulk_commit_group();
            }
          } else if (valid) {
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4)
              dst[cc * 4 + v4] = make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
          }
        }
        if (valid && p.lse != nullptr) {
          const float m_use = (m_ref == neg_inf()) ? 0.f : m_ref;
          p.lse[orow] =
              l > 0.f ? (m_use + log2f(l)) * 0.69314718055994531f : neg_inf();
        }
      }
      // this warp is done with the unit slot
      dev::tc_fence_before();
      __syncwarp();
      if (lane == 0) dev::mbar_arrive(dev::smem_u32(&sm.bar_unit_empty[slot]));
    }
  }

  // ---- teardown ----
  if (warp < 8 && lane == 0) dev::bulk_wait_group_read0();  // the staged boxes have been read
  dev::tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    dev::tc_fence_after();
    dev::tmem_dealloc(tmem, 512);
  }
}

// bf16 Q, K, V (dense or packed variable-length)
template <bool kNeg, bool kVarlen>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_bf16_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                          const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v,
                          const __grid_constant__ CUtensorMap tm_o, const Params p) {
  fwd_sm100<kNeg, kVarlen, false, false>(tm_q, tm_k, tm_v, tm_o, p);
}

// bf16 Q, K, V (dense) under a block-sparse layout
template <bool kNeg>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_bf16_sparse_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                                 const __grid_constant__ CUtensorMap tm_k,
                                 const __grid_constant__ CUtensorMap tm_v,
                                 const __grid_constant__ CUtensorMap tm_o, const Params p) {
  fwd_sm100<kNeg, false, false, true>(tm_q, tm_k, tm_v, tm_o, p);
}

// E4M3 Q, K, V with per-(b, head) descale factors (dense)
template <bool kNeg>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_fp8_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                         const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v,
                         const __grid_constant__ CUtensorMap tm_o, const Params p) {
  fwd_sm100<kNeg, false, true, false>(tm_q, tm_k, tm_v, tm_o, p);
}

}  // namespace fwd
}  // namespace attn
