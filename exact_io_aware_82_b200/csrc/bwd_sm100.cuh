// Backward pass of exact attention on sm_100a: dQ, dK, dV from Q, K, V, dO and the forward's
// row log-sum-exp, recomputing the attention weights instead of storing them.
//
// "Quadratic Complexity Bottleneck" (inferensys.com), FlashAttention section: the backward pass
// recomputes attention instead of keeping the n x n matrix; "Chapter 3.1 - The Cost of
// Attention" (llmis.ru), section 5: FlashAttention trades "somewhat more FLOPs" for memory.
// With P_ij = exp(scale * q_i.k_j - LSE_i) on visible pairs (the LSE saved by the forward makes
// P exact without a second softmax pass):
//
//     dV_j = sum_i P_ij dO_i       dP_ij = dO_i . v_j       D_i = dO_i . O_i (= sum_j P_ij dP_ij)
//     dS_ij = P_ij (dP_ij - D_i)   dK_j = scale sum_i dS_ij q_i   dQ_i = scale sum_j dS_ij k_j
//
// Three launches:
//  1. bwd_prep_kernel: D_i and LSE_i * log2(e) per query row (memory-bound, one warp per row).
//  2. bwd_dkdv_kernel: one unit per (b, kv head, 128-key block), taken by persistent CTAs (one
//     per SM) from a counter, lowest key blocks first.  A unit walks the query tiles that see
//     the block, for each of the G query heads of the group, and keeps dK and dV of its keys in
//     tensor memory for the whole walk (no atomics; GQA sums in place).  Per step, four tcgen05
//     MMAs (128 x 128 x 128, bf16 in, fp32 accumulate): S^T = K Q^T and dP^T = V dO^T into TMEM;
//     the row warps (one TMEM lane = one key each) turn them into P^T and dS^T (bf16, written
//     back over S^T and dP^T); then dV += P^T dO and dK += dS^T Q with P^T / dS^T as the A operand
//     read from TMEM.
//     It also writes each (key block, query tile) block of dS^T (bf16, the values its own
//     dK MMA used) to a workspace slot.
//  3. bwd_dq_kernel: persistent CTAs take units of (b, query head, two 128-row query tiles) and
//     compute dQ = scale dS K as a plain tensor-core product over the dS^T blocks of each tile's
//     key tiles: no recomputation and no softmax, so it is bound by reading dS (2 bytes per
//     visible pair).
// Handing dS over through HBM instead of recomputing it (or of atomically adding dQ partials)
// costs a write and a read of dS but keeps every product on the tensor core exactly once, and
// the result does not depend on the order in which CTAs finish.
//
// Roles of each 352-thread CTA: warps 0-7 are the row workers (warps w and w+4 share TMEM lanes
// 32(w%4) .. 32(w%4)+31 and split the columns), one thread of warp 8 issues the score MMAs, one
// thread of warp 10 the accumulating MMAs, and one thread of warp 9 the TMA copies.
// Tensor memory (512 columns): [0,128) S or S^T, [128,256) dP or dP^T, [256,384) dV or dQ,
// [384,512) dK.  Every wait is bounded (see common.cuh).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "dev/ptx_store.cuh"

namespace attn {
namespace bwd {

constexpr int kT = 128;  // tile rows and columns (queries and keys)
constexpr int kD = 128;  // head dimension
constexpr int kRowThreads = 256;  // warps 0-7: two warps per TMEM lane quarter
constexpr int kThreads = kRowThreads + 96;
constexpr int kMmaWarp = 8;    // issues the score MMAs (S, dP)
constexpr int kLoadWarp = 9;
constexpr int kGradWarp = 10;  // issues the accumulating MMAs (dV, dK or dQ)
constexpr uint32_t kTileBytes = kT * kD * 2;  // 32 KB, bf16
constexpr uint32_t kHalfBytes = kT * 64 * 2;  // one 128-byte-swizzled 64-column half
constexpr float kLog2e = 1.4426950408889634f;

struct Params {
  int B, Hq, Hkv, Nq, Nk, G;
  MaskSpec mask;
  float c;      // scale * log2(e)
  float scale;
  const float* lse2;  // [B][Hq][npad] LSE * log2(e); +inf for a row that sees no key or is padding
  const float* dsum;  // [B][Hq][npad] D_i = dO_i . O_i; 0 for padding rows
  __nv_bfloat16* dq;  // [B][Hq][Nq][d]
  __nv_bfloat16* dk;  // [B][Hkv][Nk][d]
  __nv_bfloat16* dv;  // [B][Hkv][Nk][d]
  int num_kblocks;    // ceil(Nk / 128)
  int num_qtiles;     // ceil(Nq / 128)
  int npad;           // num_qtiles * 128: row stride of lse2 and dsum
  // dS^T handed from the dK/dV kernel to the dQ kernel: slot (b*Hq + h) * ds_pairs + ds_off[kb] +
  // (index of the query tile in key block kb's query-tile range) holds the 128 x 128 bf16 block
  // (keys x queries) of that pair
  __nv_bfloat16* ds;
  int* ds_off;         // [num_kblocks + 1], written by the prep kernel
  long long ds_pairs;  // ds_off[num_kblocks]: blocks per (b, query head)
  unsigned int* unit_counter;  // zero at launch; the dK/dV CTAs take key-block units from it
};

// Query tiles of one key block: [s0, ns) (the global rows of the local + global mask, when
// they are apart from the rest), then [lo, hi]; the two ranges never overlap.
struct QueryTiles {
  int s0, ns, lo, hi;
  __host__ __device__ int count() const { return (ns - s0) + (hi < lo ? 0 : hi - lo + 1); }
  __host__ __device__ int tile(int j) const { return j < ns - s0 ? s0 + j : lo + (j - (ns - s0)); }
};

// Index of query tile qt in key block kb's query tiles, or -1 if they miss it.
__host__ __device__ __forceinline__ int pair_index(const QueryTiles& r, int qt) {
  if (qt >= r.s0 && qt < r.ns) return qt - r.s0;
  if (qt >= r.lo && qt <= r.hi) return (r.ns - r.s0) + (qt - r.lo);
  return -1;
}

// ------------------------------------------------------------------------------------------
// helpers
// ------------------------------------------------------------------------------------------
__device__ __forceinline__ float pos_inf() { return __int_as_float(0x7f800000); }

__host__ __device__ __forceinline__ int imin(int a, int b) { return a < b ? a : b; }
__host__ __device__ __forceinline__ int imax(int a, int b) { return a > b ? a : b; }

__host__ __device__ __forceinline__ int floor_div128(long long a) {
  return static_cast<int>(a >= 0 ? a / kT : -((-a + kT - 1) / kT));
}

// Query tiles whose rows see at least one key of [c0, c1] (off = Nk - Nq; query row i sits at
// key position i + off).
__host__ __device__ __forceinline__ QueryTiles query_tiles(const MaskSpec& m, int c0, int c1,
                                                           int off, int Nq) {
  const int nqt = (Nq + kT - 1) / kT;
  QueryTiles r{0, 0, 0, nqt - 1};
  if (m.kind == ATTN_MASK_FULL) return r;
  if (m.kind == ATTN_MASK_LOCAL_GLOBAL) {
    if (c0 < m.n_sink) return r;  // a global key is seen by every row
    // the window rows: positions p in [c0 - w, c1 + w]
    r.lo = imax(0, floor_div128(static_cast<long long>(c0) - m.window - off));
    r.hi = imin(r.hi, floor_div128(static_cast<long long>(c1) + m.window - off));
    // the global rows: positions 0 <= p < n_global, i.e. rows [max(0, -off), n_global - off)
    // of [0, Nq); they end no later than the window rows do
    const long long g0 = off < 0 ? -static_cast<long long>(off) : 0;
    long long g1 = static_cast<long long>(m.n_sink) - off;
    if (g1 > Nq) g1 = Nq;
    if (g0 >= g1) return r;  // no global row
    const int ga = static_cast<int>(g0 / kT), gb = static_cast<int>((g1 - 1) / kT);
    if (r.lo > r.hi) {  // no window row: the global rows only
      r.lo = ga;
      r.hi = gb;
    } else if (gb + 1 >= r.lo) {  // touching or overlapping: one range
      r.lo = imin(r.lo, ga);
      r.hi = imax(r.hi, gb);
    } else {  // global tiles first, apart from the window tiles
      r.s0 = ga;
      r.ns = gb + 1;
    }
    return r;
  }
  // causal: p = i + off >= key  ->  i >= c0 - off for the block's first key
  r.lo = imax(0, floor_div128(static_cast<long long>(c0) - off));
  // window: p < key + w for keys past the sinks (a block holding a sink key is seen by every
  // later row)
  if (m.kind == ATTN_MASK_SLIDING && c0 >= m.n_sink)
    r.hi = imin(r.hi, floor_div128(static_cast<long long>(c1) + m.window - 1 - off));
  return r;
}

// Producer drain: wait until the last copy issued into stage s (of `issued` copies alternating
// between two stages) has landed.
__device__ __forceinline__ void drain_stage(uint32_t bar, int issued, int s) {
  const int u = (issued - 1 - s) >= 0 ? ((issued - 1 - s) & ~1) + s : -1;
  if (u >= 0) wait_drain(bar, (u >> 1) & 1);
}

// Untiled bulk copy global -> shared (16-byte aligned addresses, size a multiple of 16),
// completion counted on an mbarrier.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void store_zero_row(__nv_bfloat16* dst, int ch) {
  uint4* d4 = reinterpret_cast<uint4*>(dst + ch * 64);
#pragma unroll
  for (int i = 0; i < 8; ++i) d4[i] = make_uint4(0u, 0u, 0u, 0u);
}

// Packed bf16 weights of a 64-column sub-step live where each column half was read: columns
// [0, 32) pack into TMEM columns [0, 16), columns [32, 64) into [32, 48), so neither warp of a
// lane quarter overwrites scores the other has yet to load.  K-step ks (16 columns) of the
// accumulating MMA therefore starts at column:
__device__ __forceinline__ uint32_t packed_col(int ks) { return ks * 8 + (ks >= 2 ? 16 : 0); }

// ------------------------------------------------------------------------------------------
// 1. D_i = dO_i . O_i and LSE_i * log2(e) per (padded) query row
// ------------------------------------------------------------------------------------------
constexpr int kPrepRowsPerBlock = 64;  // 8 warps x 8 rows per grid-stride step

__global__ void __launch_bounds__(256)
    bwd_prep_kernel(const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ dout,
                    const float* __restrict__ lse, float* __restrict__ lse2,
                    float* __restrict__ dsum, int Nq, int npad, long long padded_rows,
                    MaskSpec mask, int num_kblocks, int* __restrict__ ds_off) {
  // the dS block offsets of the key blocks (a running count of their query tiles)
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    int acc = 0;
    for (int kb = 0; kb < num_kblocks; ++kb) {
      ds_off[kb] = acc;
      const int c0 = kb * kT, c1 = imin(c0 + kT, mask.Nk) - 1;
      acc += query_tiles(mask, c0, c1, mask.Nk - Nq, Nq).count();
    }
    ds_off[num_kblocks] = acc;
  }
  // a half-warp per row (16 lanes x 16 bytes = one 256-byte row of O and of dO); a warp takes
  // groups of 8 consecutive padded rows, grid-stride (one wave of blocks), every load of a group
  // issued before the first use
  const int lane = threadIdx.x & 31, sub = lane >> 4, sl = lane & 15;
  const long long ngroups = (padded_rows + 7) / 8;
  const long long stride = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  for (long long grp = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
       grp < ngroups; grp += stride) {
    uint4 a[4], g[4];
    long long src[4];
#pragma unroll
    for (int it = 0; it < 4; ++it) {
      const long long prow = grp * 8 + 2 * it + sub;
      src[it] = -1;
      if (prow < padded_rows) {
        const int i = static_cast<int>(prow % npad);
        if (i < Nq) src[it] = (prow / npad) * Nq + i;
      }
      a[it] = src[it] >= 0 ? *reinterpret_cast<const uint4*>(o + src[it] * kD + sl * 8)
                           : make_uint4(0u, 0u, 0u, 0u);
      g[it] = src[it] >= 0 ? *reinterpret_cast<const uint4*>(dout + src[it] * kD + sl * 8)
                           : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int it = 0; it < 4; ++it) {
      const uint32_t aw[4] = {a[it].x, a[it].y, a[it].z, a[it].w};
      const uint32_t gw[4] = {g[it].x, g[it].y, g[it].z, g[it].w};
      float acc = 0.f;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        acc = fmaf(__uint_as_float(aw[w] << 16), __uint_as_float(gw[w] << 16), acc);
        acc = fmaf(__uint_as_float(aw[w] & 0xffff0000u), __uint_as_float(gw[w] & 0xffff0000u), acc);
      }
#pragma unroll
      for (int sh = 8; sh > 0; sh >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, sh);
      const long long prow = grp * 8 + 2 * it + sub;
      if (sl == 0 && prow < padded_rows) {
        if (src[it] >= 0) {
          dsum[prow] = acc;
          const float l = lse[src[it]];
          lse2[prow] = (l == -pos_inf()) ? pos_inf() : l * kLog2e;
        } else {  // padding row past Nq
          dsum[prow] = 0.f;
          lse2[prow] = pos_inf();
        }
      }
    }
  }
}

// ------------------------------------------------------------------------------------------
// The two main kernels run the same software pipeline over sub-steps of 64 rows: sub-step m is
// half h = m & 1 of tile step m >> 1, and its two score-like products (S and dP, 128 x 64 fp32)
// go to TMEM buffer m & 1.  One thread issues those score MMAs as soon as their buffer is free
// (the accumulating MMAs of sub-step m-2, which read the bf16 weights stored there, have
// completed: barrier bar_free), another issues the accumulating MMAs of a sub-step as soon as
// the row warps have released its weights, so the tensor core computes sub-step m+1 (and the
// accumulating products of m-1) while the row warps turn sub-step m into bf16 weights.
// Tensor memory: S buffers at columns [0,64) and [64,128), dP buffers at [128,192) and
// [192,256), accumulators at [256,384) (dV or dQ) and [384,512) (dK).
// ------------------------------------------------------------------------------------------
constexpr int kSub = 64;                         // rows of a sub-step (columns of its scores)
constexpr uint32_t kSubBytes = kSub * 128;       // rows of a sub-step inside one 64-column half

// ------------------------------------------------------------------------------------------
// 2. dK, dV: one CTA per (b, kv head, key block)
// ------------------------------------------------------------------------------------------
// dS^T of one sub-step leaves through shared memory: each row warp stages its 32 keys x 32
// queries (64-byte rows, 64-byte swizzle) and stores them with one TMA box.
constexpr uint32_t kDsBoxBytes = 32 * 32 * 2;

struct __align__(1024) SmemKV {
  uint8_t k[kTileBytes];
  uint8_t v[kTileBytes];
  uint8_t q[2][kTileBytes];
  uint8_t dout[2][kTileBytes];
  uint8_t ds_stage[kRowThreads / 32][kDsBoxBytes];  // one box per row warp
  float lse2[2][kT];  // per stage: the query tile's LSE * log2(e) and D, copied with Q and dO
  float dsum[2][kT];
  uint64_t bar_kv, bar_kvempty, bar_qfull[2], bar_qempty[2], bar_s[2], bar_p[2], bar_free[2];
  uint64_t bar_done, bar_drain[2];
  uint64_t bar_unit_full[2], bar_unit_empty[2];
  int unit[2];  // published key-block units (-1: no more)
  uint32_t tmem_base;
  int abort;
};
constexpr size_t kSmemKVBytes = sizeof(SmemKV) + 1024;
static_assert(kSmemKVBytes <= 227 * 1024, "shared memory of the dK/dV kernel");

// The readers of a unit slot: the two MMA threads and the 8 row warps.
constexpr uint32_t kKVUnitReaders = 10;

// Key block kb of (b, kv head hk) for unit u: lowest blocks first (under a causal mask they have
// the most query tiles), the (b, kv head) pairs of one block adjacent.
struct KVUnit {
  int kb, bk, b, hk, c0, c1;
  QueryTiles qr;
  int nqt, nsteps;
};
__device__ __forceinline__ KVUnit kv_unit(const Params& p, int u) {
  KVUnit r;
  const int nbk = p.B * p.Hkv;
  r.kb = u / nbk;
  r.bk = u % nbk;
  r.b = r.bk / p.Hkv;
  r.hk = r.bk % p.Hkv;
  r.c0 = r.kb * kT;
  r.c1 = min(r.c0 + kT, p.Nk) - 1;
  r.qr = query_tiles(p.mask, r.c0, r.c1, p.Nk - p.Nq, p.Nq);
  r.nqt = r.qr.count();
  r.nsteps = r.nqt * p.G;  // step n: query head hk*G + n / nqt, query tile qr.tile(n % nqt)
  return r;
}

// Persistent: one CTA per SM takes key-block units from p.unit_counter (the last taker sets it
// back to zero).  The producer publishes each unit in one of two slots; the barrier phases, the
// Q/dO stage ring and the sub-step count run on across units.  A unit's K and V are loaded once
// the previous unit's last score products have completed (bar_kvempty), while the accumulating
// products and the row warps finish that unit; its first accumulating product, which overwrites
// dV and dK in TMEM, waits for the row warps' first weights of the unit, which they release only
// after reading out the previous unit's dV and dK.
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_do,
                    const __grid_constant__ CUtensorMap tm_ds,
                    const __grid_constant__ CUtensorMap tm_dk,
                    const __grid_constant__ CUtensorMap tm_dv, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  SmemKV& sm = *reinterpret_cast<SmemKV*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                          ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int off = p.Nk - p.Nq;

  if (tid == 0) {
    dev::mbar_init(dev::smem_u32(&sm.bar_kv), 1);
    dev::mbar_init(dev::smem_u32(&sm.bar_kvempty), 1);
    for (int s = 0; s < 2; ++s) {
      dev::mbar_init(dev::smem_u32(&sm.bar_qfull[s]), 1);
      dev::mbar_init(dev::smem_u32(&sm.bar_qempty[s]), 1);
      dev::mbar_init(dev::smem_u32(&sm.bar_s[s]), 1);
      dev::mbar_init(dev::smem_u32(&sm.bar_p[s]), kRowThreads);
      dev::mbar_init(dev::smem_u32(&sm.bar_free[s]), 1);
      dev::mbar_init(dev::smem_u32(&sm.bar_drain[s]), 1);
      dev::mbar_init(dev::smem_u32(&sm.bar_unit_full[s]), 1);
      dev::mbar_init(dev::smem_u32(&sm.bar_unit_empty[s]), kKVUnitReaders);
    }
    dev::mbar_init(dev::smem_u32(&sm.bar_done), 1);
    sm.abort = 0;
    dev::fence_barrier_init();
  }
  if (warp == kLoadWarp && lane == 0) {
    dev::tma_prefetch_desc(&tm_q);
    dev::tma_prefetch_desc(&tm_k);
    dev::tma_prefetch_desc(&tm_v);
    dev::tma_prefetch_desc(&tm_do);
    dev::tma_prefetch_desc(&tm_ds);
    dev::tma_prefetch_desc(&tm_dk);
    dev::tma_prefetch_desc(&tm_dv);
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
  const int units = p.num_kblocks * p.B * p.Hkv;

  if (warp == kLoadWarp) {
    // ============================ unit fetch + TMA producer ============================
    if (lane == 0) {
      int published = 0, kv_loads = 0, issued = 0;
      bool ok = true, exhausted = false;
      while (ok) {
        const int slot = published & 1;
        if (published >= 2 && !wait_bounded(dev::smem_u32(&sm.bar_unit_empty[slot]),
                                             ((published - 2) >> 1) & 1, abort)) {
          ok = false;
          break;
        }
        const int f = static_cast<int>(atomicAdd(p.unit_counter, 1u));
        if (f >= units) {
          if (f == units + static_cast<int>(gridDim.x) - 1) atomicExch(p.unit_counter, 0u);
          exhausted = true;
        }
        sm.unit[slot] = exhausted ? -1 : f;
        dev::mbar_arrive(dev::smem_u32(&sm.bar_unit_full[slot]));
        if (exhausted) break;
        ++published;
        const KVUnit u = kv_unit(p, f);
        if (u.nsteps == 0) continue;
        // K and V once the previous unit's score products have read them for good
        if (kv_loads > 0 &&
            !wait_bounded(dev::smem_u32(&sm.bar_kvempty), (kv_loads - 1) & 1, abort)) {
          ok = false;
          break;
        }
        const uint32_t bkv = dev::smem_u32(&sm.bar_kv);
        dev::mbar_arrive_expect_tx(bkv, 2 * kTileBytes);
        for (int half = 0; half < 2; ++half) {
          dev::tma_load_3d(dev::smem_u32(sm.k) + half * kHalfBytes, &tm_k, bkv, half * 64, u.c0, u.bk);
          dev::tma_load_3d(dev::smem_u32(sm.v) + half * kHalfBytes, &tm_v, bkv, half * 64, u.c0, u.bk);
        }
        ++kv_loads;
        for (int n = 0; n < u.nsteps; ++n) {
          const int g = issued;  // position in the Q/dO stage ring
          const int s = g & 1;
          if (!wait_bounded(dev::smem_u32(&sm.bar_qempty[s]), ((g >> 1) & 1) ^ 1, abort)) {
            ok = false;
            break;
          }
          const int hq = u.hk * p.G + n / u.nqt;
          const int r0 = u.qr.tile(n % u.nqt) * kT;
          const uint32_t bq = dev::smem_u32(&sm.bar_qfull[s]);
          const size_t vrow = static_cast<size_t>(u.b * p.Hq + hq) * p.npad + r0;
          dev::mbar_arrive_expect_tx(bq, 2 * kTileBytes + 2 * kT * 4);
          for (int half = 0; half < 2; ++half) {
            dev::tma_load_3d(dev::smem_u32(sm.q[s]) + half * kHalfBytes, &tm_q, bq, half * 64, r0,
                             u.b * p.Hq + hq);
            dev::tma_load_3d(dev::smem_u32(sm.dout[s]) + half * kHalfBytes, &tm_do, bq, half * 64,
                             r0, u.b * p.Hq + hq);
          }
          bulk_load(dev::smem_u32(sm.lse2[s]), p.lse2 + vrow, kT * 4, bq);
          bulk_load(dev::smem_u32(sm.dsum[s]), p.dsum + vrow, kT * 4, bq);
          ++issued;
        }
      }
      // a producer that gave up still takes its share of the counter, so that the last taker
      // resets it
      if (!exhausted) {
        while (true) {
          const int f = static_cast<int>(atomicAdd(p.unit_counter, 1u));
          if (f >= units) {
            if (f == units + static_cast<int>(gridDim.x) - 1) atomicExch(p.unit_counter, 0u);
            break;
          }
        }
      }
      if (kv_loads > 0) wait_drain(dev::smem_u32(&sm.bar_kv), (kv_loads - 1) & 1);
      for (int s = 0; s < 2; ++s) drain_stage(dev::smem_u32(&sm.bar_qfull[s]), issued, s);
    }
  } else if (warp == kMmaWarp || warp == kGradWarp) {
    // ========================= tcgen05.mma issuers (two threads) ==========================
    if (lane == 0) {
      constexpr uint32_t idesc_kk = dev::idesc_bf16_f32(kT, kSub, 0, 0);  // both K-major, N = 64
      constexpr uint32_t idesc_tm = dev::idesc_bf16_f32(kT, kD, 0, 1);    // A in TMEM, B MN-major
      const int role = warp == kMmaWarp ? 0 : 1;
      // operand descriptors of the two stages: K-major (score products) and MN-major
      // (accumulating products) views of Q and dO
      uint64_t dqk[2], dok[2], dqm[2], dom[2];
      for (int s = 0; s < 2; ++s) {
        dqk[s] = dev::smem_desc(dev::smem_u32(sm.q[s]), 16, 1024, dev::kSwizzle128B);
        dok[s] = dev::smem_desc(dev::smem_u32(sm.dout[s]), 16, 1024, dev::kSwizzle128B);
        dqm[s] = dev::smem_desc(dev::smem_u32(sm.q[s]), kHalfBytes, 1024, dev::kSwizzle128B);
        dom[s] = dev::smem_desc(dev::smem_u32(sm.dout[s]), kHalfBytes, 1024, dev::kSwizzle128B);
      }
      const uint64_t dka = dev::smem_desc(dev::smem_u32(sm.k), 16, 1024, dev::kSwizzle128B);
      const uint64_t dva = dev::smem_desc(dev::smem_u32(sm.v), 16, 1024, dev::kSwizzle128B);
      bool ok = true;
      int taken = 0;  // units read from the slots
      int mg = 0;     // sub-steps of all earlier units (the barrier phases run on)
      int kv_waits = 0;
      while (ok) {
        const int slot = taken & 1;
        if (!(ok = wait_bounded(dev::smem_u32(&sm.bar_unit_full[slot]), (taken >> 1) & 1, abort)))
          break;
        const int f = sm.unit[slot];
        ++taken;
        if (f < 0) break;
        const int nsub = 2 * kv_unit(p, f).nsteps;
        if (nsub > 0) {
          if (role == 0) {
            // S^T = K Q_h^T and dP^T = V dO_h^T for sub-step m (queries 64h .. 64h+63 of its tile)
            ok = wait_bounded(dev::smem_u32(&sm.bar_kv), kv_waits & 1, abort);
            ++kv_waits;
            for (int ml = 0; ok && ml < nsub; ++ml) {
              const int m = mg + ml;
              const int n = m >> 1, h = m & 1, s = n & 1;
              // buffer m & 1 is free once the accumulating MMAs of sub-step m - 2 have completed
              if (m >= 2 && !(ok = wait_bounded(dev::smem_u32(&sm.bar_free[m & 1]),
                                                ((m >> 1) - 1) & 1, abort)))
                break;
              if (h == 0 &&
                  !(ok = wait_bounded(dev::smem_u32(&sm.bar_qfull[s]), (n >> 1) & 1, abort)))
                break;
              dev::tc_fence_after();
              const uint32_t t_st = tmem + (m & 1) * kSub, t_dpt = tmem + 128 + (m & 1) * kSub;
              const uint32_t hoff = (h * kSubBytes) >> 4;
              const uint64_t bq = (s ? dqk[1] : dqk[0]) + hoff, bo = (s ? dok[1] : dok[0]) + hoff;
#pragma unroll
              for (int ks = 0; ks < kD / 16; ++ks) {
                const uint32_t koff = ((ks >> 2) * kHalfBytes + (ks & 3) * 32) >> 4;
                dev::umma_ss(t_st, dka + koff, bq + koff, idesc_kk, ks > 0 ? 1u : 0u);
              }
#pragma unroll
              for (int ks = 0; ks < kD / 16; ++ks) {
                const uint32_t koff = ((ks >> 2) * kHalfBytes + (ks & 3) * 32) >> 4;
                dev::umma_ss(t_dpt, dva + koff, bo + koff, idesc_kk, ks > 0 ? 1u : 0u);
              }
              dev::umma_commit(dev::smem_u32(&sm.bar_s[m & 1]));
            }
            // the unit's K and V are read for good once these products complete
            if (ok) dev::umma_commit(dev::smem_u32(&sm.bar_kvempty));
          } else {
            // dV += P^T dO_h and dK += dS^T Q_h (K = the 64 queries of the sub-step)
            for (int ml = 0; ok && ml < nsub; ++ml) {
              const int m = mg + ml;
              const int n = m >> 1, h = m & 1, s = n & 1;
              if (!(ok = wait_bounded(dev::smem_u32(&sm.bar_p[m & 1]), (m >> 1) & 1, abort))) break;
              dev::tc_fence_after();
              const uint32_t t_st = tmem + (m & 1) * kSub, t_dpt = tmem + 128 + (m & 1) * kSub;
              const uint64_t bo = s ? dom[1] : dom[0], bq = s ? dqm[1] : dqm[0];
#pragma unroll
              for (int ks = 0; ks < kSub / 16; ++ks) {
                const uint32_t acc = (ml > 0 || ks > 0) ? 1u : 0u;
                const uint32_t boff = (h * kSubBytes + ks * 16 * 128) >> 4;
                dev::umma_ts(tmem + 256, t_st + packed_col(ks), bo + boff, idesc_tm, acc);
                dev::umma_ts(tmem + 384, t_dpt + packed_col(ks), bq + boff, idesc_tm, acc);
              }
              dev::umma_commit(dev::smem_u32(&sm.bar_free[m & 1]));
              if (h == 1) dev::umma_commit(dev::smem_u32(&sm.bar_qempty[s]));  // stage s read for good
            }
            // the accumulators are final once this thread's MMAs have completed (every score MMA
            // completed before the row warps released the weights these read)
            if (ok) dev::umma_commit(dev::smem_u32(&sm.bar_done));
          }
          mg += nsub;
        }
        // this thread has issued every product of the unit
        dev::mbar_arrive(dev::smem_u32(&sm.bar_unit_empty[slot]));
      }
      dev::umma_commit(dev::smem_u32(&sm.bar_drain[role]));
      wait_drain(dev::smem_u32(&sm.bar_drain[role]), 0);
    }
  } else {
    // ============== row workers: one key each, two warps per key (column halves) ==============
    const int r = (warp & 3) * 32 + lane;  // TMEM lane = key c0 + r
    const int ch = warp >> 2;              // this warp's 32 of the 64 columns of a sub-step
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const float c = p.c;
    bool ok = true;
    int taken = 0;  // units read from the slots
    int mg = 0;     // sub-steps of all earlier units
    int dones = 0;  // units whose accumulators were read
    while (ok) {
      const int slot = taken & 1;
      ok = wait_bounded(dev::smem_u32(&sm.bar_unit_full[slot]), (taken >> 1) & 1, abort);
      if (!(ok = __all_sync(0xffffffffu, ok))) break;
      const int f = sm.unit[slot];
      ++taken;
      if (f < 0) break;
      const KVUnit u = kv_unit(p, f);
      const int j = u.c0 + r;
      const int nsub = 2 * u.nsteps;
      const long long ds_base = u.nsteps > 0 ? p.ds_off[u.kb] : 0;
      for (int ml = 0; ml < nsub; ++ml) {
        const int m = mg + ml;
        const int nl = ml >> 1, h = m & 1, s = (m >> 1) & 1, n = m >> 1;
        const int r0 = u.qr.tile(nl % u.nqt) * kT + h * kSub;  // first query row of the sub-step
        // the stage's LSE / D vectors came with its Q and dO tiles; the stage cannot be refilled
        // before this tile's weights are released, so its phase is still this tile's
        ok = wait_bounded(dev::smem_u32(&sm.bar_qfull[s]), (n >> 1) & 1, abort) &&
             wait_bounded(dev::smem_u32(&sm.bar_s[m & 1]), (m >> 1) & 1, abort);
        if (!(ok = __all_sync(0xffffffffu, ok))) break;
        dev::tc_fence_after();
        const uint32_t t_st = tmem + lane_off + (m & 1) * kSub + ch * 32;
        const uint32_t t_dpt = tmem + lane_off + 128 + (m & 1) * kSub + ch * 32;
        uint32_t sr[32], dr[32];
        dev::tmem_ld32(t_st, sr);
        dev::tmem_ld32(t_dpt, dr);

        // visible query columns of key j among this warp's 32 (columns past Nq: LSE = +inf):
        // [lo, hi], and for the local + global mask also the global rows [glo, ghi]
        const int P0 = r0 + off;
        uint32_t vis = ~0u;
        if (!block_visible(p.mask, P0, kSub, u.c0, kT)) {
          int lo = -1, hi = kT, glo = 0, ghi = -1;
          if (j >= p.mask.Nk) {
            hi = -1;
          } else if (p.mask.kind == ATTN_MASK_LOCAL_GLOBAL) {
            if (j >= p.mask.n_sink) {  // a global key is seen by every row
              lo = clamp_col(static_cast<long long>(j) - p.mask.window - P0);  // p >= j - w
              hi = clamp_col(static_cast<long long>(j) + p.mask.window - P0);  // p <= j + w
              glo = clamp_col(-static_cast<long long>(P0));                  // p >= 0
              ghi = clamp_col(static_cast<long long>(p.mask.n_sink) - 1 - P0);  // p < n_global
            }
          } else if (p.mask.kind != ATTN_MASK_FULL) {
            lo = clamp_col(static_cast<long long>(j) - P0);  // p >= j
            if (p.mask.kind == ATTN_MASK_SLIDING && j >= p.mask.n_sink)
              hi = clamp_col(static_cast<long long>(j) + p.mask.window - 1 - P0);  // p < j + w
          }
          vis = (cols_upto(hi, ch) & ~cols_upto(lo - 1, ch)) |
                (cols_upto(ghi, ch) & ~cols_upto(glo - 1, ch));
        }
        const float4* l2v = reinterpret_cast<const float4*>(sm.lse2[s] + h * kSub + ch * 32);
        const float4* ddv = reinterpret_cast<const float4*>(sm.dsum[s] + h * kSub + ch * 32);
        dev::tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) asm volatile("" : "+r"(sr[e]), "+r"(dr[e]));
        uint32_t pk[16], dk16[16];
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4) {
          const float4 l4 = l2v[e4], d4 = ddv[e4];
          const float lv[4] = {l4.x, l4.y, l4.z, l4.w}, dvv[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
          for (int e2 = 0; e2 < 4; e2 += 2) {
            const int e = e4 * 4 + e2;
            float p0 = dev::ex2_approx(fmaf(__uint_as_float(sr[e]), c, -lv[e2]));
            float p1 = dev::ex2_approx(fmaf(__uint_as_float(sr[e + 1]), c, -lv[e2 + 1]));
            p0 = ((vis >> e) & 1u) ? p0 : 0.f;
            p1 = ((vis >> (e + 1)) & 1u) ? p1 : 0.f;
            const float d0 = p0 * (__uint_as_float(dr[e]) - dvv[e2]);
            const float d1 = p1 * (__uint_as_float(dr[e + 1]) - dvv[e2 + 1]);
            pk[e >> 1] = dev::pack_bf16x2(p0, p1);
            dk16[e >> 1] = dev::pack_bf16x2(d0, d1);
          }
        }
        // P^T over S^T and dS^T over dP^T, packed into the first 16 of the 32 columns this warp
        // has just read (see packed_col)
        dev::tmem_st16(t_st, pk);
        dev::tmem_st16(t_dpt, dk16);
        {
          // the same bf16 dS^T values into this (key block, query tile) block for the dQ kernel:
          // rows 32 (warp & 3) .. +31 (keys), columns 64h + 32ch .. +31 (queries), staged in this
          // warp's box (64-byte swizzle: 16-byte chunk c of row r sits at chunk c ^ ((r >> 1) & 3))
          // once the box's previous store has read it, then one TMA store
          const int hq = u.hk * p.G + nl / u.nqt;
          const long long slot_ds =
              static_cast<long long>(u.b * p.Hq + hq) * p.ds_pairs + ds_base + nl % u.nqt;
          const uint32_t box = dev::smem_u32(sm.ds_stage[warp]);
          if (lane == 0) dev::bulk_wait_group_read0();  // the box's previous store has read it
          __syncwarp();
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4)
            dev::st_shared_v4(box + lane * 64 + (static_cast<uint32_t>(v4 ^ ((lane >> 1) & 3)) << 4),
                              dk16[4 * v4], dk16[4 * v4 + 1], dk16[4 * v4 + 2], dk16[4 * v4 + 3]);
          dev::fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            dev::tma_store_3d(&tm_ds, box, h * kSub + ch * 32, (warp & 3) * 32,
                              static_cast<int>(slot_ds));
            dev::bulk_commit_group();
          }
        }
        dev::tmem_wait_st();
        dev::tc_fence_before();
        dev::mbar_arrive(dev::smem_u32(&sm.bar_p[m & 1]));
      }
      mg += nsub;

      // ---- epilogue: dV and scale * dK rows of this unit's keys, bf16, a column half per warp ----
      // dV and dK leave TMEM before this warp releases the next unit's first weights (whose
      // accumulating product overwrites them)
      const bool valid = j < p.Nk;
      const size_t krow = static_cast<size_t>(u.bk) * p.Nk + j;
      __nv_bfloat16* dst_v = p.dv + krow * kD;
      __nv_bfloat16* dst_k = p.dk + krow * kD;
      if (u.nsteps == 0) {
        if (valid) {
          store_zero_row(dst_v, ch);
          store_zero_row(dst_k, ch);
        }
      } else if (ok) {
        ok = wait_bounded(dev::smem_u32(&sm.bar_done), dones & 1, abort);
        if ((ok = __all_sync(0xffffffffu, ok))) {
          dev::tc_fence_after();
          // dV then scale * dK, 32 keys x 32 columns at a time through this warp's box (as the
          // dS^T blocks), stored by TMA; keys past Nk are clipped by the tensor maps
#pragma unroll 1
          for (int w2 = 0; w2 < 4; ++w2) {
            const int which = w2 >> 1, cc = 2 * ch + (w2 & 1);
            uint32_t a[32];
            dev::tmem_ld32(tmem + lane_off + (which ? 384 : 256) + cc * 32, a);
            dev::tmem_wait_ld_regs(a);
            const float mul = which ? p.scale : 1.f;
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 32; e += 2)
              pk[e >> 1] = dev::pack_bf16x2(__uint_as_float(a[e]) * mul, __uint_as_float(a[e + 1]) * mul);
            const uint32_t box = dev::smem_u32(sm.ds_stage[warp]);
            if (lane == 0) dev::bulk_wait_group_read0();
            __syncwarp();
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4)
              dev::st_shared_v4(box + lane * 64 + (static_cast<uint32_t>(v4 ^ ((lane >> 1) & 3)) << 4),
                                pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
            dev::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              dev::tma_store_3d(which ? &tm_dk : &tm_dv, box, cc * 32, u.c0 + (warp & 3) * 32, u.bk);
              dev::bulk_commit_group();
            }
          }
        }
      }
      if (u.nsteps > 0) ++dones;
      dev::tc_fence_before();
      __syncwarp();
      if (lane == 0) dev::mbar_arrive(dev::smem_u32(&sm.bar_unit_empty[slot]));
    }
    // every staged box has been read by its store before the CTA can end
    if (lane == 0) dev::bulk_wait_group_read0();
    __syncwarp();
  }

  // ---- teardown ----
  dev::tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    dev::tc_fence_after();
    dev::tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------------------------------
// 3. dQ = scale dS K over the dS^T blocks the dK/dV kernel wrote.  A unit is a (b, query head,
//    pair of query tiles): tile qt = nqt-1-i (heavy under a causal mask) and tile i (light), so
//    units carry similar work.  Persistent CTAs (one per SM) take units from a counter.  dS^T
//    blocks and K tiles stream through a 3-stage ring (a unit's first tile's blocks, then its
//    second's, the ring running on across units); one thread issues the MMAs (A = dS read
//    MN-major from the [keys][queries] block, B = K MN-major) into one 128-column TMEM
//    accumulator per tile, the two accumulator pairs alternating between units so that warps
//    0-7 store one unit's dQ (staged in shared-memory boxes, stored by TMA) while the next
//    unit's products run.
// ------------------------------------------------------------------------------------------
constexpr int kDqStages = 3;
constexpr uint32_t kDqBoxBytes = 32 * 32 * 2;  // 32 rows x 32 columns, 64-byte swizzle

struct __align__(1024) SmemQ {
  uint8_t ds[kDqStages][kTileBytes];
  uint8_t k[kDqStages][kTileBytes];
  uint8_t stage[8][2][kDqBoxBytes];  // two output boxes per store warp, used in turn
  uint64_t bar_full[kDqStages], bar_empty[kDqStages], bar_drain;
  uint64_t bar_done[2];     // accumulator pair a: the unit's products completed + flags written
  uint64_t bar_accfree[2];  // accumulator pair a: read out by the store warps
  uint64_t bar_unit_full[2], bar_unit_empty[2];
  int unit[2];              // published units (-1: no more)
  int any[2];               // per accumulator pair: bit t = some dS block contributed to tile t
  uint32_t tmem_base;
  int abort;
};
constexpr size_t kSmemQBytes = sizeof(SmemQ) + 1024;
static_assert(kSmemQBytes <= 227 * 1024, "shared memory of the dQ kernel");

// The readers of a unit slot: the MMA thread and the 8 store warps.
constexpr uint32_t kQUnitReaders = 9;

__global__ void __launch_bounds__(kThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_ds,
                  const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_dq, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  SmemQ& sm = *reinterpret_cast<SmemQ*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                        ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nbh = p.B * p.Hq;
  const int off = p.Nk - p.Nq;
  const int units = ((p.num_qtiles + 1) / 2) * nbh;

  // unit f: (b, h) and its one or two query tiles with their key-tile ranges
  struct QUnit {
    int bh, bkv, ntiles, nsteps;
    int qts[2], nks[2];
    TileRange trs[2];
  };
  auto q_unit = [&](int f) {
    QUnit u;
    const int pi = f / nbh;
    u.bh = f % nbh;
    const int b = u.bh / p.Hq, h = u.bh % p.Hq;
    u.bkv = b * p.Hkv + h / p.G;
    u.qts[0] = p.num_qtiles - 1 - pi;
    u.qts[1] = pi;
    u.ntiles = u.qts[0] == u.qts[1] ? 1 : 2;
    u.nks[0] = u.nks[1] = 0;
    u.trs[1] = TileRange{0, 0, -1};
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      if (t >= u.ntiles) break;
      const int r0 = u.qts[t] * kT, last_row = min(r0 + kT, p.Nq) - 1;
      u.trs[t] = key_tiles(p.mask, r0 + off, last_row + off, kT);
      u.nks[t] = u.trs[t].count();
    }
    u.nsteps = u.nks[0] + (u.ntiles > 1 ? u.nks[1] : 0);
    return u;
  };
  // step jj of unit u: tile t = jj < nks[0] ? 0 : 1 and its key tile; a pair outside the key
  // block's query-tile range has no visible entry and no dS block (slot -1); the producer and
  // the MMA thread walk the same list
  auto step_slot = [&](const QUnit& u, int jj, int& t, int& kt) -> long long {
    t = jj < u.nks[0] ? 0 : 1;
    kt = t ? u.trs[1].tile(jj - u.nks[0]) : u.trs[0].tile(jj);
    const int c0 = kt * kT, c1 = min(c0 + kT, p.Nk) - 1;
    const int idx = pair_index(query_tiles(p.mask, c0, c1, off, p.Nq), t ? u.qts[1] : u.qts[0]);
    if (idx < 0) return -1;
    return static_cast<long long>(u.bh) * p.ds_pairs + p.ds_off[kt] + idx;
  };

  if (tid == 0) {
    for (int s = 0; s < kDqStages; ++s) {
      dev::mbar_init(dev::smem_u32(&sm.bar_full[s]), 1);
      dev::mbar_init(dev::smem_u32(&sm.bar_empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      dev::mbar_init(dev::smem_u32(&sm.bar_done[a]), 2);  // the MMA commit and the flags
      dev::mbar_init(dev::smem_u32(&sm.bar_accfree[a]), 8);
      dev::mbar_init(dev::smem_u32(&sm.bar_unit_full[a]), 1);
      dev::mbar_init(dev::smem_u32(&sm.bar_unit_empty[a]), kQUnitReaders);
    }
    dev::mbar_init(dev::smem_u32(&sm.bar_drain), 1);
    sm.abort = 0;
    dev::fence_barrier_init();
  }
  if (warp == kLoadWarp && lane == 0) {
    dev::tma_prefetch_desc(&tm_ds);
    dev::tma_prefetch_desc(&tm_k);
    dev::tma_prefetch_desc(&tm_dq);
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

  if (warp == kLoadWarp) {
    // ============================ unit fetch + TMA producer ============================
    if (lane == 0) {
      int published = 0, u = 0;  // u: copies started (the stage ring runs on across units)
      bool ok = true, exhausted = false;
      while (ok) {
        const int slot = published & 1;
        if (published >= 2 && !wait_bounded(dev::smem_u32(&sm.bar_unit_empty[slot]),
                                             ((published - 2) >> 1) & 1, abort)) {
          ok = false;
          break;
        }
        const int f = static_cast<int>(atomicAdd(p.unit_counter, 1u));
        if (f >= units) {
          if (f == units + static_cast<int>(gridDim.x) - 1) atomicExch(p.unit_counter, 0u);
          exhausted = true;
        }
        sm.unit[slot] = exhausted ? -1 : f;
        dev::mbar_arrive(dev::smem_u32(&sm.bar_unit_full[slot]));
        if (exhausted) break;
        ++published;
        const QUnit qu = q_unit(f);
        for (int jj = 0; jj < qu.nsteps; ++jj) {
          int t, kt;
          const long long dslot = step_slot(qu, jj, t, kt);
          if (dslot < 0) continue;
          const int s = u % kDqStages;
          if (!wait_bounded(dev::smem_u32(&sm.bar_empty[s]), ((u / kDqStages) & 1) ^ 1, abort)) {
            ok = false;
            break;
          }
          const uint32_t bf = dev::smem_u32(&sm.bar_full[s]);
          dev::mbar_arrive_expect_tx(bf, 2 * kTileBytes);
          for (int half = 0; half < 2; ++half) {
            dev::tma_load_3d(dev::smem_u32(sm.ds[s]) + half * kHalfBytes, &tm_ds, bf, half * 64, 0,
                             static_cast<int>(dslot));
            dev::tma_load_3d(dev::smem_u32(sm.k[s]) + half * kHalfBytes, &tm_k, bf, half * 64,
                             kt * kT, qu.bkv);
          }
          ++u;
        }
      }
      if (!exhausted) {
        // a producer that gave up still takes its share of the counter, so that the last taker
        // resets it
        while (true) {
          const int f = static_cast<int>(atomicAdd(p.unit_counter, 1u));
          if (f >= units) {
            if (f == units + static_cast<int>(gridDim.x) - 1) atomicExch(p.unit_counter, 0u);
            break;
          }
        }
      }
      // drain: the last copy into each stage has landed
      for (int s = 0; s < kDqStages; ++s) {
        const int last = (u - 1 - s) >= 0 ? (u - 1 - s) / kDqStages * kDqStages + s : -1;
        if (last >= 0) wait_drain(dev::smem_u32(&sm.bar_full[s]), (last / kDqStages) & 1);
      }
    }
  } else if (warp == kMmaWarp) {
    // ============================= tcgen05.mma issuer ==============================
    if (lane == 0) {
      constexpr uint32_t idesc = dev::idesc_bf16_f32(kT, kD, 1, 1);  // A and B MN-major
      bool ok = true;
      int u = 0, taken = 0;
      while (ok) {
        const int slot = taken & 1;
        if (!(ok = wait_bounded(dev::smem_u32(&sm.bar_unit_full[slot]), (taken >> 1) & 1, abort)))
          break;
        const int f = sm.unit[slot];
        const int un = taken++;  // this CTA's unit number: accumulator pair un & 1
        if (f < 0) break;
        const QUnit qu = q_unit(f);
        const int a = un & 1;
        // the pair's previous unit (two back) has been read out
        if (un >= 2 &&
            !(ok = wait_bounded(dev::smem_u32(&sm.bar_accfree[a]), ((un - 2) >> 1) & 1, abort)))
          break;
        int used[2] = {0, 0};
        for (int jj = 0; ok && jj < qu.nsteps; ++jj) {
          int t, kt;
          if (step_slot(qu, jj, t, kt) < 0) continue;
          const int s = u % kDqStages;
          if (!(ok = wait_bounded(dev::smem_u32(&sm.bar_full[s]), (u / kDqStages) & 1, abort))) break;
          dev::tc_fence_after();
          const uint64_t da = dev::smem_desc(dev::smem_u32(sm.ds[s]), kHalfBytes, 1024, dev::kSwizzle128B);
          const uint64_t db = dev::smem_desc(dev::smem_u32(sm.k[s]), kHalfBytes, 1024, dev::kSwizzle128B);
          const int first = t ? used[1] == 0 : used[0] == 0;
#pragma unroll
          for (int ks = 0; ks < kT / 16; ++ks)  // 16 keys (2 KB of each block) per MMA
            dev::umma_ss(tmem + a * 256 + t * 128, da + ((ks * 2048) >> 4),
                         db + ((ks * 2048) >> 4), idesc, (!first || ks > 0) ? 1u : 0u);
          dev::umma_commit(dev::smem_u32(&sm.bar_empty[s]));
          if (t) ++used[1]; else ++used[0];
          ++u;
        }
        if (!ok) break;
        // the products of the unit are done once this commit arrives; the flags follow
        dev::umma_commit(dev::smem_u32(&sm.bar_done[a]));
        sm.any[a] = (used[0] > 0 ? 1 : 0) | (used[1] > 0 ? 2 : 0);
        dev::mbar_arrive(dev::smem_u32(&sm.bar_done[a]));
        dev::mbar_arrive(dev::smem_u32(&sm.bar_unit_empty[slot]));
      }
      dev::umma_commit(dev::smem_u32(&sm.bar_drain));
      wait_drain(dev::smem_u32(&sm.bar_drain), 0);
    }
  } else if (warp < 8) {
    // ========= store: scale * dQ of each tile, a column half per warp, by TMA boxes =========
    const int r = (warp & 3) * 32 + lane;
    const int ch = warp >> 2;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    bool ok = true;
    int taken = 0, nbox = 0;
    while (ok) {
      const int slot = taken & 1;
      ok = wait_bounded(dev::smem_u32(&sm.bar_unit_full[slot]), (taken >> 1) & 1, abort);
      if (!(ok = __all_sync(0xffffffffu, ok))) break;
      const int f = sm.unit[slot];
      const int un = taken++;
      if (f < 0) break;
      const QUnit qu = q_unit(f);
      const int a = un & 1;
      ok = wait_bounded(dev::smem_u32(&sm.bar_done[a]), (un >> 1) & 1, abort);
      if (!(ok = __all_sync(0xffffffffu, ok))) break;
      dev::tc_fence_after();
      const int flags = sm.any[a];
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        if (t >= qu.ntiles) break;
        const int row0 = (t ? qu.qts[1] : qu.qts[0]) * kT;
        const int i = row0 + r;
        const bool valid = i < p.Nq;
        __nv_bfloat16* dst = p.dq + (static_cast<size_t>(qu.bh) * p.Nq + i) * kD;
        if (!(flags & (1 << t))) {
          if (valid) store_zero_row(dst, ch);
          continue;
        }
#pragma unroll 1
        for (int cc = 2 * ch; cc < 2 * ch + 2; ++cc) {
          uint32_t acc[32];
          dev::tmem_ld32(tmem + lane_off + a * 256 + t * 128 + cc * 32, acc);
          dev::tmem_wait_ld_regs(acc);
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 32; e += 2)
            pk[e >> 1] = dev::pack_bf16x2(__uint_as_float(acc[e]) * p.scale,
                                          __uint_as_float(acc[e + 1]) * p.scale);
          // 32 rows x 32 columns through this warp's box (64-byte swizzle: 16-byte chunk c of
          // row r at chunk c ^ ((r >> 1) & 3)), rewritten once the store before last from it
          // has read it; rows past Nq are clipped by the tensor map
          const uint32_t box = dev::smem_u32(sm.stage[warp][nbox & 1]);
          if (lane == 0) dev::bulk_wait_group_read1();
          __syncwarp();
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4)
            dev::st_shared_v4(box + lane * 64 + (static_cast<uint32_t>(v4 ^ ((lane >> 1) & 3)) << 4),
                              pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
          dev::fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            dev::tma_store_3d(&tm_dq, box, cc * 32, row0 + (warp & 3) * 32, qu.bh);
            dev::bulk_commit_group();
          }
          ++nbox;
        }
      }
      // this warp has read the accumulator pair and is done with the unit
      dev::tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        dev::mbar_arrive(dev::smem_u32(&sm.bar_accfree[a]));
        dev::mbar_arrive(dev::smem_u32(&sm.bar_unit_empty[slot]));
      }
    }
    // every staged box has been read by its store before the CTA can end
    if (lane == 0) dev::bulk_wait_group_read0();
    __syncwarp();
  }

  // ---- teardown ----
  dev::tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    dev::tc_fence_after();
    dev::tmem_dealloc(tmem, 512);
  }
}

}  // namespace bwd
}  // namespace attn
