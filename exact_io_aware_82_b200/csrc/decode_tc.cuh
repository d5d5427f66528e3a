// Split-K decode on the tensor cores, contiguous or paged KV cache.
//
// The method is that of decode.cuh ("Attention Research" (learning-materials), section 1: a
// decode step reads the whole KV cache, so it is bound by HBM bandwidth; section 2:
// FlashDecoding splits the keys of one decode step across thread blocks; the splits are merged
// exactly by the log-sum-exp combine of decode.cuh).  What changes is who does the arithmetic:
// here the K and V tiles stream through shared memory by TMA and both products run on the
// tensor core, so the CUDA cores only see G scores per key instead of 2 G d multiply-adds per
// key (which kept decode.cuh issue-bound).
//
// One CTA = one split (at most kMaxTiles tiles of 128 keys) of one (sequence, kv head); the G
// query heads of the group are the N = 16 columns (G real, the rest padding) of
//   S^T = K_t Q^T        (M = 128 keys, N = 16 heads, K = d; A = K tile, B = Q, both K-major)
// so every score of the split lands in tensor memory (lane = key, 16 columns per tile).  With
// all scores present the split's maximum is exact: P = 2^(s c - m) needs no rescaling, is
// written to shared memory as bf16 in the layout of a K-major operand, and
//   O^T += V_t^T P_t^T   (M = 128 = d, N = 16 heads, K = keys; A = V tile, MN-major)
// accumulates the split's output in tensor memory (lane = head-dimension index).
//
// Warps: 0-3 softmax and epilogue (thread i owns TMEM lane i: key i of every tile, then output
// column i), 4 the single-thread tcgen05.mma issuer (and the TMEM allocation), 5 the TMA
// producer (Q once, then every K tile, then every V tile, through a 2-stage ring).  Two CTAs
// fit on one SM, so one CTA's set-up and epilogue overlap the other's streaming.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "decode.cuh"
#include "dev/ptx_store.cuh"

namespace attn {
namespace dtc {

constexpr int kD = 128;
constexpr int kTile = 128;                    // keys per tile
constexpr int kMaxTiles = 8;                  // tiles per split
constexpr int kMaxChunk = kTile * kMaxTiles;  // keys per split
constexpr int kN = 16;                        // MMA N: the group's query heads, padded
constexpr int kSoftThreads = 128;
constexpr int kThreads = kSoftThreads + 64;
constexpr int kMmaWarp = 4;
constexpr int kLoadWarp = 5;
constexpr int kStages = 2;
constexpr uint32_t kTileBytes = kTile * kD * 2;      // 32 KB, bf16
constexpr uint32_t kHalfBytes = kTile * 64 * 2;      // one 128-byte-swizzled column half
constexpr uint32_t kQHalfBytes = kN * 64 * 2;        // 2 KB
constexpr uint32_t kPBlockBytes = kN * 64 * 2;       // P^T rows of 64 keys: 16 x 128 bytes
constexpr uint32_t kPTileBytes = 2 * kPBlockBytes;   // 4 KB per tile of 128 keys
constexpr uint32_t kTmemCols = 256;                  // S^T: kMaxTiles x 16 columns; O^T: 16
constexpr uint32_t kOCol = kMaxTiles * kN;
// Paged caches take this kernel from 64-key pages up: with 16-key pages the 16 boxes per tile
// streamed slower than the CUDA-core kernel's loads (4.7 vs 5.5 TB/s); with 64- and 256-key
// pages faster (6.2-6.3 vs 5.1-5.4 TB/s).
constexpr int kMinTcPageShift = 6;

struct __align__(1024) Smem {
  uint8_t ring[kStages][kTileBytes];
  uint8_t p[kMaxTiles][kPTileBytes];
  uint8_t q[2][kQHalfBytes];
  float red_max[4][8];
  float red_sum[4][8];
  uint64_t bar_q, bar_full[kStages], bar_empty[kStages], bar_s, bar_p, bar_o, bar_drain;
  uint32_t tmem_base;
  int abort;
};
constexpr size_t kSmemBytes = sizeof(Smem) + 1024;  // + slack to align the base to 1024 B
static_assert(2 * (kSmemBytes + 1024) <= 228 * 1024, "two CTAs per SM");

__device__ __forceinline__ void softmax_bar_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kSoftThreads) : "memory");
}

// Q: [B * Hq][d] (one token per sequence); partials as decode.cuh: ws_o [B][Hq][splits][d]
// (O_s / l_s), ws_lse [B][Hq][splits] (natural log).
// kPaged = false: K, V [B][Hkv][Nk][d], maps (d, Nk, B * Hkv) read as 128-key boxes.
// kPaged = true: the paged cache of decode.cuh, K, V [num_pages][page_size][Hkv][d], maps
// (d, num_pages * page_size, Hkv) read as boxes of min(page_size, 32) keys (chunks are whole
// multiples of 32 keys, so a box never crosses a page); a page number outside the cache is not
// followed (the box is taken past the last row, which reads as zero) and is flagged.
template <int G, bool kPaged>
__global__ void __launch_bounds__(kThreads, 2)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, float* __restrict__ ws_o,
                     float* __restrict__ ws_lse, int Hq, int Hkv, int Nk, int chunk, int splits,
                     float c, dec::Paged pg) {
  static_assert(G == 1 || G == 2 || G == 4 || G == 8, "query heads per kv head");
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                      ~uintptr_t(1023));
  const int s = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int j0 = s * chunk;
  // keys of this sequence: Nk (contiguous cache) or its own length (paged cache)
  const int len = kPaged ? max(0, min(__ldg(pg.seq_lens + b), Nk)) : Nk;
  const int n = max(0, min(len - j0, chunk));  // keys of this split
  const int T = (n + kTile - 1) / kTile;
  auto out_row = [&](int g) { return (static_cast<size_t>(b) * Hq + hk * G + g) * splits + s; };

  if (n == 0) {
    // a split past the last key: an empty partial, which the combine gives no weight
    for (int idx = tid; idx < G * kD; idx += kThreads) {
      const size_t row = out_row(idx / kD);
      ws_o[row * kD + idx % kD] = 0.f;
      if (idx % kD == 0) ws_lse[row] = -INFINITY;
    }
    return;
  }

  // ---- set-up ----
  if (tid == 0) {
    dev::mbar_init(dev::smem_u32(&sm.bar_q), 1);
    for (int st = 0; st < kStages; ++st) {
      dev::mbar_init(dev::smem_u32(&sm.bar_full[st]), 1);
      dev::mbar_init(dev::smem_u32(&sm.bar_empty[st]), 1);
    }
    dev::mbar_init(dev::smem_u32(&sm.bar_s), 1);
    dev::mbar_init(dev::smem_u32(&sm.bar_p), kSoftThreads);
    dev::mbar_init(dev::smem_u32(&sm.bar_o), 1);
    dev::mbar_init(dev::smem_u32(&sm.bar_drain), 1);
    sm.abort = 0;
    dev::fence_barrier_init();
  }
  // P^T starts as zeros: the rows of padding heads are never written
  for (int idx = tid; idx < T * static_cast<int>(kPTileBytes / 16); idx += kThreads)
    dev::st_shared_v4(dev::smem_u32(&sm.p[0][0]) + idx * 16, 0u, 0u, 0u, 0u);
  dev::fence_proxy_async_smem();
  if (warp == kLoadWarp && lane == 0) {
    dev::tma_prefetch_desc(&tm_q);
    dev::tma_prefetch_desc(&tm_k);
    dev::tma_prefetch_desc(&tm_v);
  }
  if (warp == kMmaWarp) {
    dev::tmem_alloc(dev::smem_u32(&sm.tmem_base), kTmemCols);
    dev::tmem_relinquish();
  }
  dev::tc_fence_before();
  __syncthreads();
  dev::tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort = &sm.abort;

  if (warp == kLoadWarp) {
    // ================================ TMA producer ================================
    if (lane == 0) {
      const uint32_t bq = dev::smem_u32(&sm.bar_q);
      dev::mbar_arrive_expect_tx(bq, 2 * kQHalfBytes);
      for (int half = 0; half < 2; ++half)
        dev::tma_load_3d(dev::smem_u32(sm.q[half]), &tm_q, bq, half * 64, b * Hq + hk * G, 0);
      int issued = 0;
      for (int u = 0; u < 2 * T; ++u) {  // K tiles 0..T-1, then V tiles 0..T-1
        const int st = u & 1;
        if (!wait_bounded(dev::smem_u32(&sm.bar_empty[st]), ((u >> 1) & 1) ^ 1, abort)) break;
        const uint32_t bf = dev::smem_u32(&sm.bar_full[st]);
        dev::mbar_arrive_expect_tx(bf, kTileBytes);
        const CUtensorMap* map = u < T ? &tm_k : &tm_v;
        const int row = j0 + (u < T ? u : u - T) * kTile;  // rows past Nk read as zero
        if constexpr (!kPaged) {
          for (int half = 0; half < 2; ++half)
            dev::tma_load_3d(dev::smem_u32(sm.ring[st]) + half * kHalfBytes, map, bf, half * 64,
                             row, b * Hkv + hk);
        } else {
          // pieces of min(page_size, 32) keys, each inside one page
          const int psize = 1 << pg.page_shift;
          const int piece = psize < 32 ? psize : 32;
          const long long rows_total = static_cast<long long>(pg.num_pages) << pg.page_shift;
          for (int r = 0; r < kTile; r += piece) {
            const int key = row + r;  // logical key of the piece's first row
            int tok = static_cast<int>(rows_total);  // past the last row: reads as zero
            if (key < len) {
              const int lp = key >> pg.page_shift;
              const int phys = lp < pg.max_pages ? __ldg(pg.block_table + static_cast<size_t>(b) * pg.max_pages + lp) : -1;
              if (phys >= 0 && phys < pg.num_pages)
                tok = (phys << pg.page_shift) + (key & (psize - 1));
              else
                atomicExch(&g_device_error, ATTN_ERR_INVALID_ARG);
            }
            for (int half = 0; half < 2; ++half)
              dev::tma_load_3d(dev::smem_u32(sm.ring[st]) + half * kHalfBytes + r * 128, map, bf,
                               half * 64, tok, hk);
          }
        }
        ++issued;
      }
      // ---- drain: every copy this thread started has landed before the CTA ends ----
      wait_drain(bq, 0);
      for (int st = 0; st < kStages; ++st) {
        const int u = (issued - 1 - st) >= 0 ? ((issued - 1 - st) & ~1) + st : -1;
        if (u >= 0) wait_drain(dev::smem_u32(&sm.bar_full[st]), (u >> 1) & 1);
      }
    }
  } else if (warp == kMmaWarp) {
    // ============================= tcgen05.mma issuer ==============================
    if (lane == 0) {
      constexpr uint32_t idesc_s = dev::idesc_bf16_f32(kTile, kN, 0, 0);  // K tile, Q: K-major
      constexpr uint32_t idesc_o = dev::idesc_bf16_f32(kD, kN, 1, 0);     // V^T MN-major, P^T K-major
      const uint64_t dq = dev::smem_desc(dev::smem_u32(sm.q[0]), 16, 1024, dev::kSwizzle128B);
      bool ok = wait_bounded(dev::smem_u32(&sm.bar_q), 0, abort);
      for (int t = 0; ok && t < T; ++t) {
        const int st = t & 1;
        if (!(ok = wait_bounded(dev::smem_u32(&sm.bar_full[st]), (t >> 1) & 1, abort))) break;
        dev::tc_fence_after();
        const uint64_t a0 = dev::smem_desc(dev::smem_u32(sm.ring[st]), 16, 1024, dev::kSwizzle128B);
#pragma unroll
        for (int ks = 0; ks < kD / 16; ++ks) {
          const uint32_t ka = ((ks >> 2) * kHalfBytes + (ks & 3) * 32) >> 4;
          const uint32_t kb = ((ks >> 2) * kQHalfBytes + (ks & 3) * 32) >> 4;
          dev::umma_ss(tmem + t * kN, a0 + ka, dq + kb, idesc_s, ks > 0 ? 1u : 0u);
        }
        dev::umma_commit(dev::smem_u32(&sm.bar_empty[st]));
      }
      if (ok) dev::umma_commit(dev::smem_u32(&sm.bar_s));
      if (ok) ok = wait_bounded(dev::smem_u32(&sm.bar_p), 0, abort);
      for (int t = 0; ok && t < T; ++t) {
        const int u = T + t, st = u & 1;
        if (!(ok = wait_bounded(dev::smem_u32(&sm.bar_full[st]), (u >> 1) & 1, abort))) break;
        dev::tc_fence_after();
        const uint64_t a0 =
            dev::smem_desc(dev::smem_u32(sm.ring[st]), kHalfBytes, 1024, dev::kSwizzle128B);
        const uint64_t b0 = dev::smem_desc(dev::smem_u32(sm.p[t]), 16, 1024, dev::kSwizzle128B);
#pragma unroll
        for (int ks = 0; ks < kTile / 16; ++ks) {
          const uint32_t ka = (ks * 16 * 128) >> 4;  // 16 keys of 128-byte rows
          const uint32_t kb = ((ks >> 2) * kPBlockBytes + (ks & 3) * 32) >> 4;
          dev::umma_ss(tmem + kOCol, a0 + ka, b0 + kb, idesc_o, (t > 0 || ks > 0) ? 1u : 0u);
        }
        dev::umma_commit(dev::smem_u32(&sm.bar_empty[st]));
      }
      if (ok) dev::umma_commit(dev::smem_u32(&sm.bar_o));
      // drain: every MMA issued above has completed once this commit arrives
      dev::umma_commit(dev::smem_u32(&sm.bar_drain));
      wait_drain(dev::smem_u32(&sm.bar_drain), 0);
    }
  } else {
    // ================ softmax and epilogue: thread i owns TMEM lane i ================
    const int i = tid;
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    bool ok = wait_bounded(dev::smem_u32(&sm.bar_s), 0, abort);
    ok = __all_sync(0xffffffffu, ok);
    // scores of key t * 128 + i, in log2 units (-inf past the split's last key)
    float x[kMaxTiles][G];
    float mx[G];
#pragma unroll
    for (int g = 0; g < G; ++g) mx[g] = -INFINITY;
    if (ok) {
      dev::tc_fence_after();
      uint32_t raw[kMaxTiles][G];
#pragma unroll
      for (int t = 0; t < kMaxTiles; ++t)
        if (t < T) dev::tmem_ld_n<G>(tmem + lane_off + t * kN, raw[t]);
      dev::tmem_wait_ld();
#pragma unroll
      for (int t = 0; t < kMaxTiles; ++t)
#pragma unroll
        for (int g = 0; g < G; ++g) {
          asm volatile("" : "+r"(raw[t][g]));
          const bool in = t < T && t * kTile + i < n;
          x[t][g] = in ? __uint_as_float(raw[t][g]) * c : -INFINITY;
          mx[g] = fmaxf(mx[g], x[t][g]);
        }
    }
    // the split's maximum per head: warp shuffles, then the four warps through shared memory
#pragma unroll
    for (int g = 0; g < G; ++g) {
#pragma unroll
      for (int sh = 16; sh > 0; sh >>= 1) mx[g] = fmaxf(mx[g], __shfl_xor_sync(0xffffffffu, mx[g], sh));
      if (lane == 0) sm.red_max[warp][g] = mx[g];
    }
    softmax_bar_sync();
    float m[G], sum[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      m[g] = fmaxf(fmaxf(sm.red_max[0][g], sm.red_max[1][g]), fmaxf(sm.red_max[2][g], sm.red_max[3][g]));
      sum[g] = 0.f;
    }
    if (ok) {
      // P^T[g][key] = 2^(x - m) as bf16: tile t, key block i / 64 (2 KB), row g (128 bytes),
      // 16-byte chunk (i % 64) / 8 XOR g (the 128-byte swizzle), element i % 8
      const uint32_t kk = static_cast<uint32_t>(i & 63);
      const uint32_t in_blk = (i >> 6) * kPBlockBytes + (kk & 7) * 2;
#pragma unroll
      for (int t = 0; t < kMaxTiles; ++t) {
        if (t >= T) break;
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float pr = dev::ex2_approx(x[t][g] - m[g]);  // 0 for keys past the split
          sum[g] += pr;
          const uint32_t off = t * kPTileBytes + in_blk + g * 128 + ((((kk >> 3) ^ g) & 7) << 4);
          *reinterpret_cast<__nv_bfloat16*>(&sm.p[0][0] + off) = __float2bfloat16_rn(pr);
        }
      }
      dev::fence_proxy_async_smem();  // the tensor core reads P through the async proxy
      dev::mbar_arrive(dev::smem_u32(&sm.bar_p));
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
#pragma unroll
      for (int sh = 16; sh > 0; sh >>= 1) sum[g] += __shfl_xor_sync(0xffffffffu, sum[g], sh);
      if (lane == 0) sm.red_sum[warp][g] = sum[g];
    }
    softmax_bar_sync();
    float l[G];
#pragma unroll
    for (int g = 0; g < G; ++g) l[g] = sm.red_sum[0][g] + sm.red_sum[1][g] + sm.red_sum[2][g] + sm.red_sum[3][g];

    // ---- epilogue: thread i writes head-dimension column i of O_s / l_s for every head ----
    if (ok) ok = wait_bounded(dev::smem_u32(&sm.bar_o), 0, abort);
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
      dev::tc_fence_after();
      uint32_t o[G];
      dev::tmem_ld_n<G>(tmem + lane_off + kOCol, o);
      dev::tmem_wait_ld_regs(o);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const size_t row = out_row(g);
        ws_o[row * kD + i] = __uint_as_float(o[g]) / l[g];  // l >= 1: the maximum's own weight
        if (i == g) ws_lse[row] = (m[g] + log2f(l[g])) * 0.69314718055994531f;
      }
    }
  }

  // ---- teardown ----
  dev::tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    dev::tc_fence_after();
    dev::tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace dtc
}  // namespace attn
