// Split-K decode: one new query token per sequence against a long KV cache, contiguous or paged.
//
// "Attention Research" (learning-materials), section 1: decode reads the whole O(S) KV cache
// every step, so it is bound by HBM bandwidth; section 2: FlashDecoding splits the keys of a
// decode step across thread blocks ("split-K over keys").  Each split produces a partial
// output normalised by its own softmax sum together with its log-sum-exp; the combine merges
// the splits exactly, O = sum_s exp(lse_s - LSE) O_s with LSE = ln sum_s exp(lse_s), which is
// the online-softmax rescaling of "FlashAttention and sparse attention" (grasp.study),
// section 1, applied once per split.
//
// Split kernel: grid (splits, Hkv, B), 256 threads.  The G query heads of a kv group share
// every K/V byte read.  A half-warp covers one 256-byte key (or value) row with 16-byte loads,
// so every load instruction of a warp reads two whole rows (fully coalesced); thread lane%16
// owns head-dimension slice [8*(lane%16), 8*(lane%16)+8) for the whole kernel and keeps the
// matching slice of the G query vectors in registers.  Scores are finished with a
// reduce-scatter across the 16 lanes of a row, written to shared memory, turned into
// probabilities, and the value pass accumulates P V per slice; partial sums of the 16
// half-warps are reduced through shared memory at the end.
#pragma once

#include <cuda_bf16.h>

#include "common.cuh"

namespace attn {
namespace dec {

constexpr int kD = 128;
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxScoreFloats = 8192;  // per-CTA score buffer: chunk * G floats (32 KB)

// keys each half-warp loads per pass iteration: U * G = 32 partial dot products per thread
template <int G>
__host__ __device__ constexpr int unroll() { return G == 1 ? 16 : 32 / G; }
template <int G>
__host__ __device__ constexpr int keys_per_iter() { return 2 * unroll<G>() * kWarps; }
template <int G>
__host__ __device__ constexpr int max_chunk() { return kMaxScoreFloats / G; }

__host__ __device__ constexpr int smem_floats(int G, int chunk) {
  return (chunk * G > kWarps * G * kD) ? chunk * G : kWarps * G * kD;
}

// Paged KV cache ("Attention Research", section 2: FlashInfer's paged KV): key j of sequence b
// is row (j mod page_size) of page block_table[b][j / page_size]; a page holds page_size rows
// of [Hkv][d] (token-major).  A referenced page outside [0, num_pages) is never dereferenced:
// it reads as zero rows and records ATTN_ERR_INVALID_ARG in g_device_error.
struct Paged {
  const int* block_table;  // [B][max_pages]
  const int* seq_lens;     // [B]
  int max_pages;
  int num_pages;
  int page_shift;          // log2(page_size)
};

// The chunk of one split spans at most this many pages (chunk <= max_chunk<1>() keys and
// page_size >= kMinPageSize), plus one for a chunk that starts mid-page.
constexpr int kMinPageSize = 8;
constexpr int kMaxChunkPages = kMaxScoreFloats / kMinPageSize + 1;

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// The G scores of one key in the shared score buffer ([chunk][G] floats, 16-byte aligned).
template <int G>
__device__ __forceinline__ void load_scores(const float* p, float (&sc)[G]) {
  if constexpr (G % 4 == 0) {
#pragma unroll
    for (int i = 0; i < G; i += 4) {
      const float4 x = *reinterpret_cast<const float4*>(p + i);
      sc[i] = x.x, sc[i + 1] = x.y, sc[i + 2] = x.z, sc[i + 3] = x.w;
    }
  } else if constexpr (G == 2) {
    const float2 x = *reinterpret_cast<const float2*>(p);
    sc[0] = x.x, sc[1] = x.y;
  } else {
    sc[0] = p[0];
  }
}
template <int G>
__device__ __forceinline__ void store_scores(float* p, const float (&sc)[G]) {
  if constexpr (G % 4 == 0) {
#pragma unroll
    for (int i = 0; i < G; i += 4)
      *reinterpret_cast<float4*>(p + i) = make_float4(sc[i], sc[i + 1], sc[i + 2], sc[i + 3]);
  } else if constexpr (G == 2) {
    *reinterpret_cast<float2*>(p) = make_float2(sc[0], sc[1]);
  } else {
    p[0] = sc[0];
  }
}

// kPage: 0 = contiguous cache; 1 = paged, any page size; 2 = paged, pages of at least 2U keys
// (one page lookup per warp iteration).
template <int G, int kPage>
__device__ __forceinline__ void decode_split(const __nv_bfloat16* __restrict__ q,
                                             const __nv_bfloat16* __restrict__ k,
                                             const __nv_bfloat16* __restrict__ v,
                                             float* __restrict__ ws_o, float* __restrict__ ws_lse,
                                             int Hq, int Hkv, int Nk, int chunk, int splits,
                                             float c, Paged pg) {
  constexpr int U = unroll<G>();
  constexpr int NV = U * G;        // partial dot products per thread per iteration
  constexpr int PER_LANE = NV / 16;  // fully reduced scores each lane ends with
  extern __shared__ __align__(16) float smem[];  // scores/probabilities [chunk][G], later the
                                                 // P V partials
  __shared__ float red_m[kWarps][G];
  __shared__ float stat[2][G];     // max (log2 units) and sum per head

  const int s = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int half = lane >> 4, sl = lane & 15;
  const int j0 = s * chunk;
  // keys of this sequence: Nk (contiguous cache) or its own length (paged cache)
  constexpr bool kPaged = kPage != 0;
  const int len = kPaged ? max(0, min(__ldg(pg.seq_lens + b), Nk)) : Nk;
  const int n = max(0, min(len - j0, chunk));
  // contiguous cache: this thread's column slice of key row j0 of (b, hk)
  const size_t kv_row0 = kPaged ? 0 : (static_cast<size_t>(b) * Hkv + hk) * Nk + j0;
  const __nv_bfloat16* kb = k + kv_row0 * kD + 8 * sl;
  const __nv_bfloat16* vb = v + kv_row0 * kD + 8 * sl;
  // paged: the physical pages of this chunk, looked up once into shared memory
  __shared__ int pages[kPaged ? kMaxChunkPages : 1];
  const int page0 = j0 >> pg.page_shift;
  if (kPaged) {
    const int npg = n > 0 ? ((j0 + n - 1) >> pg.page_shift) - page0 + 1 : 0;
    for (int i = tid; i < npg; i += kThreads) {
      const int lp = page0 + i;
      const int phys = lp < pg.max_pages ? __ldg(pg.block_table + static_cast<size_t>(b) * pg.max_pages + lp) : -1;
      const bool ok = phys >= 0 && phys < pg.num_pages;
      if (!ok) atomicExch(&g_device_error, ATTN_ERR_INVALID_ARG);  // read as zero rows instead
      pages[i] = ok ? phys : -1;
    }
    __syncthreads();
  }
  // row `key` of this chunk in a cache tensor (contiguous: base + key rows; paged: via pages[])
  auto row = [&](const __nv_bfloat16* cache, const __nv_bfloat16* base, int key) -> const __nv_bfloat16* {
    if (!kPaged) return base + static_cast<size_t>(key) * kD;
    const int L = j0 + key;
    const int phys = pages[(L >> pg.page_shift) - page0];
    if (phys < 0) return nullptr;
    const size_t r = (static_cast<size_t>(phys) << pg.page_shift) + (L & ((1 << pg.page_shift) - 1));
    return cache + (r * Hkv + hk) * kD + 8 * sl;
  };
  auto load = [&](const __nv_bfloat16* p) { return p ? ldg_stream(p) : make_uint4(0, 0, 0, 0); };
  // paged, pages of at least 2U keys: the 2U keys a warp loads per iteration start at a multiple
  // of 2U (chunks are multiples of 32 keys), so they share one page; one lookup per iteration,
  // then a fixed stride of Hkv rows between consecutive keys
  constexpr bool one_page = kPage == 2;
  const size_t key_stride = static_cast<size_t>(Hkv) * kD;
  auto load_keys = [&](const __nv_bfloat16* cache, const __nv_bfloat16* base, int kw, uint4 (&r)[U]) {
    if constexpr (one_page) {
      const int L = j0 + kw;
      const int phys = kw < n ? pages[(L >> pg.page_shift) - page0] : -1;
      const size_t r0 = (static_cast<size_t>(phys < 0 ? 0 : phys) << pg.page_shift) +
                        (L & ((1 << pg.page_shift) - 1));
      const __nv_bfloat16* p = cache + ((r0 + half) * Hkv + hk) * kD + 8 * sl;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int key = kw + 2 * u + half;
        r[u] = (phys >= 0 && key < n) ? ldg_stream(p + 2 * u * key_stride) : make_uint4(0, 0, 0, 0);
      }
    } else {
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int key = kw + 2 * u + half;
        r[u] = key < n ? load(row(cache, base, key)) : make_uint4(0, 0, 0, 0);
      }
    }
  };

  // this thread's slice of the G query vectors, pre-multiplied by scale * log2(e)
  float qf[G][8];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const uint4 u = *reinterpret_cast<const uint4*>(
        q + (static_cast<size_t>(b) * Hq + hk * G + g) * kD + 8 * sl);
    bf16x8_to_f32(u, qf[g]);
#pragma unroll
    for (int e = 0; e < 8; ++e) qf[g][e] *= c;
  }

  // ---------------- pass 1: scores (log2 units) into shared memory ----------------
  for (int base = 0; base < n; base += keys_per_iter<G>()) {
    const int kw = base + warp * 2 * U;  // first key of this warp's group
    uint4 kr[U];
    load_keys(k, kb, kw, kr);
    float part[NV];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      float kf[8];
      bf16x8_to_f32(kr[u], kf);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float acc = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) acc = fmaf(qf[g][e], kf[e], acc);
        part[u * G + g] = acc;
      }
    }
    // reduce-scatter over the 16 lanes of each row: after the step with lane bit m, a lane
    // keeps the half of the vector selected by that bit; a lane ends with entries
    // 2*sl*PER_LANE/2 ... i.e. indices [sl * PER_LANE, sl * PER_LANE + PER_LANE)
#pragma unroll
    for (int m = 8, width = NV; m >= 1; m >>= 1, width >>= 1) {
      const bool upper = (sl & m) != 0;
#pragma unroll
      for (int i = 0; i < width / 2; ++i) {
        const float lo = part[i], hi = part[i + width / 2];
        const float send = upper ? lo : hi;
        const float keep = upper ? hi : lo;
        part[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
      }
    }
    if constexpr (PER_LANE == 2 && G >= 2) {
      // the lane's two scores are heads g, g + 1 of one key: one 8-byte store (a warp's
      // stores then fill 256 consecutive bytes)
      const int idx = sl * 2;  // = u * G + g
      const int u = idx / G, g = idx % G;
      const int key = kw + 2 * u + half;
      if (key < n) *reinterpret_cast<float2*>(smem + key * G + g) = make_float2(part[0], part[1]);
    } else {
#pragma unroll
      for (int i = 0; i < PER_LANE; ++i) {
        const int idx = sl * PER_LANE + i;  // = u * G + g
        const int u = idx / G, g = idx % G;
        const int key = kw + 2 * u + half;
        if (key < n) smem[key * G + g] = part[i];
      }
    }
  }
  __syncthreads();

  // ---------------- softmax statistics per head ----------------
  // a key's G scores are read and written as one unit (16-byte words for G >= 4), so that the
  // lanes of a warp touch consecutive words instead of every G-th one (bank conflicts)
  float mx[G];
#pragma unroll
  for (int g = 0; g < G; ++g) mx[g] = -INFINITY;
  for (int key = tid; key < n; key += kThreads) {
    float sc[G];
    load_scores<G>(smem + key * G, sc);
#pragma unroll
    for (int g = 0; g < G; ++g) mx[g] = fmaxf(mx[g], sc[g]);
  }
#pragma unroll
  for (int g = 0; g < G; ++g) {
#pragma unroll
    for (int sh = 16; sh > 0; sh >>= 1) mx[g] = fmaxf(mx[g], __shfl_xor_sync(0xffffffffu, mx[g], sh));
    if (lane == 0) red_m[warp][g] = mx[g];
  }
  __syncthreads();
  if (tid < G) {
    float m = -INFINITY;
    for (int w = 0; w < kWarps; ++w) m = fmaxf(m, red_m[w][tid]);
    stat[0][tid] = m;
  }
  __syncthreads();
  float sum[G];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    mx[g] = stat[0][g];
    sum[g] = 0.f;
  }
  for (int key = tid; key < n; key += kThreads) {
    float sc[G];
    load_scores<G>(smem + key * G, sc);
#pragma unroll
    for (int g = 0; g < G; ++g) {
      sc[g] = exp2f(sc[g] - mx[g]);
      sum[g] += sc[g];
    }
    store_scores<G>(smem + key * G, sc);
  }
#pragma unroll
  for (int g = 0; g < G; ++g) {
#pragma unroll
    for (int sh = 16; sh > 0; sh >>= 1) sum[g] += __shfl_xor_sync(0xffffffffu, sum[g], sh);
  }
  __syncthreads();  // every thread has read red_m; reuse it for the sums
  if (lane == 0)
#pragma unroll
    for (int g = 0; g < G; ++g) red_m[warp][g] = sum[g];
  __syncthreads();
  if (tid < G) {
    float t = 0.f;
    for (int w = 0; w < kWarps; ++w) t += red_m[w][tid];
    stat[1][tid] = t;
  }

  // ---------------- pass 2: O_s = sum_j p_j V_j per head-dimension slice ----------------
  float acc[G][8];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[g][e] = 0.f;
  for (int base = 0; base < n; base += keys_per_iter<G>()) {
    const int kw = base + warp * 2 * U;
    uint4 vr[U];
    load_keys(v, vb, kw, vr);
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int key = kw + 2 * u + half;
      if (key < n) {
        float vf[8];
        bf16x8_to_f32(vr[u], vf);
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float pr = smem[key * G + g];
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[g][e] = fmaf(pr, vf[e], acc[g][e]);
        }
      }
    }
  }
  // combine the two half-warps, then the 8 warps through shared memory
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[g][e] += __shfl_xor_sync(0xffffffffu, acc[g][e], 16);
  __syncthreads();  // all probabilities consumed; the score buffer becomes the partial buffer
  if (half == 0)
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float4* dst = reinterpret_cast<float4*>(smem + (warp * G + g) * kD + 8 * sl);
      dst[0] = make_float4(acc[g][0], acc[g][1], acc[g][2], acc[g][3]);
      dst[1] = make_float4(acc[g][4], acc[g][5], acc[g][6], acc[g][7]);
    }
  __syncthreads();
  for (int idx = tid; idx < G * kD; idx += kThreads) {
    const int g = idx / kD, dcol = idx % kD;
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) t += smem[(w * G + g) * kD + dcol];
    const float l = stat[1][g];
    const size_t row = (static_cast<size_t>(b) * Hq + hk * G + g) * splits + s;
    ws_o[row * kD + dcol] = l > 0.f ? t / l : 0.f;
    if (dcol == 0)
      ws_lse[row] = l > 0.f ? (stat[0][g] + log2f(l)) * 0.69314718055994531f : -INFINITY;
  }
}

// Contiguous cache: [B][Hkv][Nk][d].
template <int G>
__global__ void __launch_bounds__(kThreads)
    decode_split_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                        const __nv_bfloat16* __restrict__ v, float* __restrict__ ws_o,
                        float* __restrict__ ws_lse, int Hq, int Hkv, int Nk, int chunk,
                        int splits, float c) {
  decode_split<G, 0>(q, k, v, ws_o, ws_lse, Hq, Hkv, Nk, chunk, splits, c, Paged{});
}

// Paged cache (kPage 1 or 2); registers capped so that as many CTAs stay resident per SM as the
// contiguous kernel of the same G gets (three at G = 4 with one lookup per iteration, two otherwise).
template <int G, int kPage>
__global__ void __launch_bounds__(kThreads, (G == 4 && kPage == 2) ? 3 : 2)
    decode_split_paged_kernel(const __nv_bfloat16* __restrict__ q,
                              const __nv_bfloat16* __restrict__ k,
                              const __nv_bfloat16* __restrict__ v, float* __restrict__ ws_o,
                              float* __restrict__ ws_lse, int Hq, int Hkv, int Nk, int chunk,
                              int splits, float c, Paged pg) {
  decode_split<G, kPage>(q, k, v, ws_o, ws_lse, Hq, Hkv, Nk, chunk, splits, c, pg);
}

// Combine: grid B * Hq, one thread per head-dimension column.
__global__ void __launch_bounds__(kD)
    decode_combine_kernel(const float* __restrict__ ws_o, const float* __restrict__ ws_lse,
                          __nv_bfloat16* __restrict__ o, float* __restrict__ lse, int splits) {
  const int bh = blockIdx.x, dcol = threadIdx.x;
  const float* L = ws_lse + static_cast<size_t>(bh) * splits;
  float M = -INFINITY;
  for (int s = 0; s < splits; ++s) M = fmaxf(M, L[s]);
  float out = 0.f, tot = -INFINITY;
  if (M != -INFINITY) {
    float z = 0.f;
    for (int s = 0; s < splits; ++s) z += expf(L[s] - M);
    tot = M + logf(z);
    const float* Os = ws_o + static_cast<size_t>(bh) * splits * kD + dcol;
    for (int s = 0; s < splits; ++s) {
      const float w = expf(L[s] - tot);
      out = fmaf(w, Os[static_cast<size_t>(s) * kD], out);
    }
  }
  o[static_cast<size_t>(bh) * kD + dcol] = __float2bfloat16_rn(out);
  if (dcol == 0 && lse != nullptr) lse[bh] = tot;
}

}  // namespace dec
}  // namespace attn
