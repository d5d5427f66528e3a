// fp32 exact attention forward (CUDA cores, fp32 arithmetic throughout).
//
// Same method as the bf16 tensor-core kernel - K/V tiles staged in shared memory, online
// softmax with a running max and running sum, earlier partial outputs rescaled when the max
// grows ("FlashAttention and sparse attention" (grasp.study), section 1) - for fp32 inputs,
// which the tensor-core path does not take.
//
// Grid (ceil(Nq / rows), Hq, B); 8 warps per CTA, each warp owns 4 (d = 64) or 2 (d = 128)
// query rows.  Per key tile of
// 32 keys: lane l scores key l against the warp's rows (K tile padded to avoid bank
// conflicts), the row statistics are reduced with warp shuffles, and lane l accumulates output
// columns l, l+32, ... of P V.
#pragma once

#include "common.cuh"

namespace attn {
namespace f32 {

constexpr int kKeys = 32;         // keys per shared-memory tile
constexpr int kWarps = 8;
// query rows per CTA: 32 at d = 64, 16 at d = 128 (static shared memory stays under 48 KB)
template <int D>
__host__ __device__ constexpr int rows_per_cta() { return D == 128 ? 16 : 32; }

struct Params {
  int B, Hq, Hkv, Nq, Nk, G;
  MaskSpec mask;
  float c;  // scale * log2(e)
};

template <int D>
__global__ void __launch_bounds__(kWarps * 32)
    fwd_f32_kernel(const float* __restrict__ q, const float* __restrict__ k,
                   const float* __restrict__ v, float* __restrict__ o, float* __restrict__ lse,
                   const Params p) {
  constexpr int kCols = D / 32;  // output columns per lane
  constexpr int kRows = rows_per_cta<D>();
  constexpr int kRowsPerWarp = kRows / kWarps;
  __shared__ float qs[kRows][D];
  __shared__ float ks[kKeys][D + 1];
  __shared__ float vs[kKeys][D];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int r0 = blockIdx.x * kRows;
  const int h = blockIdx.y, b = blockIdx.z;
  const size_t bh = static_cast<size_t>(b) * p.Hq + h;
  const size_t bkv = static_cast<size_t>(b) * p.Hkv + h / p.G;
  const int off = p.Nk - p.Nq;
  const float* qb = q + bh * p.Nq * D;
  const float* kb = k + bkv * p.Nk * D;
  const float* vb = v + bkv * p.Nk * D;

  for (int e = tid; e < kRows * D; e += kWarps * 32) {
    const int r = e / D, cidx = e % D;
    qs[r][cidx] = (r0 + r < p.Nq) ? qb[static_cast<size_t>(r0 + r) * D + cidx] : 0.f;
  }

  float m[kRowsPerWarp], l[kRowsPerWarp], acc[kRowsPerWarp][kCols];
#pragma unroll
  for (int i = 0; i < kRowsPerWarp; ++i) {
    m[i] = -INFINITY;
    l[i] = 0.f;
#pragma unroll
    for (int cidx = 0; cidx < kCols; ++cidx) acc[i][cidx] = 0.f;
  }

  const int last_row = min(r0 + kRows, p.Nq) - 1;
  const TileRange tr = key_tiles(p.mask, r0 + off, last_row + off, kKeys);
  const int nt = tr.count();

  for (int j = 0; j < nt; ++j) {
    const int key0 = tr.tile(j) * kKeys;
    __syncthreads();
    for (int e = tid; e < kKeys * D; e += kWarps * 32) {
      const int r = e / D, cidx = e % D;
      const bool in = key0 + r < p.Nk;
      ks[r][cidx] = in ? kb[static_cast<size_t>(key0 + r) * D + cidx] : 0.f;
      vs[r][cidx] = in ? vb[static_cast<size_t>(key0 + r) * D + cidx] : 0.f;
    }
    __syncthreads();

#pragma unroll
    for (int i = 0; i < kRowsPerWarp; ++i) {
      const int row = warp * kRowsPerWarp + i;
      const int prow = r0 + row + off;
      float s = 0.f;
#pragma unroll 8
      for (int t = 0; t < D; ++t) s = fmaf(qs[row][t], ks[lane][t], s);
      const bool vis = key_visible(p.mask, prow, key0 + lane);
      const float x = vis ? s * p.c : -INFINITY;
      float tmax = x;
#pragma unroll
      for (int sh = 16; sh > 0; sh >>= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, sh));
      const float m_new = fmaxf(m[i], tmax);
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      const float alpha = exp2f(m[i] - m_use);  // 0 while the row has seen no visible key
      const float pj = vis ? exp2f(x - m_use) : 0.f;
      float psum = pj;
#pragma unroll
      for (int sh = 16; sh > 0; sh >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, sh);
      l[i] = l[i] * alpha + psum;
      m[i] = m_new;
#pragma unroll
      for (int cidx = 0; cidx < kCols; ++cidx) acc[i][cidx] *= alpha;
#pragma unroll 4
      for (int jj = 0; jj < kKeys; ++jj) {
        const float pb = __shfl_sync(0xffffffffu, pj, jj);
#pragma unroll
        for (int cidx = 0; cidx < kCols; ++cidx)
          acc[i][cidx] = fmaf(pb, vs[jj][lane + 32 * cidx], acc[i][cidx]);
      }
    }
  }

#pragma unroll
  for (int i = 0; i < kRowsPerWarp; ++i) {
    const int grow = r0 + warp * kRowsPerWarp + i;
    if (grow >= p.Nq) continue;
    const float inv = l[i] > 0.f ? 1.f / l[i] : 0.f;
    float* orow = o + (bh * p.Nq + grow) * D;
#pragma unroll
    for (int cidx = 0; cidx < kCols; ++cidx) orow[lane + 32 * cidx] = acc[i][cidx] * inv;
    if (lane == 0 && lse != nullptr)
      lse[bh * p.Nq + grow] = l[i] > 0.f ? (m[i] + log2f(l[i])) * 0.69314718055994531f : -INFINITY;
  }
}

// ------------------------------------------------------------------------------------------
// Small problems (the K and V rows of one kv head fit in shared memory, e.g. n = 256, d = 64):
// the tiled kernel above then runs a handful of CTAs through a long dependent chain of key
// tiles.  Here every CTA copies the kv head's whole K and V into shared memory at once and each
// warp computes one query row: all scores of the row (lane = key within a 32-key chunk, four
// independent partial sums per dot product), the exact row max and sum by warp shuffles, then
// P V (lane = output columns, each weight broadcast from its lane).  Same definition and
// results as the tiled kernel; no online rescaling is needed since the whole row is at hand.
// ------------------------------------------------------------------------------------------
constexpr int kSmallWarps = 8;     // query rows per CTA
constexpr int kSmallMaxChunks = 16;  // keys per row: at most 16 x 32 = 512
template <int D>
__host__ __device__ constexpr int small_stride() { return D + 4; }  // padded row (floats)
template <int D>
__host__ __device__ constexpr size_t small_smem_bytes(int Nk) {
  return static_cast<size_t>(Nk) * small_stride<D>() * 2 * sizeof(float);
}

template <int D>
__global__ void __launch_bounds__(kSmallWarps * 32)
    fwd_f32_small_kernel(const float* __restrict__ q, const float* __restrict__ k,
                         const float* __restrict__ v, float* __restrict__ o,
                         float* __restrict__ lse, const Params p) {
  constexpr int S = small_stride<D>();
  constexpr int kCols = D / 32;
  extern __shared__ float4 smem_f4[];
  float* ks = reinterpret_cast<float*>(smem_f4);
  float* vs = ks + static_cast<size_t>(p.Nk) * S;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.y, b = blockIdx.z;
  const size_t bh = static_cast<size_t>(b) * p.Hq + h;
  const size_t bkv = static_cast<size_t>(b) * p.Hkv + h / p.G;
  const float4* kb = reinterpret_cast<const float4*>(k + bkv * p.Nk * D);
  const float4* vb = reinterpret_cast<const float4*>(v + bkv * p.Nk * D);
  for (int e = tid; e < p.Nk * (D / 4); e += kSmallWarps * 32) {
    const int r = e / (D / 4), c4 = e % (D / 4);
    *reinterpret_cast<float4*>(ks + r * S + 4 * c4) = __ldg(kb + e);
    *reinterpret_cast<float4*>(vs + r * S + 4 * c4) = __ldg(vb + e);
  }
  __syncthreads();

  const int row = blockIdx.x * kSmallWarps + warp;
  if (row >= p.Nq) return;
  const int prow = row + p.Nk - p.Nq;
  const float4* qr = reinterpret_cast<const float4*>(q + (bh * p.Nq + row) * D);
  float qv[D];
#pragma unroll
  for (int c4 = 0; c4 < D / 4; ++c4) {
    const float4 x = __ldg(qr + c4);
    qv[4 * c4] = x.x, qv[4 * c4 + 1] = x.y, qv[4 * c4 + 2] = x.z, qv[4 * c4 + 3] = x.w;
  }
  const int nchunks = (p.Nk + 31) / 32;
  float sc[kSmallMaxChunks];
  float mx = -INFINITY;
#pragma unroll
  for (int cix = 0; cix < kSmallMaxChunks; ++cix) {
    sc[cix] = -INFINITY;
    if (cix >= nchunks) continue;
    const int key = cix * 32 + lane;
    if (key < p.Nk && key_visible(p.mask, prow, key)) {
      const float* kr = ks + key * S;
      float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
      for (int t = 0; t < D; t += 4) {
        const float4 kk = *reinterpret_cast<const float4*>(kr + t);
        a0 = fmaf(qv[t], kk.x, a0);
        a1 = fmaf(qv[t + 1], kk.y, a1);
        a2 = fmaf(qv[t + 2], kk.z, a2);
        a3 = fmaf(qv[t + 3], kk.w, a3);
      }
      sc[cix] = ((a0 + a1) + (a2 + a3)) * p.c;  // log2 units
      mx = fmaxf(mx, sc[cix]);
    }
  }
#pragma unroll
  for (int sh = 16; sh > 0; sh >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, sh));
  float l = 0.f;
  const float m_use = mx == -INFINITY ? 0.f : mx;
#pragma unroll
  for (int cix = 0; cix < kSmallMaxChunks; ++cix) {
    sc[cix] = cix < nchunks ? exp2f(sc[cix] - m_use) : 0.f;  // 0 for masked keys
    l += sc[cix];
  }
#pragma unroll
  for (int sh = 16; sh > 0; sh >>= 1) l += __shfl_xor_sync(0xffffffffu, l, sh);
  float acc[kCols];
#pragma unroll
  for (int cc = 0; cc < kCols; ++cc) acc[cc] = 0.f;
#pragma unroll
  for (int cix = 0; cix < kSmallMaxChunks; ++cix) {
    if (cix >= nchunks) break;
    const int keys = min(32, p.Nk - cix * 32);
#pragma unroll 4
    for (int jj = 0; jj < keys; ++jj) {
      const float pj = __shfl_sync(0xffffffffu, sc[cix], jj);
      const float* vr = vs + (cix * 32 + jj) * S;
#pragma unroll
      for (int cc = 0; cc < kCols; ++cc) acc[cc] = fmaf(pj, vr[lane + 32 * cc], acc[cc]);
    }
  }
  const float inv = l > 0.f ? 1.f / l : 0.f;
  float* orow = o + (bh * p.Nq + row) * D;
#pragma unroll
  for (int cc = 0; cc < kCols; ++cc) orow[lane + 32 * cc] = acc[cc] * inv;
  if (lane == 0 && lse != nullptr)
    lse[bh * p.Nq + row] = l > 0.f ? (mx + log2f(l)) * 0.69314718055994531f : -INFINITY;
}

}  // namespace f32
}  // namespace attn
