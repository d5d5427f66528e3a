// Shared device-side pieces: the device error flag, bounded mbarrier waits and the mask predicate.
#pragma once

#include <cstdint>

#include "../../include/attn.h"
#include "dev/ptx.cuh"

namespace attn {

// Set (never cleared on the device) when a bounded wait expires (ATTN_ERR_DEVICE_TIMEOUT) or a
// kernel met an index it refused to follow (ATTN_ERR_INVALID_ARG: a paged-cache page number
// outside the cache); read and cleared by the host through attn_get_device_error().
__device__ int g_device_error = 0;

// Longest a role may wait on one barrier before it gives up: 2^32 SM clocks (about 2 s at the
// B200's top clock).  A legitimate wait in these kernels lasts microseconds.
constexpr long long kWaitLimitCycles = 1ll << 32;

// Wait for the completion of phase `parity` of an mbarrier, bounded in time.  Returns false if
// the wait expired or another role of the CTA already gave up (shared flag *abort != 0); the
// first role to expire records ATTN_ERR_DEVICE_TIMEOUT in g_device_error and raises *abort.
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile int* abort,
                                             long long limit = kWaitLimitCycles) {
  if (dev::mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (dev::mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (clock64() - t0 > limit) {
      atomicExch(&g_device_error, ATTN_ERR_DEVICE_TIMEOUT);
      *abort = 1;
      return false;
    }
  }
}

// Same, for the drain at the end of a CTA: ignores the abort flag, only the time limit.
__device__ __forceinline__ bool wait_drain(uint32_t bar, uint32_t parity) {
  if (dev::mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (clock64() - t0 < kWaitLimitCycles) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (dev::mbar_try_wait(bar, parity)) return true;
  }
  atomicExch(&g_device_error, ATTN_ERR_DEVICE_TIMEOUT);
  return false;
}

// Mask shared by every kernel.  p = key position of the query row (i + Nk - Nq), j = key index.
struct MaskSpec {
  int kind;    // ATTN_MASK_*
  int window;  // sliding: window width w (keys p-w+1 .. p); local+global: w keys on each side
  int n_sink;  // sliding: always-visible sink keys 0 .. n_sink-1 (still causal);
               // local+global: the global tokens 0 .. n_sink-1 (as keys and as queries)
  int Nk;      // keys >= Nk are padding
};

__host__ __device__ __forceinline__ bool is_global_row(const MaskSpec& m, int p) {
  return p >= 0 && p < m.n_sink;
}

__device__ __forceinline__ bool key_visible(const MaskSpec& m, int p, int j) {
  if (j >= m.Nk) return false;
  if (m.kind == ATTN_MASK_FULL) return true;
  if (m.kind == ATTN_MASK_LOCAL_GLOBAL) {
    if (j < m.n_sink || is_global_row(m, p)) return true;
    const long long d = static_cast<long long>(p) - j;
    return d <= m.window && -d <= m.window;
  }
  if (j > p) return false;
  if (m.kind == ATTN_MASK_CAUSAL) return true;
  return (j > p - m.window) || (j < m.n_sink);
}

// Columns 32w .. 32w+31 of a 128-column tile that are <= x, as bits (bit i = column 32w + i).
__device__ __forceinline__ uint32_t cols_upto(int x, int w) {
  const int k = x - 32 * w;
  return k < 0 ? 0u : (k >= 31 ? 0xffffffffu : (2u << k) - 1u);
}

// clamp a 64-bit column bound into [-1, 128] (every bound outside a tile acts the same)
__host__ __device__ __forceinline__ int clamp_col(long long x) {
  return x < -1 ? -1 : (x > 128 ? 128 : static_cast<int>(x));
}

// Visible keys of the query at position p among the columns key0 .. key0+127 of a tile:
// (lo <= col <= hi) or col < sk, bounds clamped to [-1, 128].  Sliding-window sinks stop at the
// causal bound; global keys of the local + global mask do not.
__device__ __forceinline__ void row_cols(const MaskSpec& m, int p, int key0, int& hi, int& lo,
                                         int& sk) {
  const long long kNone = -(1ll << 40);
  long long last = m.Nk - 1, first = kNone, sink = kNone;
  if (m.kind == ATTN_MASK_CAUSAL) {
    last = p < last ? p : last;
  } else if (m.kind == ATTN_MASK_SLIDING) {
    last = p < last ? p : last;
    first = static_cast<long long>(p) - m.window + 1;
    sink = m.n_sink < last + 1 ? m.n_sink : last + 1;
  } else if (m.kind == ATTN_MASK_LOCAL_GLOBAL && !is_global_row(m, p)) {
    const long long right = static_cast<long long>(p) + m.window;
    last = right < last ? right : last;
    first = static_cast<long long>(p) - m.window;
    sink = m.n_sink < m.Nk ? m.n_sink : m.Nk;
  }
  hi = clamp_col(last - key0);
  lo = clamp_col(first - key0);
  sk = clamp_col(sink - key0);
}

// The 32 columns 32w .. 32w+31 of that set, as bits.
__device__ __forceinline__ uint32_t row_bits(int hi, int lo, int sk, int w) {
  return (cols_upto(hi, w) & ~cols_upto(lo - 1, w)) | cols_upto(sk - 1, w);
}

// Is every pair of the block (query positions P0 .. P0+rows-1) x (keys c0 .. c0+cols-1)
// visible?  Conservative: rows past Nq count as visible (callers zero or skip them).
__host__ __device__ __forceinline__ bool block_visible(const MaskSpec& m, int P0, int rows, int c0,
                                                      int cols) {
  const long long c1 = static_cast<long long>(c0) + cols - 1;
  const long long P1 = static_cast<long long>(P0) + rows - 1;
  if (c1 >= m.Nk) return false;
  if (m.kind == ATTN_MASK_FULL) return true;
  if (m.kind == ATTN_MASK_LOCAL_GLOBAL)
    return c1 < m.n_sink || (P0 >= 0 && P1 < m.n_sink) ||
           (c0 >= P1 - m.window && c1 <= P0 + static_cast<long long>(m.window));
  if (c1 > P0) return false;
  if (m.kind == ATTN_MASK_CAUSAL) return true;
  return (c0 > P1 - m.window) || (c1 < m.n_sink);
}

// Range of key tiles (of `tile` keys) a block of query positions [p_lo, p_hi] must visit:
// the sink tiles [0, ns) that precede the window, then the contiguous tiles [lo, hi].
// Returns the number of tiles (0 if no key is visible to any of the rows).
struct TileRange {
  int ns, lo, hi;
  __host__ __device__ int count() const { return hi < lo ? ns : ns + (hi - lo + 1); }
  __host__ __device__ int tile(int j) const { return j < ns ? j : lo + (j - ns); }
};

__host__ __device__ inline TileRange key_tiles(const MaskSpec& m, int p_lo, int p_hi, int tile) {
  TileRange r{0, 0, -1};
  if (m.Nk <= 0) return r;
  const int last_key = m.Nk - 1;
  if (m.kind == ATTN_MASK_FULL) {
    r.lo = 0;
    r.hi = last_key / tile;
    return r;
  }
  if (m.kind == ATTN_MASK_LOCAL_GLOBAL) {
    // a global row sees every key; otherwise the window tiles and the global-key tiles
    const int g_lo = p_lo > 0 ? p_lo : 0, g_hi = p_hi < m.n_sink - 1 ? p_hi : m.n_sink - 1;
    if (g_lo <= g_hi) {
      r.hi = last_key / tile;
      return r;
    }
    const int g_keys = m.n_sink < m.Nk ? m.n_sink : m.Nk;
    const int g_tiles = (g_keys + tile - 1) / tile;
    long long first = static_cast<long long>(p_lo) - m.window;
    long long last = static_cast<long long>(p_hi) + m.window;
    if (first < 0) first = 0;
    if (last > last_key) last = last_key;
    if (first > last) {  // no window key: the global keys only
      r.ns = g_tiles;
      r.lo = g_tiles;
      r.hi = g_tiles - 1;
      return r;
    }
    r.lo = static_cast<int>(first / tile);
    r.hi = static_cast<int>(last / tile);
    if (g_tiles >= r.lo) {  // global tiles run into the window: one contiguous range
      r.lo = 0;
      if (g_tiles - 1 > r.hi) r.hi = g_tiles - 1;
    } else {
      r.ns = g_tiles;
    }
    return r;
  }
  if (p_hi < 0) return r;  // every row precedes the first key
  r.hi = (p_hi < last_key ? p_hi : last_key) / tile;
  if (m.kind == ATTN_MASK_CAUSAL) {
    r.lo = 0;
    return r;
  }
  int first = p_lo - m.window + 1;
  if (first < 0) first = 0;
  if (first > last_key) first = last_key;
  r.lo = first / tile;
  if (r.lo > r.hi) r.lo = r.hi;
  int sink_tiles = (m.n_sink + tile - 1) / tile;
  r.ns = sink_tiles < r.lo ? sink_tiles : r.lo;
  return r;
}

}  // namespace attn
