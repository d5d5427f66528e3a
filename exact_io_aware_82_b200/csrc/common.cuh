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
  int window;  // sliding window width w (keys p-w+1 .. p)
  int n_sink;  // always-visible sink keys 0 .. n_sink-1 (still causal)
  int Nk;      // keys >= Nk are padding
};

__device__ __forceinline__ bool key_visible(const MaskSpec& m, int p, int j) {
  if (j >= m.Nk) return false;
  if (m.kind == ATTN_MASK_FULL) return true;
  if (j > p) return false;
  if (m.kind == ATTN_MASK_CAUSAL) return true;
  return (j > p - m.window) || (j < m.n_sink);
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
