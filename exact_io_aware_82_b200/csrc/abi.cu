// C ABI of the exact attention library (declared in include/attn.h): argument validation,
// device checks, TMA descriptor encoding and kernel launches.  No allocation happens here and
// no pointer is kept after a call returns.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <algorithm>
#include <cstring>
#include <mutex>

#include "../../include/attn.h"
#include "bwd_sm100.cuh"
#include "common.cuh"
#include "decode.cuh"
#include "decode_tc.cuh"
#include "fwd_f32.cuh"
#include "fwd_sm100.cuh"

namespace attn {
namespace {

constexpr int kMaxDevices = 64;
constexpr float kLog2e = 1.4426950408889634f;

struct DeviceInfo {
  bool probed = false;
  bool sm100 = false;
  int num_sms = 0;
  bool fwd_configured = false;
  bool bwd_configured = false;
  bool dtc_configured = false;
};

std::mutex g_mutex;
DeviceInfo g_devices[kMaxDevices];
thread_local const char* g_last_detail = "no error";

// Maps a CUDA runtime result to a status, remembering the runtime's text for
// attn_last_error_detail().
int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return ATTN_OK;
  g_last_detail = cudaGetErrorString(e);
  return ATTN_ERR_CUDA;
}
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

// Work-unit counters of the persistent prefill and backward kernels, one per stream that launches
// them: calls on one stream run one after another and can share a counter, calls on different
// streams may overlap and must not.  A counter is zero between launches (the last CTA of a launch
// to take from it sets it back).  Past kCounterSlots streams on one device, a stream shares the
// counter of an earlier one.
constexpr int kCounterSlots = 1024;
static __device__ unsigned int g_unit_counters[kCounterSlots];

struct CounterTable {
  unsigned int* base = nullptr;
  cudaStream_t stream[kCounterSlots] = {};
  int used = 0;
};
CounterTable g_counter_tables[kMaxDevices];

// The counter of `st` on the current device.
int unit_counter(cudaStream_t st, unsigned int** out) {
  int dev = 0;
  int rc = cuda_status(cudaGetDevice(&dev));
  if (rc != ATTN_OK) return rc;
  if (dev < 0 || dev >= kMaxDevices) return ATTN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mutex);
  CounterTable& tab = g_counter_tables[dev];
  if (tab.base == nullptr) {
    void* p = nullptr;
    rc = cuda_status(cudaGetSymbolAddress(&p, g_unit_counters));
    if (rc != ATTN_OK) return rc;
    tab.base = static_cast<unsigned int*>(p);
  }
  int slot = -1;
  for (int i = 0; i < tab.used; ++i)
    if (tab.stream[i] == st) {
      slot = i;
      break;
    }
  if (slot < 0) {
    if (tab.used < kCounterSlots) {
      slot = tab.used++;
      tab.stream[slot] = st;
    } else {
      slot = static_cast<int>(reinterpret_cast<uintptr_t>(st) % kCounterSlots);
    }
  }
  *out = tab.base + slot;
  return ATTN_OK;
}

// Looks up the current device once: compute capability 10.x and the SM count; raises the
// dynamic shared memory limit of the tensor-core kernel on first use.
int current_device(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cuda_status(cudaGetLastError());
  if (dev < 0 || dev >= kMaxDevices) return ATTN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceInfo& info = g_devices[dev];
  if (!info.probed) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return ATTN_ERR_CUDA;
    info.sm100 = (major == 10 && minor == 0);
    info.num_sms = sms;
    info.probed = true;
  }
  if (!info.sm100) return ATTN_ERR_UNSUPPORTED;
  *out = &info;
  return ATTN_OK;
}

int configure_fwd(DeviceInfo* info) {
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!info->fwd_configured) {
    void (*kernels[6])(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, fwd::Params) = {
        fwd::fwd_bf16_sm100_kernel<false, false>, fwd::fwd_bf16_sm100_kernel<true, false>,
        fwd::fwd_bf16_sm100_kernel<false, true>,  fwd::fwd_bf16_sm100_kernel<true, true>,
        fwd::fwd_fp8_sm100_kernel<false>,         fwd::fwd_fp8_sm100_kernel<true>};
    for (auto* kern : kernels) {
      const int rc = cuda_status(cudaFuncSetAttribute(
          kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(fwd::kSmemBytes)));
      if (rc != ATTN_OK) return rc;
    }
    void (*sparse_kernels[2])(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, fwd::Params) = {
        fwd::fwd_bf16_sparse_sm100_kernel<false>, fwd::fwd_bf16_sparse_sm100_kernel<true>};
    for (auto* kern : sparse_kernels) {
      const int rc = cuda_status(cudaFuncSetAttribute(kern,
                                                      cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                      static_cast<int>(fwd::kSmemBytesSparse)));
      if (rc != ATTN_OK) return rc;
    }
    info->fwd_configured = true;
  }
  if (g_encode == nullptr) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault,
                                         &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr)
      return ATTN_ERR_CUDA;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  return ATTN_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Raises the dynamic shared memory limit of the tensor-core decode kernels on first use (and
// looks up the tensor-map encoder, as configure_fwd does).
int configure_decode_tc(DeviceInfo* info) {
  int rc = configure_fwd(info);
  if (rc != ATTN_OK) return rc;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!info->dtc_configured) {
    void (*kernels[8])(CUtensorMap, CUtensorMap, CUtensorMap, float*, float*, int, int, int, int,
                       int, float, dec::Paged) = {
        dtc::decode_tc_kernel<1, false>, dtc::decode_tc_kernel<2, false>,
        dtc::decode_tc_kernel<4, false>, dtc::decode_tc_kernel<8, false>,
        dtc::decode_tc_kernel<1, true>,  dtc::decode_tc_kernel<2, true>,
        dtc::decode_tc_kernel<4, true>,  dtc::decode_tc_kernel<8, true>};
    for (auto* kern : kernels) {
      rc = cuda_status(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            static_cast<int>(dtc::kSmemBytes)));
      if (rc != ATTN_OK) return rc;
    }
    info->dtc_configured = true;
  }
  return ATTN_OK;
}

// Raises the dynamic shared memory limit of the backward kernels on first use.
int configure_bwd(DeviceInfo* info) {
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!info->bwd_configured) {
    int rc = cuda_status(cudaFuncSetAttribute(bwd::bwd_dkdv_kernel,
                                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              static_cast<int>(bwd::kSmemKVBytes)));
    if (rc != ATTN_OK) return rc;
    rc = cuda_status(cudaFuncSetAttribute(bwd::bwd_dq_kernel,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          static_cast<int>(bwd::kSmemQBytes)));
    if (rc != ATTN_OK) return rc;
    info->bwd_configured = true;
  }
  return ATTN_OK;
}

// Backward workspace, in this order: LSE * log2(e) and D per query row (fp32, rows padded to
// whole 128-row tiles); the dS block offsets of the key blocks (int32, num_kblocks + 1); the
// dS^T blocks (bf16 128 x 128, one per visible (key block, query tile) pair and query head).
struct BwdLayout {
  size_t npad, pairs, off_bytes, ds_offset, total;
};

BwdLayout bwd_layout(int B, int Hq, int Nq, int Nk, const MaskSpec& m) {
  BwdLayout L{};
  const int nqt = (Nq + bwd::kT - 1) / bwd::kT, nkb = (Nk + bwd::kT - 1) / bwd::kT;
  L.npad = static_cast<size_t>(nqt) * bwd::kT;
  size_t pairs = 0;
  for (int kb = 0; kb < nkb; ++kb) {
    const int c0 = kb * bwd::kT, c1 = (c0 + bwd::kT < Nk ? c0 + bwd::kT : Nk) - 1;
    pairs += static_cast<size_t>(bwd::query_tiles(m, c0, c1, Nk - Nq, Nq).count());
  }
  L.pairs = pairs;
  const size_t vec = 2 * static_cast<size_t>(B) * Hq * L.npad * sizeof(float);
  L.off_bytes = (static_cast<size_t>(nkb) + 1) * sizeof(int);
  L.ds_offset = (vec + L.off_bytes + 255) & ~size_t(255);
  L.total = L.ds_offset + static_cast<size_t>(B) * Hq * pairs * bwd::kT * bwd::kT * 2;
  return L;
}

// Common argument rules of the forward entry points.
int check_fwd_args(const void* q, const void* k, const void* v, const void* o, int B, int Hq,
                   int Hkv, int Nq, int Nk, int mask_kind, int window, int n_sink, float scale) {
  if (B < 0 || Nq < 0 || Nk < 0 || Hq < 1 || Hkv < 1) return ATTN_ERR_INVALID_ARG;
  // a pointer may be NULL only when its tensor holds no element
  const bool q_empty = B == 0 || Nq == 0, kv_empty = B == 0 || Nk == 0;
  if ((!q_empty && (q == nullptr || o == nullptr)) || (!kv_empty && (k == nullptr || v == nullptr)))
    return ATTN_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (mask_kind < ATTN_MASK_FULL || mask_kind > ATTN_MASK_LOCAL_GLOBAL) return ATTN_ERR_INVALID_ARG;
  if (mask_kind == ATTN_MASK_SLIDING && window < 1) return ATTN_ERR_INVALID_ARG;
  if (mask_kind == ATTN_MASK_LOCAL_GLOBAL && window < 0) return ATTN_ERR_INVALID_ARG;
  if (n_sink < 0) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  return ATTN_OK;
}

MaskSpec make_mask(int mask_kind, int window, int n_sink, int Nk) {
  MaskSpec m;
  m.kind = mask_kind;
  const bool windowed = mask_kind == ATTN_MASK_SLIDING || mask_kind == ATTN_MASK_LOCAL_GLOBAL;
  m.window = windowed ? window : 0;
  m.n_sink = windowed ? n_sink : 0;
  m.Nk = Nk;
  return m;
}

// O = 0 and LSE = -inf for rows that can see no key at all (Nk = 0).
template <typename T>
__global__ void fill_empty_kernel(T* o, float* lse, size_t rows, int d) {
  const size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x;
  if (i < rows * d) o[i] = T(0.f);
  if (lse != nullptr && i < rows) lse[i] = -INFINITY;
}

template <typename T>
int launch_fill_empty(T* o, float* lse, size_t rows, int d, cudaStream_t stream) {
  const size_t n = rows * static_cast<size_t>(d);
  if (n == 0) return ATTN_OK;
  const unsigned blocks = static_cast<unsigned>((n + 255) / 256);
  fill_empty_kernel<T><<<blocks, 256, 0, stream>>>(o, lse, rows, d);
  return cuda_status(cudaGetLastError());
}

// 3-D tiled TMA map over a [heads][rows][128] bf16 tensor: box of 64 columns x box_rows rows,
// 128-byte swizzle (the layout tcgen05.mma descriptors read).  Rows past `rows` read as zero
// and are not written.
int encode_map(CUtensorMap* map, const void* base, int rows, int heads, uint32_t box_rows = 128) {
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(fwd::kD), static_cast<cuuint64_t>(rows),
                              static_cast<cuuint64_t>(heads)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(fwd::kD) * 2,
                                 static_cast<cuuint64_t>(rows) * fwd::kD * 2};
  const cuuint32_t box[3] = {64, box_rows, 1};
  const cuuint32_t estride[3] = {1, 1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                        strides, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ATTN_OK : ATTN_ERR_CUDA;
}

// 3-D tiled TMA map over [heads][rows][128] E4M3 codes (one byte each), read as boxes of the full
// 128-byte row width x 128 rows x 1 head with the 128-byte swizzle.
int encode_map_e4m3(CUtensorMap* map, const void* base, int rows, int heads) {
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(fwd::kD), static_cast<cuuint64_t>(rows),
                              static_cast<cuuint64_t>(heads)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(fwd::kD),
                                 static_cast<cuuint64_t>(rows) * fwd::kD};
  const cuuint32_t box[3] = {128, 128, 1};
  const cuuint32_t estride[3] = {1, 1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims,
                        strides, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ATTN_OK : ATTN_ERR_CUDA;
}

// 3-D tiled TMA map over a token-major packed [rows][heads][128] bf16 tensor, read as boxes of
// 64 columns x 1 head x 128 rows (same shared-memory layout as encode_map).
int encode_map_packed(CUtensorMap* map, const void* base, int rows, int heads,
                      uint32_t box_rows = 128) {
  // dimensions (d, rows, heads): rows second, so that a box is a 64 x 128 block of one head as
  // in the dense map (a box that is one element wide in its second dimension copies measurably
  // slower); the row stride (heads * d) exceeds the head stride (d)
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(fwd::kD), static_cast<cuuint64_t>(rows),
                              static_cast<cuuint64_t>(heads)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(heads) * fwd::kD * 2,
                                 static_cast<cuuint64_t>(fwd::kD) * 2};
  const cuuint32_t box[3] = {64, box_rows, 1};
  const cuuint32_t estride[3] = {1, 1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                        strides, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ATTN_OK : ATTN_ERR_CUDA;
}

// TMA map of a prefill output (bf16, d = 128): dense [heads][rows][128] or packed
// [rows][heads][128], written as boxes of 32 columns x 32 rows x 1 head staged with the 64-byte
// swizzle (one box per softmax warp and column quarter).
int encode_map_out(CUtensorMap* map, void* base, int rows, int heads, bool packed) {
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(fwd::kD), static_cast<cuuint64_t>(rows),
                              static_cast<cuuint64_t>(heads)};
  const cuuint64_t strides[2] = {
      packed ? static_cast<cuuint64_t>(heads) * fwd::kD * 2 : static_cast<cuuint64_t>(fwd::kD) * 2,
      packed ? static_cast<cuuint64_t>(fwd::kD) * 2 : static_cast<cuuint64_t>(rows) * fwd::kD * 2};
  const cuuint32_t box[3] = {32, 32, 1};
  const cuuint32_t estride[3] = {1, 1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, estride,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ATTN_OK : ATTN_ERR_CUDA;
}

constexpr int kMaxSplits = 256;

int decode_splits(int B, int Hkv, int Nk, int G, int requested, int num_sms) {
  int max_chunk;
  switch (G) {
    case 1: max_chunk = dec::max_chunk<1>(); break;
    case 2: max_chunk = dec::max_chunk<2>(); break;
    case 4: max_chunk = dec::max_chunk<4>(); break;
    default: max_chunk = dec::max_chunk<8>(); break;
  }
  const int min_splits = Nk > 0 ? (Nk + max_chunk - 1) / max_chunk : 1;
  int s = requested;
  if (s <= 0) {
    // chunks of whole 128-key tiles, at most the tensor-core kernel's dtc::kMaxChunk keys, and
    // small enough for about 4 CTAs per SM (2 are resident at a time)
    const long long groups = B * Hkv > 0 ? static_cast<long long>(B) * Hkv : 1;
    const long long want = (4LL * num_sms + groups - 1) / groups;
    long long chunk = Nk > 0 ? (Nk + want - 1) / want : 1;
    chunk = (chunk + dtc::kTile - 1) / dtc::kTile * dtc::kTile;
    if (chunk > dtc::kMaxChunk) chunk = dtc::kMaxChunk;
    s = Nk > 0 ? static_cast<int>((Nk + chunk - 1) / chunk) : 1;
  }
  if (s < min_splits) s = min_splits;
  if (s < 1) s = 1;
  if (s > kMaxSplits) s = kMaxSplits;
  return s;
}

size_t decode_ws_bytes(int B, int Hq, int splits) {
  const size_t rows = static_cast<size_t>(B) * Hq * splits;
  return rows * dec::kD * sizeof(float) + ((rows * sizeof(float) + 15) & ~size_t(15));
}

template <int G>
void launch_decode_split(dim3 grid, int chunk, cudaStream_t stream, const __nv_bfloat16* q,
                         const __nv_bfloat16* k, const __nv_bfloat16* v, float* ws_o,
                         float* ws_lse, int Hq, int Hkv, int Nk, int splits, float c,
                         const dec::Paged* pg) {
  const size_t smem = static_cast<size_t>(dec::smem_floats(G, chunk)) * sizeof(float);
  if (pg == nullptr)
    dec::decode_split_kernel<G><<<grid, dec::kThreads, smem, stream>>>(
        q, k, v, ws_o, ws_lse, Hq, Hkv, Nk, chunk, splits, c);
  else if ((1 << pg->page_shift) >= 2 * dec::unroll<G>())
    dec::decode_split_paged_kernel<G, 2><<<grid, dec::kThreads, smem, stream>>>(
        q, k, v, ws_o, ws_lse, Hq, Hkv, Nk, chunk, splits, c, *pg);
  else
    dec::decode_split_paged_kernel<G, 1><<<grid, dec::kThreads, smem, stream>>>(
        q, k, v, ws_o, ws_lse, Hq, Hkv, Nk, chunk, splits, c, *pg);
}

// Split kernel + combine over a contiguous cache (pg == nullptr; Nk keys per sequence) or a
// paged one (Nk = the longest sequence).  Arguments are already checked.
int decode_run(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
               int Hkv, int Nk, float scale, int num_splits, void* workspace,
               size_t workspace_bytes, cudaStream_t st, const DeviceInfo* info,
               const dec::Paged* pg) {
  const int G = Hq / Hkv;
  const int splits = decode_splits(B, Hkv, Nk, G, num_splits, info->num_sms);
  const size_t need = decode_ws_bytes(B, Hq, splits);
  if (workspace == nullptr || workspace_bytes < need || !aligned16(workspace))
    return ATTN_ERR_WORKSPACE;
  int chunk = (Nk + splits - 1) / splits;
  // paged: chunks of whole 32-key groups (the kernel's one-lookup-per-iteration path needs the
  // chunk starts aligned); a multiple of 32 keeps chunk <= the kernel's largest chunk, and
  // splits past the last key see no keys
  if (pg != nullptr) chunk = (chunk + 31) & ~31;
  float* ws_o = static_cast<float*>(workspace);
  float* ws_lse = ws_o + static_cast<size_t>(B) * Hq * splits * dec::kD;
  const float c = scale * kLog2e;
  const dim3 grid(splits, Hkv, B);
  if (chunk <= dtc::kMaxChunk && (pg == nullptr || pg->page_shift >= dtc::kMinTcPageShift)) {
    // chunks of at most kMaxChunk keys, contiguous or in pages of at least 64 keys: the
    // tensor-core split kernel
    int rc = configure_decode_tc(const_cast<DeviceInfo*>(info));
    if (rc != ATTN_OK) return rc;
    CUtensorMap tq, tk, tv;
    if (encode_map(&tq, q, B * Hq, 1, dtc::kN) != ATTN_OK) return ATTN_ERR_UNSUPPORTED;
    if (pg == nullptr) {
      if (encode_map(&tk, k, Nk, B * Hkv) != ATTN_OK || encode_map(&tv, v, Nk, B * Hkv) != ATTN_OK)
        return ATTN_ERR_UNSUPPORTED;
    } else {
      const long long rows = static_cast<long long>(pg->num_pages) << pg->page_shift;
      const uint32_t piece = (1u << pg->page_shift) < 32u ? (1u << pg->page_shift) : 32u;
      if (rows > 0x7fffffffLL || encode_map_packed(&tk, k, static_cast<int>(rows), Hkv, piece) != ATTN_OK ||
          encode_map_packed(&tv, v, static_cast<int>(rows), Hkv, piece) != ATTN_OK)
        return ATTN_ERR_UNSUPPORTED;
    }
    const dec::Paged pgv = pg != nullptr ? *pg : dec::Paged{};
    const bool paged = pg != nullptr;
#define ATTN_LAUNCH_DTC(GG)                                                                      \
  do {                                                                                           \
    if (paged)                                                                                   \
      dtc::decode_tc_kernel<GG, true><<<grid, dtc::kThreads, dtc::kSmemBytes, st>>>(             \
          tq, tk, tv, ws_o, ws_lse, Hq, Hkv, Nk, chunk, splits, c, pgv);                         \
    else                                                                                         \
      dtc::decode_tc_kernel<GG, false><<<grid, dtc::kThreads, dtc::kSmemBytes, st>>>(            \
          tq, tk, tv, ws_o, ws_lse, Hq, Hkv, Nk, chunk, splits, c, pgv);                         \
  } while (0)
    switch (G) {
      case 1: ATTN_LAUNCH_DTC(1); break;
      case 2: ATTN_LAUNCH_DTC(2); break;
      case 4: ATTN_LAUNCH_DTC(4); break;
      default: ATTN_LAUNCH_DTC(8); break;
    }
#undef ATTN_LAUNCH_DTC
    rc = cuda_status(cudaGetLastError());
    if (rc != ATTN_OK) return rc;
    dec::decode_combine_kernel<<<B * Hq, dec::kD, 0, st>>>(
        ws_o, ws_lse, static_cast<__nv_bfloat16*>(o), lse, splits);
    return cuda_status(cudaGetLastError());
  }
  const auto* qb = static_cast<const __nv_bfloat16*>(q);
  const auto* kb = static_cast<const __nv_bfloat16*>(k);
  const auto* vb = static_cast<const __nv_bfloat16*>(v);
  switch (G) {
    case 1: launch_decode_split<1>(grid, chunk, st, qb, kb, vb, ws_o, ws_lse, Hq, Hkv, Nk, splits, c, pg); break;
    case 2: launch_decode_split<2>(grid, chunk, st, qb, kb, vb, ws_o, ws_lse, Hq, Hkv, Nk, splits, c, pg); break;
    case 4: launch_decode_split<4>(grid, chunk, st, qb, kb, vb, ws_o, ws_lse, Hq, Hkv, Nk, splits, c, pg); break;
    default: launch_decode_split<8>(grid, chunk, st, qb, kb, vb, ws_o, ws_lse, Hq, Hkv, Nk, splits, c, pg); break;
  }
  int rc = cuda_status(cudaGetLastError());
  if (rc != ATTN_OK) return rc;
  dec::decode_combine_kernel<<<B * Hq, dec::kD, 0, st>>>(ws_o, ws_lse,
                                                         static_cast<__nv_bfloat16*>(o), lse, splits);
  return cuda_status(cudaGetLastError());
}

__global__ void timeout_probe_kernel(long long limit) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    dev::mbar_init(dev::smem_u32(&bar), 1);
    abort_flag = 0;
    dev::fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) wait_bounded(dev::smem_u32(&bar), 0, &abort_flag, limit);
  __syncthreads();
}

// The CTAs of a prefill launch.  With an even group size a CTA takes the same 128 rows of two
// query heads that read one kv head, so its two query tiles see the same keys and every key
// tile feeds both; otherwise a CTA takes 256 consecutive rows of one head.
struct FwdSchedule {
  int head_pair, num_qblocks;
  long long units;
};

FwdSchedule fwd_schedule(int batch, int Hq, int Hkv, int rows) {
  FwdSchedule sc;
  sc.head_pair = (Hq / Hkv) % 2 == 0 ? 1 : 0;
  const int per_cta = sc.head_pair ? fwd::kBM : fwd::kRowsPerCta;
  sc.num_qblocks = (rows + per_cta - 1) / per_cta;
  sc.units = static_cast<long long>(sc.num_qblocks) * batch * (sc.head_pair ? Hq / 2 : Hq);
  return sc;
}

}  // namespace
}  // namespace attn

using namespace attn;

extern "C" {

int attn_abi_version(void) { return 1; }

const char* attn_last_error_detail(void) { return g_last_detail; }

const char* attn_status_string(int status) {
  switch (status) {
    case ATTN_OK: return "ok";
    case ATTN_ERR_INVALID_ARG: return "invalid argument";
    case ATTN_ERR_UNSUPPORTED: return "unsupported configuration (head dim, group size, alignment or device)";
    case ATTN_ERR_CUDA: return "CUDA runtime error";
    case ATTN_ERR_WORKSPACE: return "decode workspace missing or too small";
    case ATTN_ERR_DEVICE_TIMEOUT: return "a bounded device-side wait expired";
    default: return "unknown status";
  }
}

int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
             int Hkv, int Nq, int Nk, int d, int mask_kind, int window, int n_sink, float scale,
             attn_stream_t stream) {
  int rc = check_fwd_args(q, k, v, o, B, Hq, Hkv, Nq, Nk, mask_kind, window, n_sink, scale);
  if (rc != ATTN_OK) return rc;
  if (d != fwd::kD) return ATTN_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return ATTN_ERR_UNSUPPORTED;
  if (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u)) return ATTN_ERR_UNSUPPORTED;
  DeviceInfo* info = nullptr;
  if ((rc = current_device(&info)) != ATTN_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (B == 0 || Nq == 0) return ATTN_OK;
  if (Nk == 0)
    return launch_fill_empty(static_cast<__nv_bfloat16*>(o), lse,
                             static_cast<size_t>(B) * Hq * Nq, d, st);
  const FwdSchedule sc = fwd_schedule(B, Hq, Hkv, Nq);
  if (sc.units > 0x7fffffffLL - 4096) return ATTN_ERR_UNSUPPORTED;
  if ((rc = configure_fwd(info)) != ATTN_OK) return rc;

  CUtensorMap tq, tk, tv, to;
  if (encode_map(&tq, q, Nq, B * Hq) != ATTN_OK || encode_map(&tk, k, Nk, B * Hkv) != ATTN_OK ||
      encode_map(&tv, v, Nk, B * Hkv) != ATTN_OK || encode_map_out(&to, o, Nq, B * Hq, false) != ATTN_OK)
    return ATTN_ERR_UNSUPPORTED;
  fwd::Params p{};
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Nq = Nq;
  p.Nk = Nk;
  p.G = Hq / Hkv;
  p.mask = make_mask(mask_kind, window, n_sink, Nk);
  // scale = 0 makes every visible weight equal; a tiny positive c gives exactly that (every
  // exp2 argument rounds to 0) while masked scores (-inf) still map to weight 0
  p.c = scale * kLog2e;
  if (p.c == 0.f) p.c = 1e-30f;
  p.num_qblocks = sc.num_qblocks;
  p.head_pair = sc.head_pair;
  p.units = static_cast<int>(sc.units);
  if ((rc = unit_counter(st, &p.unit_counter)) != ATTN_OK) return rc;
  p.front_heavy = (mask_kind == ATTN_MASK_LOCAL_GLOBAL && n_sink > 0) ? 1 : 0;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.cu_q = nullptr;
  p.cu_k = nullptr;
  const dim3 grid(static_cast<unsigned>(std::min<long long>(sc.units, info->num_sms)));
  if (scale < 0.f)
    fwd::fwd_bf16_sm100_kernel<true, false><<<grid, fwd::kThreads, fwd::kSmemBytes, st>>>(tq, tk, tv, to, p);
  else
    fwd::fwd_bf16_sm100_kernel<false, false><<<grid, fwd::kThreads, fwd::kSmemBytes, st>>>(tq, tk, tv, to, p);
  return cuda_status(cudaGetLastError());
}

int attn_fwd_block_sparse(const void* q, const void* k, const void* v, void* o, float* lse,
                          const uint8_t* block_mask, int mask_heads, int B, int Hq, int Hkv,
                          int Nq, int Nk, int d, int mask_kind, int window, int n_sink,
                          float scale, attn_stream_t stream) {
  int rc = check_fwd_args(q, k, v, o, B, Hq, Hkv, Nq, Nk, mask_kind, window, n_sink, scale);
  if (rc != ATTN_OK) return rc;
  if (mask_heads != 1 && mask_heads != Hq) return ATTN_ERR_INVALID_ARG;
  if (B > 0 && Nq > 0 && Nk > 0 && block_mask == nullptr) return ATTN_ERR_INVALID_ARG;
  if (d != fwd::kD) return ATTN_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return ATTN_ERR_UNSUPPORTED;
  if (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u)) return ATTN_ERR_UNSUPPORTED;
  const int mask_qtiles = (Nq + fwd::kBM - 1) / fwd::kBM, mask_ktiles = (Nk + fwd::kBN - 1) / fwd::kBN;
  if (mask_ktiles > fwd::kMaxSparseTiles) return ATTN_ERR_UNSUPPORTED;
  DeviceInfo* info = nullptr;
  if ((rc = current_device(&info)) != ATTN_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (B == 0 || Nq == 0) return ATTN_OK;
  if (Nk == 0)
    return launch_fill_empty(static_cast<__nv_bfloat16*>(o), lse,
                             static_cast<size_t>(B) * Hq * Nq, d, st);
  const FwdSchedule sc = fwd_schedule(B, Hq, Hkv, Nq);
  if (sc.units > 0x7fffffffLL - 4096) return ATTN_ERR_UNSUPPORTED;
  if ((rc = configure_fwd(info)) != ATTN_OK) return rc;
  CUtensorMap tq, tk, tv, to;
  if (encode_map(&tq, q, Nq, B * Hq) != ATTN_OK || encode_map(&tk, k, Nk, B * Hkv) != ATTN_OK ||
      encode_map(&tv, v, Nk, B * Hkv) != ATTN_OK || encode_map_out(&to, o, Nq, B * Hq, false) != ATTN_OK)
    return ATTN_ERR_UNSUPPORTED;
  fwd::Params p{};
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Nq = Nq;
  p.Nk = Nk;
  p.G = Hq / Hkv;
  p.mask = make_mask(mask_kind, window, n_sink, Nk);
  p.c = scale * kLog2e;
  if (p.c == 0.f) p.c = 1e-30f;
  p.num_qblocks = sc.num_qblocks;
  p.head_pair = sc.head_pair;
  p.units = static_cast<int>(sc.units);
  if ((rc = unit_counter(st, &p.unit_counter)) != ATTN_OK) return rc;
  p.front_heavy = (mask_kind == ATTN_MASK_FULL || mask_kind == ATTN_MASK_LOCAL_GLOBAL) ? 1 : 0;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.block_mask = block_mask;
  p.mask_heads = mask_heads;
  p.mask_qtiles = mask_qtiles;
  p.mask_ktiles = mask_ktiles;
  const dim3 grid(static_cast<unsigned>(std::min<long long>(sc.units, info->num_sms)));
  if (scale < 0.f)
    fwd::fwd_bf16_sparse_sm100_kernel<true><<<grid, fwd::kThreads, fwd::kSmemBytesSparse, st>>>(tq, tk, tv, to, p);
  else
    fwd::fwd_bf16_sparse_sm100_kernel<false><<<grid, fwd::kThreads, fwd::kSmemBytesSparse, st>>>(tq, tk, tv, to, p);
  return cuda_status(cudaGetLastError());
}

int attn_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                    const int* cu_seqlens_q, const int* cu_seqlens_k, int num_seqs, int Hq,
                    int Hkv, int total_q, int total_k, int max_seqlen_q, int d, int mask_kind,
                    int window, int n_sink, float scale, attn_stream_t stream) {
  if (num_seqs < 0 || total_q < 0 || total_k < 0 || max_seqlen_q < 0) return ATTN_ERR_INVALID_ARG;
  if (num_seqs > 0 && (cu_seqlens_q == nullptr || cu_seqlens_k == nullptr)) return ATTN_ERR_INVALID_ARG;
  // the packed tensors play the role of one batch row each for the common checks
  int rc = check_fwd_args(q, k, v, o, num_seqs > 0 ? 1 : 0, Hq, Hkv, total_q, total_k, mask_kind,
                          window, n_sink, scale);
  if (rc != ATTN_OK) return rc;
  if (d != fwd::kD) return ATTN_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return ATTN_ERR_UNSUPPORTED;
  if (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u)) return ATTN_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(cu_seqlens_q) & 3u) || (reinterpret_cast<uintptr_t>(cu_seqlens_k) & 3u))
    return ATTN_ERR_UNSUPPORTED;
  DeviceInfo* info = nullptr;
  if ((rc = current_device(&info)) != ATTN_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (num_seqs == 0 || total_q == 0 || max_seqlen_q == 0) return ATTN_OK;
  if (total_k == 0)
    return launch_fill_empty(static_cast<__nv_bfloat16*>(o), lse, static_cast<size_t>(total_q) * Hq, d, st);
  const FwdSchedule sc = fwd_schedule(num_seqs, Hq, Hkv, max_seqlen_q);
  if (sc.units > 0x7fffffffLL - 4096) return ATTN_ERR_UNSUPPORTED;
  if ((rc = configure_fwd(info)) != ATTN_OK) return rc;
  CUtensorMap tq, tk, tv, to;
  if (encode_map_packed(&tq, q, total_q, Hq) != ATTN_OK || encode_map_packed(&tk, k, total_k, Hkv) != ATTN_OK ||
      encode_map_packed(&tv, v, total_k, Hkv) != ATTN_OK ||
      encode_map_out(&to, o, total_q, Hq, true) != ATTN_OK)
    return ATTN_ERR_UNSUPPORTED;
  fwd::Params p{};
  p.B = num_seqs;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Nq = total_q;
  p.Nk = total_k;
  p.G = Hq / Hkv;
  p.mask = make_mask(mask_kind, window, n_sink, total_k);
  p.c = scale * kLog2e;
  if (p.c == 0.f) p.c = 1e-30f;
  p.num_qblocks = sc.num_qblocks;
  p.head_pair = sc.head_pair;
  p.units = static_cast<int>(sc.units);
  if ((rc = unit_counter(st, &p.unit_counter)) != ATTN_OK) return rc;
  p.front_heavy = (mask_kind == ATTN_MASK_LOCAL_GLOBAL && n_sink > 0) ? 1 : 0;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.cu_q = cu_seqlens_q;
  p.cu_k = cu_seqlens_k;
  const dim3 grid(static_cast<unsigned>(std::min<long long>(sc.units, info->num_sms)));
  if (scale < 0.f)
    fwd::fwd_bf16_sm100_kernel<true, true><<<grid, fwd::kThreads, fwd::kSmemBytes, st>>>(tq, tk, tv, to, p);
  else
    fwd::fwd_bf16_sm100_kernel<false, true><<<grid, fwd::kThreads, fwd::kSmemBytes, st>>>(tq, tk, tv, to, p);
  return cuda_status(cudaGetLastError());
}

int attn_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse,
                 const float* descale_q, const float* descale_k, const float* descale_v, int B,
                 int Hq, int Hkv, int Nq, int Nk, int d, int mask_kind, int window, int n_sink,
                 float scale, attn_stream_t stream) {
  int rc = check_fwd_args(q, k, v, o, B, Hq, Hkv, Nq, Nk, mask_kind, window, n_sink, scale);
  if (rc != ATTN_OK) return rc;
  const bool q_empty = B == 0 || Nq == 0, kv_empty = B == 0 || Nk == 0;
  if (!q_empty && (descale_q == nullptr || (!kv_empty && (descale_k == nullptr ||
                                                          descale_v == nullptr))))
    return ATTN_ERR_INVALID_ARG;
  if (d != fwd::kD) return ATTN_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return ATTN_ERR_UNSUPPORTED;
  if (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u)) return ATTN_ERR_UNSUPPORTED;
  DeviceInfo* info = nullptr;
  if ((rc = current_device(&info)) != ATTN_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (q_empty) return ATTN_OK;
  if (Nk == 0)
    return launch_fill_empty(static_cast<__nv_bfloat16*>(o), lse, static_cast<size_t>(B) * Hq * Nq, d, st);
  const FwdSchedule sc = fwd_schedule(B, Hq, Hkv, Nq);
  if (sc.units > 0x7fffffffLL - 4096) return ATTN_ERR_UNSUPPORTED;
  if ((rc = configure_fwd(info)) != ATTN_OK) return rc;
  CUtensorMap tq, tk, tv, to;
  if (encode_map_e4m3(&tq, q, Nq, B * Hq) != ATTN_OK || encode_map_e4m3(&tk, k, Nk, B * Hkv) != ATTN_OK ||
      encode_map_e4m3(&tv, v, Nk, B * Hkv) != ATTN_OK || encode_map_out(&to, o, Nq, B * Hq, false) != ATTN_OK)
    return ATTN_ERR_UNSUPPORTED;
  fwd::Params p{};
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Nq = Nq;
  p.Nk = Nk;
  p.G = Hq / Hkv;
  p.mask = make_mask(mask_kind, window, n_sink, Nk);
  p.c = scale * kLog2e;
  if (p.c == 0.f) p.c = 1e-30f;
  p.num_qblocks = sc.num_qblocks;
  p.head_pair = sc.head_pair;
  p.units = static_cast<int>(sc.units);
  if ((rc = unit_counter(st, &p.unit_counter)) != ATTN_OK) return rc;
  p.front_heavy = (mask_kind == ATTN_MASK_LOCAL_GLOBAL && n_sink > 0) ? 1 : 0;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.cu_q = nullptr;
  p.cu_k = nullptr;
  p.descale_q = descale_q;
  p.descale_k = descale_k;
  p.descale_v = descale_v;
  const dim3 grid(static_cast<unsigned>(std::min<long long>(sc.units, info->num_sms)));
  if (scale < 0.f)
    fwd::fwd_fp8_sm100_kernel<true><<<grid, fwd::kThreads, fwd::kSmemBytes, st>>>(tq, tk, tv, to, p);
  else
    fwd::fwd_fp8_sm100_kernel<false><<<grid, fwd::kThreads, fwd::kSmemBytes, st>>>(tq, tk, tv, to, p);
  return cuda_status(cudaGetLastError());
}

int attn_fwd_f32(const float* q, const float* k, const float* v, float* o, float* lse, int B,
                 int Hq, int Hkv, int Nq, int Nk, int d, int mask_kind, int window, int n_sink,
                 float scale, attn_stream_t stream) {
  int rc = check_fwd_args(q, k, v, o, B, Hq, Hkv, Nq, Nk, mask_kind, window, n_sink, scale);
  if (rc != ATTN_OK) return rc;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return ATTN_ERR_UNSUPPORTED;
  DeviceInfo* info = nullptr;
  if ((rc = current_device(&info)) != ATTN_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (B == 0 || Nq == 0) return ATTN_OK;
  if (Nk == 0) return launch_fill_empty(o, lse, static_cast<size_t>(B) * Hq * Nq, d, st);
  if (Hq > 65535 || B > 65535) return ATTN_ERR_UNSUPPORTED;
  f32::Params p;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Nq = Nq;
  p.Nk = Nk;
  p.G = Hq / Hkv;
  p.mask = make_mask(mask_kind, window, n_sink, Nk);
  p.c = scale * kLog2e;
  // the kv head's whole K and V in shared memory (at most 512 keys, about 200 KB): one warp per
  // query row; otherwise the tiled kernel
  const size_t small_bytes = d == 64 ? f32::small_smem_bytes<64>(Nk) : f32::small_smem_bytes<128>(Nk);
  if (Nk <= 32 * f32::kSmallMaxChunks && small_bytes <= 200 * 1024) {
    const dim3 grid((Nq + f32::kSmallWarps - 1) / f32::kSmallWarps, Hq, B);
    if (d == 64) {
      rc = cuda_status(cudaFuncSetAttribute(f32::fwd_f32_small_kernel<64>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            static_cast<int>(small_bytes)));
      if (rc != ATTN_OK) return rc;
      f32::fwd_f32_small_kernel<64><<<grid, f32::kSmallWarps * 32, small_bytes, st>>>(q, k, v, o, lse, p);
    } else {
      rc = cuda_status(cudaFuncSetAttribute(f32::fwd_f32_small_kernel<128>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            static_cast<int>(small_bytes)));
      if (rc != ATTN_OK) return rc;
      f32::fwd_f32_small_kernel<128><<<grid, f32::kSmallWarps * 32, small_bytes, st>>>(q, k, v, o, lse, p);
    }
    return cuda_status(cudaGetLastError());
  }
  if (d == 64) {
    dim3 grid((Nq + f32::rows_per_cta<64>() - 1) / f32::rows_per_cta<64>(), Hq, B);
    f32::fwd_f32_kernel<64><<<grid, f32::kWarps * 32, 0, st>>>(q, k, v, o, lse, p);
  } else {
    dim3 grid((Nq + f32::rows_per_cta<128>() - 1) / f32::rows_per_cta<128>(), Hq, B);
    f32::fwd_f32_kernel<128><<<grid, f32::kWarps * 32, 0, st>>>(q, k, v, o, lse, p);
  }
  return cuda_status(cudaGetLastError());
}

int attn_decode_num_splits(int B, int Hq, int Hkv, int Nk, int d) {
  (void)d;
  if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || Nk < 0) return ATTN_ERR_INVALID_ARG;
  DeviceInfo* info = nullptr;
  const int num_sms = current_device(&info) == ATTN_OK ? info->num_sms : 148;
  return decode_splits(B, Hkv, Nk, Hq / Hkv, 0, num_sms);
}

size_t attn_decode_workspace_bytes(int B, int Hq, int Hkv, int Nk, int d, int num_splits) {
  if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || Nk < 0 || d != dec::kD) return 0;
  DeviceInfo* info = nullptr;
  const int num_sms = current_device(&info) == ATTN_OK ? info->num_sms : 148;
  const int splits = decode_splits(B, Hkv, Nk, Hq / Hkv, num_splits, num_sms);
  return decode_ws_bytes(B, Hq, splits);
}

int attn_decode(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                int Hkv, int Nk, int d, float scale, int num_splits, void* workspace,
                size_t workspace_bytes, attn_stream_t stream) {
  if (B < 0 || Nk < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (B > 0 && (q == nullptr || o == nullptr || (Nk > 0 && (k == nullptr || v == nullptr))))
    return ATTN_ERR_INVALID_ARG;
  if (num_splits < 0 || !std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  if (d != dec::kD) return ATTN_ERR_UNSUPPORTED;
  const int G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return ATTN_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return ATTN_ERR_UNSUPPORTED;
  DeviceInfo* info = nullptr;
  int rc = current_device(&info);
  if (rc != ATTN_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (B == 0) return ATTN_OK;
  if (Nk == 0)
    return launch_fill_empty(static_cast<__nv_bfloat16*>(o), lse, static_cast<size_t>(B) * Hq, d, st);
  if (B > 65535 || Hkv > 65535) return ATTN_ERR_UNSUPPORTED;
  return decode_run(q, k, v, o, lse, B, Hq, Hkv, Nk, scale, num_splits, workspace,
                    workspace_bytes, st, info, nullptr);
}

int attn_decode_paged(const void* q, const void* k_cache, const void* v_cache, void* o,
                      float* lse, const int* block_table, const int* seq_lens, int B, int Hq,
                      int Hkv, int num_pages, int page_size, int max_pages_per_seq,
                      int max_seq_len, int d, float scale, int num_splits, void* workspace,
                      size_t workspace_bytes, attn_stream_t stream) {
  if (B < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || num_pages < 0 || max_pages_per_seq < 0 ||
      max_seq_len < 0)
    return ATTN_ERR_INVALID_ARG;
  if (page_size < dec::kMinPageSize || page_size > (1 << 20) || (page_size & (page_size - 1)) != 0)
    return ATTN_ERR_INVALID_ARG;
  if (static_cast<long long>(max_seq_len) > static_cast<long long>(max_pages_per_seq) * page_size)
    return ATTN_ERR_INVALID_ARG;
  if (num_splits < 0 || !std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  const bool any_keys = max_seq_len > 0 && num_pages > 0;
  if (B > 0 && (q == nullptr || o == nullptr || seq_lens == nullptr)) return ATTN_ERR_INVALID_ARG;
  if (B > 0 && any_keys && (k_cache == nullptr || v_cache == nullptr || block_table == nullptr))
    return ATTN_ERR_INVALID_ARG;
  if (d != dec::kD) return ATTN_ERR_UNSUPPORTED;
  const int G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return ATTN_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o))
    return ATTN_ERR_UNSUPPORTED;
  DeviceInfo* info = nullptr;
  int rc = current_device(&info);
  if (rc != ATTN_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (B == 0) return ATTN_OK;
  if (!any_keys)
    return launch_fill_empty(static_cast<__nv_bfloat16*>(o), lse, static_cast<size_t>(B) * Hq, d, st);
  if (B > 65535 || Hkv > 65535) return ATTN_ERR_UNSUPPORTED;
  int shift = 0;
  while ((1 << shift) < page_size) ++shift;
  const dec::Paged pg{block_table, seq_lens, max_pages_per_seq, num_pages, shift};
  return decode_run(q, k_cache, v_cache, o, lse, B, Hq, Hkv, max_seq_len, scale, num_splits,
                    workspace, workspace_bytes, st, info, &pg);
}

size_t attn_bwd_workspace_bytes(int B, int Hq, int Nq, int Nk, int mask_kind, int window,
                                int n_sink) {
  if (B < 1 || Hq < 1 || Nq < 0 || Nk < 0) return 0;
  if (mask_kind < ATTN_MASK_FULL || mask_kind > ATTN_MASK_LOCAL_GLOBAL || n_sink < 0 ||
      (mask_kind == ATTN_MASK_SLIDING && window < 1) ||
      (mask_kind == ATTN_MASK_LOCAL_GLOBAL && window < 0))
    return 0;
  return bwd_layout(B, Hq, Nq, Nk, make_mask(mask_kind, window, n_sink, Nk)).total;
}

int attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
             const void* dout, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Nq,
             int Nk, int d, int mask_kind, int window, int n_sink, float scale, void* workspace,
             size_t workspace_bytes, attn_stream_t stream) {
  int rc = check_fwd_args(q, k, v, o, B, Hq, Hkv, Nq, Nk, mask_kind, window, n_sink, scale);
  if (rc != ATTN_OK) return rc;
  const bool q_empty = B == 0 || Nq == 0, kv_empty = B == 0 || Nk == 0;
  if (!q_empty && (lse == nullptr || dout == nullptr || dq == nullptr)) return ATTN_ERR_INVALID_ARG;
  if (!kv_empty && (dk == nullptr || dv == nullptr)) return ATTN_ERR_INVALID_ARG;
  if (d != bwd::kD) return ATTN_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || (reinterpret_cast<uintptr_t>(lse) & 3u))
    return ATTN_ERR_UNSUPPORTED;
  DeviceInfo* info = nullptr;
  if ((rc = current_device(&info)) != ATTN_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (B == 0) return ATTN_OK;
  const size_t q_bytes = static_cast<size_t>(B) * Hq * Nq * d * 2;
  const size_t kv_bytes = static_cast<size_t>(B) * Hkv * Nk * d * 2;
  // no query: every key gets zero gradients; no key: every query does
  if (Nq == 0 || Nk == 0) {
    if (Nq == 0 && Nk > 0) {
      if ((rc = cuda_status(cudaMemsetAsync(dk, 0, kv_bytes, st))) != ATTN_OK) return rc;
      return cuda_status(cudaMemsetAsync(dv, 0, kv_bytes, st));
    }
    if (Nq > 0) return cuda_status(cudaMemsetAsync(dq, 0, q_bytes, st));
    return ATTN_OK;
  }
  const int nqt = (Nq + bwd::kT - 1) / bwd::kT, nkb = (Nk + bwd::kT - 1) / bwd::kT;
  const long long units_q = static_cast<long long>((nqt + 1) / 2) * B * Hq;  // query-tile pairs
  const long long units_kv = static_cast<long long>(nkb) * B * Hkv;
  if (units_q > 0x7fffffffLL - 4096 || units_kv > 0x7fffffffLL - 4096) return ATTN_ERR_UNSUPPORTED;
  const MaskSpec mask = make_mask(mask_kind, window, n_sink, Nk);
  const BwdLayout L = bwd_layout(B, Hq, Nq, Nk, mask);
  if (static_cast<double>(B) * Hq * static_cast<double>(L.pairs) > 2147483647.0)
    return ATTN_ERR_UNSUPPORTED;  // dS block index of the dQ kernel's tensor map
  if (workspace == nullptr || workspace_bytes < L.total || !aligned16(workspace))
    return ATTN_ERR_WORKSPACE;
  if ((rc = configure_fwd(info)) != ATTN_OK) return rc;  // the tensor-map encoder
  if ((rc = configure_bwd(info)) != ATTN_OK) return rc;
  CUtensorMap tq, tk, tv, tdo;
  if (encode_map(&tq, q, Nq, B * Hq) != ATTN_OK || encode_map(&tk, k, Nk, B * Hkv) != ATTN_OK ||
      encode_map(&tv, v, Nk, B * Hkv) != ATTN_OK || encode_map(&tdo, dout, Nq, B * Hq) != ATTN_OK)
    return ATTN_ERR_UNSUPPORTED;
  bwd::Params p;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Nq = Nq;
  p.Nk = Nk;
  p.G = Hq / Hkv;
  p.mask = mask;
  p.scale = scale;
  p.c = scale * kLog2e;
  p.num_kblocks = nkb;
  p.num_qtiles = nqt;
  p.npad = nqt * bwd::kT;
  float* lse2 = static_cast<float*>(workspace);
  float* dsum = lse2 + static_cast<size_t>(B) * Hq * p.npad;
  p.lse2 = lse2;
  p.dsum = dsum;
  p.dq = static_cast<__nv_bfloat16*>(dq);
  p.dk = static_cast<__nv_bfloat16*>(dk);
  p.dv = static_cast<__nv_bfloat16*>(dv);
  p.ds_off = reinterpret_cast<int*>(dsum + static_cast<size_t>(B) * Hq * p.npad);
  p.ds = reinterpret_cast<__nv_bfloat16*>(static_cast<uint8_t*>(workspace) + L.ds_offset);
  p.ds_pairs = static_cast<long long>(L.pairs);
  if ((rc = unit_counter(st, &p.unit_counter)) != ATTN_OK) return rc;
  // dS^T blocks as a 3-D tensor (queries, keys, block) for the dQ kernel's TMA loads
  CUtensorMap tds;
  {
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(bwd::kT), static_cast<cuuint64_t>(bwd::kT),
                                static_cast<cuuint64_t>(B) * Hq * (L.pairs > 0 ? L.pairs : 1)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(bwd::kT) * 2,
                                   static_cast<cuuint64_t>(bwd::kT) * bwd::kT * 2};
    const cuuint32_t box[3] = {64, 128, 1};
    const cuuint32_t estride[3] = {1, 1, 1};
    if (g_encode(&tds, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, p.ds, dims, strides, box, estride,
                 CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                 CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return ATTN_ERR_UNSUPPORTED;
  }
  // the same blocks as the dK/dV kernel writes them: boxes of 32 queries x 32 keys, one per row
  // warp and sub-step, staged with the 64-byte swizzle
  CUtensorMap tds_out;
  {
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(bwd::kT), static_cast<cuuint64_t>(bwd::kT),
                                static_cast<cuuint64_t>(B) * Hq * (L.pairs > 0 ? L.pairs : 1)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(bwd::kT) * 2,
                                   static_cast<cuuint64_t>(bwd::kT) * bwd::kT * 2};
    const cuuint32_t box[3] = {32, 32, 1};
    const cuuint32_t estride[3] = {1, 1, 1};
    if (g_encode(&tds_out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, p.ds, dims, strides, box, estride,
                 CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                 CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return ATTN_ERR_UNSUPPORTED;
  }
  // dQ, dK and dV as boxes of 32 columns x 32 rows staged with the 64-byte swizzle
  CUtensorMap tdq, tdk, tdv;
  if (encode_map_out(&tdq, dq, Nq, B * Hq, false) != ATTN_OK ||
      encode_map_out(&tdk, dk, Nk, B * Hkv, false) != ATTN_OK ||
      encode_map_out(&tdv, dv, Nk, B * Hkv, false) != ATTN_OK)
    return ATTN_ERR_UNSUPPORTED;
  const long long prow = static_cast<long long>(B) * Hq * p.npad;
  // one wave (4 blocks of 8 warps per SM at 64 registers a thread), grid-stride over the row groups
  const long long prep_blocks = std::min<long long>((prow + bwd::kPrepRowsPerBlock - 1) /
                                                        bwd::kPrepRowsPerBlock,
                                                    4LL * info->num_sms);
  bwd::bwd_prep_kernel<<<static_cast<unsigned>(prep_blocks), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dout), lse, lse2,
      dsum, Nq, p.npad, prow, mask, nkb, p.ds_off);
  if ((rc = cuda_status(cudaGetLastError())) != ATTN_OK) return rc;
  // persistent: one CTA per SM walking the key-block units
  bwd::bwd_dkdv_kernel<<<static_cast<unsigned>(std::min<long long>(units_kv, info->num_sms)),
                         bwd::kThreads, bwd::kSmemKVBytes, st>>>(tq, tk, tv, tdo, tds_out, tdk,
                                                                 tdv, p);
  if ((rc = cuda_status(cudaGetLastError())) != ATTN_OK) return rc;
  bwd::bwd_dq_kernel<<<static_cast<unsigned>(std::min<long long>(units_q, info->num_sms)),
                       bwd::kThreads, bwd::kSmemQBytes, st>>>(tds, tk, tdq, p);
  return cuda_status(cudaGetLastError());
}

int attn_get_device_error(attn_stream_t stream) {
  int rc = cuda_status(cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)));
  if (rc != ATTN_OK) return rc;
  int flag = 0;
  if ((rc = cuda_status(cudaMemcpyFromSymbol(&flag, g_device_error, sizeof(int)))) != ATTN_OK)
    return rc;
  if (flag != 0) {
    const int zero = 0;
    if ((rc = cuda_status(cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int)))) != ATTN_OK)
      return rc;
    return flag;
  }
  return ATTN_OK;
}

int attn_debug_timeout_probe(long long limit_cycles, attn_stream_t stream) {
  if (limit_cycles < 1 || limit_cycles > (1ll << 34)) return ATTN_ERR_INVALID_ARG;
  DeviceInfo* info = nullptr;
  int rc = current_device(&info);
  if (rc != ATTN_OK) return rc;
  timeout_probe_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(limit_cycles);
  return cuda_status(cudaGetLastError());
}

}  // extern "C"

// ------------------------------------------------------------------------------------------
// Decode without allocation: the same split-K decode, with its partial results kept in a
// fixed array that the library owns instead of a caller-provided workspace.
// ------------------------------------------------------------------------------------------
namespace attn {
namespace {

// Every GPU that loads this library holds this array until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[ATTN_DECODE_NOALLOC_MAX_BYTES];

void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device, looked up once per device (in
// host code the array's name is only a host-side stand-in, never a device address).  The
// address is kept for the process's life: the header rules out use across a device reset.
int noalloc_scratch(void** out) {
  int dev = 0;
  int rc = cuda_status(cudaGetDevice(&dev));
  if (rc != ATTN_OK) return rc;
  if (dev < 0 || dev >= kMaxDevices) return ATTN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    rc = cuda_status(cudaGetSymbolAddress(&p, g_noalloc_scratch));
    if (rc != ATTN_OK) return rc;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return ATTN_OK;
}

}  // namespace
}  // namespace attn

extern "C" int attn_decode_noalloc(const void* q, const void* k, const void* v, void* o,
                                   float* lse, int B, int Hq, int Hkv, int Nk, int d,
                                   float scale, int num_splits, attn_stream_t stream) {
  // same argument rules as attn_decode; the scratch size is checked before anything runs
  if (B < 0 || Nk < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (num_splits < 0) return ATTN_ERR_INVALID_ARG;
  if (d != dec::kD) return ATTN_ERR_UNSUPPORTED;
  DeviceInfo* info = nullptr;
  int rc = current_device(&info);
  if (rc != ATTN_OK) return rc;
  const int G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return ATTN_ERR_UNSUPPORTED;
  if (B > 0 && Nk > 0) {
    const int splits = decode_splits(B, Hkv, Nk, G, num_splits, info->num_sms);
    if (decode_ws_bytes(B, Hq, splits) > ATTN_DECODE_NOALLOC_MAX_BYTES) return ATTN_ERR_WORKSPACE;
  }
  void* scratch = nullptr;
  if ((rc = noalloc_scratch(&scratch)) != ATTN_OK) return rc;
  return attn_decode(q, k, v, o, lse, B, Hq, Hkv, Nk, d, scale, num_splits, scratch,
                     ATTN_DECODE_NOALLOC_MAX_BYTES, stream);
}
