/*
 * attn.h - C ABI of the exact IO-aware attention library for NVIDIA B200 (sm_100a).
 *
 * Operation (all entry points): for every batch b, query head h and query row i,
 *
 *     O[b,h,i,:]  = sum_j P_ij V[b,hk,j,:],   P_ij = exp(s_ij) / sum_{visible j'} exp(s_ij'),
 *     s_ij        = scale * Q[b,h,i,:] . K[b,hk,j,:]   over the keys j visible to row i,
 *     LSE[b,h,i]  = ln sum_{visible j} exp(s_ij)       (natural log),
 *
 * i.e. scaled dot-product attention softmax(Q K^T / sqrt(d)) V with Q, K, V of shape (n, d)
 * ("Chapter 3.1 - The Cost of Attention", section 2), computed exactly, FlashAttention-style:
 * Q/K/V tiles pass through on-chip memory and an online (running max / running sum) softmax
 * is used, so the n x n score matrix never reaches HBM ("FlashAttention and sparse
 * attention", section 1: tiling, kernel fusion and online softmax; same page as above,
 * section 5).
 *
 * Masks (mask_kind), with p_i = i + Nk - Nq the key position of query row i (bottom-right
 * alignment when Nq != Nk):
 *   ATTN_MASK_FULL     every key visible;
 *   ATTN_MASK_CAUSAL   key j visible iff j <= p_i;
 *   ATTN_MASK_SLIDING  causal, and (p_i - window < j  or  j < n_sink): a left window of `window`
 *                      keys including the diagonal ("Quadratic Complexity Bottleneck",
 *                      sliding-window attention) plus n_sink always-visible sink tokens at key
 *                      positions 0..n_sink-1 ("Attention Research", section 4).
 *   ATTN_MASK_LOCAL_GLOBAL  not causal: key j visible iff |p_i - j| <= window (window keys on
 *                      each side), or j < n_sink, or 0 <= p_i < n_sink: the first n_sink
 *                      tokens are global, they see and are seen by every token (Longformer;
 *                      "Chapter 3.1 - The Cost of Attention", section 3; "Quadratic Complexity
 *                      Bottleneck", sliding window: W tokens to the left and right).
 * Rows with no visible key get O = 0 and LSE = -inf.
 * GQA ("Quadratic Complexity Bottleneck", grouped-query attention): Hq = G * Hkv and query head
 * h reads kv head hk = h / G (contiguous groups); Hkv = 1 is multi-query attention.
 *
 * Layouts: contiguous, row-major, head dimension innermost.
 *   Q, O  [B][Hq][Nq][d]      K, V  [B][Hkv][Nk][d]      LSE  [B][Hq][Nq] fp32
 *
 * Ownership and execution: every pointer is a DEVICE pointer owned by the caller (a tensor with
 * no element may be passed as NULL; LSE may always be NULL when not wanted); the library
 * never allocates, frees or keeps a pointer after the call returns.  Calls only enqueue work
 * on `stream` (asynchronous, reentrant); results are valid once the stream reaches them.
 * No CPU fallback exists: without an sm_100 device a call returns ATTN_ERR_UNSUPPORTED.
 *
 * Errors: a call that returns non-zero has launched nothing (except ATTN_ERR_CUDA, returned
 * when a launch itself failed).  Device-side waits are bounded; if one expires the kernel
 * stops early, records the event in a device flag and `attn_get_device_error` reports
 * ATTN_ERR_DEVICE_TIMEOUT after the stream has been synchronised (the same flag reports an
 * out-of-range page number met by attn_decode_paged).
 */
#ifndef EXACT_ATTN_B200_ATTN_H
#define EXACT_ATTN_B200_ATTN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ATTN_API __attribute__((visibility("default")))
#else
#define ATTN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t (NULL = the legacy default stream). */
typedef struct CUstream_st *attn_stream_t;

enum attn_mask_kind {
  ATTN_MASK_FULL = 0,
  ATTN_MASK_CAUSAL = 1,
  ATTN_MASK_SLIDING = 2,
  ATTN_MASK_LOCAL_GLOBAL = 3
};

enum attn_status {
  ATTN_OK = 0,
  ATTN_ERR_INVALID_ARG = -1,    /* null pointer, negative size, Hq % Hkv != 0, bad mask, ... */
  ATTN_ERR_UNSUPPORTED = -2,    /* head dim, group size, alignment or device not supported */
  ATTN_ERR_CUDA = -3,           /* a CUDA runtime call or launch failed */
  ATTN_ERR_WORKSPACE = -4,      /* decode workspace missing or too small */
  ATTN_ERR_DEVICE_TIMEOUT = -5  /* a bounded device-side wait expired (see attn_get_device_error) */
};

/* Version of this ABI (bumped on any incompatible change). */
ATTN_API int attn_abi_version(void);

/* Human-readable text for a status code (static storage, never NULL). */
ATTN_API const char *attn_status_string(int status);

/* The CUDA runtime's text for the last ATTN_ERR_CUDA returned on the calling thread
 * (static storage, never NULL; "no error" if there was none). */
ATTN_API const char *attn_last_error_detail(void);

/*
 * The prefill calls (attn_fwd, attn_fwd_block_sparse, attn_fwd_varlen, attn_fwd_fp8) and
 * attn_bwd run persistent grids whose CTAs take work from a 4-byte counter in device memory
 * that the library owns: one counter per stream (up to 1024 streams per device; later streams
 * share the counter of an earlier one, and two streams that share one must not run these calls
 * at the same time).  Calls on one stream are ordered and share its counter; a CUDA graph that captured a
 * call keeps the counter of the capturing stream, so two launches of such graphs must not run at
 * the same time.  The counter is back at zero when a call's kernel ends, also when it ended on
 * ATTN_ERR_DEVICE_TIMEOUT.  attn_bwd's dK/dV and dQ kernels use the same counter.  The first
 * such call on a device looks the counters' address up (make it before any stream capture) and
 * keeps it for the life of the process: do not use the library across a device reset.
 */

/*
 * attn_fwd - bf16 prefill / full forward.
 *   q, o   bf16 [B][Hq][Nq][d];  k, v  bf16 [B][Hkv][Nk][d];  lse fp32 [B][Hq][Nq] or NULL.
 *   B >= 0, Nq >= 0, Nk >= 0 (B = 0 or Nq = 0: nothing to do; Nk = 0: O = 0, LSE = -inf),
 *   Hq >= 1, Hkv >= 1, Hq % Hkv == 0, d == 128.
 *   mask_kind in attn_mask_kind; window >= 1 for ATTN_MASK_SLIDING, >= 0 for
 *   ATTN_MASK_LOCAL_GLOBAL (ignored otherwise); n_sink >= 0 (sinks or global tokens, used by
 *   those two masks only); scale finite (1/sqrt(d) in the usual case).
 *   All pointers 16-byte aligned.  Accumulation is fp32; O is rounded to bf16 once.
 */
ATTN_API int attn_fwd(const void *q, const void *k, const void *v, void *o, float *lse, int B, int Hq,
             int Hkv, int Nq, int Nk, int d, int mask_kind, int window, int n_sink, float scale,
             attn_stream_t stream);

/*
 * attn_fwd_block_sparse - attn_fwd under a fixed block-sparse layout ("Quadratic Complexity
 * Bottleneck", sparse attention patterns: the sequence cut into blocks, attention computed
 * within and between selected blocks; the selection is the caller's).
 *   block_mask  DEVICE uint8 [mask_heads][ceil(Nq / 128)][ceil(Nk / 128)]: entry (hm, qt, kt)
 *               != 0 selects query rows [128 qt, 128 qt + 128) against keys [128 kt, 128 kt + 128)
 *               of head h, hm = h when mask_heads == Hq, hm = 0 when mask_heads == 1 (one
 *               layout for every head); shared by the batch.  Read only, not kept.
 *   A key is visible to a query row iff its block is selected and the mask (mask_kind, window,
 *   n_sink) admits it; a row with no visible key gets O = 0 and LSE = -inf.
 *   mask_heads == 1 or Hq (else ATTN_ERR_INVALID_ARG); block_mask may be NULL only when there
 *   is nothing to compute; ceil(Nk / 128) <= 4096 (else ATTN_ERR_UNSUPPORTED).
 *   Other arguments, layouts and rules as attn_fwd.
 */
ATTN_API int attn_fwd_block_sparse(const void *q, const void *k, const void *v, void *o,
                                   float *lse, const uint8_t *block_mask, int mask_heads, int B,
                                   int Hq, int Hkv, int Nq, int Nk, int d, int mask_kind,
                                   int window, int n_sink, float scale, attn_stream_t stream);

/*
 * attn_fwd_varlen - attn_fwd on packed variable-length sequences ("What Lost, and Why", the note
 * on sequence packing: several sequences concatenated in one batch row, attention masked block
 * diagonally so that it resets at every boundary given by cu_seqlens).
 *   q, o  bf16 [total_q][Hq][d];  k, v  bf16 [total_k][Hkv][d];  lse fp32 [total_q][Hq] or NULL
 *   (token-major packing).  cu_seqlens_q / cu_seqlens_k: DEVICE int32 arrays of num_seqs + 1
 *   non-decreasing offsets; sequence s owns query rows [cu_seqlens_q[s], cu_seqlens_q[s+1]) and
 *   key rows [cu_seqlens_k[s], cu_seqlens_k[s+1]), and is masked on its own exactly as attn_fwd
 *   masks one (b, h) slice (p_i = i + Nk_s - Nq_s).  max_seqlen_q >= every Nq_s (host value; rows
 *   past it are not computed).  Rows outside every sequence are not written.
 *   Other arguments and rules as attn_fwd (d == 128, GQA by Hq / Hkv, the same masks).
 */
ATTN_API int attn_fwd_varlen(const void *q, const void *k, const void *v, void *o, float *lse,
                             const int *cu_seqlens_q, const int *cu_seqlens_k, int num_seqs,
                             int Hq, int Hkv, int total_q, int total_k, int max_seqlen_q, int d,
                             int mask_kind, int window, int n_sink, float scale,
                             attn_stream_t stream);

/*
 * attn_fwd_fp8 - attn_fwd on E4M3 (8-bit floating point) Q, K, V ("Attention Research",
 * section 2: FlashAttention-3's FP8 path, and FP8/FP4 attention numerics as remaining work).
 *   q bytes [B][Hq][Nq][d], k, v bytes [B][Hkv][Nk][d]: E4M3 codes (1 sign, 4 exponent bits
 *   with bias 7, 3 mantissa bits, largest finite 448); element (b, h, i, t) of Q stands for
 *   descale_q[b*Hq + h] * E4M3(q[b][h][i][t]), likewise K and V with descale_k, descale_v
 *   [B][Hkv] (device fp32 arrays, every factor > 0).  o bf16 [B][Hq][Nq][d], lse fp32 or NULL.
 *   Both products run on the tensor cores as E4M3 x E4M3 with fp32 accumulation; the weights P
 *   (times 128) are rounded to E4M3 for the P V product, the row sums stay fp32.  Masks,
 *   scale and the other rules as attn_fwd (dense layout only).
 */
ATTN_API int attn_fwd_fp8(const void *q, const void *k, const void *v, void *o, float *lse,
                          const float *descale_q, const float *descale_k, const float *descale_v,
                          int B, int Hq, int Hkv, int Nq, int Nk, int d, int mask_kind, int window,
                          int n_sink, float scale, attn_stream_t stream);

/*
 * attn_fwd_f32 - the same operation on fp32 Q, K, V, O (fp32 arithmetic throughout).
 *   d in {64, 128}; all other arguments and rules as attn_fwd.
 */
ATTN_API int attn_fwd_f32(const float *q, const float *k, const float *v, float *o, float *lse, int B,
                 int Hq, int Hkv, int Nq, int Nk, int d, int mask_kind, int window, int n_sink,
                 float scale, attn_stream_t stream);

/*
 * attn_bwd - backward pass of attn_fwd: dQ, dK, dV for a given dO, recomputing the attention
 * weights from the forward's LSE instead of storing them ("Quadratic Complexity Bottleneck",
 * FlashAttention section: the backward pass recomputes attention; "Chapter 3.1 - The Cost of
 * Attention", section 5).  With P_ij = exp(scale q_i.k_j - LSE_i) on visible pairs:
 *   dV_j = sum_i P_ij dO_i,  dS_ij = P_ij (dO_i.v_j - dO_i.O_i),
 *   dK_j = scale sum_i dS_ij q_i,  dQ_i = scale sum_j dS_ij k_j  (GQA: dK, dV sum over the group).
 *   q, o, dout, dq  bf16 [B][Hq][Nq][d];  k, v, dk, dv  bf16 [B][Hkv][Nk][d];
 *   lse  fp32 [B][Hq][Nq], the forward's LSE for the same inputs, mask and scale (required).
 *   d == 128; mask, window, n_sink, scale as attn_fwd.  dq, dk, dv are fully written (rows and
 *   keys that see nothing get zeros).
 *   workspace: device scratch of at least attn_bwd_workspace_bytes(B, Hq, Nq, Nk, mask_kind,
 *   window, n_sink) bytes, 16-byte aligned, overwritten before it is read.  Besides two fp32
 *   values per query row it holds dS, the weight gradient, as bf16 for every 128 x 128 (query
 *   tile, key block) pair that has a visible entry: the dK/dV kernel writes it, the dQ kernel
 *   reads it (about 2 bytes per visible pair and query head, e.g. 285 MB for B=4, H=16,
 *   causal n=2048).
 * Errors: as attn_fwd; ATTN_ERR_WORKSPACE for a missing or short workspace.  Three kernels are
 * queued on `stream`; the result does not depend on their scheduling (no atomics).
 */
ATTN_API size_t attn_bwd_workspace_bytes(int B, int Hq, int Nq, int Nk, int mask_kind, int window,
                                         int n_sink);

ATTN_API int attn_bwd(const void *q, const void *k, const void *v, const void *o, const float *lse,
                      const void *dout, void *dq, void *dk, void *dv, int B, int Hq, int Hkv,
                      int Nq, int Nk, int d, int mask_kind, int window, int n_sink, float scale,
                      void *workspace, size_t workspace_bytes, attn_stream_t stream);

/*
 * Decode: one new query token per sequence against a contiguous KV cache, split-K over the
 * keys with a log-sum-exp combine ("Attention Research", section 2: split-K over keys for
 * decode; "Quadratic Complexity Bottleneck", KV cache).  Every cached key is visible.
 *   q, o   bf16 [B][Hq][1][d];  k, v  bf16 [B][Hkv][Nk][d];  lse fp32 [B][Hq] or NULL.
 *   d == 128; G = Hq / Hkv in {1, 2, 4, 8}; num_splits = 0 picks a split count for the device.
 *   workspace: caller-owned device scratch of at least attn_decode_workspace_bytes(...) bytes
 *   (same B, Hq, Hkv, Nk, d, num_splits), 16-byte aligned; every call overwrites the part it
 *   uses before reading it, so it needs no clearing.  attn_decode_workspace_bytes returns 0 for
 *   arguments attn_decode would reject.
 */
ATTN_API size_t attn_decode_workspace_bytes(int B, int Hq, int Hkv, int Nk, int d, int num_splits);

ATTN_API int attn_decode(const void *q, const void *k, const void *v, void *o, float *lse, int B, int Hq,
                int Hkv, int Nk, int d, float scale, int num_splits, void *workspace,
                size_t workspace_bytes, attn_stream_t stream);

/*
 * attn_decode_paged - decode against a paged KV cache ("Attention Research", section 2: FlashInfer
 * lists paged KV among its kernel variants, after the reading list's PagedAttention entry).  The
 * cache is a pool of fixed-size pages shared by all sequences; a per-sequence block table says
 * which page holds each run of page_size consecutive keys.  Same split-K decode and combine as
 * attn_decode; every key of a sequence is visible.
 *   q, o        bf16 [B][Hq][1][d] (device);  lse fp32 [B][Hq] or NULL.
 *   k_cache, v_cache  bf16 [num_pages][page_size][Hkv][d] (device): key j of sequence b lives at
 *               page block_table[b][j / page_size], row j % page_size.
 *   block_table int32 [B][max_pages_per_seq] (device); entries past a sequence's last page are
 *               never read.
 *   seq_lens    int32 [B] (device): keys of each sequence, clamped on the device to
 *               [0, max_seq_len]; a sequence of length 0 gets O = 0, LSE = -inf.
 *   max_seq_len an upper bound of seq_lens (host); it sets the split count and the workspace size
 *               and must not exceed max_pages_per_seq * page_size.
 *   page_size   a power of two, 8 <= page_size <= 2^20.
 *   workspace   as attn_decode, sized by attn_decode_workspace_bytes(B, Hq, Hkv, max_seq_len, d,
 *               num_splits).
 * Errors: as attn_decode for shapes, alignment and workspace; ATTN_ERR_INVALID_ARG for a bad
 * page_size or max_seq_len.  A block-table entry that a sequence uses and that lies outside
 * [0, num_pages) is not followed: those keys read as zero vectors and the device flag records
 * ATTN_ERR_INVALID_ARG (see attn_get_device_error).
 */
ATTN_API int attn_decode_paged(const void *q, const void *k_cache, const void *v_cache, void *o,
                               float *lse, const int *block_table, const int *seq_lens, int B,
                               int Hq, int Hkv, int num_pages, int page_size, int max_pages_per_seq,
                               int max_seq_len, int d, float scale, int num_splits,
                               void *workspace, size_t workspace_bytes, attn_stream_t stream);

/*
 * attn_decode_noalloc - attn_decode for callers that cannot allocate device memory.
 *
 * Some callers must not call cudaMalloc themselves: code that runs where an allocation (which
 * can synchronise the whole device) would stall other work, code whose device memory is all
 * owned and budgeted up front by a host framework or pool allocator, or a plugin that is handed
 * tensors but no allocator.  This variant takes the same arguments as attn_decode minus the
 * workspace: the split partials go to a fixed array of ATTN_DECODE_NOALLOC_MAX_BYTES bytes
 * that the library defines in device memory (every GPU that loads the library holds it until
 * the process exits).  The library calls no allocation routine here.
 *
 * Limits and rules:
 *  - a call whose partials would need more than ATTN_DECODE_NOALLOC_MAX_BYTES (see
 *    attn_decode_workspace_bytes) returns ATTN_ERR_WORKSPACE and launches nothing; a smaller
 *    num_splits lowers the need;
 *  - the first call on each device looks up the array's device address (and may make CUDA load
 *    the library's device code on that device); make that first call before any stream capture;
 *  - that address is kept for the life of the process: do not use the library across a device
 *    reset (cudaDeviceReset, or a primary context torn down and made again), after which the
 *    kept address would no longer name the array;
 *  - all calls on a device share the one array, which keeps the last call's contents; every call
 *    writes the part it reads, so nothing needs clearing, but two calls that overlap on the GPU
 *    (different streams, or different host threads, without ordering between them) race on it.
 * The pages describe no counterpart of this entry point; it exists for callers only.
 */
#define ATTN_DECODE_NOALLOC_MAX_BYTES (64u << 20)

ATTN_API int attn_decode_noalloc(const void *q, const void *k, const void *v, void *o, float *lse,
                                 int B, int Hq, int Hkv, int Nk, int d, float scale,
                                 int num_splits, attn_stream_t stream);

/* The split count attn_decode uses for num_splits = 0 on the current device. */
ATTN_API int attn_decode_num_splits(int B, int Hq, int Hkv, int Nk, int d);

/*
 * Reads and clears the device error flag of the current device after synchronising `stream`.
 * Returns ATTN_OK, ATTN_ERR_DEVICE_TIMEOUT (a bounded wait expired), ATTN_ERR_INVALID_ARG (a
 * paged decode met a page number outside its cache), or ATTN_ERR_CUDA if the synchronisation
 * failed.
 */
ATTN_API int attn_get_device_error(attn_stream_t stream);

/*
 * Test hook: wait on an mbarrier that nothing will complete, with a wait limit of
 * `limit_cycles` SM clocks, to exercise the bounded-wait path.  The kernel returns normally
 * and records ATTN_ERR_DEVICE_TIMEOUT in the device flag.
 */
ATTN_API int attn_debug_timeout_probe(long long limit_cycles, attn_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* EXACT_ATTN_B200_ATTN_H */
