"""Work accounting for the attention workloads: visible (query, key) pairs, FLOPs and bytes.

Closed forms only (no enumeration), so the benchmark can count work at any size.  The test
suite pins every closed form against brute-force enumeration of the mask definition.

Mask definitions (the same reading the library implements):
  FULL     every key is visible;
  CAUSAL   key j is visible to query row i iff j <= p_i, with p_i = i + Nk - Nq
           (bottom-right alignment when Nq != Nk);
  SLIDING  causal, and either p_i - w < j (a left window of w keys including the diagonal,
           "each token attends to w neighbouring tokens" in "Quadratic Complexity Bottleneck",
           sparse-attention section) or j < n_sink (always-visible sink tokens, "Attention
           Research", section 4).

FLOPs count 4*d per visible pair (2*d for Q K^T, 2*d for P V), the standard count for the
forward pass of "Chapter 3.1 - The Cost of Attention", section 2; masked pairs and tile padding
are not credited.
"""

from __future__ import annotations

MASK_FULL, MASK_CAUSAL, MASK_SLIDING, MASK_LOCAL_GLOBAL = 0, 1, 2, 3


def _sum_min_w(lo: int, hi: int, w: int) -> int:
    """sum_{x=lo}^{hi} min(w, x) for integers 0 <= lo, with hi < lo meaning an empty sum."""
    if hi < lo:
        return 0
    total = 0
    a, b = lo, min(hi, w)
    if a <= b:
        total += (a + b) * (b - a + 1) // 2
    a = max(lo, w + 1)
    if a <= hi:
        total += w * (hi - a + 1)
    return total


def visible_pairs(Nq: int, Nk: int, mask_kind: int, window: int = 0, n_sink: int = 0) -> int:
    """Visible (query, key) pairs of one (b, h) slice."""
    if Nq <= 0 or Nk <= 0:
        return 0
    off = Nk - Nq
    if mask_kind == MASK_FULL:
        return Nq * Nk
    # causal row i sees keys 0..p_i (p_i = i + off) clipped to [0, Nk): count c_i = clip(p_i + 1)
    p_lo, p_hi = off, Nq - 1 + off  # p ranges over [p_lo, p_hi]; p_hi = Nk - 1
    lo = max(p_lo, -1)
    if mask_kind == MASK_CAUSAL:
        # sum over p of max(0, p + 1), p <= Nk - 1 always
        a = max(lo, 0)
        if a > p_hi:
            return 0
        return (a + 1 + p_hi + 1) * (p_hi - a + 1) // 2
    if mask_kind == MASK_LOCAL_GLOBAL:
        return _local_global_pairs(Nq, Nk, window, n_sink)
    if mask_kind != MASK_SLIDING:
        raise ValueError("mask_kind")
    w, s = window, n_sink
    a = max(lo, 0)
    if a > p_hi:
        return 0
    # window part: min(w, p + 1) keys for each p in [a, p_hi]
    total = _sum_min_w(a + 1, p_hi + 1, w)
    # sinks outside the window: keys j < s with j <= p - w  ->  max(0, min(s, p - w + 1))
    total += _sum_min_w(max(a - w + 1, 0), p_hi - w + 1, s) if s > 0 else 0
    return total


def attn_flops(B: int, Hq: int, Nq: int, Nk: int, d: int, mask_kind: int, window: int = 0,
               n_sink: int = 0) -> int:
    """Unmasked forward FLOPs: 4*d per visible pair, over every (b, query head)."""
    return 4 * d * B * Hq * visible_pairs(Nq, Nk, mask_kind, window, n_sink)


def attn_fwd_bytes(B: int, Hq: int, Hkv: int, Nq: int, Nk: int, d: int, elem: int = 2) -> int:
    """Unique HBM bytes of one forward call: Q, K, V read once, O written once, fp32 LSE."""
    return elem * d * (2 * B * Hq * Nq + 2 * B * Hkv * Nk) + 4 * B * Hq * Nq


def decode_bytes(B: int, Hq: int, Hkv: int, Nk: int, d: int, elem: int = 2) -> int:
    """Algorithmic bytes of one decode call: the K and V cache once (shared by the G query heads
    of a group), Q read, O written, fp32 LSE written."""
    return elem * d * 2 * B * Hkv * Nk + elem * d * 2 * B * Hq + 4 * B * Hq


def decode_paged_bytes(B: int, Hq: int, Hkv: int, Nk: int, d: int, page_size: int,
                       elem: int = 2) -> int:
    """Algorithmic bytes of one paged decode call with every sequence Nk keys long: the decode
    bytes plus the block-table entries it follows (int32, one per page of each sequence) and
    the int32 sequence lengths."""
    pages = (Nk + page_size - 1) // page_size
    return decode_bytes(B, Hq, Hkv, Nk, d, elem) + 4 * B * pages + 4 * B


def attn_bwd_flops(B: int, Hq: int, Nq: int, Nk: int, d: int, mask_kind: int, window: int = 0,
                   n_sink: int = 0) -> int:
    """Algorithmic FLOPs of the backward pass: five d-long products per visible pair (recomputed
    score, dP, and the dV, dK, dQ contributions), 2 * d each, i.e. 10 * d = 2.5 x the forward.
    The extra score and dP recomputation of a split dQ kernel is not credited."""
    return 10 * d * B * Hq * visible_pairs(Nq, Nk, mask_kind, window, n_sink)


def _local_global_pairs(Nq: int, Nk: int, w: int, g: int) -> int:
    """Bidirectional window of w keys on each side plus g global tokens, counted row by row:
    a global row (0 <= p < g) sees all Nk keys; another row sees the window [p - w, p + w]
    clipped to the keys, plus the global keys outside it."""
    import numpy as np

    p = np.arange(Nq, dtype=np.int64) + (Nk - Nq)
    G = min(g, Nk)
    lo = np.maximum(p - w, 0)
    hi = np.minimum(p + w, Nk - 1)
    win = np.maximum(hi - lo + 1, 0)
    inter = np.where(hi >= lo, np.maximum(np.minimum(hi, G - 1) - lo + 1, 0), 0)
    rows = win + (G - inter)
    rows = np.where((p >= 0) & (p < g), Nk, rows)
    return int(rows.sum())


def _visible_in(p, c0: int, c1: int, mask_kind: int, w: int, s: int, Nk: int):
    """Visible keys in [c0, c1] (inclusive, c1 < Nk) for each query position in the array p."""
    import numpy as np

    def span(lo, hi):  # size of [max(lo, c0), min(hi, c1)] for array bounds lo, hi
        return np.maximum(0, np.minimum(hi, c1) - np.maximum(lo, c0) + 1)

    p = np.asarray(p, dtype=np.int64)
    if mask_kind == MASK_FULL:
        return np.full(p.shape, c1 - c0 + 1, dtype=np.int64)
    if mask_kind == MASK_CAUSAL:
        return span(np.zeros_like(p), p)
    if mask_kind == MASK_SLIDING:
        win = span(p - w + 1, p)  # window keys, causal by construction
        sinks = span(np.zeros_like(p), np.minimum(p, s - 1))  # sinks, causal
        both = span(np.maximum(p - w + 1, 0), np.minimum(p, s - 1))  # sinks inside the window
        return win + sinks - both
    if mask_kind == MASK_LOCAL_GLOBAL:
        g = min(s, Nk)
        glob_row = (p >= 0) & (p < s)
        win = span(p - w, p + w)
        gk = span(np.zeros_like(p), np.full(p.shape, g - 1))
        both = span(np.maximum(p - w, 0), np.minimum(p + w, g - 1))
        return np.where(glob_row, c1 - c0 + 1, win + gk - both)
    raise ValueError("mask_kind")


def block_sparse_pairs(block_mask, Nq: int, Nk: int, mask_kind: int, window: int = 0,
                       n_sink: int = 0, Hq: int = 1, block: int = 128) -> int:
    """Visible pairs of one batch row under a block-sparse layout, summed over the Hq query
    heads: a pair counts when its block is selected (block_mask [1 or Hq][qtiles][ktiles]; a
    single layout serves every head) and the base mask admits it."""
    import numpy as np

    bm = np.asarray(block_mask) != 0
    off = Nk - Nq
    total = 0
    for hm in range(bm.shape[0]):
        heads = Hq if bm.shape[0] == 1 else 1
        for qt, kt in zip(*np.nonzero(bm[hm])):
            r0, r1 = qt * block, min(Nq, (qt + 1) * block)
            c0, c1 = kt * block, min(Nk, (kt + 1) * block) - 1
            if r0 >= r1 or c0 > c1:
                continue
            p = np.arange(r0, r1, dtype=np.int64) + off
            total += heads * int(_visible_in(p, c0, c1, mask_kind, window, n_sink, Nk).sum())
    return total

