"""Pins for the fp64 oracle: each test checks it against something other than itself.

Sources of truth used here: closed forms of softmax attention, invariants of the definition
(row-stochastic weights, key-permutation invariance, linearity in V, GQA as repeated heads),
an independent 50-digit Decimal brute force on tiny inputs with the mask enumerated from its set
definition, and the figures the pages print (tests/golden/page_figures.json).  A plausible slip
in the oracle (a dropped scale, a transposed operand, a wrong head index, an off-by-one in a
mask edge, a missing max subtraction) fails at least one of them.
"""

import json
import math
import os
from decimal import Decimal, getcontext

import numpy as np
import pytest

import synth
from exact_io_aware_82_b200 import accounting as acc
from oracle import oracle as O

FULL, CAUSAL, SLIDING, LOCAL = O.MASK_FULL, O.MASK_CAUSAL, O.MASK_SLIDING, O.MASK_LOCAL_GLOBAL
GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_figures.json")


def rnd(seed, tid, shape):
    return synth.normal_f32(seed, tid, shape).astype(np.float64)


def visible_set(p, Nk, mask, w, s):
    """Mask as a set, written from the set definitions (not from the oracle's predicate)."""
    if mask == FULL:
        return set(range(Nk))
    if mask == LOCAL:
        # Longformer: w neighbours on either side; s global tokens (positions 0..s-1) that see
        # every key and are seen by every query
        if 0 <= p < s:
            return set(range(Nk))
        return set(j for j in range(Nk) if abs(p - j) <= w) | set(range(min(s, Nk)))
    past = set(range(0, min(p, Nk - 1) + 1)) if p >= 0 else set()
    if mask == CAUSAL:
        return past
    window = set(range(max(p - w + 1, 0), p + 1))
    sinks = set(range(0, s))
    return (window | sinks) & past


# --------------------------------------------------------------------------------------------
# P1  Q = 0 (or scale = 0): O_i is the mean of V over the visible keys, LSE_i = ln(#visible)
# --------------------------------------------------------------------------------------------
@pytest.mark.parametrize("mask,w,s,Nq,Nk", [
    (FULL, 0, 0, 7, 11), (CAUSAL, 0, 0, 9, 9), (CAUSAL, 0, 0, 5, 12), (CAUSAL, 0, 0, 12, 5),
    (SLIDING, 3, 0, 10, 10), (SLIDING, 4, 2, 13, 13), (SLIDING, 2, 3, 6, 15),
    (LOCAL, 2, 0, 11, 11), (LOCAL, 1, 2, 12, 12), (LOCAL, 3, 1, 6, 14), (LOCAL, 2, 2, 14, 6)])
def test_zero_query_gives_mean_of_visible_values(mask, w, s, Nq, Nk):
    d = 5
    q = np.zeros((1, 2, Nq, d))
    k = rnd(11, 1, (1, 1, Nk, d))
    v = rnd(11, 2, (1, 1, Nk, d))
    o, lse = O.attention(q, k, v, mask, w, s, scale=0.37)
    for h in range(2):
        for i in range(Nq):
            vis = sorted(visible_set(i + Nk - Nq, Nk, mask, w, s))
            if not vis:
                assert np.all(o[0, h, i] == 0) and lse[0, h, i] == -np.inf
                continue
            np.testing.assert_allclose(o[0, h, i], v[0, 0, vis].mean(axis=0), rtol=0, atol=1e-13)
            assert abs(lse[0, h, i] - math.log(len(vis))) < 1e-13


def test_scale_zero_is_uniform():
    q, k, v = rnd(3, 0, (1, 1, 6, 4)), rnd(3, 1, (1, 1, 6, 4)), rnd(3, 2, (1, 1, 6, 4))
    o, lse = O.attention(q, k, v, FULL, scale=0.0)
    np.testing.assert_allclose(o[0, 0], np.broadcast_to(v[0, 0].mean(axis=0), (6, 4)), atol=1e-14)
    np.testing.assert_allclose(lse, math.log(6), atol=1e-14)


# --------------------------------------------------------------------------------------------
# P2  one-hot: a peaked softmax is a hard lookup (Chapter 3.1, section 4)
# --------------------------------------------------------------------------------------------
def test_one_hot_lookup():
    n, d = 256, 64
    k = rnd(2, 1, (1, 1, n, d))
    v = rnd(2, 2, (1, 1, n, d))
    target = (np.arange(n) * 37 + 11) % n
    q = 20.0 * k[:, :, target, :]
    o, _ = O.attention(q, k, v, FULL, scale=1.0 / 8.0)
    np.testing.assert_allclose(o[0, 0], v[0, 0, target], rtol=0, atol=1e-6)


# --------------------------------------------------------------------------------------------
# P3  row-stochastic weights; V = I exposes P itself
# --------------------------------------------------------------------------------------------
@pytest.mark.parametrize("mask,w,s", [(FULL, 0, 0), (CAUSAL, 0, 0), (SLIDING, 3, 2), (LOCAL, 2, 1),
                                      (LOCAL, 0, 0)])
def test_weights_are_row_stochastic_and_masked(mask, w, s):
    n = 12
    q, k = rnd(4, 0, (1, 1, n, n)), rnd(4, 1, (1, 1, n, n))
    v = np.eye(n)[None, None]  # d = Nk = n and V = I: O_i is the weight row P_i
    P, _ = O.attention(q, k, v, mask, w, s, scale=0.9)
    P = P[0, 0]
    assert np.all(P >= 0)
    np.testing.assert_allclose(P.sum(axis=1), 1.0, atol=1e-12)
    for i in range(n):
        vis = visible_set(i, n, mask, w, s)
        for j in range(n):
            if j not in vis:
                assert P[i, j] == 0.0
            else:
                assert P[i, j] > 0.0
    o1, _ = O.attention(q, k, np.full((1, 1, n, n), -2.5), mask, w, s, scale=0.9)
    np.testing.assert_allclose(o1, -2.5, atol=1e-12)


# --------------------------------------------------------------------------------------------
# P4  key permutation invariance (full mask)
# --------------------------------------------------------------------------------------------
def test_key_permutation_invariance():
    q, k, v = rnd(5, 0, (2, 3, 17, 8)), rnd(5, 1, (2, 3, 29, 8)), rnd(5, 2, (2, 3, 29, 8))
    perm = np.random.default_rng(0).permutation(29)
    o1, l1 = O.attention(q, k, v, FULL)
    o2, l2 = O.attention(q, k[:, :, perm], v[:, :, perm], FULL)
    np.testing.assert_allclose(o1, o2, atol=1e-12)
    np.testing.assert_allclose(l1, l2, atol=1e-12)
    # and a non-trivial check that K is used row-wise: swapping only K (not V) changes O
    o3, _ = O.attention(q, k[:, :, perm], v, FULL)
    assert np.max(np.abs(o3 - o1)) > 1e-3


# --------------------------------------------------------------------------------------------
# P5  causal rows 0 and 1 in closed form
# --------------------------------------------------------------------------------------------
def test_causal_first_rows_closed_form():
    d = 16
    scale = 0.25
    q, k, v = rnd(6, 0, (1, 1, 8, d)), rnd(6, 1, (1, 1, 8, d)), rnd(6, 2, (1, 1, 8, d))
    o, lse = O.attention(q, k, v, CAUSAL, scale=scale)
    q0, q1 = q[0, 0, 0], q[0, 0, 1]
    k0, k1 = k[0, 0, 0], k[0, 0, 1]
    v0, v1 = v[0, 0, 0], v[0, 0, 1]
    np.testing.assert_allclose(o[0, 0, 0], v0, atol=1e-15)
    assert abs(lse[0, 0, 0] - scale * float(q0 @ k0)) < 1e-13
    a, b = scale * float(q1 @ k0), scale * float(q1 @ k1)
    w0 = 1.0 / (1.0 + math.exp(b - a))
    np.testing.assert_allclose(o[0, 0, 1], w0 * v0 + (1 - w0) * v1, atol=1e-13)
    assert abs(lse[0, 0, 1] - np.logaddexp(a, b)) < 1e-13


# --------------------------------------------------------------------------------------------
# P6  brute force on tiny inputs: 50-digit Decimal, no max subtraction, mask from set definition
# --------------------------------------------------------------------------------------------
def _decimal_attention(q, k, v, Nq, Nk, d, mask, w, s, scale, keep=None):
    """keep(i, j), if given, further restricts the visible set (block-sparse layouts)."""
    getcontext().prec = 50
    sc = Decimal(repr(scale))
    out, lses = [], []
    for i in range(Nq):
        vis = sorted(j for j in visible_set(i + Nk - Nq, Nk, mask, w, s) if keep is None or keep(i, j))
        if not vis:
            out.append([0.0] * d)
            lses.append(-math.inf)
            continue
        ex = {}
        for j in vis:
            dot = sum(Decimal(repr(float(q[i, t]))) * Decimal(repr(float(k[j, t]))) for t in range(d))
            ex[j] = (sc * dot).exp()
        den = sum(ex.values())
        row = []
        for t in range(d):
            num = sum(ex[j] * Decimal(repr(float(v[j, t]))) for j in vis)
            row.append(float(num / den))
        out.append(row)
        lses.append(float(den.ln()))
    return np.array(out), np.array(lses)


@pytest.mark.parametrize("Nq,Nk,d,mask,w,s", [
    (4, 4, 3, FULL, 0, 0), (5, 5, 4, CAUSAL, 0, 0), (3, 6, 2, CAUSAL, 0, 0), (6, 3, 2, CAUSAL, 0, 0),
    (6, 6, 3, SLIDING, 2, 0), (6, 6, 4, SLIDING, 2, 1), (5, 6, 3, SLIDING, 1, 2),
    (6, 6, 3, SLIDING, 6, 0), (1, 6, 4, FULL, 0, 0), (7, 7, 3, LOCAL, 1, 1), (5, 8, 2, LOCAL, 2, 2),
    (8, 5, 3, LOCAL, 1, 0)])
def test_brute_force_decimal(Nq, Nk, d, mask, w, s):
    q, k, v = rnd(7, 0, (1, 1, Nq, d)), rnd(7, 1, (1, 1, Nk, d)), rnd(7, 2, (1, 1, Nk, d))
    scale = 1.0 / math.sqrt(d)
    o, lse = O.attention(q, k, v, mask, w, s, scale)
    eo, el = _decimal_attention(q[0, 0], k[0, 0], v[0, 0], Nq, Nk, d, mask, w, s, scale)
    np.testing.assert_allclose(o[0, 0], eo, rtol=0, atol=1e-14)
    fin = np.isfinite(el)
    np.testing.assert_allclose(lse[0, 0][fin], el[fin], rtol=0, atol=1e-14)
    assert np.all(lse[0, 0][~fin] == -np.inf)


# --------------------------------------------------------------------------------------------
# P7  online = direct: per-chunk results merged with the online-softmax / LSE recurrence
#     (tiling + online softmax, "FlashAttention and sparse attention", section 1;
#     split-K over keys for decode, "Attention Research", section 2)
# --------------------------------------------------------------------------------------------
@pytest.mark.parametrize("cuts", [[5], [1, 2, 30], [13, 14, 20, 40], list(range(1, 47, 7))])
def test_chunked_merge_equals_direct(cuts):
    q, k, v = rnd(8, 0, (1, 2, 3, 8)), rnd(8, 1, (1, 2, 47, 8)), rnd(8, 2, (1, 2, 47, 8))
    o, lse = O.attention(q, k, v, FULL)
    edges = [0] + cuts + [47]
    parts = [O.attention(q, k[:, :, a:b], v[:, :, a:b], FULL, scale=1 / math.sqrt(8))
             for a, b in zip(edges[:-1], edges[1:]) if b > a]
    L = np.logaddexp.reduce(np.stack([p[1] for p in parts]), axis=0)
    M = sum(np.exp(p[1] - L)[..., None] * p[0] for p in parts)
    np.testing.assert_allclose(M, o, atol=1e-12)
    np.testing.assert_allclose(L, lse, atol=1e-12)


# --------------------------------------------------------------------------------------------
# P8  mask reductions
# --------------------------------------------------------------------------------------------
def test_mask_reductions():
    n, d = 23, 6
    q, k, v = rnd(9, 0, (1, 2, n, d)), rnd(9, 1, (1, 2, n, d)), rnd(9, 2, (1, 2, n, d))
    oc, lc = O.attention(q, k, v, CAUSAL)
    for w in (n, n + 5):
        ow, lw = O.attention(q, k, v, SLIDING, w, 0)
        np.testing.assert_array_equal(ow, oc)
        np.testing.assert_array_equal(lw, lc)
    os_, ls_ = O.attention(q, k, v, SLIDING, 1, n)  # every key is a sink -> causal
    np.testing.assert_array_equal(os_, oc)
    o1, l1 = O.attention(q, k, v, SLIDING, 1, 0)  # window 1 -> the diagonal only
    np.testing.assert_allclose(o1, v, atol=1e-15)
    np.testing.assert_allclose(l1, np.einsum("bhid,bhid->bhi", q, k) / math.sqrt(d), atol=1e-13)
    of, lf = O.attention(q, k, v, FULL)
    np.testing.assert_allclose(of[:, :, -1], oc[:, :, -1], atol=1e-15)
    np.testing.assert_allclose(lf[:, :, -1], lc[:, :, -1], atol=1e-15)
    # local + global: a window covering every key, or every token global, is the full mask;
    # w = 0 without globals is the diagonal; one global token at 0 makes row 0 a full row and
    # column 0 visible to every row
    for w, g in ((n, 0), (n + 3, 2), (0, n), (1, n + 1)):
        ol, ll = O.attention(q, k, v, LOCAL, w, g)
        np.testing.assert_array_equal(ol, of)
        np.testing.assert_array_equal(ll, lf)
    o0, l0 = O.attention(q, k, v, LOCAL, 0, 0)
    np.testing.assert_allclose(o0, v, atol=1e-15)
    np.testing.assert_allclose(l0, np.einsum("bhid,bhid->bhi", q, k) / math.sqrt(d), atol=1e-13)
    og, lg = O.attention(q, k, v, LOCAL, 0, 1)
    np.testing.assert_array_equal(og[:, :, 0], of[:, :, 0])
    np.testing.assert_allclose(lg[:, :, 1:], np.logaddexp(
        np.einsum("bhid,bhd->bhi", q[:, :, 1:], k[:, :, 0]) / math.sqrt(d),
        np.einsum("bhid,bhid->bhi", q[:, :, 1:], k[:, :, 1:]) / math.sqrt(d)), atol=1e-13)


# --------------------------------------------------------------------------------------------
# P9  GQA = MHA over repeat-interleaved K/V; decode = last causal prefill row
# --------------------------------------------------------------------------------------------
@pytest.mark.parametrize("G", [1, 2, 4])
def test_gqa_equals_repeated_heads(G):
    Hkv, n, d = 2, 19, 8
    q = rnd(10, 0, (2, Hkv * G, n, d))
    k, v = rnd(10, 1, (2, Hkv, n, d)), rnd(10, 2, (2, Hkv, n, d))
    og, lg = O.attention(q, k, v, SLIDING, 5, 2)
    om, lm = O.attention(q, np.repeat(k, G, axis=1), np.repeat(v, G, axis=1), SLIDING, 5, 2)
    np.testing.assert_array_equal(og, om)
    np.testing.assert_array_equal(lg, lm)
    if G > 1:  # the grouping is contiguous (h -> h // G), not strided (h -> h % Hkv)
        ob, _ = O.attention(q, np.tile(k, (1, G, 1, 1)), np.tile(v, (1, G, 1, 1)), SLIDING, 5, 2)
        assert np.max(np.abs(ob - og)) > 1e-3


def test_decode_is_last_causal_row():
    n, d = 31, 8
    q, k, v = rnd(12, 0, (2, 4, n, d)), rnd(12, 1, (2, 2, n, d)), rnd(12, 2, (2, 2, n, d))
    oc, lc = O.attention(q, k, v, CAUSAL)
    od, ld = O.attention(q[:, :, -1:], k, v, FULL)
    np.testing.assert_array_equal(od[:, :, 0], oc[:, :, -1])
    odc, _ = O.attention(q[:, :, -1:], k, v, CAUSAL)  # bottom-right alignment: same thing
    np.testing.assert_array_equal(odc, od)


def test_rows_api_matches_full():
    q, k, v = rnd(13, 0, (2, 4, 9, 8)), rnd(13, 1, (2, 2, 9, 8)), rnd(13, 2, (2, 2, 9, 8))
    o, lse = O.attention(q, k, v, SLIDING, 3, 1)
    rows = [0, 5, 17, 40, 71]
    orow, lrow = O.attention_rows(q, k, v, rows, SLIDING, 3, 1)
    np.testing.assert_array_equal(orow, o.reshape(-1, 8)[rows])
    np.testing.assert_array_equal(lrow, lse.reshape(-1)[rows])


# --------------------------------------------------------------------------------------------
# P10  linearity in V
# --------------------------------------------------------------------------------------------
def test_linearity_in_v():
    q, k = rnd(14, 0, (1, 2, 10, 8)), rnd(14, 1, (1, 2, 10, 8))
    v1, v2 = rnd(14, 2, (1, 2, 10, 8)), rnd(15, 2, (1, 2, 10, 8))
    o1, _ = O.attention(q, k, v1, CAUSAL)
    o2, _ = O.attention(q, k, v2, CAUSAL)
    o3, _ = O.attention(q, k, 1.5 * v1 - 0.25 * v2, CAUSAL)
    np.testing.assert_allclose(o3, 1.5 * o1 - 0.25 * o2, atol=1e-13)


# --------------------------------------------------------------------------------------------
# P11  counting: enumeration vs closed forms vs the figures the pages print
# --------------------------------------------------------------------------------------------
@pytest.mark.parametrize("Nq,Nk", [(1, 1), (7, 7), (5, 12), (12, 5), (128, 128), (129, 300)])
@pytest.mark.parametrize("mask,w,s", [(FULL, 0, 0), (CAUSAL, 0, 0), (SLIDING, 1, 0),
                                      (SLIDING, 4, 0), (SLIDING, 4, 3), (SLIDING, 50, 60),
                                      (SLIDING, 400, 4), (LOCAL, 0, 0), (LOCAL, 3, 0), (LOCAL, 3, 2),
                                      (LOCAL, 40, 70), (LOCAL, 200, 5)])
def test_pair_counts_closed_form(Nq, Nk, mask, w, s):
    brute = sum(len(visible_set(i + Nk - Nq, Nk, mask, w, s)) for i in range(Nq))
    assert O.visible_pairs(Nq, Nk, mask, w, s) == brute
    assert acc.visible_pairs(Nq, Nk, mask, w, s) == brute


def test_pair_counts_at_workload_sizes():
    assert acc.visible_pairs(256, 256, FULL) == 65536
    assert acc.visible_pairs(2048, 2048, CAUSAL) == 2098176 == O.visible_pairs(2048, 2048, CAUSAL)
    assert acc.visible_pairs(8192, 8192, CAUSAL) == 33558528
    assert acc.visible_pairs(32768, 32768, SLIDING, 4096, 4) == 125945850
    assert O.visible_pairs(32768, 32768, SLIDING, 4096, 4) == 125945850
    assert acc.visible_pairs(1, 32768, FULL) == 32768
    # FLOP totals of the benchmark workloads (4*d per visible pair)
    assert acc.attn_flops(4, 16, 2048, 2048, 128, CAUSAL) == 68753031168
    assert acc.attn_flops(2, 32, 8192, 8192, 128, CAUSAL) == 1099645845504
    assert acc.decode_bytes(64, 32, 8, 32768, 128) == 8589934592 + 2 * 128 * 2 * 64 * 32 + 4 * 64 * 32
    # local + global workload: the row-wise count against the oracle's enumeration
    assert acc.visible_pairs(32768, 32768, LOCAL, 2048, 4) == 130299884
    assert O.visible_pairs(32768, 32768, LOCAL, 2048, 4) == 130299884
    # backward: five products of 2*d per visible pair, 2.5x the forward
    assert acc.attn_bwd_flops(4, 16, 2048, 2048, 128, CAUSAL) == 171882577920
    assert 2 * acc.attn_bwd_flops(4, 16, 2048, 2048, 128, CAUSAL) == 5 * acc.attn_flops(
        4, 16, 2048, 2048, 128, CAUSAL)
    # paged: plus one int32 block-table entry per 16-key page and one int32 length per sequence
    assert acc.decode_paged_bytes(64, 32, 8, 32768, 128, 16) == \
        acc.decode_bytes(64, 32, 8, 32768, 128) + 4 * 64 * 2048 + 4 * 64


def test_page_figures():
    g = json.load(open(GOLDEN))
    n = g["score_entries_n1000"]["n"]
    assert O.visible_pairs(n, n, FULL) == g["score_entries_n1000"]["value"]
    assert O.visible_pairs(2 * 300, 2 * 300, FULL) == g["double_context_factor"]["value"] * O.visible_pairs(300, 300, FULL)
    f = g["ctx_2k_to_128k_factor"]
    assert acc.visible_pairs(f["n_large"], f["n_large"], FULL) == f["value"] * acc.visible_pairs(f["n_small"], f["n_small"], FULL)
    f = g["ctx_1k_to_32k_factor"]
    assert acc.visible_pairs(f["n_large"], f["n_large"], FULL) == f["value"] * acc.visible_pairs(f["n_small"], f["n_small"], FULL)
    f = g["full_vs_window_ratio"]
    # a steady-state row (p >= w - 1) of the window mask sees exactly w keys; a full row sees n
    n, w = f["n"], f["w"]
    per_row = acc.visible_pairs(1, n, SLIDING, w, 0)
    assert per_row == w
    assert round(acc.visible_pairs(1, n, FULL) / per_row) == f["value"]
    f = g["score_matrix_bytes_64k_fp32"]
    nbytes = acc.visible_pairs(f["n"], f["n"], FULL) * f["bytes_per_entry"]
    assert round(nbytes / 2**30) == f["value_gb_approx"]
