"""Pins of the block-sparse oracle (oracle_attn_block_sparse) to things other than itself.

A fixed block-sparse layout selects, per query head (or for all heads), which (block of query
rows, block of keys) pairs are attended ("Quadratic Complexity Bottleneck", sparse attention
patterns: attention within and between selected blocks); a key is visible when its block is
selected and the base mask admits it.  Pins:
- every block selected: the dense oracle (pinned on its own in test_oracle_pins.py), every base
  mask, GQA, Nq != Nk both ways;
- block-diagonal and one-block-per-row layouts over a full base mask: the dense oracle run on
  the selected slices of Q, K, V as separate problems;
- an unselected row of blocks: O = 0 and LSE = -inf; Q = 0: the mean of V over the visible set
  and LSE = ln #visible, with the set enumerated here from the definition;
- per-head layouts: each head equals the shared-layout oracle given that head's layout;
- 50-digit Decimal brute force on tiny inputs with non-square blocks (block_q != block_k);
- planted slips in copies of the C source (key blocks one key too wide, row block taken from
  the key position, the base mask dropped, the layout's head taken as the kv head), each of
  which one of the pins above catches.
"""

import ctypes
import math
import os
import shutil
import subprocess
import tempfile

import numpy as np
import pytest

from oracle import oracle as O

from .test_oracle_pins import _decimal_attention, rnd, visible_set

FULL, CAUSAL, SLIDING, LOCAL = O.MASK_FULL, O.MASK_CAUSAL, O.MASK_SLIDING, O.MASK_LOCAL_GLOBAL


def layout(seed, heads, nqb, nkb, density=0.5):
    r = np.random.default_rng(seed)
    return (r.random((heads, nqb, nkb)) < density).astype(np.uint8)


def nblocks(n, b):
    return -(-n // b)


def all_selected_check():
    cases = [(FULL, 0, 0, 9, 11), (CAUSAL, 0, 0, 10, 10), (CAUSAL, 0, 0, 6, 13), (CAUSAL, 0, 0, 13, 6),
             (SLIDING, 3, 2, 12, 12), (LOCAL, 2, 1, 11, 9)]
    for mask, w, s, Nq, Nk in cases:
        q, k, v = rnd(71, 0, (2, 4, Nq, 3)), rnd(71, 1, (2, 2, Nk, 3)), rnd(71, 2, (2, 2, Nk, 3))
        bm = np.ones((1, nblocks(Nq, 4), nblocks(Nk, 3)), np.uint8)
        o, lse = O.attention_block_sparse(q, k, v, bm, mask, w, s, 0.7, block_q=4, block_k=3)
        ro, rl = O.attention(q, k, v, mask, w, s, 0.7)
        np.testing.assert_allclose(o, ro, rtol=0, atol=1e-15)
        np.testing.assert_array_equal(lse, rl)


def test_all_blocks_selected_is_the_dense_oracle():
    all_selected_check()


def sliced_check():
    # block-diagonal over a full base mask: row block r sees key block r only
    bq = bk = 4
    N, d = 14, 3
    q, k, v = rnd(72, 0, (1, 2, N, d)), rnd(72, 1, (1, 1, N, d)), rnd(72, 2, (1, 1, N, d))
    nb = nblocks(N, 4)
    bm = np.eye(nb, dtype=np.uint8)[None]
    o, lse = O.attention_block_sparse(q, k, v, bm, FULL, scale=0.8, block_q=bq, block_k=bk)
    for r in range(nb):
        a, b = r * bq, min(N, (r + 1) * bq)
        ro, rl = O.attention(q[:, :, a:b], k[:, :, a:b], v[:, :, a:b], FULL, scale=0.8)
        np.testing.assert_allclose(o[:, :, a:b], ro, rtol=0, atol=1e-15)
        np.testing.assert_allclose(lse[:, :, a:b], rl, rtol=0, atol=1e-15)
    # one key block per row block, not on the diagonal, non-square blocks, Nq != Nk
    Nq, Nk, bq, bk = 10, 17, 3, 5
    q, k, v = rnd(73, 0, (1, 1, Nq, d)), rnd(73, 1, (1, 1, Nk, d)), rnd(73, 2, (1, 1, Nk, d))
    nqb, nkb = nblocks(Nq, bq), nblocks(Nk, bk)
    pick = [(3 * r + 1) % nkb for r in range(nqb)]
    bm = np.zeros((1, nqb, nkb), np.uint8)
    for r, c in enumerate(pick):
        bm[0, r, c] = 1
    o, lse = O.attention_block_sparse(q, k, v, bm, FULL, scale=0.6, block_q=bq, block_k=bk)
    for r, c in enumerate(pick):
        a, b = r * bq, min(Nq, (r + 1) * bq)
        ka, kb = c * bk, min(Nk, (c + 1) * bk)
        ro, rl = O.attention(q[:, :, a:b], k[:, :, ka:kb], v[:, :, ka:kb], FULL, scale=0.6)
        np.testing.assert_allclose(o[:, :, a:b], ro, rtol=0, atol=1e-15)
        np.testing.assert_allclose(lse[:, :, a:b], rl, rtol=0, atol=1e-15)


def test_selected_slices_are_separate_problems():
    sliced_check()


def mean_check():
    # Q = 0: O_i = mean of V over the visible set, LSE_i = ln #visible (-inf, O = 0 if empty)
    for mask, w, s, Nq, Nk, bq, bk in ((CAUSAL, 0, 0, 11, 11, 3, 2), (SLIDING, 4, 2, 9, 13, 2, 3),
                                       (LOCAL, 2, 1, 12, 8, 4, 3), (FULL, 0, 0, 7, 10, 2, 4)):
        Hq, Hkv, d = 4, 2, 3
        q = np.zeros((1, Hq, Nq, d))
        k, v = rnd(74, 1, (1, Hkv, Nk, d)), rnd(74, 2, (1, Hkv, Nk, d))
        bm = layout(74 + Nq, Hq, nblocks(Nq, bq), nblocks(Nk, bk))
        bm[1, 0, :] = 0  # an unselected row of blocks
        o, lse = O.attention_block_sparse(q, k, v, bm, mask, w, s, 1.3, block_q=bq, block_k=bk)
        for h in range(Hq):
            for i in range(Nq):
                vis = [j for j in visible_set(i + Nk - Nq, Nk, mask, w, s) if bm[h, i // bq, j // bk]]
                if not vis:
                    assert np.all(o[0, h, i] == 0) and lse[0, h, i] == -np.inf
                    continue
                np.testing.assert_allclose(o[0, h, i], v[0, h // 2, vis].mean(axis=0), rtol=0, atol=1e-14)
                assert abs(lse[0, h, i] - math.log(len(vis))) < 1e-14


def test_zero_query_mean_over_the_selected_keys():
    mean_check()


def per_head_check():
    Nq, Nk, d, Hq, Hkv, bq, bk = 9, 12, 3, 4, 2, 4, 3
    q, k, v = rnd(75, 0, (2, Hq, Nq, d)), rnd(75, 1, (2, Hkv, Nk, d)), rnd(75, 2, (2, Hkv, Nk, d))
    bm = layout(75, Hq, nblocks(Nq, bq), nblocks(Nk, bk), 0.6)
    o, lse = O.attention_block_sparse(q, k, v, bm, CAUSAL, scale=0.5, block_q=bq, block_k=bk)
    for h in range(Hq):
        g = h // (Hq // Hkv)
        ro, rl = O.attention_block_sparse(q[:, h:h + 1], k[:, g:g + 1], v[:, g:g + 1], bm[h:h + 1],
                                          CAUSAL, scale=0.5, block_q=bq, block_k=bk)
        np.testing.assert_array_equal(o[:, h:h + 1], ro)
        np.testing.assert_array_equal(lse[:, h:h + 1], rl)


def test_per_head_layouts():
    per_head_check()


DECIMAL_CASES = [
    # Nq, Nk, d, mask, w, s, block_q, block_k
    (6, 7, 3, FULL, 0, 0, 2, 3),
    (7, 7, 2, CAUSAL, 0, 0, 3, 2),
    (5, 8, 3, CAUSAL, 0, 0, 2, 3),
    (8, 5, 2, SLIDING, 2, 1, 3, 2),
    (7, 6, 2, LOCAL, 1, 1, 2, 4),
]


def decimal_check(case, seed=76):
    Nq, Nk, d, mask, w, s, bq, bk = case
    q, k, v = rnd(seed, 0, (1, 1, Nq, d)), rnd(seed, 1, (1, 1, Nk, d)), rnd(seed, 2, (1, 1, Nk, d))
    bm = layout(seed + Nq * 10 + Nk, 1, nblocks(Nq, bq), nblocks(Nk, bk), 0.6)
    scale = 1.0 / math.sqrt(d)
    o, lse = O.attention_block_sparse(q, k, v, bm, mask, w, s, scale, block_q=bq, block_k=bk)
    eo, el = _decimal_attention(q[0, 0], k[0, 0], v[0, 0], Nq, Nk, d, mask, w, s, scale,
                                keep=lambda i, j: bm[0, i // bq, j // bk] != 0)
    np.testing.assert_allclose(o[0, 0], eo, rtol=0, atol=1e-14)
    fin = np.isfinite(el)
    np.testing.assert_allclose(lse[0, 0][fin], el[fin], rtol=0, atol=1e-14)
    assert np.all(lse[0, 0][~fin] == -np.inf)


@pytest.mark.parametrize("case", DECIMAL_CASES)
def test_brute_force_decimal(case):
    decimal_check(case)


def test_rejects_bad_layouts():
    q, k, v = rnd(77, 0, (1, 4, 5, 2)), rnd(77, 1, (1, 2, 6, 2)), rnd(77, 2, (1, 2, 6, 2))
    with pytest.raises(ValueError):
        O.attention_block_sparse(q, k, v, np.ones((2, 3, 2)), block_q=2, block_k=3)  # 2 heads of 4
    with pytest.raises(ValueError):
        O.attention_block_sparse(q, k, v, np.ones((1, 3, 3)), block_q=2, block_k=3)  # nkb = 2


# ------------------------------------------------------------------------------------------
# planted slips in copies of the C source
# ------------------------------------------------------------------------------------------
MUTANTS = {
    "key_block_size_off_by_one": ("kblocks[j / block_k]", "kblocks[j / (block_k + 1)]"),
    "row_block_from_position": ("(hm * nqb + i / block_q) * nkb",
                                "(hm * nqb + (i + Nk - Nq > 0 ? i + Nk - Nq : 0) / block_q) * nkb"),
    "base_mask_dropped": ("(unsigned char)(oracle_visible(p, j, mask_kind, window, n_sink) &&",
                          "(unsigned char)((kblocks != NULL || oracle_visible(p, j, mask_kind, window, n_sink)) &&"),
    "layout_head_is_kv_head": ("int64_t hm = mask_heads == 1 ? 0 : h;", "int64_t hm = mask_heads == 1 ? 0 : hk;"),
}


def _checks():
    yield "all_selected", all_selected_check
    yield "sliced", sliced_check
    yield "mean", mean_check
    yield "per_head", per_head_check
    for c in DECIMAL_CASES:
        yield "decimal %s" % (c,), lambda c=c: decimal_check(c)


@pytest.fixture(scope="module")
def tmpdir():
    d = tempfile.mkdtemp(prefix="oracle_block_mutants_")
    yield d
    shutil.rmtree(d, ignore_errors=True)


def test_unmutated_block_sparse_passes_every_check():
    for _, fn in _checks():
        fn()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_block_sparse_mutant_is_caught(name, tmpdir, monkeypatch):
    old, new = MUTANTS[name]
    src = open(os.path.join(os.path.dirname(O.__file__), "oracle.c")).read()
    assert src.count(old) == 1, "mutation site missing or ambiguous: " + name
    path_c, path_so = os.path.join(tmpdir, name + ".c"), os.path.join(tmpdir, name + ".so")
    open(path_c, "w").write(src.replace(old, new))
    subprocess.check_call(["gcc", "-O1", "-std=c99", "-fopenmp", "-fPIC", "-shared", "-o", path_so,
                           path_c, "-lm"])
    O._load()
    real = O._lib
    lib = ctypes.CDLL(path_so)
    for fn in ("oracle_attn", "oracle_attn_rows", "oracle_visible_pairs", "oracle_visible",
               "oracle_attn_bwd", "oracle_attn_block_sparse"):
        getattr(lib, fn).argtypes = getattr(real, fn).argtypes
        getattr(lib, fn).restype = getattr(real, fn).restype
    monkeypatch.setattr(O, "_lib", lib)
    caught = []
    for cname, fn in _checks():
        try:
            fn()
        except AssertionError:
            caught.append(cname)
    assert caught, "mutant %s slipped through every pin" % name
