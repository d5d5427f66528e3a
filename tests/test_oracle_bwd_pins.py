"""Pins of the backward oracle (oracle_attn_bwd) to things other than itself.

- Central finite differences of the scalar L = sum(dO * O), with O from the forward oracle
  (pinned on its own in test_oracle_pins.py), at tiny sizes: every mask, GQA, Nq != Nk in both
  directions, rows with no visible key, scales other than 1/sqrt(d) including a negative one.
- scale = 0 in closed form: the weights are uniform over the visible set (enumerated from the
  set definition), so dV_j = sum over the rows that see j of dO_i / |visible(i)| and dQ = dK = 0.
- Invariants: every row of dS sums to zero, so sum_j dK_j = 0 for each (b, kv head); the rows
  of P sum to one, so sum_j dV_j = sum of dO over the rows that see any key (all G heads).
- Planted slips in copies of the C source (a dropped scale, D_i left out, a flipped sign,
  unnormalised weights, strided GQA, a wrong D_i), each of which one of the pins above catches.
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

from .test_oracle_pins import rnd, visible_set

FULL, CAUSAL, SLIDING = O.MASK_FULL, O.MASK_CAUSAL, O.MASK_SLIDING


def finite_difference_grads(q, k, v, dout, mask, w, s, scale, h=1e-6):
    def loss(qq, kk, vv):
        o, _ = O.attention(qq, kk, vv, mask, w, s, scale)
        return float((o * dout).sum())

    grads = []
    for which in range(3):
        x = (q, k, v)[which]
        g = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            args_p, args_m = [q, k, v], [q, k, v]
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p[which], args_m[which] = xp, xm
            g[idx] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        grads.append(g)
    return grads


FD_CASES = [
    # Nq, Nk, d, mask, window, n_sink, Hq, Hkv, scale
    (4, 5, 3, FULL, 0, 0, 1, 1, 0.7),
    (5, 5, 3, CAUSAL, 0, 0, 2, 1, 1 / math.sqrt(3)),
    (3, 6, 2, CAUSAL, 0, 0, 1, 1, 0.9),          # Nq < Nk: bottom-right alignment
    (6, 3, 2, CAUSAL, 0, 0, 1, 1, 0.9),          # Nq > Nk: the first rows see no key
    (7, 7, 3, SLIDING, 2, 2, 4, 2, 0.6),         # window + sinks, GQA with two kv heads
    (5, 5, 2, SLIDING, 1, 0, 2, 2, -0.8),        # diagonal only, negative scale
    (4, 6, 3, FULL, 0, 0, 4, 2, -0.5),
    (7, 7, 3, O.MASK_LOCAL_GLOBAL, 1, 1, 2, 1, 0.8),  # bidirectional window + a global token
    (5, 8, 2, O.MASK_LOCAL_GLOBAL, 2, 0, 1, 1, 0.7),
]


def fd_check(case, seed=61):
    Nq, Nk, d, mask, w, s, Hq, Hkv, scale = case
    q, k, v = rnd(seed, 0, (1, Hq, Nq, d)), rnd(seed, 1, (1, Hkv, Nk, d)), rnd(seed, 2, (1, Hkv, Nk, d))
    dout = rnd(seed, 3, (1, Hq, Nq, d))
    dq, dk, dv = O.attention_bwd(q, k, v, dout, mask, w, s, scale)
    nq, nk, nv = finite_difference_grads(q, k, v, dout, mask, w, s, scale)
    np.testing.assert_allclose(dq, nq, atol=2e-7)
    np.testing.assert_allclose(dk, nk, atol=2e-7)
    np.testing.assert_allclose(dv, nv, atol=2e-7)


@pytest.mark.parametrize("case", FD_CASES)
def test_backward_equals_finite_differences(case):
    fd_check(case)


def scale_zero_check(seed=62):
    Nq, Nk, d, Hq, Hkv = 6, 8, 3, 4, 2
    G = Hq // Hkv
    for mask, w, s in ((FULL, 0, 0), (CAUSAL, 0, 0), (SLIDING, 3, 1)):
        q, k, v = rnd(seed, 0, (1, Hq, Nq, d)), rnd(seed, 1, (1, Hkv, Nk, d)), rnd(seed, 2, (1, Hkv, Nk, d))
        dout = rnd(seed, 3, (1, Hq, Nq, d))
        dq, dk, dv = O.attention_bwd(q, k, v, dout, mask, w, s, 0.0)
        assert np.all(dq == 0) and np.all(dk == 0)
        want = np.zeros_like(dv)
        for h in range(Hq):
            for i in range(Nq):
                vis = visible_set(i + Nk - Nq, Nk, mask, w, s)
                for j in vis:
                    want[0, h // G, j] += dout[0, h, i] / len(vis)
        np.testing.assert_allclose(dv, want, atol=1e-13)


def test_scale_zero_closed_form():
    scale_zero_check()


def invariant_check(seed=63):
    Nq, Nk, d, Hq, Hkv = 9, 11, 4, 4, 2
    G = Hq // Hkv
    for mask, w, s in ((FULL, 0, 0), (CAUSAL, 0, 0), (SLIDING, 4, 2)):
        q, k, v = rnd(seed, 0, (2, Hq, Nq, d)), rnd(seed, 1, (2, Hkv, Nk, d)), rnd(seed, 2, (2, Hkv, Nk, d))
        dout = rnd(seed, 3, (2, Hq, Nq, d))
        dq, dk, dv = O.attention_bwd(q, k, v, dout, mask, w, s, 0.4)
        np.testing.assert_allclose(dk.sum(axis=2), 0.0, atol=1e-12)
        seen = np.array([len(visible_set(i + Nk - Nq, Nk, mask, w, s)) > 0 for i in range(Nq)])
        for b in range(2):
            for hk in range(Hkv):
                want = sum(dout[b, hk * G + g][seen].sum(axis=0) for g in range(G))
                np.testing.assert_allclose(dv[b, hk].sum(axis=0), want, atol=1e-12)


def test_gradient_sums():
    invariant_check()


# ------------------------------------------------------------------------------------------
# planted slips in copies of the C source
# ------------------------------------------------------------------------------------------
MUTANTS = {
    "dk_without_scale": ("dkj[t] += scale * ds * qi[t];", "dkj[t] += ds * qi[t];"),
    "ds_without_D": ("const double ds = pij * (dpv - Dv[r]);", "const double ds = pij * dpv;"),
    "dq_sign": ("dqi[t] += scale * ds * Kb[j * (int64_t)d + t];",
                "dqi[t] -= scale * ds * Kb[j * (int64_t)d + t];"),
    "unnormalised_p": ("const double pij = exp(scale * sc - lse[r]);", "const double pij = exp(scale * sc);"),
    "strided_gqa": ("const int64_t h = hk * G + g;", "const int64_t h = g * Hkv + hk;"),
    "wrong_D": ("D += s[j] * dp[j];", "D += dp[j];"),
}


def _checks():
    yield "fd_causal_gqa", lambda: fd_check(FD_CASES[4])
    yield "fd_full_gqa", lambda: fd_check(FD_CASES[6])
    yield "scale_zero", scale_zero_check
    yield "sums", invariant_check


@pytest.fixture(scope="module")
def tmpdir():
    d = tempfile.mkdtemp(prefix="oracle_bwd_mutants_")
    yield d
    shutil.rmtree(d, ignore_errors=True)


def test_unmutated_backward_passes_every_check():
    for _, fn in _checks():
        fn()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_backward_mutant_is_caught(name, tmpdir, monkeypatch):
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
               "oracle_attn_bwd"):
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
