"""Plant mistakes in a copy of the oracle (on the CPU) and check that the pins catch each one.

Every mutant below is a plausible slip: a dropped scale, an off-by-one at a window or sink edge,
strided instead of contiguous GQA grouping, a missing term in the LSE, top-left instead of
bottom-right causal alignment, a wrong value row.  The checks are the same kinds of pins as in
test_oracle_pins.py (closed forms, brute force, invariants), run against the mutant library.
"""

import math
import os
import shutil
import subprocess
import tempfile

import numpy as np
import pytest

from oracle import oracle as O

from .test_oracle_pins import _decimal_attention, rnd, visible_set

FULL, CAUSAL, SLIDING = O.MASK_FULL, O.MASK_CAUSAL, O.MASK_SLIDING

MUTANTS = {
    "drop_scale": ("s[j] = scale * acc;", "s[j] = acc;"),
    "window_edge": ("if (j > p - window) return 1;", "if (j >= p - window) return 1;"),
    "sink_edge": ("if (j < n_sink) return 1;", "if (j <= n_sink) return 1;"),
    "strided_gqa": ("int64_t hk = h / G;", "int64_t hk = h % Hkv;"),
    "lse_without_max": ("*lse = m + log(l);", "*lse = log(l);"),
    "top_left_causal": ("i + (int64_t)Nk - Nq, mask_kind", "i, mask_kind"),
    "wrong_value_row": ("o[t] += pj * V[j * (int64_t)d + t];", "o[t] += pj * V[(Nk - 1 - j) * (int64_t)d + t];"),
    "unnormalised": ("double pj = s[j] / l;", "double pj = s[j];"),
    "local_one_sided": ("return j >= p - window && j <= p + window;", "return j >= p - window && j <= p;"),
    "local_window_edge": ("return j >= p - window && j <= p + window;",
                          "return j > p - window && j <= p + window;"),
    "local_no_global_query": ("if (p >= 0 && p < n_sink) return 1;  /* global query */", ""),
    "local_no_global_key": ("if (j < n_sink) return 1;            /* global key */", ""),
}


def _checks():
    """Yield (name, callable) pins; each callable raises AssertionError on a mismatch."""
    def brute(Nq, Nk, d, mask, w, s, Hq=1, Hkv=1):
        def run():
            q, k, v = rnd(21, 0, (1, Hq, Nq, d)), rnd(21, 1, (1, Hkv, Nk, d)), rnd(21, 2, (1, Hkv, Nk, d))
            scale = 1.0 / math.sqrt(d)
            o, lse = O.attention(q, k, v, mask, w, s, scale)
            G = Hq // Hkv
            for h in range(Hq):
                eo, el = _decimal_attention(q[0, h], k[0, h // G], v[0, h // G], Nq, Nk, d, mask, w, s, scale)
                np.testing.assert_allclose(o[0, h], eo, atol=1e-12)
                fin = np.isfinite(el)
                np.testing.assert_allclose(lse[0, h][fin], el[fin], atol=1e-12)
        return run

    yield "brute_full", brute(4, 5, 3, FULL, 0, 0)
    yield "brute_causal_rect", brute(3, 6, 2, CAUSAL, 0, 0)
    yield "brute_sliding_sinks", brute(7, 7, 3, SLIDING, 2, 2)
    yield "brute_gqa", brute(3, 4, 2, CAUSAL, 0, 0, Hq=4, Hkv=2)
    yield "brute_local_global", brute(7, 7, 3, O.MASK_LOCAL_GLOBAL, 1, 1)

    def zero_q():
        Nq = Nk = 9
        q = np.zeros((1, 1, Nq, 4))
        v = rnd(22, 2, (1, 1, Nk, 4))
        o, lse = O.attention(q, rnd(22, 1, (1, 1, Nk, 4)), v, SLIDING, 3, 1, 0.5)
        for i in range(Nq):
            vis = sorted(visible_set(i, Nk, SLIDING, 3, 1))
            np.testing.assert_allclose(o[0, 0, i], v[0, 0, vis].mean(axis=0), atol=1e-13)
            assert abs(lse[0, 0, i] - math.log(len(vis))) < 1e-13
    yield "zero_q", zero_q


def _build_mutant(tmpdir, name, old, new):
    src = open(os.path.join(os.path.dirname(O.__file__), "oracle.c")).read()
    assert src.count(old) >= 1, "mutation site missing: " + name
    path_c = os.path.join(tmpdir, name + ".c")
    path_so = os.path.join(tmpdir, name + ".so")
    open(path_c, "w").write(src.replace(old, new))
    subprocess.check_call(["gcc", "-O1", "-std=c99", "-fopenmp", "-fPIC", "-shared", "-o",
                           path_so, path_c, "-lm"])
    return path_so


@pytest.fixture(scope="module")
def tmpdir():
    d = tempfile.mkdtemp(prefix="oracle_mutants_")
    yield d
    shutil.rmtree(d, ignore_errors=True)


def test_unmutated_oracle_passes_every_check():
    for name, fn in _checks():
        fn()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmpdir, monkeypatch):
    import ctypes

    old, new = MUTANTS[name]
    so = _build_mutant(tmpdir, name, old, new)
    O._load()  # make sure the signatures are known, then swap in the mutant
    real = O._lib
    lib = ctypes.CDLL(so)
    for fn in ("oracle_attn", "oracle_attn_rows", "oracle_visible_pairs", "oracle_visible"):
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
