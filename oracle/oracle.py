"""Python front end of the fp64 exact-attention oracle (``oracle.c``).

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the benchmark's CPU-baseline leg
are the only callers.  Nothing here touches CUDA.  Inputs are widened to fp64 exactly (bf16 and
fp32 values are representable in fp64), so the oracle measures kernel error and not input
quantisation.
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

MASK_FULL, MASK_CAUSAL, MASK_SLIDING, MASK_LOCAL_GLOBAL = 0, 1, 2, 3

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile liboracle.so with gcc + OpenMP (host only, no CUDA)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        dp = ctypes.POINTER(ctypes.c_double)
        lib.oracle_attn.argtypes = [dp, dp, dp, dp, dp] + [ctypes.c_int] * 9 + [ctypes.c_double]
        lib.oracle_attn.restype = ctypes.c_int
        lib.oracle_attn_rows.argtypes = ([dp, dp, dp] + [ctypes.c_int] * 9 + [ctypes.c_double,
                                         ctypes.POINTER(ctypes.c_int64), ctypes.c_int64, dp, dp])
        lib.oracle_attn_rows.restype = ctypes.c_int
        lib.oracle_visible_pairs.argtypes = [ctypes.c_int] * 5
        lib.oracle_visible_pairs.restype = ctypes.c_int64
        lib.oracle_visible.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_int,
                                       ctypes.c_int64, ctypes.c_int64]
        lib.oracle_visible.restype = ctypes.c_int
        lib.oracle_attn_bwd.argtypes = [dp] * 7 + [ctypes.c_int] * 9 + [ctypes.c_double]
        lib.oracle_attn_bwd.restype = ctypes.c_int
        lib.oracle_attn_block_sparse.argtypes = ([dp, dp, dp, dp, dp] + [ctypes.c_int] * 9 +
                                                 [ctypes.c_double, ctypes.c_void_p] +
                                                 [ctypes.c_int] * 3)
        lib.oracle_attn_block_sparse.restype = ctypes.c_int
        lib.oracle_num_threads.argtypes = []
        lib.oracle_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def attention(q, k, v, mask_kind=MASK_FULL, window=0, n_sink=0, scale=None):
    """O and LSE for every row.  q: [B,Hq,Nq,d]; k, v: [B,Hkv,Nk,d] (any real dtype).

    Returns (o [B,Hq,Nq,d] fp64, lse [B,Hq,Nq] fp64).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, Nq, d = q.shape
    _, Hkv, Nk, _ = k.shape
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    o = np.zeros((B, Hq, Nq, d), dtype=np.float64)
    lse = np.zeros((B, Hq, Nq), dtype=np.float64)
    rc = _load().oracle_attn(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, Nq, Nk, d,
                             int(mask_kind), int(window), int(n_sink), float(scale))
    if rc != 0:
        raise ValueError("oracle_attn rejected its arguments (rc=%d)" % rc)
    return o, lse


def attention_block_sparse(q, k, v, block_mask, mask_kind=MASK_FULL, window=0, n_sink=0,
                           scale=None, block_q=128, block_k=128):
    """Block-sparse O and LSE: key j is visible to row i of head h iff
    block_mask[hm, i // block_q, j // block_k] is non-zero (hm = h, or 0 for a layout shared by
    every head) and the base mask admits it.  block_mask: [1 or Hq, ceil(Nq/block_q),
    ceil(Nk/block_k)], any integer or bool dtype.  Returns (o fp64, lse fp64) as attention().
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, Nq, d = q.shape
    _, Hkv, Nk, _ = k.shape
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    bm = np.ascontiguousarray(np.asarray(block_mask) != 0, dtype=np.uint8)
    nqb, nkb = -(-Nq // block_q), -(-Nk // block_k)
    if bm.ndim != 3 or bm.shape[0] not in (1, Hq) or bm.shape[1:] != (nqb, nkb):
        raise ValueError("block_mask must be [1 or Hq, %d, %d], got %s" % (nqb, nkb, bm.shape))
    o = np.zeros((B, Hq, Nq, d), dtype=np.float64)
    lse = np.zeros((B, Hq, Nq), dtype=np.float64)
    rc = _load().oracle_attn_block_sparse(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq,
                                          Hkv, Nq, Nk, d, int(mask_kind), int(window),
                                          int(n_sink), float(scale), bm.ctypes.data,
                                          int(bm.shape[0]), int(block_q), int(block_k))
    if rc != 0:
        raise ValueError("oracle_attn_block_sparse rejected its arguments (rc=%d)" % rc)
    return o, lse


def attention_rows(q, k, v, rows, mask_kind=MASK_FULL, window=0, n_sink=0, scale=None):
    """O and LSE for the flat rows r = (b*Hq + h)*Nq + i listed in ``rows``.

    Returns (o [len(rows), d], lse [len(rows)]).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, Nq, d = q.shape
    _, Hkv, Nk, _ = k.shape
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    o = np.zeros((len(r), d), dtype=np.float64)
    lse = np.zeros(len(r), dtype=np.float64)
    rc = _load().oracle_attn_rows(_ptr(q), _ptr(k), _ptr(v), B, Hq, Hkv, Nq, Nk, d,
                                  int(mask_kind), int(window), int(n_sink), float(scale),
                                  r.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), len(r),
                                  _ptr(o), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_attn_rows rejected its arguments (rc=%d)" % rc)
    return o, lse


def attention_bwd(q, k, v, dout, mask_kind=MASK_FULL, window=0, n_sink=0, scale=None):
    """Gradients (dq, dk, dv) of a loss whose gradient with respect to O is ``dout``.

    q, dout: [B,Hq,Nq,d]; k, v: [B,Hkv,Nk,d].  Returns fp64 arrays of the same shapes.
    """
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, Hq, Nq, d = q.shape
    _, Hkv, Nk, _ = k.shape
    if dout.shape != q.shape:
        raise ValueError("dout must have the shape of q")
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    rc = _load().oracle_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(dq), _ptr(dk),
                                 _ptr(dv), B, Hq, Hkv, Nq, Nk, d, int(mask_kind), int(window),
                                 int(n_sink), float(scale))
    if rc != 0:
        raise ValueError("oracle_attn_bwd rejected its arguments (rc=%d)" % rc)
    return dq, dk, dv


def visible(p: int, j: int, mask_kind: int, window: int = 0, n_sink: int = 0) -> bool:
    return bool(_load().oracle_visible(p, j, mask_kind, window, n_sink))


def visible_pairs(Nq: int, Nk: int, mask_kind: int, window: int = 0, n_sink: int = 0) -> int:
    """Visible (query, key) pairs of one (b, h) slice, by enumeration."""
    return int(_load().oracle_visible_pairs(Nq, Nk, mask_kind, window, n_sink))


def num_threads() -> int:
    return int(_load().oracle_num_threads())
