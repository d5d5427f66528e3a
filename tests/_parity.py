"""Helpers shared by the GPU parity tests: seeded inputs, oracle calls and the tolerance check.

Tolerances (bf16 inputs, fp32 accumulation, bf16 output), as the exact-attention workloads
state them: max|dO| <= 2e-2, mean|dO| <= 2e-3, and LSE within 1e-3 relative, read as
|dLSE| <= 1e-3 * max(1, |LSE|) because LSE can sit near 0.  Rows with no visible key must give
O = 0 and LSE = -inf exactly.  fp32 inputs with fp32 arithmetic: max|dO| <= 1e-4 (fp32 rounding
over at most a few thousand terms of magnitude <= 1, with margin), same LSE rule.
"""

from __future__ import annotations

import numpy as np
import torch

import synth
from oracle import oracle as O

TOL_BF16 = dict(max_abs=2e-2, mean_abs=2e-3, lse_rel=1e-3)
TOL_F32 = dict(max_abs=1e-4, mean_abs=1e-5, lse_rel=1e-5)
# E4M3 forward: the weights 16 * P are rounded to E4M3 (3 mantissa bits) for the P V product.
# tests/test_tolerance_models.py recomputes the error of exactly that rounding against the
# oracle and checks that these limits cover it with margin.
TOL_FP8 = dict(max_abs=0.1, mean_abs=6e-3, lse_rel=1e-3)
# Backward, per gradient tensor: max|d| <= BWD_REL * max|ref| + BWD_ABS_MAX and
# mean|d| <= BWD_REL * mean|ref| + BWD_ABS_MEAN (P and dS rounded to bf16 for the tensor cores,
# D from the bf16 O, gradients rounded to bf16; the same model test covers these).
BWD_REL = 1e-2
BWD_ABS_MAX = 1e-4
BWD_ABS_MEAN = 1e-5


def bf16_inputs(seed, B, Hq, Hkv, Nq, Nk, d, device="cuda"):
    """bf16 Q, K, V drawn on the host (exact same bytes for the GPU and for the oracle).

    Returns (q, k, v) as CUDA bf16 tensors and (q64, k64, v64) as the fp64 widening."""
    host = []
    dev = []
    for tid, shape in ((synth.Q_ID, (B, Hq, Nq, d)), (synth.K_ID, (B, Hkv, Nk, d)),
                       (synth.V_ID, (B, Hkv, Nk, d))):
        bits = synth.normal_bf16_bits(seed, tid, shape)
        host.append(synth.bf16_bits_to_f32(bits).astype(np.float64).reshape(shape))
        dev.append(torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).to(device))
    return dev, host


def f32_inputs(seed, B, Hq, Hkv, Nq, Nk, d, device="cuda"):
    host, dev = [], []
    for tid, shape in ((synth.Q_ID, (B, Hq, Nq, d)), (synth.K_ID, (B, Hkv, Nk, d)),
                       (synth.V_ID, (B, Hkv, Nk, d))):
        x = synth.normal_f32(seed, tid, shape)
        host.append(x.astype(np.float64))
        dev.append(torch.from_numpy(x).to(device))
    return dev, host


def to64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def assert_close(o_gpu, lse_gpu, o_ref, lse_ref, tol, what=""):
    """Element-wise comparison against the oracle with the stated tolerances."""
    o_gpu = np.asarray(o_gpu, dtype=np.float64)
    o_ref = np.asarray(o_ref, dtype=np.float64)
    assert o_gpu.shape == o_ref.shape, (o_gpu.shape, o_ref.shape)
    assert np.all(np.isfinite(o_gpu)), what + ": non-finite output"
    err = np.abs(o_gpu - o_ref)
    mx, mean = float(err.max()) if err.size else 0.0, float(err.mean()) if err.size else 0.0
    assert mx <= tol["max_abs"], "%s: max|dO| = %.3g > %.3g" % (what, mx, tol["max_abs"])
    assert mean <= tol["mean_abs"], "%s: mean|dO| = %.3g > %.3g" % (what, mean, tol["mean_abs"])
    if lse_gpu is not None:
        lg = np.asarray(lse_gpu, dtype=np.float64).reshape(-1)
        lr = np.asarray(lse_ref, dtype=np.float64).reshape(-1)
        empty = lr == -np.inf
        assert np.all(lg[empty] == -np.inf), what + ": rows without a visible key need LSE = -inf"
        fin = ~empty
        d = np.abs(lg[fin] - lr[fin])
        bound = tol["lse_rel"] * np.maximum(1.0, np.abs(lr[fin]))
        worst = float((d / bound).max()) if d.size else 0.0
        assert worst <= 1.0, "%s: LSE error %.3g x the bound" % (what, worst)
    return mx, mean


def sample_rows(Nq, n_random, structural=(), seed=0):
    rng = np.random.default_rng(seed)
    rows = set(int(r) for r in structural if 0 <= r < Nq)
    rows.update(int(r) for r in rng.integers(0, Nq, size=n_random))
    return np.array(sorted(rows), dtype=np.int64)


def oracle_rows_one_head(q64_rows, rows, k64, v64, Nq, mask, window, n_sink, scale):
    """Oracle for selected rows i of one (b, h): q64_rows[len(rows), d] holds those rows' query
    vectors; k64/v64 [Nk, d] are the kv head's keys/values.  Builds a [1,1,Nq,d] query array
    with only the selected rows filled (the others are not evaluated)."""
    d = k64.shape[-1]
    q_full = np.zeros((1, 1, Nq, d), dtype=np.float64)
    q_full[0, 0, rows] = q64_rows
    return O.attention_rows(q_full, k64[None, None], v64[None, None], rows, mask, window, n_sink,
                            scale)
