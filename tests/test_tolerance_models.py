"""Where the E4M3 forward's and the backward's test tolerances come from.

Both GPU paths round an intermediate to a narrow type before a tensor-core product, so they
cannot meet the bf16 forward's limits: the E4M3 forward rounds the weights 16 * P to E4M3 for
the P V product, and the backward rounds P and dS to bf16 for its four products and computes
D_i = dO_i . O_i from the bf16 O.  The tests here model exactly those roundings in numpy (fp64
everywhere else) and compare the model against the fp64 oracle on the inputs the GPU tests use:
the limits in tests/_parity.py (TOL_FP8 and BWD_*) must cover the modelled error with a stated
margin.  A model, not a kernel: no code of the CUDA path is imported or run, and no GPU is used.

Readings:
- the kernels' running-max bookkeeping (the E4M3 kernel rescales whenever the max grows by more
  than four log2 units) only moves where the E4M3 subnormal range starts, so the model takes P
  relative to the row's final max; the margin covers the rest (fp32 accumulation of the
  scores and sums, the ex2 approximation, bf16 rounding of the output, which the model does
  include);
- "Chapter 3.1 - The Cost of Attention" (llmis.ru), section 5: the method computes the same
  answer as the definition up to floating-point tolerance; the tolerance is sized here.
"""

from __future__ import annotations

import math

import numpy as np
import pytest

import synth
from oracle import oracle as O

from ._parity import BWD_ABS_MAX, BWD_ABS_MEAN, BWD_REL, TOL_FP8

FULL, CAUSAL, SLIDING, LOCAL = O.MASK_FULL, O.MASK_CAUSAL, O.MASK_SLIDING, O.MASK_LOCAL_GLOBAL

# the modelled error may use at most this share of a limit
MARGIN = 1.5


def visible_matrix(Nq, Nk, mask, w, s):
    """Visibility of (query row i, key j) from the masks' set definitions, bottom-right aligned
    (query position p = i + Nk - Nq)."""
    p = np.arange(Nq)[:, None] + (Nk - Nq)
    j = np.arange(Nk)[None, :]
    if mask == FULL:
        return np.ones((Nq, Nk), bool)
    if mask == CAUSAL:
        return j <= p
    if mask == SLIDING:
        return (j <= p) & ((j > p - w) | (j < s))
    assert mask == LOCAL
    return (np.abs(p - j) <= w) | (j < s) | ((p >= 0) & (p < s))


def bf16(x):
    return synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(np.asarray(x, np.float32))).astype(np.float64)


def e4m3(x):
    return synth.e4m3_bits_to_f32(synth.f32_to_e4m3_bits(np.asarray(x, np.float64))).astype(np.float64)


def softmax_weights(S, vis):
    """exp(S - rowmax) over the visible keys (0 elsewhere) and the row sums; rows without a
    visible key get all-zero weights and a zero sum."""
    Sm = np.where(vis, S, -np.inf)
    m = Sm.max(axis=1, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)
    P = np.where(vis, np.exp(Sm - m), 0.0)
    return P, P.sum(axis=1, keepdims=True)


# ---------------------------------------------------------------------------------------------
# E4M3 forward
# ---------------------------------------------------------------------------------------------

P_SCALE_F8 = 16.0  # the weights are scaled by 16 before they are rounded to E4M3

FP8_CASES = [  # (B, Hq, Hkv, Nq, Nk, mask, w, s): the shapes tests/test_gpu_fp8.py runs
    (1, 2, 1, 512, 512, CAUSAL, 0, 0),
    (1, 2, 1, 1024, 1024, FULL, 0, 0),
    (1, 2, 1, 700, 700, SLIDING, 128, 4),
    (1, 2, 1, 700, 700, LOCAL, 64, 2),
    (1, 2, 1, 257, 333, FULL, 0, 0),
    (1, 1, 1, 2048, 2048, CAUSAL, 0, 0),
]


def fp8_model_error(B, Hq, Hkv, Nq, Nk, mask, w, s, seed=96):
    d = 128
    vals = []
    for tid, shape in ((synth.Q_ID, (B, Hq, Nq, d)), (synth.K_ID, (B, Hkv, Nk, d)),
                       (synth.V_ID, (B, Hkv, Nk, d))):
        codes, scales = synth.normal_e4m3(seed, tid, shape)
        vals.append(synth.e4m3_bits_to_f32(codes).astype(np.float64) * scales[..., None, None])
    q, k, v = vals
    scale = 1 / math.sqrt(d)
    o_ref, _ = O.attention(q, k, v, mask, w, s, scale)
    vis = visible_matrix(Nq, Nk, mask, w, s)
    G = Hq // Hkv
    errs = []
    for b in range(B):
        for h in range(Hq):
            P, l = softmax_weights(q[b, h] @ k[b, h // G].T * scale, vis)
            p8 = e4m3(P * P_SCALE_F8)  # the only narrow rounding before the product
            o = np.divide(p8 @ v[b, h // G], P_SCALE_F8 * l, out=np.zeros((Nq, d)), where=l > 0)
            errs.append(np.abs(bf16(o) - o_ref[b, h]))
    e = np.stack(errs)
    return float(e.max()), float(e.mean())


@pytest.mark.parametrize("case", FP8_CASES)
def test_fp8_tolerance_covers_the_modelled_rounding(case):
    mx, mean = fp8_model_error(*case)
    # the model must show the rounding (a model that rounds nothing proves nothing) ...
    assert mx > 1e-3 and mean > 1e-4, (mx, mean)
    # ... and the GPU test's limits must hold it with margin
    assert MARGIN * mx <= TOL_FP8["max_abs"], (case, mx)
    assert MARGIN * mean <= TOL_FP8["mean_abs"], (case, mean)


def test_fp8_bf16_tolerance_would_not_cover_it():
    """The E4M3 path needs its own limits: the bf16 forward's max limit (2e-2) is below the
    modelled E4M3 error on rows that see few keys."""
    mx, _ = fp8_model_error(1, 2, 1, 512, 512, CAUSAL, 0, 0)
    assert mx > 2e-2


# ---------------------------------------------------------------------------------------------
# backward
# ---------------------------------------------------------------------------------------------

BWD_CASES = [  # (B, Hq, Hkv, N, mask, w, s): shapes of the kind tests/test_gpu_bwd.py runs
    (1, 2, 1, 512, CAUSAL, 0, 0),
    (1, 2, 1, 1024, FULL, 0, 0),
    (1, 4, 2, 700, SLIDING, 128, 4),
    (1, 2, 1, 600, LOCAL, 64, 2),
    (1, 1, 1, 2048, CAUSAL, 0, 0),
]


def bwd_model_errors(B, Hq, Hkv, N, mask, w, s, seed=71):
    """Relative errors (max err / max|ref|, mean err / mean|ref|) of dQ, dK, dV as the kernels
    round them, against the oracle's backward."""
    d = 128
    q, k, v, do = (bf16(synth.normal_f32(seed, tid, shape)) for tid, shape in (
        (synth.Q_ID, (B, Hq, N, d)), (synth.K_ID, (B, Hkv, N, d)), (synth.V_ID, (B, Hkv, N, d)),
        (synth.DO_ID, (B, Hq, N, d))))
    scale = 1 / math.sqrt(d)
    o, _ = O.attention(q, k, v, mask, w, s, scale)
    rq, rk, rv = O.attention_bwd(q, k, v, do, mask, w, s, scale)
    vis = visible_matrix(N, N, mask, w, s)
    G = Hq // Hkv
    mq, mk, mv = np.zeros_like(rq), np.zeros_like(rk), np.zeros_like(rv)
    o16 = bf16(o)  # the forward's output as the backward receives it
    for b in range(B):
        for h in range(Hq):
            hk = h // G
            P, l = softmax_weights(q[b, h] @ k[b, hk].T * scale, vis)
            P = np.divide(P, l, out=np.zeros_like(P), where=l > 0)
            D = (do[b, h] * o16[b, h]).sum(-1)[:, None]
            dS = bf16(P * (do[b, h] @ v[b, hk].T - D))  # dS rounded for the tensor cores
            mv[b, hk] += bf16(P).T @ do[b, h]          # P rounded for dV = P^T dO
            mk[b, hk] += scale * dS.T @ q[b, h]
            mq[b, h] = scale * dS @ k[b, hk]
    out = {}
    for name, ref, got in (("dq", rq, bf16(mq)), ("dk", rk, bf16(mk)), ("dv", rv, bf16(mv))):
        err = np.abs(got - ref)
        out[name] = (float(err.max() / np.abs(ref).max()), float(err.mean() / np.abs(ref).mean()),
                     float(err.max()), float(err.mean()))
    return out


@pytest.mark.parametrize("case", BWD_CASES)
def test_bwd_tolerance_covers_the_modelled_rounding(case):
    for name, (rel_max, rel_mean, mx, mean) in bwd_model_errors(*case).items():
        # the bf16 roundings show (about 2^-9 relative per rounded product) ...
        assert rel_mean > 1e-4, (case, name, rel_mean)
        # ... and the per-tensor limits of the GPU test hold them with margin (the absolute
        # terms of those limits are ignored here: the relative part alone must suffice)
        assert MARGIN * rel_max <= BWD_REL, (case, name, rel_max)
        assert MARGIN * rel_mean <= BWD_REL, (case, name, rel_mean)
        assert BWD_ABS_MAX < 1e-2 * mx + 1e-3 and BWD_ABS_MEAN < 1e-2 * mean + 1e-3
