"""GPU parity of the backward pass (attn_bwd) against the fp64 oracle's backward.

The GPU backward gets the GPU forward's own O and LSE (the pipeline a training step runs), the
oracle recomputes everything in fp64 from the same bf16 Q, K, V, dO.

Tolerance, per gradient tensor (derived from the arithmetic): the kernels round P
and dS to bf16 for the tensor cores, compute D_i from the bf16 O, accumulate in fp32 and round
the gradients to bf16.  A numpy model of exactly those roundings against the fp64 oracle
(tests/test_tolerance_models.py, a CPU test that also checks the margin) gives, on causal, full
and sliding cases up to n = 2048, a mean error of about 0.23% of mean|ref| (the final bf16
rounding) and a max error of at most about 0.4% of max|ref|.  The test allows 1% for both:
max|d| <= 1e-2 * max|ref| + 1e-4 and mean|d| <= 1e-2 * mean|ref| + 1e-5.  The absolute terms
cover gradients that are exactly zero in real arithmetic but not in fp32: with a window of one
key, dS_ii = P_ii (dP_ii - D_i) with dP_ii = dO_i . v_i summed by the tensor core and
D_i = dO_i . O_i (O_i = v_i) summed by the prep kernel in another order, a difference of a few
fp32 ulps of |dO_i . v_i| ~ sqrt(d) (about 1e-6), times scale * |k| in dQ.
"""

import math

import numpy as np
import pytest
import torch

import synth
from exact_io_aware_82_b200 import attn as A
from exact_io_aware_82_b200 import build as Bld
from oracle import oracle as O

from ._parity import BWD_ABS_MAX, BWD_ABS_MEAN, BWD_REL, bf16_inputs, to64

pytestmark = pytest.mark.gpu
FULL, CAUSAL, SLIDING = A.MASK_FULL, A.MASK_CAUSAL, A.MASK_SLIDING


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    Bld.build()
    A.lib()
    yield
    assert A.attn_get_device_error() == 0


def grad_close(got, ref, what):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape
    assert np.all(np.isfinite(got)), what + ": non-finite gradient"
    err = np.abs(got - ref)
    mx, mean = float(err.max()) if err.size else 0.0, float(err.mean()) if err.size else 0.0
    lim_mx = BWD_REL * float(np.abs(ref).max() if ref.size else 0.0) + BWD_ABS_MAX
    lim_mean = BWD_REL * float(np.abs(ref).mean() if ref.size else 0.0) + BWD_ABS_MEAN
    assert mx <= lim_mx, "%s: max|d| = %.3g > %.3g" % (what, mx, lim_mx)
    assert mean <= lim_mean, "%s: mean|d| = %.3g > %.3g" % (what, mean, lim_mean)


def run(seed, B, Hq, Hkv, Nq, Nk, mask, w, s, scale=None):
    d = 128
    (q, k, v), (q64, k64, v64) = bf16_inputs(seed, B, Hq, Hkv, Nq, Nk, d)
    bits = synth.normal_bf16_bits(seed, synth.DO_ID, (B, Hq, Nq, d))
    do64 = synth.bf16_bits_to_f32(bits).astype(np.float64)
    do = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).cuda()
    scale = 1 / math.sqrt(d) if scale is None else scale
    o, lse = A.attn_fwd(q, k, v, mask_kind=mask, window=w, n_sink=s, scale=scale)
    dq, dk, dv = A.attn_bwd(q, k, v, o, lse, do, mask_kind=mask, window=w, n_sink=s, scale=scale)
    torch.cuda.synchronize()
    rq, rk, rv = O.attention_bwd(q64, k64, v64, do64, mask, w, s, scale)
    tag = "B%d Hq%d Hkv%d Nq%d Nk%d mask%d w%d s%d" % (B, Hq, Hkv, Nq, Nk, mask, w, s)
    grad_close(to64(dq), rq, "dq " + tag)
    grad_close(to64(dk), rk, "dk " + tag)
    grad_close(to64(dv), rv, "dv " + tag)


CASES = [
    # B, Hq, Hkv, Nq, Nk, mask, window, n_sink
    (1, 2, 2, 128, 128, FULL, 0, 0),
    (1, 2, 1, 300, 300, CAUSAL, 0, 0),      # ragged tail, GQA
    (2, 4, 2, 513, 513, CAUSAL, 0, 0),
    (1, 2, 2, 200, 450, CAUSAL, 0, 0),      # Nq < Nk: bottom-right alignment
    (1, 2, 2, 450, 200, CAUSAL, 0, 0),      # Nq > Nk: the first rows see no key
    (1, 4, 1, 700, 700, SLIDING, 200, 4),   # window + sinks, G = 4
    (1, 2, 2, 600, 600, SLIDING, 1, 0),     # diagonal only
    (1, 8, 1, 257, 333, FULL, 0, 0),        # G = 8, ragged both ways
    (1, 2, 2, 1, 700, CAUSAL, 0, 0),        # one query row
    (1, 2, 2, 700, 1, CAUSAL, 0, 0),        # one key
]


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nk,mask,w,s", CASES)
def test_bwd_against_oracle(B, Hq, Hkv, Nq, Nk, mask, w, s):
    run(81, B, Hq, Hkv, Nq, Nk, mask, w, s)


@pytest.mark.parametrize("scale", [0.05, -0.09, 0.0])
def test_bwd_other_scales(scale):
    run(82, 1, 2, 1, 300, 300, CAUSAL, 0, 0, scale=scale)


def test_bwd_empty_sides_give_zero_gradients():
    d = 128
    for Nq, Nk in ((0, 200), (200, 0)):
        q = synth.normal_torch(83, 0, (1, 2, Nq, d), device="cuda")
        k = synth.normal_torch(83, 1, (1, 2, Nk, d), device="cuda")
        v = synth.normal_torch(83, 2, (1, 2, Nk, d), device="cuda")
        do = synth.normal_torch(83, 3, (1, 2, Nq, d), device="cuda")
        o, lse = A.attn_fwd(q, k, v, mask_kind=CAUSAL)
        dq = torch.full_like(q, 3.0)
        dk = torch.full_like(k, 3.0)
        dv = torch.full_like(v, 3.0)
        A.attn_bwd(q, k, v, o, lse, do, mask_kind=CAUSAL, dq=dq, dk=dk, dv=dv)
        torch.cuda.synchronize()
        assert torch.all(dq == 0) and torch.all(dk == 0) and torch.all(dv == 0)


def test_bwd_is_deterministic():
    d = 128
    B, Hq, Hkv, N = 2, 8, 2, 1000
    q = synth.normal_torch(84, 0, (B, Hq, N, d), device="cuda")
    k = synth.normal_torch(84, 1, (B, Hkv, N, d), device="cuda")
    v = synth.normal_torch(84, 2, (B, Hkv, N, d), device="cuda")
    do = synth.normal_torch(84, 3, (B, Hq, N, d), device="cuda")
    o, lse = A.attn_fwd(q, k, v, mask_kind=CAUSAL)
    a = A.attn_bwd(q, k, v, o, lse, do, mask_kind=CAUSAL)
    b = A.attn_bwd(q, k, v, o, lse, do, mask_kind=CAUSAL)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_bwd_causal_b4_h16_n2048_sampled():
    # the benchmark's backward workload; two (b, head) slices checked against the oracle (each
    # slice's gradients depend on that slice only)
    B, H, N, d = 4, 16, 2048, 128
    q = synth.normal_torch(8, 0, (B, H, N, d), device="cuda")
    k = synth.normal_torch(8, 1, (B, H, N, d), device="cuda")
    v = synth.normal_torch(8, 2, (B, H, N, d), device="cuda")
    do = synth.normal_torch(8, 3, (B, H, N, d), device="cuda")
    o, lse = A.attn_fwd(q, k, v, mask_kind=CAUSAL)
    dq, dk, dv = A.attn_bwd(q, k, v, o, lse, do, mask_kind=CAUSAL)
    torch.cuda.synchronize()
    for b, h in ((0, 0), (3, 11)):
        sl = lambda t: to64(t[b:b + 1, h:h + 1])  # noqa: E731
        rq, rk, rv = O.attention_bwd(sl(q), sl(k), sl(v), sl(do), CAUSAL, 0, 0, 1 / math.sqrt(d))
        grad_close(sl(dq), rq, "dq b%d h%d" % (b, h))
        grad_close(sl(dk), rk, "dk b%d h%d" % (b, h))
        grad_close(sl(dv), rv, "dv b%d h%d" % (b, h))
