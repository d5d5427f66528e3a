"""GPU checks that need no oracle: properties the definition fixes at any size, determinism, and
the bounded-wait error path."""

import math

import numpy as np
import pytest
import torch

import synth
from exact_io_aware_82_b200 import attn as A
from exact_io_aware_82_b200 import build as Bld

from ._parity import TOL_BF16, assert_close, to64

pytestmark = pytest.mark.gpu
FULL, CAUSAL, SLIDING = A.MASK_FULL, A.MASK_CAUSAL, A.MASK_SLIDING


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    Bld.build()
    A.lib()


def rnd(seed, tid, shape):
    return synth.normal_torch(seed, tid, shape, device="cuda")


@pytest.mark.parametrize("mask,w,s", [(FULL, 0, 0), (CAUSAL, 0, 0), (SLIDING, 130, 3)])
def test_zero_query_gives_mean_of_visible_values(mask, w, s):
    N = 600
    q = torch.zeros(1, 2, N, 128, dtype=torch.bfloat16, device="cuda")
    k, v = rnd(20, 1, (1, 1, N, 128)), rnd(20, 2, (1, 1, N, 128))
    o, lse = A.attn_fwd(q, k, v, mask_kind=mask, window=w, n_sink=s)
    v64 = to64(v)[0, 0]
    csum = np.concatenate([np.zeros((1, 128)), np.cumsum(v64, axis=0)])
    ref = np.zeros((N, 128))
    cnt = np.zeros(N)
    for i in range(N):
        if mask == FULL:
            ref[i], cnt[i] = csum[N] / N, N
        elif mask == CAUSAL:
            ref[i], cnt[i] = csum[i + 1] / (i + 1), i + 1
        else:
            lo = max(0, i - w + 1)
            tot = csum[i + 1] - csum[lo]
            extra = max(0, min(s, lo))  # sinks left of the window
            tot = tot + csum[extra]
            c = (i + 1 - lo) + extra
            ref[i], cnt[i] = tot / c, c
    for h in range(2):
        assert_close(to64(o)[0, h], to64(lse)[0, h], ref, np.log(cnt), TOL_BF16, "Q=0 %d" % mask)


def test_constant_values_give_constant_output():
    q, k = rnd(21, 0, (2, 4, 700, 128)), rnd(21, 1, (2, 2, 700, 128))
    v = torch.full((2, 2, 700, 128), -1.5, dtype=torch.bfloat16, device="cuda")
    for mask in (FULL, CAUSAL, SLIDING):
        o, _ = A.attn_fwd(q, k, v, mask_kind=mask, window=100, n_sink=2)
        assert float((o.float() + 1.5).abs().max()) <= 1.5 * 2e-2


def test_large_window_equals_causal_and_sinks_everywhere_equal_causal():
    q, k, v = rnd(22, 0, (1, 4, 900, 128)), rnd(22, 1, (1, 2, 900, 128)), rnd(22, 2, (1, 2, 900, 128))
    oc, lc = A.attn_fwd(q, k, v, mask_kind=CAUSAL)
    ow, lw = A.attn_fwd(q, k, v, mask_kind=SLIDING, window=5000)
    assert torch.equal(oc, ow) and torch.equal(lc, lw)
    os_, ls_ = A.attn_fwd(q, k, v, mask_kind=SLIDING, window=1, n_sink=900)
    assert_close(to64(os_), to64(ls_), to64(oc), to64(lc), TOL_BF16, "all sinks")


def test_gqa_equals_repeated_heads():
    G = 4
    q, k, v = rnd(23, 0, (2, 8, 500, 128)), rnd(23, 1, (2, 2, 500, 128)), rnd(23, 2, (2, 2, 500, 128))
    og, lg = A.attn_fwd(q, k, v, mask_kind=SLIDING, window=200, n_sink=4)
    om, lm = A.attn_fwd(q, k.repeat_interleave(G, dim=1).contiguous(),
                        v.repeat_interleave(G, dim=1).contiguous(), mask_kind=SLIDING, window=200,
                        n_sink=4)
    assert torch.equal(og, om) and torch.equal(lg, lm)


def test_decode_equals_last_causal_row():
    q, k, v = rnd(24, 0, (3, 8, 1000, 128)), rnd(24, 1, (3, 2, 1000, 128)), rnd(24, 2, (3, 2, 1000, 128))
    oc, lc = A.attn_fwd(q, k, v, mask_kind=CAUSAL)
    od, ld = A.attn_decode(q[:, :, -1:].contiguous(), k, v)
    assert_close(to64(od)[:, :, 0], to64(ld), to64(oc)[:, :, -1], to64(lc)[:, :, -1], TOL_BF16,
                 "decode vs prefill")
    of, lf = A.attn_fwd(q[:, :, -1:].contiguous(), k, v, mask_kind=FULL)
    assert_close(to64(of), to64(lf), to64(oc)[:, :, -1:], to64(lc)[:, :, -1:], TOL_BF16,
                 "full Nq=1 vs prefill")


def test_linearity_in_values():
    q, k = rnd(25, 0, (1, 2, 400, 128)), rnd(25, 1, (1, 2, 400, 128))
    v1, v2 = rnd(25, 2, (1, 2, 400, 128)), rnd(26, 2, (1, 2, 400, 128))
    o1, _ = A.attn_fwd(q, k, v1, mask_kind=CAUSAL)
    o2, _ = A.attn_fwd(q, k, v2, mask_kind=CAUSAL)
    v3 = (0.5 * v1.float() - 0.25 * v2.float()).to(torch.bfloat16)
    o3, _ = A.attn_fwd(q, k, v3, mask_kind=CAUSAL)
    ref = 0.5 * to64(o1) - 0.25 * to64(o2)
    assert np.abs(to64(o3) - ref).max() <= 2e-2


def test_deterministic():
    q, k, v = rnd(27, 0, (2, 8, 1500, 128)), rnd(27, 1, (2, 2, 1500, 128)), rnd(27, 2, (2, 2, 1500, 128))
    a = A.attn_fwd(q, k, v, mask_kind=SLIDING, window=300, n_sink=4)
    b = A.attn_fwd(q, k, v, mask_kind=SLIDING, window=300, n_sink=4)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
    d1 = A.attn_decode(q[:, :, :1].contiguous(), k, v)
    d2 = A.attn_decode(q[:, :, :1].contiguous(), k, v)
    assert torch.equal(d1[0], d2[0]) and torch.equal(d1[1], d2[1])


def test_prefill_on_concurrent_streams_matches_serial():
    """The persistent prefill grids take work from one counter per stream: calls queued on two
    streams at once (so their kernels may overlap) give the same bits as the calls run one
    after another, and back-to-back calls on one stream see the counter back at zero."""
    cases = [
        (rnd(29, 0, (2, 8, 1500, 128)), rnd(29, 1, (2, 2, 1500, 128)), rnd(29, 2, (2, 2, 1500, 128)),
         dict(mask_kind=CAUSAL)),
        (rnd(30, 0, (1, 3, 2100, 128)), rnd(30, 1, (1, 1, 2100, 128)), rnd(30, 2, (1, 1, 2100, 128)),
         dict(mask_kind=SLIDING, window=500, n_sink=2)),
    ]
    serial = []
    for q, k, v, kw in cases:
        serial.append(A.attn_fwd(q, k, v, **kw))
        serial.append(A.attn_fwd(q, k, v, **kw))  # same stream, counter reused at once
    for i in range(0, len(serial), 2):
        assert torch.equal(serial[i][0], serial[i + 1][0])
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    torch.cuda.synchronize()
    outs = [[], []]
    for rep in range(4):
        for si, (q, k, v, kw) in enumerate(cases):
            with torch.cuda.stream(streams[si]):
                outs[si].append(A.attn_fwd(q, k, v, stream=streams[si], **kw))
    torch.cuda.synchronize()
    for si in range(2):
        ref_o, ref_l = serial[2 * si]
        for o, l in outs[si]:
            assert torch.equal(o, ref_o) and torch.equal(l, ref_l)
    assert A.attn_get_device_error() == 0


def test_backward_on_concurrent_streams_matches_serial():
    """The persistent backward kernels share the per-stream work counter with the prefill: two
    backward calls queued on two streams at once give the same bits as serial calls."""
    cases = []
    for seed, shape_q, shape_kv, kw in ((31, (1, 4, 700, 128), (1, 2, 700, 128), dict(mask_kind=CAUSAL)),
                                        (32, (2, 2, 500, 128), (2, 1, 500, 128),
                                         dict(mask_kind=SLIDING, window=200, n_sink=3))):
        q, k, v = rnd(seed, 0, shape_q), rnd(seed, 1, shape_kv), rnd(seed, 2, shape_kv)
        do = rnd(seed, 3, shape_q)
        o, lse = A.attn_fwd(q, k, v, **kw)
        cases.append((q, k, v, o, lse, do, kw))
    serial = [A.attn_bwd(q, k, v, o, lse, do, **kw) for q, k, v, o, lse, do, kw in cases]
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    torch.cuda.synchronize()
    outs = [[], []]
    for rep in range(3):
        for si, (q, k, v, o, lse, do, kw) in enumerate(cases):
            with torch.cuda.stream(streams[si]):
                outs[si].append(A.attn_bwd(q, k, v, o, lse, do, stream=streams[si], **kw))
    torch.cuda.synchronize()
    for si in range(2):
        for got in outs[si]:
            for x, y in zip(got, serial[si]):
                assert torch.equal(x, y)
    assert A.attn_get_device_error() == 0


def test_bounded_wait_reports_timeout_and_context_survives():
    assert A.attn_get_device_error() == 0
    A.attn_debug_timeout_probe(2_000_000)  # ~1 ms of SM clocks on an mbarrier nobody completes
    assert A.attn_get_device_error() == A.ATTN_ERR_DEVICE_TIMEOUT
    assert A.attn_get_device_error() == 0  # read-and-clear
    q, k, v = rnd(28, 0, (1, 1, 256, 128)), rnd(28, 1, (1, 1, 256, 128)), rnd(28, 2, (1, 1, 256, 128))
    o, _ = A.attn_fwd(q, k, v, mask_kind=CAUSAL)
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all()
