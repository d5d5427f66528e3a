"""GPU parity of packed variable-length attention (cu_seqlens): every sequence of the packed batch
against the fp64 oracle on its own slice, rows outside every sequence left untouched, and
agreement with the dense entry point when all sequences have the same length."""

import math

import numpy as np
import pytest
import torch

import synth
from exact_io_aware_82_b200 import attn as A
from exact_io_aware_82_b200 import build as Bld
from oracle import oracle as O

from ._parity import TOL_BF16, assert_close, to64

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


def packed(seed, lens_q, lens_k, Hq, Hkv, d=128, lead=0):
    """Packed bf16 tensors drawn on the host; ``lead`` rows before the first sequence."""
    cu_q = np.concatenate([[lead], lead + np.cumsum(lens_q)]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum(lens_k)]).astype(np.int32)
    tq, tk = int(cu_q[-1]), int(cu_k[-1])
    dev, host = [], []
    for tid, shape in ((synth.Q_ID, (tq, Hq, d)), (synth.K_ID, (tk, Hkv, d)), (synth.V_ID, (tk, Hkv, d))):
        bits = synth.normal_bf16_bits(seed, tid, shape)
        host.append(synth.bf16_bits_to_f32(bits).astype(np.float64))
        dev.append(torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).cuda())
    return dev, host, cu_q, cu_k


def check_against_oracle(o, lse, host, cu_q, cu_k, mask, w, s, what):
    q64, k64, v64 = host
    og, lg = to64(o), to64(lse)
    d = q64.shape[-1]
    for i in range(len(cu_q) - 1):
        a, b = cu_q[i], cu_q[i + 1]
        ka, kb = cu_k[i], cu_k[i + 1]
        if b == a:
            continue
        qs = q64[a:b].transpose(1, 0, 2)[None]   # [1, Hq, Nq_s, d]
        ks = k64[ka:kb].transpose(1, 0, 2)[None]
        vs = v64[ka:kb].transpose(1, 0, 2)[None]
        if kb == ka:
            ro = np.zeros_like(qs)
            rl = np.full(qs.shape[:3], -np.inf)
        else:
            ro, rl = O.attention(qs, ks, vs, mask, w, s, scale=1 / math.sqrt(d))
        assert_close(og[a:b].transpose(1, 0, 2)[None], lg[a:b].T[None], ro, rl, TOL_BF16,
                     "%s seq %d (Nq=%d, Nk=%d)" % (what, i, b - a, kb - ka))


CASES = [
    # lens_q, lens_k (None = same), Hq, Hkv, mask, window, n_sink
    ([1, 127, 128, 129, 300], None, 2, 1, CAUSAL, 0, 0),
    ([513, 0, 64, 1000, 255], None, 4, 2, CAUSAL, 0, 0),
    ([200, 700, 33], [500, 700, 90], 4, 1, CAUSAL, 0, 0),
    ([700, 129, 1100], None, 2, 2, SLIDING, 200, 4),
    ([300, 600], None, 4, 1, SLIDING, 1, 0),
    ([100, 257, 400], [300, 257, 50], 2, 1, FULL, 0, 0),
]


@pytest.mark.parametrize("lens_q,lens_k,Hq,Hkv,mask,w,s", CASES)
def test_varlen_against_oracle(lens_q, lens_k, Hq, Hkv, mask, w, s):
    lens_k = lens_q if lens_k is None else lens_k
    (q, k, v), host, cu_q, cu_k = packed(31, lens_q, lens_k, Hq, Hkv)
    o, lse = A.attn_fwd_varlen(q, k, v, torch.from_numpy(cu_q).cuda(), torch.from_numpy(cu_k).cuda(),
                               max(lens_q), mask_kind=mask, window=w, n_sink=s)
    torch.cuda.synchronize()
    check_against_oracle(o, lse, host, cu_q, cu_k, mask, w, s, "varlen")


def test_rows_outside_sequences_are_untouched():
    lens = [150, 90]
    (q, k, v), host, cu_q, cu_k = packed(32, lens, lens, 2, 1, lead=7)
    o = torch.full_like(q, 5.0)
    lse = torch.full((q.shape[0], q.shape[1]), 5.0, device="cuda")
    A.attn_fwd_varlen(q, k, v, torch.from_numpy(cu_q).cuda(), torch.from_numpy(cu_k).cuda(),
                      max(lens), o=o, lse=lse, mask_kind=CAUSAL)
    torch.cuda.synchronize()
    assert torch.all(o[:7] == 5.0) and torch.all(lse[:7] == 5.0)
    check_against_oracle(o, lse, host, cu_q, cu_k, CAUSAL, 0, 0, "lead rows")


@pytest.mark.parametrize("mask,w,s", [(CAUSAL, 0, 0), (SLIDING, 300, 4)])
def test_varlen_equals_dense_for_equal_lengths(mask, w, s):
    B, Hq, Hkv, N, d = 3, 4, 2, 777, 128
    qd = synth.normal_torch(33, synth.Q_ID, (B, Hq, N, d), device="cuda")
    kd = synth.normal_torch(33, synth.K_ID, (B, Hkv, N, d), device="cuda")
    vd = synth.normal_torch(33, synth.V_ID, (B, Hkv, N, d), device="cuda")
    od, ld = A.attn_fwd(qd, kd, vd, mask_kind=mask, window=w, n_sink=s)
    pack = lambda t: t.permute(0, 2, 1, 3).reshape(B * N, t.shape[1], d).contiguous()  # noqa: E731
    cu = torch.arange(0, (B + 1) * N, N, dtype=torch.int32, device="cuda")
    ov, lv = A.attn_fwd_varlen(pack(qd), pack(kd), pack(vd), cu, cu, N, mask_kind=mask, window=w,
                               n_sink=s)
    torch.cuda.synchronize()
    assert torch.equal(ov, pack(od))
    assert torch.equal(lv, ld.permute(0, 2, 1).reshape(B * N, Hq))
