"""GPU parity of the local + global mask (bidirectional window of w keys on each side, the first
n_global tokens global) against the fp64 oracle: bf16 and fp32 forward, packed sequences,
backward, and the full-size n = 32768 workload on sampled rows."""

import math

import numpy as np
import pytest
import torch

import synth
from exact_io_aware_82_b200 import attn as A
from exact_io_aware_82_b200 import build as Bld
from oracle import oracle as O

from ._parity import TOL_BF16, TOL_F32, assert_close, bf16_inputs, f32_inputs, to64
from .test_gpu_bwd import grad_close
from .test_gpu_parity import _full_size_check
from .test_gpu_varlen import check_against_oracle, packed

pytestmark = pytest.mark.gpu
LOCAL = A.MASK_LOCAL_GLOBAL


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    Bld.build()
    A.lib()
    yield
    assert A.attn_get_device_error() == 0


CASES = [
    # Nq, Nk, window, n_global, Hq, Hkv
    (300, 300, 0, 0, 2, 1),       # the diagonal only
    (300, 300, 1, 0, 2, 1),
    (700, 700, 64, 1, 2, 1),
    (700, 700, 128, 4, 4, 1),
    (700, 700, 200, 130, 2, 2),   # global tokens spanning more than a tile
    (1000, 1000, 300, 4, 2, 1),
    (900, 1100, 100, 4, 2, 1),    # Nq < Nk
    (1100, 900, 100, 4, 2, 1),    # Nq > Nk: rows before the first key position
    (513, 513, 2000, 0, 2, 1),    # the window covers every key: full attention
    (256, 256, 3, 300, 2, 1),     # every token global: full attention
]


@pytest.mark.parametrize("Nq,Nk,w,g,Hq,Hkv", CASES)
def test_local_global_bf16(Nq, Nk, w, g, Hq, Hkv):
    (q, k, v), (q64, k64, v64) = bf16_inputs(91, 2, Hq, Hkv, Nq, Nk, 128)
    o, lse = A.attn_fwd(q, k, v, mask_kind=LOCAL, window=w, n_sink=g)
    ro, rl = O.attention(q64, k64, v64, LOCAL, w, g, scale=1 / math.sqrt(128))
    assert_close(to64(o), to64(lse), ro, rl, TOL_BF16, "local+global %s" % ((Nq, Nk, w, g),))


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("Nq,Nk,w,g,Hq,Hkv", [(129, 129, 17, 3, 4, 1), (100, 140, 5, 2, 2, 2),
                                              (140, 100, 0, 1, 2, 1)])
def test_local_global_fp32(d, Nq, Nk, w, g, Hq, Hkv):
    (q, k, v), (q64, k64, v64) = f32_inputs(92, 2, Hq, Hkv, Nq, Nk, d)
    o, lse = A.attn_fwd_f32(q, k, v, mask_kind=LOCAL, window=w, n_sink=g)
    ro, rl = O.attention(q64, k64, v64, LOCAL, w, g, scale=1 / math.sqrt(d))
    assert_close(to64(o), to64(lse), ro, rl, TOL_F32, "fp32 local+global %s" % ((d, Nq, Nk, w, g),))


def test_local_global_packed_sequences():
    lens = [300, 700, 129, 1]
    (q, k, v), host, cu_q, cu_k = packed(93, lens, lens, 4, 2)
    o, lse = A.attn_fwd_varlen(q, k, v, torch.from_numpy(cu_q).cuda(), torch.from_numpy(cu_k).cuda(),
                               max(lens), mask_kind=LOCAL, window=64, n_sink=2)
    torch.cuda.synchronize()
    check_against_oracle(o, lse, host, cu_q, cu_k, LOCAL, 64, 2, "varlen local+global")


@pytest.mark.parametrize("Nq,Nk,w,g,Hq,Hkv", [(700, 700, 64, 2, 4, 1), (300, 450, 50, 1, 2, 2),
                                              (450, 300, 30, 0, 2, 2), (513, 513, 0, 130, 2, 1),
                                              (1100, 900, 100, 4, 2, 1)])
def test_local_global_backward(Nq, Nk, w, g, Hq, Hkv):
    d = 128
    (q, k, v), (q64, k64, v64) = bf16_inputs(94, 1, Hq, Hkv, Nq, Nk, d)
    bits = synth.normal_bf16_bits(94, synth.DO_ID, (1, Hq, Nq, d))
    do64 = synth.bf16_bits_to_f32(bits).astype(np.float64)
    do = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).cuda()
    o, lse = A.attn_fwd(q, k, v, mask_kind=LOCAL, window=w, n_sink=g)
    dq, dk, dv = A.attn_bwd(q, k, v, o, lse, do, mask_kind=LOCAL, window=w, n_sink=g)
    torch.cuda.synchronize()
    rq, rk, rv = O.attention_bwd(q64, k64, v64, do64, LOCAL, w, g, 1 / math.sqrt(d))
    tag = "local+global bwd %s" % ((Nq, Nk, w, g, Hq, Hkv),)
    grad_close(to64(dq), rq, "dq " + tag)
    grad_close(to64(dk), rk, "dk " + tag)
    grad_close(to64(dv), rv, "dv " + tag)


def test_local_global_prefill_n32768_w2048_g4():
    w = 2048
    _full_size_check(9, 1, 32, 8, 32768, LOCAL, w, 4, whole_heads=[(0, 31)], n_random=12,
                     structural=(0, 1, 3, 4, 5, w - 1, w, w + 1, w + 4, w + 5, 16384,
                                 32767 - w, 32767))
