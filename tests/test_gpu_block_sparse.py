"""GPU parity of the block-sparse forward (attn_fwd_block_sparse) against the fp64 oracle.

Layouts are seeded random selections of 128 x 128 blocks (one per head, or one shared by every
head), on top of every base mask, with GQA, Nq != Nk both ways and ragged tails; the oracle is
oracle_attn_block_sparse on the same bf16 inputs and the same layout.  Also: every block
selected gives attn_fwd's result bit for bit (the same steps in the same order); no block
selected gives O = 0, LSE = -inf; a shared layout equals per-head copies of it; and the
benchmark's workload, checked on sampled rows against the dense oracle over the keys of the
row's selected blocks (a full base mask makes that the whole visible set).
"""

import math

import numpy as np
import pytest
import torch

import synth
from exact_io_aware_82_b200 import accounting as acc
from exact_io_aware_82_b200 import attn as A
from exact_io_aware_82_b200 import build as Bld
from oracle import oracle as O

from ._parity import TOL_BF16, assert_close, bf16_inputs, to64

pytestmark = pytest.mark.gpu
FULL, CAUSAL, SLIDING, LOCAL = A.MASK_FULL, A.MASK_CAUSAL, A.MASK_SLIDING, A.MASK_LOCAL_GLOBAL


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    Bld.build()
    A.lib()
    yield
    assert A.attn_get_device_error() == 0


def random_layout(seed, heads, Nq, Nk, density):
    r = np.random.default_rng(seed)
    return (r.random((heads, -(-Nq // 128), -(-Nk // 128))) < density).astype(np.uint8)


CASES = [
    # B, Hq, Hkv, Nq, Nk, mask, window, n_sink, layout heads (1 = shared), density
    (1, 2, 1, 300, 300, FULL, 0, 0, 1, 0.5),
    (2, 4, 2, 513, 513, CAUSAL, 0, 0, 4, 0.5),
    (1, 2, 2, 200, 450, CAUSAL, 0, 0, 2, 0.6),
    (1, 2, 2, 450, 200, CAUSAL, 0, 0, 1, 0.6),
    (1, 4, 1, 700, 700, SLIDING, 200, 4, 4, 0.5),
    (1, 2, 1, 640, 640, LOCAL, 100, 3, 2, 0.4),
    (1, 8, 1, 257, 333, FULL, 0, 0, 8, 0.3),
    (1, 2, 2, 1100, 1100, CAUSAL, 0, 0, 2, 0.15),
]


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nk,mask,w,s,heads,density", CASES)
def test_block_sparse_against_oracle(B, Hq, Hkv, Nq, Nk, mask, w, s, heads, density):
    (q, k, v), (q64, k64, v64) = bf16_inputs(101, B, Hq, Hkv, Nq, Nk, 128)
    bm = random_layout(Nq * 7 + Nk, heads, Nq, Nk, density)
    o, lse = A.attn_fwd_block_sparse(q, k, v, torch.from_numpy(bm).cuda(), mask_kind=mask,
                                     window=w, n_sink=s)
    torch.cuda.synchronize()
    ro, rl = O.attention_block_sparse(q64, k64, v64, bm, mask, w, s, 1 / math.sqrt(128))
    assert_close(to64(o), to64(lse), ro, rl, TOL_BF16,
                 "block-sparse %s" % ((B, Hq, Hkv, Nq, Nk, mask, w, s, heads, density),))


@pytest.mark.parametrize("mask,w,s", [(CAUSAL, 0, 0), (SLIDING, 300, 4), (LOCAL, 200, 2), (FULL, 0, 0)])
def test_every_block_selected_is_attn_fwd_bit_for_bit(mask, w, s):
    (q, k, v), _ = bf16_inputs(102, 2, 4, 2, 777, 777, 128)
    bm = torch.ones((1, 7, 7), dtype=torch.uint8, device="cuda")
    o1, l1 = A.attn_fwd_block_sparse(q, k, v, bm, mask_kind=mask, window=w, n_sink=s)
    o2, l2 = A.attn_fwd(q, k, v, mask_kind=mask, window=w, n_sink=s)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_no_block_selected_gives_empty_rows():
    (q, k, v), _ = bf16_inputs(103, 1, 2, 1, 300, 400, 128)
    bm = torch.zeros((2, 3, 4), dtype=torch.uint8, device="cuda")
    bm[1, 1, 2] = 1  # one block of head 1: rows 128..255 see keys 256..383
    o, lse = A.attn_fwd_block_sparse(q, k, v, bm)
    torch.cuda.synchronize()
    assert torch.all(o[:, 0] == 0) and torch.all(torch.isneginf(lse[:, 0]))
    assert torch.all(o[:, 1, :128] == 0) and torch.all(o[:, 1, 256:] == 0)
    assert torch.all(torch.isfinite(lse[:, 1, 128:256]))


def test_shared_layout_equals_per_head_copies():
    (q, k, v), _ = bf16_inputs(104, 1, 4, 2, 600, 600, 128)
    bm = torch.from_numpy(random_layout(104, 1, 600, 600, 0.5)).cuda()
    o1, l1 = A.attn_fwd_block_sparse(q, k, v, bm, mask_kind=CAUSAL)
    o2, l2 = A.attn_fwd_block_sparse(q, k, v, bm.expand(4, -1, -1).contiguous(), mask_kind=CAUSAL)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_block_sparse_b1_h32_kv8_n32768_sampled():
    B, Hq, Hkv, N, d = 1, 32, 8, 32768, 128
    q = synth.normal_torch(11, 0, (B, Hq, N, d), device="cuda")
    k = synth.normal_torch(11, 1, (B, Hkv, N, d), device="cuda")
    v = synth.normal_torch(11, 2, (B, Hkv, N, d), device="cuda")
    bm = synth.block_layout_bigbird(11, N // 128, N // 128)
    o, lse = A.attn_fwd_block_sparse(q, k, v, torch.from_numpy(bm).cuda())
    torch.cuda.synchronize()
    assert acc.block_sparse_pairs(bm, N, N, FULL, Hq=Hq) > 0
    r = np.random.default_rng(12)
    rows = [(int(h), int(i)) for h, i in zip(r.integers(0, Hq, 24), r.integers(0, N, 24))]
    rows += [(0, 0), (31, N - 1), (5, 128), (7, 127)]
    for h, i in rows:
        sel = np.nonzero(bm[0, i // 128])[0]
        keys = torch.from_numpy(np.concatenate([np.arange(t * 128, (t + 1) * 128) for t in sel])).cuda()
        g = h // (Hq // Hkv)
        qi = to64(q[:, h:h + 1, i:i + 1])
        ks, vs = to64(k[:, g:g + 1, keys]), to64(v[:, g:g + 1, keys])
        ro, rl = O.attention(qi, ks, vs, FULL, scale=1 / math.sqrt(d))
        assert_close(to64(o[:, h:h + 1, i:i + 1]), to64(lse[:, h:h + 1, i:i + 1]), ro, rl,
                     TOL_BF16, "row (h %d, i %d)" % (h, i))
