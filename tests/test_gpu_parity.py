"""GPU parity: the CUDA kernels (through the C ABI) against the fp64 oracle on the same seeded
inputs.  Small cases compare every output element; the benchmark workloads at full size
compare sampled rows (whole heads plus structural and random rows) that the oracle computes
one by one."""

import math

import numpy as np
import pytest
import torch

import synth
from exact_io_aware_82_b200 import attn as A
from exact_io_aware_82_b200 import build as Bld
from oracle import oracle as O

from ._parity import (TOL_BF16, TOL_F32, assert_close, bf16_inputs, f32_inputs,
                      oracle_rows_one_head, sample_rows, to64)

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


# ------------------------------------------------------------------------------------------
# fp32 path (the single-head full-attention workload, n = 256, d = 64)
# ------------------------------------------------------------------------------------------
def test_fp32_single_head_full_workload():
    (q, k, v), (q64, k64, v64) = f32_inputs(1, 1, 1, 1, 256, 256, 64)
    o, lse = A.attn_fwd_f32(q, k, v, mask_kind=FULL)
    ro, rl = O.attention(q64, k64, v64, FULL, scale=1 / 8.0)
    assert_close(to64(o), to64(lse), ro, rl, TOL_F32, "fp32 n=256 d=64 full")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("Nq,Nk,mask,w,s,Hq,Hkv", [
    (1, 1, FULL, 0, 0, 1, 1), (33, 33, CAUSAL, 0, 0, 2, 1), (70, 150, CAUSAL, 0, 0, 4, 2),
    (150, 70, CAUSAL, 0, 0, 2, 2), (129, 129, SLIDING, 17, 3, 4, 1), (100, 100, SLIDING, 1, 0, 1, 1),
    (65, 200, FULL, 0, 0, 8, 2),
    # more than 512 keys: the tiled fp32 kernel (up to 512, the one with K/V in shared memory)
    (40, 700, SLIDING, 100, 2, 2, 1), (30, 600, FULL, 0, 0, 2, 2)])
def test_fp32_masks(d, Nq, Nk, mask, w, s, Hq, Hkv):
    (q, k, v), (q64, k64, v64) = f32_inputs(5, 2, Hq, Hkv, Nq, Nk, d)
    o, lse = A.attn_fwd_f32(q, k, v, mask_kind=mask, window=w, n_sink=s)
    ro, rl = O.attention(q64, k64, v64, mask, w, s, scale=1 / math.sqrt(d))
    assert_close(to64(o), to64(lse), ro, rl, TOL_F32, "fp32 %s" % ((d, Nq, Nk, mask, w, s),))


# ------------------------------------------------------------------------------------------
# bf16 tensor-core path: small shapes spanning several tiles and ragged tails
# ------------------------------------------------------------------------------------------
SMALL = [
    # Nq, Nk, mask, window, n_sink, Hq, Hkv
    (1, 1, FULL, 0, 0, 1, 1),
    (2, 2, CAUSAL, 0, 0, 1, 1),
    (3, 3, FULL, 0, 0, 2, 1),
    (127, 127, CAUSAL, 0, 0, 2, 2),
    (128, 128, CAUSAL, 0, 0, 2, 1),
    (129, 129, CAUSAL, 0, 0, 1, 1),
    (255, 255, FULL, 0, 0, 2, 2),
    (256, 256, CAUSAL, 0, 0, 4, 1),
    (257, 257, CAUSAL, 0, 0, 4, 4),
    (300, 300, FULL, 0, 0, 8, 1),
    (513, 513, CAUSAL, 0, 0, 4, 1),
    (100, 300, CAUSAL, 0, 0, 2, 1),
    (300, 100, CAUSAL, 0, 0, 2, 1),
    (200, 700, FULL, 0, 0, 4, 2),
    (700, 700, SLIDING, 1, 0, 2, 1),
    (700, 700, SLIDING, 128, 0, 2, 1),
    (700, 700, SLIDING, 129, 4, 2, 1),
    (700, 700, SLIDING, 200, 1, 4, 1),
    (700, 700, SLIDING, 1000, 0, 2, 2),
    (1000, 1000, SLIDING, 256, 130, 2, 1),
    (900, 1100, SLIDING, 300, 4, 4, 1),
    (1100, 900, SLIDING, 300, 4, 2, 1),
]


@pytest.mark.parametrize("Nq,Nk,mask,w,s,Hq,Hkv", SMALL)
def test_bf16_small(Nq, Nk, mask, w, s, Hq, Hkv):
    (q, k, v), (q64, k64, v64) = bf16_inputs(7, 2, Hq, Hkv, Nq, Nk, 128)
    o, lse = A.attn_fwd(q, k, v, mask_kind=mask, window=w, n_sink=s)
    ro, rl = O.attention(q64, k64, v64, mask, w, s, scale=1 / math.sqrt(128))
    assert_close(to64(o), to64(lse), ro, rl, TOL_BF16, "bf16 %s" % ((Nq, Nk, mask, w, s, Hq, Hkv),))


@pytest.mark.parametrize("scale", [0.0, -0.2, 0.5])
def test_bf16_other_scales(scale):
    (q, k, v), (q64, k64, v64) = bf16_inputs(8, 1, 2, 1, 300, 300, 128)
    o, lse = A.attn_fwd(q, k, v, mask_kind=CAUSAL, scale=scale)
    ro, rl = O.attention(q64, k64, v64, CAUSAL, scale=scale)
    assert_close(to64(o), to64(lse), ro, rl, TOL_BF16, "scale %g" % scale)


def test_bf16_without_lse_output():
    (q, k, v), (q64, k64, v64) = bf16_inputs(9, 1, 2, 2, 200, 200, 128)
    o, lse = A.attn_fwd(q, k, v, mask_kind=CAUSAL, return_lse=False)
    assert lse is None
    ro, _ = O.attention(q64, k64, v64, CAUSAL, scale=1 / math.sqrt(128))
    assert_close(to64(o), None, ro, None, TOL_BF16, "no lse")


# ------------------------------------------------------------------------------------------
# empty and degenerate inputs
# ------------------------------------------------------------------------------------------
def test_empty_inputs():
    dev = "cuda"
    z = lambda *s: torch.zeros(s, dtype=torch.bfloat16, device=dev)  # noqa: E731
    o, lse = A.attn_fwd(z(2, 2, 0, 128), z(2, 2, 5, 128), z(2, 2, 5, 128))
    assert o.shape == (2, 2, 0, 128) and lse.shape == (2, 2, 0)
    o, lse = A.attn_fwd(z(0, 2, 5, 128), z(0, 2, 5, 128), z(0, 2, 5, 128))
    assert o.numel() == 0
    q = torch.ones(1, 2, 7, 128, dtype=torch.bfloat16, device=dev)
    o = torch.full_like(q, 3.0)
    o, lse = A.attn_fwd(q, z(1, 1, 0, 128), z(1, 1, 0, 128), o=o)
    assert torch.all(o == 0) and torch.all(lse == -math.inf)
    qf = torch.ones(1, 1, 3, 64, device=dev)
    o, lse = A.attn_fwd_f32(qf, torch.zeros(1, 1, 0, 64, device=dev), torch.zeros(1, 1, 0, 64, device=dev))
    assert torch.all(o == 0) and torch.all(lse == -math.inf)
    torch.cuda.synchronize()


def test_rows_without_visible_keys():
    # Nq > Nk with a causal mask: the first Nq - Nk rows see no key at all
    (q, k, v), (q64, k64, v64) = bf16_inputs(10, 1, 2, 1, 400, 150, 128)
    o, lse = A.attn_fwd(q, k, v, mask_kind=CAUSAL)
    ro, rl = O.attention(q64, k64, v64, CAUSAL, scale=1 / math.sqrt(128))
    assert np.all(rl[:, :, :250] == -np.inf)
    assert_close(to64(o), to64(lse), ro, rl, TOL_BF16, "empty rows")
    assert torch.all(o[:, :, :250] == 0)


# ------------------------------------------------------------------------------------------
# the benchmark workloads at full size, in the launch configuration the benchmark times
# ------------------------------------------------------------------------------------------
def _full_size_check(seed, B, Hq, Hkv, N, mask, w, s, whole_heads, n_random, structural):
    d = 128
    G = Hq // Hkv
    q = synth.normal_torch(seed, synth.Q_ID, (B, Hq, N, d), device="cuda")
    k = synth.normal_torch(seed, synth.K_ID, (B, Hkv, N, d), device="cuda")
    v = synth.normal_torch(seed, synth.V_ID, (B, Hkv, N, d), device="cuda")
    o, lse = A.attn_fwd(q, k, v, mask_kind=mask, window=w, n_sink=s)
    torch.cuda.synchronize()
    scale = 1 / math.sqrt(d)
    worst = []
    for (b, h) in sorted(set(whole_heads) | {(b, h) for b in range(B) for h in range(Hq)}):
        rows = (np.arange(N) if (b, h) in whole_heads
                else sample_rows(N, n_random, structural, seed=b * 1000 + h))
        hk = h // G
        q_rows = to64(q[b, h][torch.from_numpy(rows).cuda()])
        ro, rl = oracle_rows_one_head(q_rows, rows, to64(k[b, hk]), to64(v[b, hk]), N, mask, w,
                                      s, scale)
        og = to64(o[b, h][torch.from_numpy(rows).cuda()])
        lg = to64(lse[b, h][torch.from_numpy(rows).cuda()])
        worst.append(assert_close(og, lg, ro, rl, TOL_BF16, "(b=%d, h=%d)" % (b, h)))
    return worst


def test_causal_prefill_b4_h16_n2048():
    _full_size_check(2, 4, 16, 16, 2048, CAUSAL, 0, 0, whole_heads=[(0, 0), (3, 15)],
                     n_random=24, structural=(0, 1, 127, 128, 255, 256, 2047))


def test_gqa_causal_prefill_b2_h32_kv8_n8192():
    _full_size_check(3, 2, 32, 8, 8192, CAUSAL, 0, 0, whole_heads=[(0, 0)], n_random=12,
                     structural=(0, 1, 255, 256, 4095, 8191))


def test_sliding_window_prefill_n32768_w4096_sinks4():
    w = 4096
    _full_size_check(4, 1, 32, 8, 32768, SLIDING, w, 4, whole_heads=[(0, 31)], n_random=12,
                     structural=(0, 1, 3, 4, 5, w - 1, w, w + 1, w + 2, w + 3, w + 4, 2 * w,
                                 32767))


# ------------------------------------------------------------------------------------------
# split-K decode
# ------------------------------------------------------------------------------------------
@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("Nk,splits", [(1, 0), (5, 0), (127, 3), (128, 0), (129, 2), (1000, 7),
                                        (4097, 0), (4097, 1), (20000, 0)])
def test_decode_small(G, Nk, splits):
    B, Hkv = 3, 2
    Hq = G * Hkv
    (q, k, v), (q64, k64, v64) = bf16_inputs(11, B, Hq, Hkv, 1, Nk, 128)
    o, lse = A.attn_decode(q, k, v, num_splits=splits)
    ro, rl = O.attention(q64, k64, v64, FULL, scale=1 / math.sqrt(128))
    assert_close(to64(o), to64(lse), ro, rl.reshape(B, Hq), TOL_BF16, "decode G=%d Nk=%d" % (G, Nk))


def test_decode_b64_h32_kv8_n32768():
    B, Hq, Hkv, Nk, d = 64, 32, 8, 32768, 128
    q = synth.normal_torch(5, synth.Q_ID, (B, Hq, 1, d), device="cuda")
    k = synth.normal_torch(5, synth.K_ID, (B, Hkv, Nk, d), device="cuda")
    v = synth.normal_torch(5, synth.V_ID, (B, Hkv, Nk, d), device="cuda")
    o, lse = A.attn_decode(q, k, v)
    torch.cuda.synchronize()
    for b in (0, 17, 63):
        ro, rl = O.attention(to64(q[b:b + 1]), to64(k[b:b + 1]), to64(v[b:b + 1]), FULL,
                             scale=1 / math.sqrt(d))
        assert_close(to64(o[b:b + 1]), to64(lse[b:b + 1]), ro, rl.reshape(1, Hq), TOL_BF16,
                     "decode b=%d" % b)
