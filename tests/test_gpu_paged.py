"""GPU parity of decode against a paged KV cache: each sequence's keys are gathered from its pages
on the host and the fp64 oracle runs on that contiguous copy; pages are shuffled, shared between
sequences and of several sizes; lengths include 0, 1, page boundaries and ragged tails.  Also:
bitwise agreement with the contiguous decode when the pages are laid out in order, and the
device flag for a page number outside the cache."""

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


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    Bld.build()
    A.lib()
    yield
    assert A.attn_get_device_error() == 0


def bf16_pair(seed, tid, shape):
    bits = synth.normal_bf16_bits(seed, tid, shape)
    host = synth.bf16_bits_to_f32(bits).astype(np.float64)
    dev = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).cuda()
    return dev, host


def make_table(rng, lens, page_size, num_pages, share_prefix=False):
    """Block table [B, max_pages] of distinct shuffled pages (-1 past each sequence's last page);
    with share_prefix, every sequence reuses sequence 0's first page (prefix sharing)."""
    need = [(n + page_size - 1) // page_size for n in lens]
    max_pages = max(max(need), 1)
    perm = rng.permutation(num_pages)
    table = np.full((len(lens), max_pages), -1, dtype=np.int32)
    pos = 0
    for b, m in enumerate(need):
        table[b, :m] = perm[pos:pos + m]
        pos += m
    assert pos <= num_pages
    if share_prefix:
        for b in range(1, len(lens)):
            if need[b] > 0 and need[0] > 0:
                table[b, 0] = table[0, 0]
    return table


def gather(cache64, table, b, n, page_size):
    """Keys 0..n-1 of sequence b as [Hkv, n, d] from the host copy of the cache."""
    rows = [cache64[table[b, j // page_size], j % page_size] for j in range(n)]
    if not rows:
        return np.zeros((cache64.shape[2], 0, cache64.shape[3]))
    return np.stack(rows, axis=1)


def run_case(seed, lens, Hq, Hkv, page_size, share_prefix=False, num_splits=0, extra_pages=3):
    d = 128
    B = len(lens)
    rng = np.random.default_rng(seed)
    num_pages = sum((n + page_size - 1) // page_size for n in lens) + extra_pages
    q, q64 = bf16_pair(seed, synth.Q_ID, (B, Hq, 1, d))
    kc, k64 = bf16_pair(seed, synth.K_ID, (num_pages, page_size, Hkv, d))
    vc, v64 = bf16_pair(seed, synth.V_ID, (num_pages, page_size, Hkv, d))
    table = make_table(rng, lens, page_size, num_pages, share_prefix)
    bt = torch.from_numpy(table).cuda()
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    o, lse = A.attn_decode_paged(q, kc, vc, bt, sl, max(lens), num_splits=num_splits)
    torch.cuda.synchronize()
    og, lg = to64(o), to64(lse)
    for b, n in enumerate(lens):
        kb = gather(k64, table, b, n, page_size)[None]
        vb = gather(v64, table, b, n, page_size)[None]
        if n == 0:
            ro, rl = np.zeros((1, Hq, 1, d)), np.full((1, Hq, 1), -np.inf)
        else:
            ro, rl = O.attention(q64[b:b + 1], kb, vb, O.MASK_FULL, 0, 0, scale=1 / math.sqrt(d))
        assert_close(og[b:b + 1], lg[b:b + 1, :, None], ro, rl, TOL_BF16,
                     "paged seq %d (len %d, page %d)" % (b, n, page_size))


@pytest.mark.parametrize("lens,Hq,Hkv,page_size", [
    ([1, 7, 8, 9, 300, 1024], 8, 8, 8),
    ([5000, 17, 0, 2048], 16, 8, 16),
    ([3000, 4096, 129], 16, 4, 64),
    ([9001, 1, 255, 256, 257], 32, 4, 256),
    ([12000, 600], 8, 1, 32),
])
def test_paged_decode_against_oracle(lens, Hq, Hkv, page_size):
    run_case(51, lens, Hq, Hkv, page_size)


@pytest.mark.parametrize("num_splits", [1, 3, 40])
def test_paged_decode_split_counts(num_splits):
    run_case(52, [2500, 70, 1800], 8, 2, 16, num_splits=num_splits)


def test_paged_decode_shared_prefix_pages():
    run_case(53, [700, 640, 33, 1500], 8, 2, 32, share_prefix=True)


def test_paged_decode_all_lengths_zero():
    run_case(54, [0, 0], 8, 2, 16)


def _paged_vs_contiguous(seed, B, Hq, Hkv, N, ps, splits):
    d = 128
    q = synth.normal_torch(seed, synth.Q_ID, (B, Hq, 1, d), device="cuda")
    k = synth.normal_torch(seed, synth.K_ID, (B, Hkv, N, d), device="cuda")
    v = synth.normal_torch(seed, synth.V_ID, (B, Hkv, N, d), device="cuda")
    oc, lc = A.attn_decode(q, k, v, num_splits=splits)
    npg = N // ps + 1
    to_pages = lambda t: torch.nn.functional.pad(  # noqa: E731
        t.permute(0, 2, 1, 3), (0, 0, 0, 0, 0, npg * ps - N)).reshape(B * npg, ps, Hkv, d).contiguous()
    table = torch.arange(B * npg, dtype=torch.int32, device="cuda").reshape(B, npg)
    sl = torch.full((B,), N, dtype=torch.int32, device="cuda")
    op, lp = A.attn_decode_paged(q, to_pages(k), to_pages(v), table, sl, N, num_splits=splits)
    torch.cuda.synchronize()
    return (oc, lc), (op, lp)


def test_paged_equals_contiguous_decode_bitwise():
    # pages laid out in order (page p = keys [p*ps, (p+1)*ps) of one (b, all heads) slab) give
    # the same keys in the same order; with chunks of more than 1024 keys (6144 / 4 = 1536, a
    # multiple of the paged path's 32-key granularity) both calls run the CUDA-core split
    # kernel on the same chunks, so the results are identical
    (oc, lc), (op, lp) = _paged_vs_contiguous(55, 4, 32, 8, 6144, 16, 4)
    assert torch.equal(op, oc) and torch.equal(lp, lc)


def test_paged_equals_contiguous_tensor_core_decode_bitwise():
    # chunks of at most 1024 keys (6000 / 47 -> 128, already a multiple of 32) and pages of 64
    # keys: both caches go through the tensor-core split kernel, with the same keys in the same
    # tiles, so the results are identical too
    (oc, lc), (op, lp) = _paged_vs_contiguous(57, 4, 32, 8, 6000, 64, 47)
    assert torch.equal(op, oc) and torch.equal(lp, lc)


def test_tensor_core_and_cuda_core_decode_agree():
    # the same problem through both split kernels (chunks of 128 keys vs 1536 keys)
    B, Hq, Hkv, N, d = 2, 16, 4, 6144, 128
    q = synth.normal_torch(58, synth.Q_ID, (B, Hq, 1, d), device="cuda")
    k = synth.normal_torch(58, synth.K_ID, (B, Hkv, N, d), device="cuda")
    v = synth.normal_torch(58, synth.V_ID, (B, Hkv, N, d), device="cuda")
    ot, lt = A.attn_decode(q, k, v, num_splits=48)
    oc, lc = A.attn_decode(q, k, v, num_splits=4)
    torch.cuda.synchronize()
    assert_close(to64(ot), to64(lt), to64(oc), to64(lc), TOL_BF16, "tensor-core vs CUDA-core")


@pytest.mark.parametrize("ps", [16, 64])  # the CUDA-core and the tensor-core split kernels
def test_page_number_outside_cache_is_flagged_not_followed(ps):
    d = 128
    lens = [100, 200]
    npg = (200 + ps - 1) // ps
    q = synth.normal_torch(56, synth.Q_ID, (2, 8, 1, d), device="cuda")
    kc = synth.normal_torch(56, synth.K_ID, (2 * npg + 14, ps, 2, d), device="cuda")
    vc = synth.normal_torch(56, synth.V_ID, (2 * npg + 14, ps, 2, d), device="cuda")
    table = torch.arange(2 * npg, dtype=torch.int32, device="cuda").reshape(2, npg)
    table[1, 1] = 1 << 30  # far outside the pool
    good = table.clone()
    good[1, 1] = 2 * npg + 13
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    o_bad, _ = A.attn_decode_paged(q, kc, vc, table, sl, 200)
    assert A.attn_get_device_error() == A.ATTN_ERR_INVALID_ARG
    assert A.attn_get_device_error() == 0  # reading cleared it
    o_good, _ = A.attn_decode_paged(q, kc, vc, good, sl, 200)
    torch.cuda.synchronize()
    assert torch.equal(o_bad[0], o_good[0])  # the other sequence is unaffected
    assert torch.all(torch.isfinite(o_bad[1].float()))


def test_paged_decode_b64_h32_kv8_n32768_p16():
    # the full paged-decode workload (8.6 GB of cache in 16-key pages, seeded random page order);
    # three sequences checked against the oracle on their gathered keys
    B, Hq, Hkv, N, d, ps = 64, 32, 8, 32768, 128, 16
    per_seq = N // ps
    table = torch.from_numpy(
        np.random.default_rng(7).permutation(B * per_seq).astype(np.int32).reshape(B, per_seq)).cuda()
    q = synth.normal_torch(7, synth.Q_ID, (B, Hq, 1, d), device="cuda")
    kc = synth.normal_torch(7, synth.K_ID, (B * per_seq, ps, Hkv, d), device="cuda")
    vc = synth.normal_torch(7, synth.V_ID, (B * per_seq, ps, Hkv, d), device="cuda")
    sl = torch.full((B,), N, dtype=torch.int32, device="cuda")
    o, lse = A.attn_decode_paged(q, kc, vc, table, sl, N)
    torch.cuda.synchronize()
    for b in (0, 31, 63):
        kb = kc[table[b].long()].reshape(N, Hkv, d).permute(1, 0, 2)[None]
        vb = vc[table[b].long()].reshape(N, Hkv, d).permute(1, 0, 2)[None]
        ro, rl = O.attention(to64(q[b:b + 1]), to64(kb), to64(vb), O.MASK_FULL,
                             scale=1 / math.sqrt(d))
        assert_close(to64(o[b:b + 1]), to64(lse[b:b + 1]), ro, rl.reshape(1, Hq), TOL_BF16,
                     "paged decode b=%d" % b)
