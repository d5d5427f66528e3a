"""attn_decode_noalloc: the decode entry point for callers that cannot allocate device memory.

Such callers (code whose device memory is owned and budgeted up front by a framework or pool
allocator, code that must not risk the device-wide synchronisation an allocation can cause, or
a plugin handed tensors but no allocator) cannot provide attn_decode's workspace; this variant
keeps the split partials in a fixed array inside the library.  The test calls it through the C
ABI twice in a row, on different inputs, and checks each result against the allocating entry
point attn_decode on the same inputs (and the first one also against the fp64 oracle); it also
checks that a call leaves the device's free memory unchanged.  The file is named to be
collected last.
"""

import ctypes
import math

import pytest
import torch

import synth
from exact_io_aware_82_b200 import attn as A
from exact_io_aware_82_b200 import build as Bld
from oracle import oracle as O

from ._parity import TOL_BF16, assert_close, to64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    Bld.build()
    return A.lib()


def _inputs(seed, B, Hq, Hkv, Nk, d=128):
    q = synth.normal_torch(seed, synth.Q_ID, (B, Hq, 1, d), device="cuda")
    k = synth.normal_torch(seed, synth.K_ID, (B, Hkv, Nk, d), device="cuda")
    v = synth.normal_torch(seed, synth.V_ID, (B, Hkv, Nk, d), device="cuda")
    return q, k, v


def _noalloc(lib, q, k, v, o, lse, num_splits=0):
    B, Hq, _, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    p = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    return lib.attn_decode_noalloc(p(q), p(k), p(v), p(o), p(lse), B, Hq, Hkv, Nk, d,
                                   1.0 / math.sqrt(d), num_splits,
                                   ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_noalloc_decode_matches_decode_on_two_calls_in_a_row(lib):
    # two different problems back to back: the second call must not depend on what the first
    # left in the shared scratch array
    for seed, (B, Hq, Hkv, Nk) in ((41, (8, 32, 8, 6000)), (42, (3, 16, 2, 9001))):
        q, k, v = _inputs(seed, B, Hq, Hkv, Nk)
        o = torch.full_like(q, 7.0)
        lse = torch.full((B, Hq), 7.0, dtype=torch.float32, device="cuda")
        assert _noalloc(lib, q, k, v, o, lse) == A.ATTN_OK
        ref_o, ref_lse = A.attn_decode(q, k, v)
        torch.cuda.synchronize()
        assert_close(to64(o), to64(lse), to64(ref_o), to64(ref_lse), TOL_BF16,
                     "noalloc vs decode (seed %d)" % seed)
        if seed == 41:
            ro, rl = O.attention(to64(q[:1]), to64(k[:1]), to64(v[:1]), O.MASK_FULL,
                                 scale=1 / math.sqrt(128))
            assert_close(to64(o[:1]), to64(lse[:1]), ro, rl.reshape(1, Hq), TOL_BF16,
                         "noalloc vs oracle")
    assert A.attn_get_device_error() == 0


def test_noalloc_decode_leaves_free_device_memory_unchanged(lib):
    q, k, v = _inputs(44, 4, 32, 8, 5000)
    o = torch.empty_like(q)
    lse = torch.empty((4, 32), dtype=torch.float32, device="cuda")
    assert _noalloc(lib, q, k, v, o, lse) == A.ATTN_OK  # warm-up: module and context set-up
    torch.cuda.synchronize()
    free_before, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        assert _noalloc(lib, q, k, v, o, lse) == A.ATTN_OK
    torch.cuda.synchronize()
    free_after, _ = torch.cuda.mem_get_info()
    assert free_after == free_before, (free_before, free_after)


def test_noalloc_rejects_requests_beyond_its_array(lib):
    # the partials of 64 x 32 heads over 256 splits need far more than the fixed array
    B, Hq, Hkv, Nk = 64, 32, 8, 4096
    need = A.attn_decode_workspace_bytes(B, Hq, Hkv, Nk, 128, 256)
    assert need > A.DECODE_NOALLOC_MAX_BYTES
    q, k, v = _inputs(43, B, Hq, Hkv, Nk)
    o = torch.full_like(q, 7.0)
    lse = torch.full((B, Hq), 7.0, dtype=torch.float32, device="cuda")
    assert _noalloc(lib, q, k, v, o, lse, num_splits=256) == A.ATTN_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.all(o == 7.0) and torch.all(lse == 7.0)  # nothing was launched
    with pytest.raises(A.AttnError):
        A.attn_decode_noalloc(q, k, v, num_splits=256)
