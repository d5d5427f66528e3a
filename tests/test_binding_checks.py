"""Argument checks of the Python binding, on the CPU.

The C ABI takes raw pointers and trusts the sizes it is given, so the binding must refuse any
tensor whose shape, dtype, layout or device does not match what the call will read or write,
before a pointer reaches a kernel.  Every check runs before the library is touched: with CPU
tensors a well-formed call stops at the device check ("CUDA tensors"), a malformed one at the
check that names the bad argument.
"""

import pytest
import torch

from exact_io_aware_82_b200 import attn as A

bf16, f32, i32, u8 = torch.bfloat16, torch.float32, torch.int32, torch.uint8


def t(*shape, dtype=bf16, device="cpu"):
    return torch.zeros(shape, dtype=dtype, device=device)


def raises(exc, match, fn, *args, **kw):
    with pytest.raises(exc, match=match):
        fn(*args, **kw)


def test_well_formed_calls_reach_the_device_check():
    q, k, v = t(2, 8, 5, 128), t(2, 2, 7, 128), t(2, 2, 7, 128)
    raises(ValueError, "CUDA tensors", A.attn_fwd, q, k, v)
    raises(ValueError, "CUDA tensors", A.attn_fwd, q, k, v, o=t(2, 8, 5, 128), lse=t(2, 8, 5, dtype=f32))
    raises(ValueError, "CUDA tensors", A.attn_fwd_f32, t(1, 1, 4, 64, dtype=f32),
           t(1, 1, 0, 64, dtype=f32), t(1, 1, 0, 64, dtype=f32))
    raises(ValueError, "CUDA tensors", A.attn_fwd_fp8, t(2, 8, 5, 128, dtype=u8),
           t(2, 2, 7, 128, dtype=u8), t(2, 2, 7, 128, dtype=u8), t(2, 8, dtype=f32),
           t(2, 2, dtype=f32), t(2, 2, dtype=f32))
    raises(ValueError, "CUDA tensors", A.attn_bwd, q, k, v, t(2, 8, 5, 128), t(2, 8, 5, dtype=f32),
           t(2, 8, 5, 128), dq=t(2, 8, 5, 128), dk=t(2, 2, 7, 128), dv=t(2, 2, 7, 128),
           workspace=t(64, dtype=u8))
    raises(ValueError, "CUDA tensors", A.attn_fwd_varlen, t(9, 4, 128), t(11, 2, 128),
           t(11, 2, 128), t(3, dtype=i32), t(3, dtype=i32), 6)
    raises(ValueError, "CUDA tensors", A.attn_decode, t(3, 8, 1, 128), t(3, 2, 100, 128),
           t(3, 2, 100, 128), o=t(3, 8, 1, 128), lse=t(3, 8, dtype=f32), workspace=t(16, dtype=u8))
    raises(ValueError, "CUDA tensors", A.attn_decode_noalloc, t(3, 8, 1, 128), t(3, 2, 100, 128),
           t(3, 2, 100, 128))
    raises(ValueError, "CUDA tensors", A.attn_decode_paged, t(3, 8, 1, 128), t(10, 16, 2, 128),
           t(10, 16, 2, 128), t(3, 4, dtype=i32), t(3, dtype=i32), 64)
    # empty tensors are well formed too
    raises(ValueError, "CUDA tensors", A.attn_fwd, t(0, 2, 5, 128), t(0, 2, 5, 128), t(0, 2, 5, 128))
    raises(ValueError, "CUDA tensors", A.attn_fwd, t(1, 1, 3, 128), t(1, 1, 0, 128), t(1, 1, 0, 128))


def test_forward_shape_mismatches():
    q, k, v = t(2, 8, 5, 128), t(2, 2, 7, 128), t(2, 2, 7, 128)
    raises(ValueError, "v must have shape", A.attn_fwd, q, k, t(2, 2, 6, 128))  # V shorter than K
    raises(ValueError, "k must have shape", A.attn_fwd, q, t(1, 2, 7, 128), v)  # batch
    raises(ValueError, "k must have shape", A.attn_fwd, q, t(2, 2, 7, 64), v)   # head dim
    raises(ValueError, "o must have shape", A.attn_fwd, q, k, v, o=t(2, 8, 4, 128))
    raises(ValueError, "lse must be a contiguous 3-d", A.attn_fwd, q, k, v, lse=t(2, 8, dtype=f32))
    raises(TypeError, "lse must be", A.attn_fwd, q, k, v, lse=t(2, 8, 5))
    raises(TypeError, "o must be", A.attn_fwd, q, k, v, o=t(2, 8, 5, 128, dtype=f32))
    raises(ValueError, "contiguous", A.attn_fwd, q.transpose(1, 2), k, v)
    raises(TypeError, "q must be", A.attn_fwd, q.float(), k, v)
    raises(ValueError, "o must have shape", A.attn_fwd_f32, q.float(), k.float(), v.float(),
           o=t(2, 8, 5, 64, dtype=f32))


def test_fp8_descale_shapes():
    q, k, v = t(2, 8, 5, 128, dtype=u8), t(2, 2, 7, 128, dtype=u8), t(2, 2, 7, 128, dtype=u8)
    dq, dk = t(2, 8, dtype=f32), t(2, 2, dtype=f32)
    raises(ValueError, "descale_q must have shape", A.attn_fwd_fp8, q, k, v, t(2, 2, dtype=f32), dk, dk)
    raises(ValueError, "descale_k must have shape", A.attn_fwd_fp8, q, k, v, dq, t(2, 8, dtype=f32), dk)
    raises(ValueError, "descale_v must have shape", A.attn_fwd_fp8, q, k, v, dq, dk, t(1, 2, dtype=f32))
    raises(ValueError, "v must have shape", A.attn_fwd_fp8, q, k, t(2, 2, 8, 128, dtype=u8), dq, dk, dk)


def test_backward_shape_mismatches():
    q, k, v = t(2, 8, 5, 128), t(2, 2, 7, 128), t(2, 2, 7, 128)
    o, lse, do = t(2, 8, 5, 128), t(2, 8, 5, dtype=f32), t(2, 8, 5, 128)
    raises(ValueError, "dout must have shape", A.attn_bwd, q, k, v, o, lse, t(2, 8, 4, 128))
    raises(ValueError, "o must have shape", A.attn_bwd, q, k, v, t(2, 8, 5, 64), lse, do)
    raises(ValueError, "lse must have shape", A.attn_bwd, q, k, v, o, t(2, 8, 6, dtype=f32), do)
    raises(ValueError, "dq must have shape", A.attn_bwd, q, k, v, o, lse, do, dq=t(2, 8, 5, 64))
    raises(ValueError, "dk must have shape", A.attn_bwd, q, k, v, o, lse, do, dk=t(2, 8, 7, 128))
    raises(ValueError, "dv must have shape", A.attn_bwd, q, k, v, o, lse, do, dv=t(2, 2, 6, 128))
    raises(TypeError, "workspace must be", A.attn_bwd, q, k, v, o, lse, do, workspace=t(64, dtype=f32))


def test_varlen_and_decode_mismatches():
    q, k, v = t(9, 4, 128), t(11, 2, 128), t(11, 2, 128)
    cu = t(3, dtype=i32)
    raises(ValueError, "cu_seqlens_k must have shape", A.attn_fwd_varlen, q, k, v, cu, t(4, dtype=i32), 6)
    raises(ValueError, "v must have shape", A.attn_fwd_varlen, q, k, t(10, 2, 128), cu, cu, 6)
    raises(ValueError, "k must have shape", A.attn_fwd_varlen, q, t(11, 2, 64), v, cu, cu, 6)
    raises(ValueError, "o must have shape", A.attn_fwd_varlen, q, k, v, cu, cu, 6, o=t(9, 4, 64))
    raises(ValueError, "num_seqs", A.attn_fwd_varlen, q, k, v, t(0, dtype=i32), t(0, dtype=i32), 6)

    qd, kd, vd = t(3, 8, 1, 128), t(3, 2, 100, 128), t(3, 2, 100, 128)
    raises(ValueError, "one query token", A.attn_decode, t(3, 8, 2, 128), kd, vd)
    raises(ValueError, "v must have shape", A.attn_decode, qd, kd, t(3, 2, 99, 128))
    raises(ValueError, "o must be a contiguous 4-d", A.attn_decode, qd, kd, vd, o=t(3, 8, 128))
    raises(ValueError, "lse must have shape", A.attn_decode, qd, kd, vd, lse=t(3, 9, dtype=f32))
    raises(ValueError, "v must have shape", A.attn_decode_noalloc, qd, kd, t(2, 2, 100, 128))

    kc = t(10, 16, 2, 128)
    bt, sl = t(3, 4, dtype=i32), t(3, dtype=i32)
    raises(ValueError, "v_cache must have shape", A.attn_decode_paged, qd, kc, t(10, 8, 2, 128), bt, sl, 64)
    raises(ValueError, "one row per sequence", A.attn_decode_paged, qd, kc, kc, t(2, 4, dtype=i32), sl, 64)
    raises(ValueError, "seq_lens must have shape", A.attn_decode_paged, qd, kc, kc, bt, t(4, dtype=i32), 64)
    raises(ValueError, "k_cache and v_cache", A.attn_decode_paged, qd, t(10, 16, 2, 64), kc, bt, sl, 64)


def test_tensors_on_two_devices_are_refused():
    q, k, v = t(2, 8, 5, 128), t(2, 2, 7, 128), t(2, 2, 7, 128)
    raises(ValueError, "one device", A.attn_fwd, q, k, t(2, 2, 7, 128, device="meta"))
    raises(ValueError, "one device", A.attn_fwd, q, k, v, o=t(2, 8, 5, 128, device="meta"))
    raises(ValueError, "one device", A.attn_decode, t(3, 8, 1, 128), t(3, 2, 100, 128),
           t(3, 2, 100, 128), workspace=t(16, dtype=u8, device="meta"))


def test_block_sparse_layout_checks():
    q, k, v = t(2, 8, 300, 128), t(2, 2, 450, 128), t(2, 2, 450, 128)
    raises(ValueError, "CUDA tensors", A.attn_fwd_block_sparse, q, k, v, t(1, 3, 4, dtype=u8))
    raises(ValueError, "CUDA tensors", A.attn_fwd_block_sparse, q, k, v, t(8, 3, 4, dtype=torch.bool))
    raises(ValueError, "block_mask must have shape", A.attn_fwd_block_sparse, q, k, v, t(1, 3, 3, dtype=u8))
    raises(ValueError, "block_mask must have shape", A.attn_fwd_block_sparse, q, k, v, t(1, 2, 4, dtype=u8))
    raises(ValueError, "1 or Hq", A.attn_fwd_block_sparse, q, k, v, t(2, 3, 4, dtype=u8))
    raises(TypeError, "block_mask must be", A.attn_fwd_block_sparse, q, k, v, t(1, 3, 4, dtype=i32))
    raises(ValueError, "v must have shape", A.attn_fwd_block_sparse, q, k, t(2, 2, 449, 128),
           t(1, 3, 4, dtype=u8))
