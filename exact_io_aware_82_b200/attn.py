"""Thin ctypes binding of libattn.so (the C ABI in include/attn.h).

Argument marshalling only: torch tensors are checked for device, dtype and contiguity and
passed as raw device pointers together with the current CUDA stream; every step of the
computation runs in the library's kernels.  Output and workspace tensors the caller does not
supply are allocated with torch (device memory is PyTorch's job here).  A non-zero status from
the library raises ``AttnError`` with the library's own message.  There is no fallback: if the
library is missing or no sm_100 device is present, calls raise.
"""

from __future__ import annotations

import ctypes
import math
import os

MASK_FULL, MASK_CAUSAL, MASK_SLIDING, MASK_LOCAL_GLOBAL = 0, 1, 2, 3
ATTN_OK = 0
ATTN_ERR_INVALID_ARG = -1
ATTN_ERR_UNSUPPORTED = -2
ATTN_ERR_CUDA = -3
ATTN_ERR_WORKSPACE = -4
ATTN_ERR_DEVICE_TIMEOUT = -5

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libattn.so")

# every symbol include/attn.h declares
EXPORTS = ("attn_abi_version", "attn_status_string", "attn_last_error_detail", "attn_fwd", "attn_fwd_f32",
           "attn_decode_workspace_bytes", "attn_decode", "attn_decode_num_splits",
           "attn_get_device_error", "attn_debug_timeout_probe", "attn_decode_noalloc",
           "attn_fwd_varlen", "attn_decode_paged", "attn_bwd", "attn_bwd_workspace_bytes", "attn_fwd_fp8",
           "attn_fwd_block_sparse")

# size of the library-owned scratch array behind attn_decode_noalloc (include/attn.h)
DECODE_NOALLOC_MAX_BYTES = 64 << 20

_lib = None


class AttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = "%s: %s (status %d)" % (where, status_string(status), status)
        if status == ATTN_ERR_CUDA:
            msg += ": " + lib().attn_last_error_detail().decode()
        super().__init__(msg)


def lib():
    """Load libattn.so once; raise if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libattn.so is missing (%s): build it with "
                               "`python -m exact_io_aware_82_b200.build`" % LIB_PATH)
        L = ctypes.CDLL(LIB_PATH)
        vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
        L.attn_abi_version.argtypes, L.attn_abi_version.restype = [], i
        L.attn_status_string.argtypes, L.attn_status_string.restype = [i], ctypes.c_char_p
        L.attn_last_error_detail.argtypes, L.attn_last_error_detail.restype = [], ctypes.c_char_p
        L.attn_fwd.argtypes = [vp] * 5 + [i] * 9 + [f, vp]
        L.attn_fwd.restype = i
        L.attn_fwd_f32.argtypes = [vp] * 5 + [i] * 9 + [f, vp]
        L.attn_fwd_f32.restype = i
        L.attn_decode_workspace_bytes.argtypes = [i] * 6
        L.attn_decode_workspace_bytes.restype = ctypes.c_size_t
        L.attn_decode.argtypes = [vp] * 5 + [i] * 5 + [f, i, vp, ctypes.c_size_t, vp]
        L.attn_decode.restype = i
        L.attn_decode_num_splits.argtypes, L.attn_decode_num_splits.restype = [i] * 5, i
        L.attn_get_device_error.argtypes, L.attn_get_device_error.restype = [vp], i
        L.attn_debug_timeout_probe.argtypes = [ctypes.c_longlong, vp]
        L.attn_debug_timeout_probe.restype = i
        L.attn_decode_noalloc.argtypes = [vp] * 5 + [i] * 5 + [f, i, vp]
        L.attn_decode_noalloc.restype = i
        L.attn_fwd_varlen.argtypes = [vp] * 7 + [i] * 10 + [f, vp]
        L.attn_fwd_varlen.restype = i
        L.attn_decode_paged.argtypes = [vp] * 7 + [i] * 8 + [f, i, vp, ctypes.c_size_t, vp]
        L.attn_decode_paged.restype = i
        L.attn_fwd_fp8.argtypes = [vp] * 8 + [i] * 9 + [f, vp]
        L.attn_fwd_fp8.restype = i
        L.attn_fwd_block_sparse.argtypes = [vp] * 6 + [i] * 10 + [f, vp]
        L.attn_fwd_block_sparse.restype = i
        L.attn_bwd_workspace_bytes.argtypes = [i] * 7
        L.attn_bwd_workspace_bytes.restype = ctypes.c_size_t
        L.attn_bwd.argtypes = [vp] * 9 + [i] * 9 + [f, vp, ctypes.c_size_t, vp]
        L.attn_bwd.restype = i
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().attn_status_string(int(status)).decode()


def abi_version() -> int:
    return int(lib().attn_abi_version())


def _stream_ptr(stream=None):
    import torch

    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _check(t, name, dtype, ndim, shape=None):
    """Type, dtype, rank, contiguity and (if given) exact shape of one tensor argument."""
    import torch

    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a torch.Tensor" % name)
    if t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if t.dim() != ndim or not t.is_contiguous():
        raise ValueError("%s must be a contiguous %d-d tensor" % (name, ndim))
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError("%s must have shape %s, got %s" % (name, tuple(shape), tuple(t.shape)))


def _check_out(t, name, dtype, shape):
    """An optional output / gradient tensor: None, or exactly the tensor the library writes."""
    if t is not None:
        _check(t, name, dtype, len(shape), shape)


def _check_workspace(ws, nbytes):
    import torch

    if ws is None:
        return
    _check(ws, "workspace", torch.uint8, 1)
    if ws.numel() < nbytes:
        raise ValueError("workspace holds %d bytes, the call needs %d" % (ws.numel(), nbytes))


def _device(stream, **tensors):
    """The one CUDA device that every given tensor (and the stream, if any) lives on.

    The library launches on the calling thread's current device with raw pointers, so a tensor
    on another device must be refused here rather than handed to a kernel."""
    devs = {t.device for t in tensors.values() if t is not None}
    if len(devs) != 1:
        raise ValueError("all tensors must be on one device, got %s" % ", ".join(
            "%s on %s" % (n, t.device) for n, t in tensors.items() if t is not None))
    dev = devs.pop()
    if dev.type != "cuda":
        raise ValueError("tensors must be CUDA tensors, got %s" % dev)
    if stream is not None and stream.device != dev:
        raise ValueError("stream is on %s, the tensors on %s" % (stream.device, dev))
    return dev


def _raise(rc, where):
    if rc != ATTN_OK:
        raise AttnError(rc, where)


def attn_fwd(q, k, v, o=None, lse=None, mask_kind=MASK_FULL, window=0, n_sink=0, scale=None,
             return_lse=True, stream=None):
    """Exact attention forward on bf16 tensors q [B,Hq,Nq,d], k/v [B,Hkv,Nk,d].

    Returns (o, lse) with o bf16 [B,Hq,Nq,d] and lse fp32 [B,Hq,Nq] (None if not requested).
    """
    import torch

    _check(q, "q", torch.bfloat16, 4)
    B, Hq, Nq, d = q.shape
    _check(k, "k", torch.bfloat16, 4)
    Hkv, Nk = k.shape[1], k.shape[2]
    _check(k, "k", torch.bfloat16, 4, (B, Hkv, Nk, d))
    _check(v, "v", torch.bfloat16, 4, (B, Hkv, Nk, d))
    _check_out(o, "o", torch.bfloat16, (B, Hq, Nq, d))
    _check_out(lse, "lse", torch.float32, (B, Hq, Nq))
    dev = _device(stream, q=q, k=k, v=v, o=o, lse=lse)
    with torch.cuda.device(dev):
        if o is None:
            o = torch.empty_like(q)
        if lse is None and return_lse:
            lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=dev)
        scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
        rc = lib().attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, Nq, Nk, d,
                            int(mask_kind), int(window), int(n_sink), scale, _stream_ptr(stream))
    _raise(rc, "attn_fwd")
    return o, lse


def attn_fwd_block_sparse(q, k, v, block_mask, o=None, lse=None, mask_kind=MASK_FULL, window=0,
                          n_sink=0, scale=None, return_lse=True, stream=None):
    """attn_fwd under a fixed block-sparse layout: block_mask uint8 (or bool) [1 or Hq,
    ceil(Nq/128), ceil(Nk/128)] selects the 128 x 128 blocks each head attends (one layout for
    every head when its first dimension is 1).  Returns (o, lse) as attn_fwd."""
    import torch

    _check(q, "q", torch.bfloat16, 4)
    B, Hq, Nq, d = q.shape
    _check(k, "k", torch.bfloat16, 4)
    Hkv, Nk = k.shape[1], k.shape[2]
    _check(k, "k", torch.bfloat16, 4, (B, Hkv, Nk, d))
    _check(v, "v", torch.bfloat16, 4, (B, Hkv, Nk, d))
    if isinstance(block_mask, torch.Tensor) and block_mask.dtype == torch.bool:
        block_mask = block_mask.view(torch.uint8)
    _check(block_mask, "block_mask", torch.uint8, 3)
    shape = (block_mask.shape[0], -(-Nq // 128), -(-Nk // 128))
    if block_mask.shape[0] not in (1, Hq):
        raise ValueError("block_mask must have 1 or Hq = %d layouts, got %d" % (Hq, block_mask.shape[0]))
    _check(block_mask, "block_mask", torch.uint8, 3, shape)
    _check_out(o, "o", torch.bfloat16, (B, Hq, Nq, d))
    _check_out(lse, "lse", torch.float32, (B, Hq, Nq))
    dev = _device(stream, q=q, k=k, v=v, block_mask=block_mask, o=o, lse=lse)
    with torch.cuda.device(dev):
        if o is None:
            o = torch.empty_like(q)
        if lse is None and return_lse:
            lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=dev)
        scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
        rc = lib().attn_fwd_block_sparse(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                         _ptr(block_mask), int(block_mask.shape[0]), B, Hq, Hkv,
                                         Nq, Nk, d, int(mask_kind), int(window), int(n_sink),
                                         scale, _stream_ptr(stream))
    _raise(rc, "attn_fwd_block_sparse")
    return o, lse


def attn_fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, o=None, lse=None,
                    mask_kind=MASK_FULL, window=0, n_sink=0, scale=None, return_lse=True,
                    stream=None):
    """Packed variable-length forward: q [total_q, Hq, d], k/v [total_k, Hkv, d] bf16;
    cu_seqlens_q / cu_seqlens_k int32 CUDA tensors of num_seqs + 1 offsets.

    Returns (o [total_q, Hq, d] bf16, lse [total_q, Hq] fp32).  Rows outside every sequence are
    left as they were in ``o`` / ``lse`` (allocated uninitialised when not given).
    """
    import torch

    _check(q, "q", torch.bfloat16, 3)
    total_q, Hq, d = q.shape
    _check(k, "k", torch.bfloat16, 3)
    total_k, Hkv = k.shape[0], k.shape[1]
    _check(k, "k", torch.bfloat16, 3, (total_k, Hkv, d))
    _check(v, "v", torch.bfloat16, 3, (total_k, Hkv, d))
    _check(cu_seqlens_q, "cu_seqlens_q", torch.int32, 1)
    num_seqs = cu_seqlens_q.numel() - 1
    if num_seqs < 0:
        raise ValueError("cu_seqlens_q needs num_seqs + 1 >= 1 offsets")
    _check(cu_seqlens_k, "cu_seqlens_k", torch.int32, 1, (num_seqs + 1,))
    _check_out(o, "o", torch.bfloat16, (total_q, Hq, d))
    _check_out(lse, "lse", torch.float32, (total_q, Hq))
    dev = _device(stream, q=q, k=k, v=v, cu_seqlens_q=cu_seqlens_q, cu_seqlens_k=cu_seqlens_k,
                  o=o, lse=lse)
    with torch.cuda.device(dev):
        if o is None:
            o = torch.empty_like(q)
        if lse is None and return_lse:
            lse = torch.empty((total_q, Hq), dtype=torch.float32, device=dev)
        scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
        rc = lib().attn_fwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                   _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), num_seqs, Hq, Hkv,
                                   total_q, total_k, int(max_seqlen_q), d, int(mask_kind),
                                   int(window), int(n_sink), scale, _stream_ptr(stream))
    _raise(rc, "attn_fwd_varlen")
    return o, lse


def attn_fwd_fp8(q, k, v, descale_q, descale_k, descale_v, o=None, lse=None,
                 mask_kind=MASK_FULL, window=0, n_sink=0, scale=None, return_lse=True,
                 stream=None):
    """E4M3 forward: q [B,Hq,Nq,d], k, v [B,Hkv,Nk,d] as uint8 (or float8_e4m3fn) codes;
    descale_q [B,Hq], descale_k / descale_v [B,Hkv] fp32 CUDA tensors.  Returns (o bf16, lse)."""
    import torch

    def codes(t, n):
        if not isinstance(t, torch.Tensor):
            raise TypeError("%s must be a torch.Tensor" % n)
        if t.dtype == getattr(torch, "float8_e4m3fn", None):
            t = t.view(torch.uint8)
        _check(t, n, torch.uint8, 4)
        return t

    q, k, v = codes(q, "q"), codes(k, "k"), codes(v, "v")
    B, Hq, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    _check(k, "k", torch.uint8, 4, (B, Hkv, Nk, d))
    _check(v, "v", torch.uint8, 4, (B, Hkv, Nk, d))
    _check(descale_q, "descale_q", torch.float32, 2, (B, Hq))
    _check(descale_k, "descale_k", torch.float32, 2, (B, Hkv))
    _check(descale_v, "descale_v", torch.float32, 2, (B, Hkv))
    _check_out(o, "o", torch.bfloat16, (B, Hq, Nq, d))
    _check_out(lse, "lse", torch.float32, (B, Hq, Nq))
    dev = _device(stream, q=q, k=k, v=v, descale_q=descale_q, descale_k=descale_k,
                  descale_v=descale_v, o=o, lse=lse)
    with torch.cuda.device(dev):
        if o is None:
            o = torch.empty((B, Hq, Nq, d), dtype=torch.bfloat16, device=dev)
        if lse is None and return_lse:
            lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=dev)
        scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
        rc = lib().attn_fwd_fp8(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(descale_q),
                                _ptr(descale_k), _ptr(descale_v), B, Hq, Hkv, Nq, Nk, d,
                                int(mask_kind), int(window), int(n_sink), scale,
                                _stream_ptr(stream))
    _raise(rc, "attn_fwd_fp8")
    return o, lse


def attn_fwd_f32(q, k, v, o=None, lse=None, mask_kind=MASK_FULL, window=0, n_sink=0, scale=None,
                 return_lse=True, stream=None):
    """Exact attention forward on fp32 tensors (same shapes and rules as attn_fwd)."""
    import torch

    _check(q, "q", torch.float32, 4)
    B, Hq, Nq, d = q.shape
    _check(k, "k", torch.float32, 4)
    Hkv, Nk = k.shape[1], k.shape[2]
    _check(k, "k", torch.float32, 4, (B, Hkv, Nk, d))
    _check(v, "v", torch.float32, 4, (B, Hkv, Nk, d))
    _check_out(o, "o", torch.float32, (B, Hq, Nq, d))
    _check_out(lse, "lse", torch.float32, (B, Hq, Nq))
    dev = _device(stream, q=q, k=k, v=v, o=o, lse=lse)
    with torch.cuda.device(dev):
        if o is None:
            o = torch.empty_like(q)
        if lse is None and return_lse:
            lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=dev)
        scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
        rc = lib().attn_fwd_f32(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, Nq,
                                Nk, d, int(mask_kind), int(window), int(n_sink), scale,
                                _stream_ptr(stream))
    _raise(rc, "attn_fwd_f32")
    return o, lse


def attn_bwd_workspace_bytes(B, Hq, Nq, Nk, mask_kind=MASK_FULL, window=0, n_sink=0) -> int:
    return int(lib().attn_bwd_workspace_bytes(B, Hq, Nq, Nk, int(mask_kind), int(window),
                                              int(n_sink)))


def attn_bwd(q, k, v, o, lse, dout, mask_kind=MASK_FULL, window=0, n_sink=0, scale=None,
             dq=None, dk=None, dv=None, workspace=None, stream=None):
    """Backward of attn_fwd: returns (dq, dk, dv), bf16 with the shapes of q, k, v.

    o and lse are the forward's outputs for the same q, k, v, mask and scale; dout = dL/dO.
    """
    import torch

    _check(q, "q", torch.bfloat16, 4)
    B, Hq, Nq, d = q.shape
    _check(k, "k", torch.bfloat16, 4)
    Hkv, Nk = k.shape[1], k.shape[2]
    _check(k, "k", torch.bfloat16, 4, (B, Hkv, Nk, d))
    _check(v, "v", torch.bfloat16, 4, (B, Hkv, Nk, d))
    _check(o, "o", torch.bfloat16, 4, (B, Hq, Nq, d))
    _check(dout, "dout", torch.bfloat16, 4, (B, Hq, Nq, d))
    _check(lse, "lse", torch.float32, 3, (B, Hq, Nq))
    _check_out(dq, "dq", torch.bfloat16, (B, Hq, Nq, d))
    _check_out(dk, "dk", torch.bfloat16, (B, Hkv, Nk, d))
    _check_out(dv, "dv", torch.bfloat16, (B, Hkv, Nk, d))
    _check_workspace(workspace, 0)
    dev = _device(stream, q=q, k=k, v=v, o=o, lse=lse, dout=dout, dq=dq, dk=dk, dv=dv,
                  workspace=workspace)
    with torch.cuda.device(dev):
        dq = torch.empty_like(q) if dq is None else dq
        dk = torch.empty_like(k) if dk is None else dk
        dv = torch.empty_like(v) if dv is None else dv
        if workspace is None:
            workspace = torch.empty(max(attn_bwd_workspace_bytes(B, Hq, Nq, Nk, mask_kind, window,
                                                                 n_sink), 16),
                                    dtype=torch.uint8, device=dev)
        scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
        rc = lib().attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout), _ptr(dq),
                            _ptr(dk), _ptr(dv), B, Hq, Hkv, Nq, Nk, d, int(mask_kind),
                            int(window), int(n_sink), scale, _ptr(workspace), workspace.numel(),
                            _stream_ptr(stream))
    _raise(rc, "attn_bwd")
    return dq, dk, dv


def attn_decode_workspace_bytes(B, Hq, Hkv, Nk, d, num_splits=0) -> int:
    return int(lib().attn_decode_workspace_bytes(B, Hq, Hkv, Nk, d, num_splits))


def attn_decode_num_splits(B, Hq, Hkv, Nk, d) -> int:
    return int(lib().attn_decode_num_splits(B, Hq, Hkv, Nk, d))


def _decode_query(q):
    import torch

    _check(q, "q", torch.bfloat16, 4)
    B, Hq, one, d = q.shape
    if one != 1:
        raise ValueError("decode takes one query token per sequence (q.shape[2] == 1)")
    return B, Hq, d


def attn_decode(q, k, v, o=None, lse=None, scale=None, num_splits=0, workspace=None,
                return_lse=True, stream=None):
    """Split-K decode: q [B,Hq,1,d] bf16 against the cache k/v [B,Hkv,Nk,d] bf16.

    Returns (o [B,Hq,1,d] bf16, lse [B,Hq] fp32).  ``workspace`` (a uint8 CUDA tensor of at
    least attn_decode_workspace_bytes(...) bytes) is allocated with torch when not given.
    """
    import torch

    B, Hq, d = _decode_query(q)
    _check(k, "k", torch.bfloat16, 4)
    Hkv, Nk = k.shape[1], k.shape[2]
    _check(k, "k", torch.bfloat16, 4, (B, Hkv, Nk, d))
    _check(v, "v", torch.bfloat16, 4, (B, Hkv, Nk, d))
    _check_out(o, "o", torch.bfloat16, (B, Hq, 1, d))
    _check_out(lse, "lse", torch.float32, (B, Hq))
    _check_workspace(workspace, 0)
    dev = _device(stream, q=q, k=k, v=v, o=o, lse=lse, workspace=workspace)
    with torch.cuda.device(dev):
        if o is None:
            o = torch.empty_like(q)
        if lse is None and return_lse:
            lse = torch.empty((B, Hq), dtype=torch.float32, device=dev)
        if workspace is None:
            nbytes = attn_decode_workspace_bytes(B, Hq, Hkv, Nk, d, num_splits)
            workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dev)
        scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
        rc = lib().attn_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, Nk, d,
                               scale, int(num_splits), _ptr(workspace), workspace.numel(),
                               _stream_ptr(stream))
    _raise(rc, "attn_decode")
    return o, lse


def attn_decode_paged(q, k_cache, v_cache, block_table, seq_lens, max_seq_len, o=None, lse=None,
                      scale=None, num_splits=0, workspace=None, return_lse=True, stream=None):
    """Decode against a paged cache.

    q [B,Hq,1,d] bf16; k_cache/v_cache [num_pages,page_size,Hkv,d] bf16; block_table
    [B,max_pages_per_seq] int32; seq_lens [B] int32 (device); max_seq_len an int >= every length.
    Returns (o [B,Hq,1,d] bf16, lse [B,Hq] fp32).
    """
    import torch

    B, Hq, d = _decode_query(q)
    _check(k_cache, "k_cache", torch.bfloat16, 4)
    num_pages, page_size, Hkv, dk = k_cache.shape
    if dk != d:
        raise ValueError("k_cache and v_cache must both be [num_pages, page_size, Hkv, d]")
    _check(v_cache, "v_cache", torch.bfloat16, 4, k_cache.shape)
    _check(block_table, "block_table", torch.int32, 2)
    if block_table.shape[0] != B:
        raise ValueError("block_table and seq_lens need one row per sequence")
    _check(seq_lens, "seq_lens", torch.int32, 1, (B,))
    _check_out(o, "o", torch.bfloat16, (B, Hq, 1, d))
    _check_out(lse, "lse", torch.float32, (B, Hq))
    _check_workspace(workspace, 0)
    dev = _device(stream, q=q, k_cache=k_cache, v_cache=v_cache, block_table=block_table,
                  seq_lens=seq_lens, o=o, lse=lse, workspace=workspace)
    max_seq_len = int(max_seq_len)
    with torch.cuda.device(dev):
        if o is None:
            o = torch.empty_like(q)
        if lse is None and return_lse:
            lse = torch.empty((B, Hq), dtype=torch.float32, device=dev)
        if workspace is None:
            nbytes = attn_decode_workspace_bytes(B, Hq, Hkv, max_seq_len, d, num_splits)
            workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dev)
        scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
        rc = lib().attn_decode_paged(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(o), _ptr(lse),
                                     _ptr(block_table), _ptr(seq_lens), B, Hq, Hkv, num_pages,
                                     page_size, block_table.shape[1], max_seq_len, d, scale,
                                     int(num_splits), _ptr(workspace), workspace.numel(),
                                     _stream_ptr(stream))
    _raise(rc, "attn_decode_paged")
    return o, lse


def attn_decode_noalloc(q, k, v, o=None, lse=None, scale=None, num_splits=0, return_lse=True,
                        stream=None):
    """attn_decode without a workspace, for callers that cannot allocate device memory: the
    split partials live in a fixed library-owned device array of DECODE_NOALLOC_MAX_BYTES
    (shared by every call on the device, so calls that overlap on the GPU race).  Raises
    AttnError(ATTN_ERR_WORKSPACE) when the call would need more than that array."""
    import torch

    B, Hq, d = _decode_query(q)
    _check(k, "k", torch.bfloat16, 4)
    Hkv, Nk = k.shape[1], k.shape[2]
    _check(k, "k", torch.bfloat16, 4, (B, Hkv, Nk, d))
    _check(v, "v", torch.bfloat16, 4, (B, Hkv, Nk, d))
    _check_out(o, "o", torch.bfloat16, (B, Hq, 1, d))
    _check_out(lse, "lse", torch.float32, (B, Hq))
    dev = _device(stream, q=q, k=k, v=v, o=o, lse=lse)
    with torch.cuda.device(dev):
        if o is None:
            o = torch.empty_like(q)
        if lse is None and return_lse:
            lse = torch.empty((B, Hq), dtype=torch.float32, device=dev)
        scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
        rc = lib().attn_decode_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv,
                                       Nk, d, scale, int(num_splits), _stream_ptr(stream))
    _raise(rc, "attn_decode_noalloc")
    return o, lse


def attn_get_device_error(stream=None) -> int:
    """Synchronise the stream, then read and clear the device error flag (0 = none)."""
    return int(lib().attn_get_device_error(_stream_ptr(stream)))


def attn_debug_timeout_probe(limit_cycles: int, stream=None) -> None:
    _raise(lib().attn_debug_timeout_probe(int(limit_cycles), _stream_ptr(stream)),
           "attn_debug_timeout_probe")
