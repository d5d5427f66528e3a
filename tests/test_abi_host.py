"""Host-side checks of the C ABI: the library builds and loads, exports every declared symbol,
and rejects invalid arguments with the documented status before touching the device."""

import ctypes
import os
import re

import pytest

from exact_io_aware_82_b200 import attn as A
from exact_io_aware_82_b200 import build as B

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "attn.h")


@pytest.fixture(scope="module")
def lib():
    B.build()
    return A.lib()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"ATTN_API\s+[\w\s\*]+?\b(attn_\w+)\s*\(", text)))


def test_header_declarations_match_binding():
    assert declared_functions() == sorted(A.EXPORTS)


def declared_parameters():
    """Each declared function's parameters as the ctypes class that carries them: pointers
    (and the stream handle) as c_void_p, then int, float, size_t, long long."""
    text = re.sub(r"/\*.*?\*/", " ", open(HEADER).read(), flags=re.S)
    out = {}
    for m in re.finditer(r"ATTN_API\s+[\w\s\*]+?\b(attn_\w+)\s*\(([^)]*)\)", text):
        params = " ".join(m.group(2).split())
        kinds = []
        for prm in ([] if params in ("", "void") else params.split(",")):
            prm = prm.strip()
            if "*" in prm or prm.startswith("attn_stream_t"):
                kinds.append(ctypes.c_void_p)
            elif prm.startswith("size_t"):
                kinds.append(ctypes.c_size_t)
            elif prm.startswith("long long"):
                kinds.append(ctypes.c_longlong)
            elif prm.startswith("float"):
                kinds.append(ctypes.c_float)
            elif prm.startswith("int"):
                kinds.append(ctypes.c_int)
            else:
                raise AssertionError("unexpected parameter type: " + prm)
        out[m.group(1)] = kinds
    return out


def test_binding_argtypes_match_header(lib):
    # a binding that passes one argument too many or too few would shift every argument after
    # it; each declared parameter must have an argtype of the same kind
    params = declared_parameters()
    assert sorted(params) == declared_functions()
    for name, kinds in params.items():
        got = list(getattr(lib, name).argtypes)
        assert len(got) == len(kinds), "%s: %d argtypes, header declares %d" % (name, len(got), len(kinds))
        for n, (a, b) in enumerate(zip(got, kinds)):
            assert a is b, "%s parameter %d: binding %s, header %s" % (name, n, a, b)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    # nothing else of ours leaks out of the library (hidden visibility)
    out = os.popen("nm -D --defined-only %s" % A.LIB_PATH).read()
    ours = sorted(set(re.findall(r"\b(attn_\w+)\b", out)))
    assert ours == declared_functions()


def test_status_strings(lib):
    assert A.abi_version() == 1
    for rc in (0, -1, -2, -3, -4, -5):
        assert A.status_string(rc) and A.status_string(rc) != "unknown status"
    assert A.status_string(42) == "unknown status"


P = ctypes.c_void_p(16)  # a non-null, 16-byte aligned dummy: invalid-argument paths never use it
N = ctypes.c_void_p(0)


def fwd(lib, q=P, k=P, v=P, o=P, B=1, Hq=2, Hkv=1, Nq=4, Nk=4, d=128, mask=0, w=0, s=0, scale=0.1,
        f32=False):
    fn = lib.attn_fwd_f32 if f32 else lib.attn_fwd
    return fn(q, k, v, o, N, B, Hq, Hkv, Nq, Nk, d, mask, w, s, scale, N)


@pytest.mark.parametrize("f32", [False, True])
def test_invalid_arguments_are_rejected(lib, f32):
    E = A.ATTN_ERR_INVALID_ARG
    assert fwd(lib, q=N, f32=f32) == E
    assert fwd(lib, k=N, f32=f32) == E
    assert fwd(lib, v=N, f32=f32) == E
    assert fwd(lib, o=N, f32=f32) == E
    assert fwd(lib, B=-1, f32=f32) == E
    assert fwd(lib, Nq=-1, f32=f32) == E
    assert fwd(lib, Nk=-1, f32=f32) == E
    assert fwd(lib, Hq=0, f32=f32) == E
    assert fwd(lib, Hkv=0, f32=f32) == E
    assert fwd(lib, Hq=3, Hkv=2, f32=f32) == E
    assert fwd(lib, mask=4, f32=f32) == E
    assert fwd(lib, mask=-1, f32=f32) == E
    assert fwd(lib, mask=2, w=0, f32=f32) == E
    assert fwd(lib, mask=3, w=-1, f32=f32) == E
    assert fwd(lib, mask=3, w=2, s=-1, f32=f32) == E
    assert fwd(lib, mask=2, w=4, s=-1, f32=f32) == E
    assert fwd(lib, scale=float("nan"), f32=f32) == E
    assert fwd(lib, scale=float("inf"), f32=f32) == E


def test_unsupported_shapes_are_rejected(lib):
    U = A.ATTN_ERR_UNSUPPORTED
    assert fwd(lib, d=64) == U
    assert fwd(lib, d=96, f32=True) == U
    assert fwd(lib, q=ctypes.c_void_p(24)) == U  # misaligned
    dec = lib.attn_decode
    assert dec(P, P, P, P, N, 1, 16, 1, 8, 128, 0.1, 0, P, 1 << 20, N) == U  # G = 16
    assert dec(P, P, P, P, N, 1, 4, 1, 8, 64, 0.1, 0, P, 1 << 20, N) == U  # d = 64
    E = A.ATTN_ERR_INVALID_ARG
    assert dec(N, P, P, P, N, 1, 4, 1, 8, 128, 0.1, 0, P, 1 << 20, N) == E
    assert dec(P, P, P, P, N, 1, 4, 3, 8, 128, 0.1, 0, P, 1 << 20, N) == E
    assert dec(P, P, P, P, N, 1, 4, 1, 8, 128, 0.1, -1, P, 1 << 20, N) == E
    assert lib.attn_decode_workspace_bytes(1, 4, 3, 8, 128, 0) == 0
    assert lib.attn_decode_workspace_bytes(64, 32, 8, 32768, 128, 16) == 64 * 32 * 16 * 129 * 4


def paged(lib, q=P, k=P, v=P, o=P, bt=P, sl=P, B=2, Hq=8, Hkv=2, num_pages=10, ps=16, max_pages=4,
          max_len=64, d=128, scale=0.1, splits=0):
    return lib.attn_decode_paged(q, k, v, o, N, bt, sl, B, Hq, Hkv, num_pages, ps, max_pages,
                                 max_len, d, scale, splits, P, 1 << 20, N)


def test_paged_decode_invalid_arguments_are_rejected(lib):
    E = A.ATTN_ERR_INVALID_ARG
    for ps in (0, 4, 12, 24, 1 << 21):
        assert paged(lib, ps=ps) == E
    assert paged(lib, max_len=65) == E          # beyond max_pages * page_size
    assert paged(lib, max_len=-1) == E
    assert paged(lib, num_pages=-1) == E
    assert paged(lib, max_pages=-1) == E
    assert paged(lib, B=-1) == E
    assert paged(lib, Hq=3) == E
    assert paged(lib, q=N) == E
    assert paged(lib, sl=N) == E
    assert paged(lib, bt=N) == E
    assert paged(lib, k=N) == E
    assert paged(lib, splits=-1) == E
    assert paged(lib, scale=float("nan")) == E


def bwd(lib, q=P, k=P, v=P, o=P, lse=P, do=P, dq=P, dk=P, dv=P, B=1, Hq=2, Hkv=1, Nq=4, Nk=4,
        d=128, mask=1, w=0, s=0, scale=0.1, ws=P, ws_bytes=1 << 20):
    return lib.attn_bwd(q, k, v, o, lse, do, dq, dk, dv, B, Hq, Hkv, Nq, Nk, d, mask, w, s, scale,
                        ws, ws_bytes, N)


def test_bwd_invalid_arguments_are_rejected(lib):
    E = A.ATTN_ERR_INVALID_ARG
    for name in ("q", "k", "v", "o", "lse", "do", "dq", "dk", "dv"):
        assert bwd(lib, **{name: N}) == E, name
    assert bwd(lib, B=-1) == E
    assert bwd(lib, Hq=3, Hkv=2) == E
    assert bwd(lib, mask=2, w=0) == E
    assert bwd(lib, scale=float("nan")) == E
    assert bwd(lib, d=64) == A.ATTN_ERR_UNSUPPORTED


def test_bwd_workspace_size():
    def expect(B, Hq, Nq, Nk, pairs):
        npad = (Nq + 127) // 128 * 128
        vec = 2 * B * Hq * npad * 4
        off = ((Nk + 127) // 128 + 1) * 4
        return (vec + off + 255) // 256 * 256 + B * Hq * pairs * 128 * 128 * 2

    # causal n = 2048: key block kb is seen by query tiles kb .. 15, 136 pairs per head
    assert A.attn_bwd_workspace_bytes(4, 16, 2048, 2048, A.MASK_CAUSAL) == expect(4, 16, 2048, 2048, 136)
    # full, 300 x 300: 3 key blocks x 3 query tiles
    assert A.attn_bwd_workspace_bytes(1, 2, 300, 300, A.MASK_FULL) == expect(1, 2, 300, 300, 9)
    # window of one key: each key block meets its own query tile only
    assert A.attn_bwd_workspace_bytes(1, 2, 512, 512, A.MASK_SLIDING, 1, 0) == expect(1, 2, 512, 512, 4)
    assert A.attn_bwd_workspace_bytes(0, 2, 300, 300, A.MASK_FULL) == 0
    assert A.attn_bwd_workspace_bytes(1, 2, 300, 300, A.MASK_SLIDING, 0, 0) == 0  # bad window


def test_fp8_invalid_arguments_are_rejected(lib):
    E = A.ATTN_ERR_INVALID_ARG

    def fp8(q=P, k=P, v=P, o=P, dq=P, dk=P, dv=P, mask=1, w=0, s=0, scale=0.1, d=128):
        return lib.attn_fwd_fp8(q, k, v, o, N, dq, dk, dv, 1, 2, 1, 4, 4, d, mask, w, s, scale, N)

    for name in ("q", "k", "v", "o", "dq", "dk", "dv"):
        assert fp8(**{name: N}) == E, name
    assert fp8(mask=5) == E
    assert fp8(scale=float("inf")) == E
    assert fp8(d=64) == A.ATTN_ERR_UNSUPPORTED
