"""The kernels' integer mask logic, compiled for the host and checked against the oracle.

The CUDA kernels decide which (query tile, key tile) blocks to visit, which blocks need no
element mask, and which keys of a tile each row sees, with integer helpers in the library's
headers (the MaskSpec region of common.cuh; QueryTiles, query_tiles and pair_index in
bwd_sm100.cuh).  Those helpers are plain integer C++: this test cuts them out of the headers,
compiles them with g++
into tests/host_mask_check.cpp together with the oracle's visibility predicate, and checks them
exhaustively (every row and key) on a few hundred problem shapes: every mask kind, Nq = Nk and
Nq != Nk both ways, ragged tails, windows and sink / global counts on either side of a tile
edge.  The GPU parity tests cover the same logic through the kernels, on fewer shapes.
"""

import itertools
import os
import re
import shutil
import subprocess
import tempfile

import pytest

from oracle import oracle as O

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(ROOT, "exact_io_aware_82_b200", "csrc")


def _function(src, name):
    """Source text of the __host__ __device__ function `name` (signature to closing brace)."""
    m = re.search(r"__host__ __device__[^;{}]*?\b%s\(" % re.escape(name), src)
    assert m, "function %s not found" % name
    i = src.index("{", m.end())
    depth = 0
    for j in range(i, len(src)):
        depth += {"{": 1, "}": -1}.get(src[j], 0)
        if depth == 0:
            return src[m.start():j + 1]
    raise AssertionError("unbalanced braces in " + name)


def _struct(src, name):
    """Source text of `struct name { ... };`."""
    i = src.index("struct %s {" % name)
    return src[i:src.index("};", i) + 2]


def mask_logic_source():
    common = open(os.path.join(CSRC, "common.cuh")).read()
    start = common.index("// Mask shared by every kernel.")
    end = common.rindex("}  // namespace attn")
    bwd = open(os.path.join(CSRC, "bwd_sm100.cuh")).read()
    parts = [common[start:end]]
    parts.append(_struct(bwd, "QueryTiles"))
    parts += [_function(bwd, n) for n in ("imin", "imax", "floor_div128", "query_tiles", "pair_index")]
    return "\n".join(parts)


def configs():
    F, C, S, L = O.MASK_FULL, O.MASK_CAUSAL, O.MASK_SLIDING, O.MASK_LOCAL_GLOBAL
    shapes = [(1, 1), (1, 300), (300, 1), (128, 128), (129, 129), (300, 300), (200, 450),
              (450, 200), (513, 513), (256, 700), (700, 256), (640, 640)]
    out = []
    for nq, nk in shapes:
        out.append((F, nq, nk, 0, 0))
        out.append((C, nq, nk, 0, 0))
        for w, s in itertools.product((1, 2, 127, 128, 129, 200, 1000), (0, 1, 4, 130)):
            out.append((S, nq, nk, w, s))
        for w, s in itertools.product((0, 1, 50, 127, 128, 300), (0, 1, 4, 128, 130)):
            out.append((L, nq, nk, w, s))
    return out


@pytest.fixture(scope="module")
def checker():
    if shutil.which("g++") is None or shutil.which("gcc") is None:
        pytest.skip("g++ / gcc not available")
    d = tempfile.mkdtemp(prefix="mask_check_")
    try:
        with open(os.path.join(d, "mask_logic.inc"), "w") as f:
            f.write(mask_logic_source())
        obj = os.path.join(d, "oracle.o")
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-fopenmp", "-c", "-o", obj,
                               os.path.join(ROOT, "oracle", "oracle.c")])
        exe = os.path.join(d, "mask_check")
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-fopenmp", "-I", d, "-I",
                               os.path.join(ROOT, "include"), "-o", exe,
                               os.path.join(HERE, "host_mask_check.cpp"), obj, "-lm"])
        yield exe
    finally:
        shutil.rmtree(d, ignore_errors=True)


def run(exe, cfgs):
    text = "".join("%d %d %d %d %d\n" % c for c in cfgs)
    return subprocess.run([exe], input=text, capture_output=True, text=True, timeout=600)


def test_mask_logic_matches_oracle_everywhere(checker):
    cfgs = configs()
    r = run(checker, cfgs)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
    ok, n, pairs = r.stdout.split()
    assert ok == "ok" and int(n) == len(cfgs) and int(pairs) > 10 ** 7


@pytest.mark.parametrize("old,new", [
    # a sliding window one key too wide, as the kernel would compute it
    ("first = static_cast<long long>(p) - m.window + 1;", "first = static_cast<long long>(p) - m.window;"),
    # sinks that ignore the causal bound
    ("sink = m.n_sink < last + 1 ? m.n_sink : last + 1;", "sink = m.n_sink;"),
    # a key-tile range that drops the tile holding the last visible key
    ("r.hi = (p_hi < last_key ? p_hi : last_key) / tile;", "r.hi = (p_hi < last_key ? p_hi : last_key) / tile - (p_hi > 0);"),
    # query tiles of a key block counted from the wrong side of the diagonal
    ("r.lo = imax(0, floor_div128(static_cast<long long>(c0) - off));",
     "r.lo = imax(0, floor_div128(static_cast<long long>(c1) - off));"),
    # global query rows counted from row 0 although rows before -off sit at negative positions
    ("const long long g0 = off < 0 ? -static_cast<long long>(off) : 0;", "const long long g0 = 0;"),
])
def test_checker_catches_planted_slips(checker, old, new, tmp_path):
    # the same build with one slip planted in a copy of the extracted helpers
    src = mask_logic_source()
    assert src.count(old) == 1, old
    (tmp_path / "mask_logic.inc").write_text(src.replace(old, new))
    obj = tmp_path / "oracle.o"
    subprocess.check_call(["gcc", "-O2", "-std=c99", "-fopenmp", "-c", "-o", str(obj),
                           os.path.join(ROOT, "oracle", "oracle.c")])
    exe = tmp_path / "mask_check"
    subprocess.check_call(["g++", "-O2", "-std=c++17", "-fopenmp", "-I", str(tmp_path), "-I",
                           os.path.join(ROOT, "include"), "-o", str(exe),
                           os.path.join(HERE, "host_mask_check.cpp"), str(obj), "-lm"])
    cfgs = [c for c in configs() if c[1] in (300, 513, 450, 200)]
    r = run(str(exe), cfgs)
    assert r.returncode != 0 and "FAIL" in r.stdout
