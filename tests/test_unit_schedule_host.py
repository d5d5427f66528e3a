"""The prefill kernels' work units, compiled for the host and checked for exact coverage.

The persistent prefill grid decodes a unit index into two 128-row query tiles (the same rows of
two query heads that share a kv head, or 256 consecutive rows of one head) and the key tiles they
visit.  This test cuts that logic out of the library's sources (decode_unit and its structs from
the forward header, fwd_schedule from the launch code, the integer mask helpers from the common
header), compiles it with g++ into tests/host_unit_check.cpp and checks, for dense and packed
variable-length problems under every mask kind, that every query row of every head is covered by
exactly one unit tile, that a unit's tiles read one kv head, and that a unit's key range holds
every key its rows see.  The GPU parity tests cover the same units through the kernels.
"""

import os
import re
import shutil
import subprocess
import tempfile

import pytest

from .test_mask_tiles_host import mask_logic_source

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(ROOT, "exact_io_aware_82_b200", "csrc")


def _braced(src, start):
    """Text from `start` to the brace that closes the first '{' after it (and a ';' after it)."""
    i = src.index("{", start)
    depth = 0
    for j in range(i, len(src)):
        depth += {"{": 1, "}": -1}.get(src[j], 0)
        if depth == 0:
            end = j + 1
            if src[end:end + 1] == ";":
                end += 1
            return src[start:end]
    raise AssertionError("unbalanced braces")


def unit_logic_source():
    fwd = open(os.path.join(CSRC, "fwd_sm100.cuh")).read()
    abi = open(os.path.join(CSRC, "abi.cu")).read()
    parts = [mask_logic_source(), "namespace fwd {"]
    for name in ("kBM", "kBN", "kRowsPerCta"):
        m = re.search(r"^constexpr int %s = [^;]*;" % name, fwd, re.M)
        assert m, name
        parts.append(m.group(0))
    parts.append(_braced(fwd, fwd.index("struct Params {")))
    parts.append(_braced(fwd, fwd.index("struct Unit {")))
    i = fwd.index("__device__ __forceinline__ bool in_range(")
    parts.append(_braced(fwd, i))
    i = fwd.index("template <bool kVarlen, bool kSparse>\n__device__ __forceinline__ bool decode_unit(")
    parts.append(_braced(fwd, i))
    parts.append("}  // namespace fwd")
    parts.append(_braced(abi, abi.index("struct FwdSchedule {")))
    parts.append(_braced(abi, abi.index("FwdSchedule fwd_schedule(")))
    return "\n".join(parts)


def build(tmpdir, logic):
    with open(os.path.join(tmpdir, "unit_logic.inc"), "w") as f:
        f.write(logic)
    exe = os.path.join(tmpdir, "unit_check")
    subprocess.check_call(["g++", "-O2", "-std=c++17", "-I", tmpdir, "-I",
                           os.path.join(ROOT, "include"), "-o", exe,
                           os.path.join(HERE, "host_unit_check.cpp")])
    return exe


@pytest.fixture(scope="module")
def checker():
    if shutil.which("g++") is None:
        pytest.skip("g++ not available")
    d = tempfile.mkdtemp(prefix="unit_check_")
    try:
        yield build(d, unit_logic_source())
    finally:
        shutil.rmtree(d, ignore_errors=True)


def test_units_cover_every_row_once(checker):
    r = subprocess.run([checker], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
    ok, n, rows = r.stdout.split()
    assert ok == "ok" and int(n) > 500 and int(rows) > 10 ** 6


@pytest.mark.parametrize("old,new", [
    # head pairs taken as heads 2i and 2i + 2 (the second tile reads another kv head's rows)
    ("u.h = (unit % nbh) % groups * heads_cta;", "u.h = (unit % nbh) % groups * heads_cta * 2 % p.Hq;"),
    # the last query block of a head forgotten
    ("const int qb = p.front_heavy ? unit / nbh : p.num_qblocks - 1 - unit / nbh;",
     "const int qb = p.front_heavy ? unit / nbh : p.num_qblocks - 2 - unit / nbh;"),
    # rows of a unit measured against the wrong end of a packed sequence
    ("if (u.r0 >= u.nq) return false;", "if (u.r0 > u.nq) return false;"),
])
def test_checker_catches_planted_slips(old, new, tmp_path):
    logic = unit_logic_source()
    assert logic.count(old) == 1, old
    exe = build(str(tmp_path), logic.replace(old, new))
    r = subprocess.run([exe], capture_output=True, text=True, timeout=600)
    assert r.returncode != 0 and "FAIL" in r.stdout
