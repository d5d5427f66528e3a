"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle harness.

This module only draws numbers; it holds none of the attention arithmetic.

Generator (counter based, so any element can be drawn on its own and any
device produces the same stream):

    key   = (seed << 40) ^ (tensor_id << 32) ^ idx          (idx < 2**32)
    x     = splitmix64(key)                                  (Steele, Lea & Flood, 2014)
    u1    = ((x >> 40) + 0.5) / 2**24                        in (0, 1)
    u2    = ((x >> 16) & 0xFFFFFF) / 2**24                   in [0, 1)
    z     = sqrt(-2 ln u1) * cos(2 pi u2)                    Box-Muller, fp64
    value = fp32(z), then bf16 by round-to-nearest-even for the bf16 workloads

Tensor ids: Q = 0, K = 1, V = 2.  ``idx`` is the flat row-major element index.
The workloads draw Q, K and V iid N(0, 1), as the configurations of the exact
attention benchmark state.
"""

from __future__ import annotations

import numpy as np

Q_ID, K_ID, V_ID = 0, 1, 2
DO_ID = 3  # dL/dO of the backward pass

_GOLDEN = 0x9E3779B97F4A7C15
_M1 = 0xBF58476D1CE4E5B9
_M2 = 0x94D049BB133111EB
_MASK64 = (1 << 64) - 1
_CHUNK = 1 << 24


def splitmix64_np(z: np.ndarray) -> np.ndarray:
    """SplitMix64 finaliser over a uint64 array (wrapping arithmetic)."""
    z = z.astype(np.uint64, copy=True)
    with np.errstate(over="ignore"):
        z += np.uint64(_GOLDEN)
        z = (z ^ (z >> np.uint64(30))) * np.uint64(_M1)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(_M2)
        z = z ^ (z >> np.uint64(31))
    return z


def _keys(seed: int, tensor_id: int, start: int, count: int) -> np.ndarray:
    if start + count > (1 << 32):
        raise ValueError("element index must stay below 2**32")
    base = ((seed << 40) ^ (tensor_id << 32)) & _MASK64
    idx = np.arange(start, start + count, dtype=np.uint64)
    return idx ^ np.uint64(base)


def _box_muller(x: np.ndarray) -> np.ndarray:
    u1 = ((x >> np.uint64(40)).astype(np.float64) + 0.5) * (1.0 / (1 << 24))
    u2 = ((x >> np.uint64(16)) & np.uint64(0xFFFFFF)).astype(np.float64) * (1.0 / (1 << 24))
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)


def normal_f32(seed: int, tensor_id: int, shape) -> np.ndarray:
    """iid N(0,1) drawn in fp64 and rounded once to fp32."""
    n = int(np.prod(shape, dtype=np.int64))
    out = np.empty(n, dtype=np.float32)
    for s in range(0, n, _CHUNK):
        c = min(_CHUNK, n - s)
        out[s:s + c] = _box_muller(splitmix64_np(_keys(seed, tensor_id, s, c))).astype(np.float32)
    return out.reshape(shape)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (round to nearest, ties to even); returns the uint16 bit patterns."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (b + np.uint64(0x7FFF) + ((b >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def normal_bf16_bits(seed: int, tensor_id: int, shape) -> np.ndarray:
    """iid N(0,1) as bf16 bit patterns (uint16), drawn as in ``normal_f32`` and rounded once."""
    return f32_to_bf16_bits(normal_f32(seed, tensor_id, shape)).reshape(shape)


# --------------------------------------------------------------------------------------------
# FP8 E4M3 (1 sign, 4 exponent bits with bias 7, 3 mantissa bits, no infinities, largest
# finite 448, code 0x7F / 0xFF is NaN) for the FP8 workloads' inputs.
# --------------------------------------------------------------------------------------------
E4M3_MAX = 448.0


def _e4m3_magnitudes() -> np.ndarray:
    """Values of the non-negative finite codes 0x00 .. 0x7E, increasing with the code."""
    codes = np.arange(0x7F, dtype=np.int64)
    e, m = codes >> 3, codes & 7
    return np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))


def f32_to_e4m3_bits(x: np.ndarray) -> np.ndarray:
    """Round to the nearest E4M3 value (ties to an even code), saturating at +-448; uint8 codes."""
    x = np.asarray(x, dtype=np.float64)
    mags = _e4m3_magnitudes()
    a = np.minimum(np.abs(x), E4M3_MAX)
    i = np.clip(np.searchsorted(mags, a), 1, len(mags) - 1)
    lo, hi = mags[i - 1], mags[i]
    down, up = a - lo, hi - a
    code = np.where(down < up, i - 1, np.where(up < down, i, np.where((i - 1) % 2 == 0, i - 1, i)))
    code = np.where(a >= E4M3_MAX, 0x7E, code)
    return (code | np.where(np.signbit(x), 0x80, 0)).astype(np.uint8)


def e4m3_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact values of E4M3 codes (NaN codes are not produced by f32_to_e4m3_bits)."""
    b = np.asarray(bits, dtype=np.uint8).astype(np.int64)
    mag = np.append(_e4m3_magnitudes(), np.nan)[b & 0x7F]
    return np.where(b & 0x80, -mag, mag).astype(np.float32)


def normal_e4m3(seed: int, tensor_id: int, shape, head_axes: int = 2):
    """iid N(0,1) (as ``normal_f32``) quantised to E4M3 with one scale per slice over the first
    ``head_axes`` axes (per (b, head)): scale = amax / 448, code = E4M3(x / scale).

    Returns (codes uint8 of ``shape``, scales float32 of shape[:head_axes]); the represented
    values are scale * e4m3_bits_to_f32(codes)."""
    x = normal_f32(seed, tensor_id, shape).astype(np.float64)
    lead = tuple(shape[:head_axes])
    flat = x.reshape(lead + (-1,))
    amax = np.abs(flat).max(axis=-1)
    scales = (np.maximum(amax, 1e-30) / E4M3_MAX).astype(np.float32)
    codes = f32_to_e4m3_bits(flat / scales.astype(np.float64)[..., None])
    return codes.reshape(shape), scales


# --------------------------------------------------------------------------------------------
# torch implementation of the same counter-based stream (used to fill large device buffers
# directly on the GPU; equality with the numpy stream is checked on the CPU by the tests).
# --------------------------------------------------------------------------------------------

def block_layout_bigbird(seed: int, n_qtiles: int, n_ktiles: int, n_random: int = 3) -> np.ndarray:
    """A fixed block-sparse layout [1][n_qtiles][n_ktiles] (uint8) in the BigBird style: the
    three blocks around the diagonal, the first block row and column (global), and n_random
    further key blocks per block row, drawn without replacement from the seeded generator."""
    bm = np.zeros((1, n_qtiles, n_ktiles), np.uint8)
    r = np.random.default_rng(seed)
    for qt in range(n_qtiles):
        bm[0, qt, max(0, qt - 1):min(n_ktiles, qt + 2)] = 1
        bm[0, qt, r.choice(n_ktiles, size=min(n_random, n_ktiles), replace=False)] = 1
    bm[0, 0, :] = 1
    bm[0, :, 0] = 1
    return bm


def _s64(c: int) -> int:
    c &= _MASK64
    return c - (1 << 64) if c >= (1 << 63) else c


def _lsr(x, k: int):
    import torch  # noqa: F401

    return (x >> k) & ((1 << (64 - k)) - 1)


def splitmix64_torch(z):
    """SplitMix64 on an int64 tensor, interpreting the bits as uint64 (wrapping)."""
    z = z + _s64(_GOLDEN)
    z = (z ^ _lsr(z, 30)) * _s64(_M1)
    z = (z ^ _lsr(z, 27)) * _s64(_M2)
    return z ^ _lsr(z, 31)


def normal_torch(seed: int, tensor_id: int, shape, dtype=None, device="cpu"):
    """Fill a tensor of ``shape`` on ``device`` with the same stream as ``normal_f32``.

    ``dtype`` is torch.float32 or torch.bfloat16 (bf16 by round-to-nearest-even from fp32).
    """
    import math

    import torch

    dtype = torch.bfloat16 if dtype is None else dtype
    n = 1
    for s in shape:
        n *= int(s)
    if n > (1 << 32):
        raise ValueError("element index must stay below 2**32")
    out = torch.empty(n, dtype=dtype, device=device)
    base = _s64((seed << 40) ^ (tensor_id << 32))
    chunk = 1 << 26
    for s in range(0, n, chunk):
        c = min(chunk, n - s)
        idx = torch.arange(s, s + c, dtype=torch.int64, device=device)
        x = splitmix64_torch(idx ^ base)
        u1 = (_lsr(x, 40).to(torch.float64) + 0.5) * (1.0 / (1 << 24))
        u2 = (_lsr(x, 16) & 0xFFFFFF).to(torch.float64) * (1.0 / (1 << 24))
        z = torch.sqrt(-2.0 * torch.log(u1)) * torch.cos((2.0 * math.pi) * u2)
        out[s:s + c] = z.to(torch.float32).to(dtype)
        del idx, x, u1, u2, z
    return out.view(*shape)
