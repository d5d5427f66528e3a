"""The seeded input generator: numpy and torch streams agree, bf16 rounding is RNE, moments."""

import numpy as np
import torch

import synth


def test_splitmix64_reference_values():
    # SplitMix64 seeded with 0: the first outputs of the published generator
    # (state advances by the golden gamma before each finalisation).
    z = np.array([0, 0x9E3779B97F4A7C15], dtype=np.uint64)
    out = synth.splitmix64_np(z)
    assert int(out[0]) == 0xE220A8397B1DCDAF
    assert int(out[1]) == 0x6E789E6AA1B965F4


def test_numpy_and_torch_streams_agree():
    shape = (3, 5, 33, 64)
    a = synth.normal_f32(7, synth.K_ID, shape)
    b = synth.normal_torch(7, synth.K_ID, shape, dtype=torch.float32).numpy()
    assert np.array_equal(a.view(np.uint32), b.view(np.uint32))
    bits = synth.normal_bf16_bits(7, synth.K_ID, shape)
    tb = synth.normal_torch(7, synth.K_ID, shape, dtype=torch.bfloat16).view(torch.int16).numpy()
    assert np.array_equal(bits.view(np.int16), tb)


def test_bf16_rounding_matches_torch_rne():
    x = np.concatenate([synth.normal_f32(1, 0, (4096,)) * 37.0,
                        np.array([1.0 + 2**-8, 1.0 + 3 * 2**-8, -1.0 - 2**-8, 0.0, -0.0], np.float32)])
    ours = synth.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    back = synth.bf16_bits_to_f32(ours)
    assert np.array_equal(back, torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_streams_are_distinct_and_normal():
    q = synth.normal_f32(2, synth.Q_ID, (1 << 18,))
    k = synth.normal_f32(2, synth.K_ID, (1 << 18,))
    q3 = synth.normal_f32(3, synth.Q_ID, (1 << 18,))
    assert abs(q.mean()) < 0.01 and abs(q.std() - 1.0) < 0.01
    assert abs(np.corrcoef(q, k)[0, 1]) < 0.01 and abs(np.corrcoef(q, q3)[0, 1]) < 0.01
    # tails of N(0,1): P(|z| > 3) = 0.0027
    assert abs(np.mean(np.abs(q) > 3.0) - 0.0027) < 0.0006


def test_e4m3_codes_round_trip_and_order():
    codes = np.arange(256, dtype=np.uint8)
    finite = codes[(codes & 0x7F) != 0x7F]
    vals = synth.e4m3_bits_to_f32(finite)
    assert np.array_equal(synth.f32_to_e4m3_bits(vals)[vals != 0], finite[vals != 0])
    mags = synth.e4m3_bits_to_f32(np.arange(0x7F, dtype=np.uint8)).astype(np.float64)
    assert np.all(np.diff(mags) > 0)
    # published anchors of the format: smallest subnormal, smallest normal, one, largest finite
    assert mags[1] == 2.0 ** -9 and mags[8] == 2.0 ** -6 and mags[0x38] == 1.0 and mags[-1] == 448.0


def test_e4m3_rounding_matches_torch():
    import torch

    rng = np.random.default_rng(5)
    x = np.concatenate([rng.standard_normal(20000) * 30, rng.uniform(-448, 448, 20000),
                        rng.standard_normal(5000) * 1e-3]).astype(np.float32)
    ours = synth.f32_to_e4m3_bits(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)
    assert synth.f32_to_e4m3_bits(np.array([1000.0, -1e9]))[0] == 0x7E  # saturates at 448


def test_normal_e4m3_per_head_scales():
    codes, scales = synth.normal_e4m3(3, synth.Q_ID, (2, 3, 50, 16))
    assert codes.shape == (2, 3, 50, 16) and scales.shape == (2, 3)
    x = synth.normal_f32(3, synth.Q_ID, (2, 3, 50, 16)).astype(np.float64)
    deq = synth.e4m3_bits_to_f32(codes).astype(np.float64) * scales[..., None, None]
    # every element within half an E4M3 step (relative 2^-4) of the drawn value, amax exact-ish
    rel = np.abs(deq - x) / np.maximum(np.abs(x), 2.0 ** -6 * scales.max())
    assert rel.max() <= 2.0 ** -4 + 1e-6
    assert np.all(np.abs(synth.e4m3_bits_to_f32(codes)).reshape(2, 3, -1).max(axis=-1) == 448.0)
