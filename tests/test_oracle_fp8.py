"""Pins for O3 (the smoothed FP8 E4M3 emulation), independent of the oracle's own arithmetic:
torch's float8_e4m3fn conversion (a library routine) for the rounding, hand-derived ties and
saturation cases, the format's bit layout decoded by torch, exact rational sums for the scores,
and a lossless case where O3 must equal the plain definition O1."""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from oracle import fp8_emulation as f8

RNG = np.random.default_rng(88)


def _torch_e4m3(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_rounding_matches_torch_float8_e4m3fn():
    # every E4M3 value, the midpoints between neighbours, points just off them, and random values
    grid = _torch_e4m3(np.linspace(-448, 448, 20001))
    vals = np.unique(np.concatenate([grid, torch.arange(0, 256, dtype=torch.uint8)
                                     .view(torch.float8_e4m3fn).to(torch.float64).numpy()]))
    vals = vals[np.isfinite(vals) & (np.abs(vals) <= 448)]
    mids = (vals[1:] + vals[:-1]) / 2
    x = np.concatenate([vals, mids, np.nextafter(mids.astype(np.float32), np.float32(np.inf)),
                        np.nextafter(mids.astype(np.float32), np.float32(-np.inf)),
                        RNG.uniform(-448, 448, 20000), RNG.uniform(-0.05, 0.05, 20000),
                        RNG.uniform(-2e-3, 2e-3, 5000)]).astype(np.float32)
    x = x[np.abs(x) <= 448]
    np.testing.assert_array_equal(f8.e4m3_round(x), _torch_e4m3(x))


@pytest.mark.parametrize("x,want", [
    (1.0625, 1.0),            # halfway between 1.0 (m=0) and 1.125 (m=1): even m=0
    (1.1875, 1.25),           # halfway between 1.125 (m=1) and 1.25 (m=2): even m=2
    (3 * 2.0 ** -10, 2.0 ** -8),  # subnormals m 2^-9: 1.5 -> even 2
    (2.0 ** -10, 0.0),        # halfway between 0 and 2^-9: even 0
    (2.0 ** -6, 2.0 ** -6),   # smallest normal
    (241.0, 240.0),           # spacing 16 in [128, 256)
    (248.0, 256.0),           # halfway between 240 (m=7) and 256 (next binade, m=0): even
    (450.0, 448.0),           # saturates
    (480.0, 448.0),           # halfway to 512, which does not exist: saturates
    (-3.3, -3.25),
])
def test_rounding_hand_cases(x, want):
    assert f8.e4m3_round(np.float32(x)) == want


def test_sign_of_zero_is_kept():
    assert np.signbit(f8.e4m3_round(np.float32(-0.0)))
    assert f8.e4m3_bits(np.array([-0.0]))[0] == 0x80
    assert f8.e4m3_bits(f8.e4m3_round(np.array([-1e-5], np.float32)))[0] == 0x80  # rounds to -0


def test_bit_layout():
    vals = np.array([1.0, 448.0, 2.0 ** -9, -2.0, 0.0, 2.0 ** -6, 7 * 2.0 ** -9, 1.75])
    want = np.array([0x38, 0x7E, 0x01, 0xC0, 0x00, 0x08, 0x07, 0x3E], dtype=np.uint8)
    np.testing.assert_array_equal(f8.e4m3_bits(vals), want)
    # and the library decodes every pattern the encoder produces back to the value
    x = f8.e4m3_round(RNG.uniform(-448, 448, 5000).astype(np.float32))
    dec = torch.from_numpy(f8.e4m3_bits(x)).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(dec, x)


def test_quant_block_scale_and_extremes():
    x = RNG.standard_normal(128 * 64).astype(np.float32)
    codes, scale = f8.quant_block(x)
    amax = np.float32(np.abs(x).max())
    assert scale == np.float32(amax / np.float32(448))
    assert np.abs(codes).max() == 448.0
    assert codes[np.argmax(np.abs(x))] == np.sign(x[np.argmax(np.abs(x))]) * 448.0
    z, zs = f8.quant_block(np.zeros(10, np.float32))
    assert zs == 0 and not z.any()


def test_scores_are_exact_sums():
    q = RNG.standard_normal((1, 2, 5, 16)).astype(np.float32)
    k = RNG.standard_normal((1, 1, 7, 16)).astype(np.float32)
    q8, _, k8, _, _, _ = f8.prepass(torch.from_numpy(q).to(torch.bfloat16), torch.from_numpy(k).to(torch.bfloat16), 0.25)
    acc = q8[0, 1] @ k8[0, 0].T
    for i in range(5):
        for j in range(7):
            exact = sum(Fraction(float(a)) * Fraction(float(b)) for a, b in zip(q8[0, 1, i], k8[0, 0, j]))
            assert Fraction(float(acc[i, j])) == exact


def test_lossless_case_equals_exact_attention():
    """Q and K that are E4M3 values times a power of two, with block maxima at 448 times that
    power, and K's channel means exactly zero (rows come in +-pairs): smoothing and quantisation
    are exact, and O3 must equal O1 bit for bit."""
    N, d = 128, 32
    qv = f8.e4m3_round(RNG.uniform(-448, 448, (N, d)).astype(np.float32))
    qv[0, 0] = 448.0
    kv = f8.e4m3_round(RNG.uniform(-448, 448, (N // 2, d)).astype(np.float32))
    kv[0, 0] = -448.0
    kv = np.concatenate([kv, -kv])
    q = torch.tensor(qv * 2.0 ** -6, dtype=torch.float32)[None, None]
    k = torch.tensor(kv * 2.0 ** -7, dtype=torch.float32)[None, None]
    v = torch.tensor(RNG.standard_normal((N, d)), dtype=torch.float32)[None, None]
    q8, sq, k8, sk, mean, bias = f8.prepass(q, k, 0.125)
    assert not np.any(mean) and not np.any(bias)
    np.testing.assert_array_equal(q8[0, 0], qv)
    np.testing.assert_array_equal(k8[0, 0], kv)
    assert sq[0, 0, 0] == np.float32(2.0 ** -6) and sk[0, 0, 0] == np.float32(2.0 ** -7)
    for causal in (False, True):
        O3, L3 = f8.attention_fp8(q8, sq, k8, sk, bias, v, 0.125, causal)
        O1, L1 = oracle.attention(q, k, v, 0.125, causal)
        np.testing.assert_array_equal(O3, O1)
        np.testing.assert_array_equal(L3, L1)
