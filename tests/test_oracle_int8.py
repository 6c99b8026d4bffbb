"""Pins for the INT8 emulation O2, independent of the oracle's own code.

The float32 / float64 rounding steps are re-derived with exact rational
arithmetic (fractions.Fraction plus an explicit round-to-nearest-even), the
integer scores by pure-Python sums, and the sum order of the K mean by
hand-built cases whose sequential float64 result differs from the exact sum.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle

RNG = np.random.default_rng(99)
torch.manual_seed(5)


def _rne(x: Fraction, mant_bits: int, emin: int) -> Fraction:
    """Round a rational to the nearest binary float (ties to even)."""
    if x == 0:
        return Fraction(0)
    sign = -1 if x < 0 else 1
    a = abs(x)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, emin)
    quantum = Fraction(2) ** (e - mant_bits)
    n = a / quantum
    fl = n.numerator // n.denominator
    rem = n - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return sign * fl * quantum


def rne32(x):
    return _rne(Fraction(x), 23, -126)


def rne64(x):
    return _rne(Fraction(x), 52, -1022)


def rint_even(x: Fraction) -> int:
    fl = x.numerator // x.denominator
    rem = x - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return fl


def test_rational_rounding_helper_against_hardware():
    """The helper itself must agree with IEEE float32/float64 on known values."""
    for v in RNG.standard_normal(200):
        assert rne32(Fraction(float(v))) == Fraction(float(np.float32(v)))
    assert rne64(Fraction(1, 3)) == Fraction(1 / 3)
    assert rne32(Fraction(1, 3)) == Fraction(float(np.float32(1 / 3)))


def test_golden_quant_blocks(golden_dir):
    spec = json.load(open(os.path.join(golden_dir, "quant_blocks.json")))
    for case in spec["cases"]:
        codes, scale = oracle.quant_block(np.array(case["x"], np.float32))
        assert codes.tolist() == case["codes"], case["name"]
        assert float(scale) == case["scale"], case["name"]


def _quant_exact(xs):
    """Exact-arithmetic restatement of one block's quantisation."""
    amax = max(abs(Fraction(float(x))) for x in xs)
    if amax == 0:
        return [0] * len(xs), Fraction(0)
    scale = rne32(amax / 127)
    inv = rne32(Fraction(127) / amax)
    codes = [max(-127, min(127, rint_even(rne32(Fraction(float(x)) * inv)))) for x in xs]
    return codes, scale


def test_quant_block_matches_exact_arithmetic():
    for trial in range(30):
        n = int(RNG.integers(1, 200))
        x = (RNG.standard_normal(n) * 10 ** RNG.uniform(-3, 3)).astype(np.float32)
        codes, scale = oracle.quant_block(x)
        ec, es = _quant_exact(x)
        assert codes.tolist() == ec
        assert Fraction(float(scale)) == es


def test_quant_invariants():
    q = torch.randn(2, 3, 300, 64).to(torch.bfloat16)
    q8, sq = oracle.quant_q(q)
    assert sq.shape == (2, 3, 3)
    assert np.abs(q8.astype(int)).max() <= 127
    qf = q.to(torch.float32).numpy()
    for t in range(3):
        blk = q8[:, :, t * 128:(t + 1) * 128].astype(int)
        # every non-zero block reaches +-127 exactly once its amax element is coded
        assert (np.abs(blk).reshape(6, -1).max(axis=1) == 127).all()
        recon = blk * sq[:, :, t][:, :, None, None]
        err = np.abs(recon - qf[:, :, t * 128:(t + 1) * 128])
        # |code*scale - x| <= scale/2, up to float32 rounding of inv and the product
        assert (err <= sq[:, :, t][:, :, None, None] * (0.5 + 1e-5) + 1e-12).all()


def test_k_mean_matches_exact_sum_when_sums_are_exact():
    """bf16 N(0,1) values have 8 significant bits in a narrow exponent range,
    so every float64 partial sum is exact and the order cannot matter: the
    mean is float32(float64(exact_sum / N))."""
    k = (torch.randn(1, 2, 300, 16) * 2 + 0.5).to(torch.bfloat16)
    mean = oracle.k_channel_mean(k)
    kf = k.to(torch.float64).numpy()
    for h in range(2):
        for c in range(16):
            exact = sum(Fraction(float(x)) for x in kf[0, h, :, c])
            assert Fraction(float(mean[0, h, c])) == rne32(rne64(exact / 300))


def test_k_mean_sum_order_within_and_across_blocks():
    """Hand-built: 2^60 + 1 - 2^60 is 0 in sequential float64, 1 exactly.

    Within one block: tokens (2^60, 1, -2^60) give partial 0, mean 0 (an
    exact or pairwise sum would give 1/3).  Across blocks: block partials
    (2^60, 1, -2^60) in ascending order also give total 0."""
    big = 2.0 ** 60
    k = np.zeros((1, 1, 3, 2))
    k[0, 0, :, 0] = [big, 1.0, -big]
    k[0, 0, :, 1] = [1.0, 2.0, 4.0]  # exact: 7/3 rounded to float64 then float32
    mean = oracle.k_channel_mean(k)
    assert mean[0, 0, 0] == 0.0
    assert Fraction(float(mean[0, 0, 1])) == rne32(rne64(Fraction(7, 3)))
    k = np.zeros((1, 1, 257, 1))
    k[0, 0, 0, 0] = big      # block 0
    k[0, 0, 128, 0] = 1.0    # block 1
    k[0, 0, 256, 0] = -big   # block 2 (ragged: one token)
    assert oracle.k_channel_mean(k)[0, 0, 0] == 0.0
    # ...whereas the same three values inside one block in another order keep the 1
    k = np.zeros((1, 1, 3, 1))
    k[0, 0, :, 0] = [big, -big, 1.0]
    assert Fraction(float(oracle.k_channel_mean(k)[0, 0, 0])) == rne32(rne64(Fraction(1, 3)))


def test_smoothing_matches_exact_arithmetic_and_centres_k():
    k = (torch.randn(1, 1, 200, 8) + 3.0 * torch.randn(1, 1, 1, 8)).to(torch.bfloat16)
    mean = oracle.k_channel_mean(k)
    k8, sk = oracle.smooth_quant_k(k, mean)
    kf = k.to(torch.float32).numpy()
    for t, (lo, hi) in enumerate([(0, 128), (128, 200)]):
        ks = [rne32(Fraction(float(kf[0, 0, i, c])) - Fraction(float(mean[0, 0, c])))
              for i in range(lo, hi) for c in range(8)]
        codes, scale = _quant_exact([float(x) for x in ks])
        assert k8[0, 0, lo:hi].reshape(-1).tolist() == codes
        assert Fraction(float(sk[0, 0, t])) == scale
    ks = kf - mean[:, :, None, :]
    assert np.abs(ks.mean(axis=2)).max() < 1e-5


def test_scores_int32_brute_force():
    q8 = RNG.integers(-127, 128, (1, 4, 9, 16)).astype(np.int8)
    k8 = RNG.integers(-127, 128, (1, 2, 9, 16)).astype(np.int8)
    for h in range(4):
        acc = oracle.scores_int32(q8, k8, 0, h)
        g = h // 2
        for i in range(9):
            for j in range(9):
                assert acc[i, j] == sum(int(q8[0, h, i, c]) * int(k8[0, g, j, c]) for c in range(16))
    worst = oracle.scores_int32(np.full((1, 1, 1, 128), -127, np.int8), np.full((1, 1, 1, 128), -127, np.int8), 0, 0)
    assert worst[0, 0] == 128 * 127 * 127 < 2**31


def test_lse_bias_restores_user_lse():
    """Removing a vector c from every key shifts row i's scores by scale*q_i.c;
    bias = scale*q_i.mean puts it back, so lse(K - mean) + bias = lse(K)."""
    q = torch.randn(1, 4, 70, 16).to(torch.bfloat16)
    k = (torch.randn(1, 2, 70, 16) + 2.0).to(torch.bfloat16)
    v = torch.randn(1, 2, 70, 16).to(torch.bfloat16)
    mean = oracle.k_channel_mean(k)
    bias = oracle.lse_bias(q, mean, 0.25)
    ksm = k.to(torch.float64).numpy() - mean[:, :, None, :].astype(np.float64)
    O, L = oracle.attention(q, k, v, 0.25, True)
    O2, L2 = oracle.attention(q, ksm, v, 0.25, True)
    np.testing.assert_allclose(O2, O, atol=1e-12)
    np.testing.assert_allclose(L2 + bias, L, atol=1e-11)
    # brute-force the bias of one row
    qf = q.to(torch.float64).numpy()
    want = 0.25 * math.fsum(qf[0, 3, 5, c] * float(mean[0, 1, c]) for c in range(16))
    assert abs(bias[0, 3, 5] - want) < 1e-14


def _exact_int_blocks(n, d, scales):
    """Integer-valued blocks whose quantisation is exact: block t holds
    multiples of scales[t] up to 127*scales[t], with the maximum present."""
    x = np.zeros((n, d))
    for t, s in enumerate(scales):
        lo, hi = t * 128, min(n, (t + 1) * 128)
        x[lo:hi] = RNG.integers(-126, 127, (hi - lo, d)) * s
        x[lo, 0] = 127 * s
    return x


@pytest.mark.parametrize("causal", [False, True])
def test_int8_attention_equals_exact_when_quantisation_is_lossless(causal):
    """When codes*scale reproduce Q and K exactly and the K mean is 0,
    the dequantised scores are the true scores: O2's attention must equal O1.
    Blocks use scales 1 and 2, so a misplaced or dropped block scale fails."""
    n, d = 200, 8
    q = _exact_int_blocks(n, d, [1.0, 2.0])[None, None]

    def pm_block(rows, s):  # rows r and -r: every column sums to exactly 0
        half = RNG.integers(-126, 127, (rows // 2, d)) * s
        half[0, 0] = 127 * s
        return np.concatenate([half, -half])

    k = np.concatenate([pm_block(128, 2.0), pm_block(72, 1.0)])[None, None]
    v = RNG.standard_normal((1, 1, n, d))
    mean = oracle.k_channel_mean(k)
    assert np.all(mean == 0)
    k8, sk = oracle.smooth_quant_k(k, mean)
    q8, sq = oracle.quant_q(q)
    np.testing.assert_array_equal(k8.astype(float) * np.repeat(sk, 128, axis=2)[:, :, :n, None], k)
    np.testing.assert_array_equal(q8.astype(float) * np.repeat(sq, 128, axis=2)[:, :, :n, None], q)
    bias = oracle.lse_bias(q, mean, 0.003)
    O, L = oracle.attention_int8(q8, sq, k8, sk, bias, v, 0.003, causal)
    Oe, Le = oracle.attention(q, k, v, 0.003, causal)
    np.testing.assert_allclose(O, Oe, atol=1e-12)
    np.testing.assert_allclose(L, Le, atol=1e-10)
