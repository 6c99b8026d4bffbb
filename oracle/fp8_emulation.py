"""O3: CPU emulation of the smoothed FP8 (E4M3) Q K^T mode.

The SageAttention article ("又快又准，即插即用！清华8比特量化Attention，两倍加速于FlashAttention2，各端到端任务
均不掉点！", section 技术方案) smooths K by its per-channel mean and quantises Q and K per block
before an 8-bit Q K^T; it weighs INT8 against FP8 for that product.  This module is the FP8
variant: the same smoothing, the same 128-token blocks and the same lse bias as O2
(``int8_emulation``), with E4M3 codes in place of INT8 ones.

E4M3 (the "fn" variant: 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits, no
infinities): normal values (1 + m/8) 2^(e-7) for e = 1..15 (m = 0..6 when e = 15), subnormals
m 2^-9, largest finite 448, smallest positive 2^-9.  Readings taken here:
  * scale = amax / 448 and inv = 448 / amax (each one IEEE float32 division), so the block's
    largest magnitude maps to the largest finite E4M3 value; an all-zero block has scale 0 and
    codes 0;
  * code = E4M3(fl32(x * inv)): one float32 multiply, then round to nearest E4M3 value with
    ties to even, saturating at +-448 (values here never exceed 448 by more than the float32
    rounding of the multiply);
  * scores = sum_c q8 * k8 of the code VALUES, exact (each product has at most 8 significant
    bits and exponents within 2^-18 .. 2^17, so a float64 sum of 128 of them is exact), then
    s = scale * acc * sq * sk in float64, as in O2.

Every step is IEEE binary32 / binary64 with round-to-nearest-even.
"""
from __future__ import annotations

import numpy as np

from .exact import _f64, _kv_head
from .int8_emulation import QBLOCK, _nblocks, k_channel_mean, lse_bias

E4M3_MAX = 448.0
_MIN_NORMAL_EXP = -6   # smallest normal binade 2^-6
_MANT_BITS = 3


def e4m3_round(x) -> np.ndarray:
    """Nearest E4M3 value of each element (ties to even), saturated to +-448, as float64.

    In the binade [2^e, 2^(e+1)) (e >= -6) the E4M3 values are spaced 2^(e-3); below 2^-6 they
    are the subnormals, spaced 2^-9.  Dividing by the spacing is exact (a power of two), rint
    rounds half to even, and the product is exact again; a value that rounds up to the next
    binade lands on its first value, which is the correct result.  The sign of zero is kept.
    """
    x = np.asarray(x, dtype=np.float64)
    ax = np.abs(x)
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    # log2 of a float64 can be off by one ulp near a power of two: fix e so 2^e <= ax < 2^(e+1)
    e = np.where(np.exp2(e) > ax, e - 1, e)
    e = np.where(np.exp2(e + 1) <= ax, e + 1, e)
    e = np.maximum(e, _MIN_NORMAL_EXP)
    q = np.exp2(e - _MANT_BITS)
    y = np.rint(x / q) * q
    y = np.clip(y, -E4M3_MAX, E4M3_MAX)
    return np.where(ax == 0, x, y)  # keep +0 / -0 exactly


def e4m3_bits(vals) -> np.ndarray:
    """The E4M3 bit pattern (uint8) of values that are exactly representable (e.g. from
    e4m3_round): sign << 7 | exponent field << 3 | mantissa field."""
    v = np.asarray(vals, dtype=np.float64)
    sign = np.signbit(v).astype(np.uint8) << 7
    a = np.abs(v)
    out = np.zeros(v.shape, dtype=np.uint8)
    sub = a < 2.0 ** _MIN_NORMAL_EXP
    m_sub = np.rint(a / 2.0 ** -9)
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.where(np.exp2(e) > a, e - 1, e)
    e = np.where(np.exp2(e + 1) <= a, e + 1, e)
    m_norm = np.rint((a / np.exp2(e) - 1.0) * 8.0)
    field = np.where(sub, m_sub, ((e + 7) * 8 + m_norm))
    if not np.array_equal(np.where(sub, m_sub * 2.0 ** -9, (1 + m_norm / 8.0) * np.exp2(e)), a):
        raise ValueError("value not representable in E4M3")
    out[...] = field.astype(np.uint8)
    return out | sign


def quant_block(x32: np.ndarray):
    """FP8 quantisation of one block of float32 values: (code values float64, scale float32)."""
    x32 = np.asarray(x32, dtype=np.float32)
    amax = np.float32(np.max(np.abs(x32))) if x32.size else np.float32(0)
    if amax == 0:
        return np.zeros(x32.shape), np.float32(0)
    scale = np.float32(amax / np.float32(E4M3_MAX))
    inv = np.float32(np.float32(E4M3_MAX) / amax)
    prod = (x32 * inv).astype(np.float32)
    return e4m3_round(prod), scale


def _quant(x32):
    B, H, N, d = x32.shape
    codes = np.zeros((B, H, N, d))
    sc = np.zeros((B, H, _nblocks(N)), np.float32)
    for b in range(B):
        for h in range(H):
            for t in range(_nblocks(N)):
                lo, hi = t * QBLOCK, min(N, (t + 1) * QBLOCK)
                codes[b, h, lo:hi], sc[b, h, t] = quant_block(x32[b, h, lo:hi])
    return codes, sc


def prepass(q, k, scale):
    """(q8, sq, k8, sk, mean, bias): code VALUES (float64 arrays) and float32 scales; the mean
    and the lse bias are O2's."""
    mean = k_channel_mean(k)
    k32 = _f64(k).astype(np.float32)
    ks = (k32 - np.asarray(mean, np.float32)[:, :, None, :]).astype(np.float32)
    k8, sk = _quant(ks)
    q8, sq = _quant(_f64(q).astype(np.float32))
    return q8, sq, k8, sk, mean, lse_bias(q, mean, scale)


def attention_fp8(q8, sq, k8, sk, bias, v, scale, causal, rows=None):
    """Attention from the FP8 scores, float64 from the (exact) code products on:
    s[i, j] = scale * acc[i, j] * sq[block(i)] * sk[block(j)], O1's masked softmax and P V,
    lse = lse(s) + bias[i].  Returns (O [B, Hq, R, d], lse [B, Hq, R])."""
    v = _f64(v)
    B, Hq, N, d = q8.shape
    Hkv = k8.shape[1]
    rows = np.arange(N) if rows is None else np.asarray(rows)
    qblk = rows // QBLOCK
    kblk = np.arange(N) // QBLOCK
    O = np.empty((B, Hq, len(rows), v.shape[3]))
    L = np.empty((B, Hq, len(rows)))
    for b in range(B):
        for h in range(Hq):
            g = _kv_head(h, Hq, Hkv)
            acc = q8[b, h][rows] @ k8[b, g].T
            s = scale * acc * sq[b, h][qblk][:, None].astype(np.float64) \
                * sk[b, g][kblk][None, :].astype(np.float64)
            if causal:
                s = np.where(np.arange(N)[None, :] > rows[:, None], -np.inf, s)
            m = s.max(axis=1, keepdims=True)
            P = np.exp(s - m)
            l = P.sum(axis=1, keepdims=True)
            O[b, h] = (P @ v[b, g]) / l
            L[b, h] = m[:, 0] + np.log(l[:, 0]) + np.asarray(bias)[b, h][rows]
    return O, L
