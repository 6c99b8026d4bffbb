"""O2: bit-exact CPU emulation of the SageAttention-style INT8 pre-pass.

Follows the SageAttention article "又快又准，即插即用！清华8比特量化Attention，
两倍加速于FlashAttention2，各端到端任务均不掉点！", section 技术方案:
  (1) smoothing: K <- K - mean(K), which leaves softmax(Q K^T) unchanged;
  (2) Q and K are quantised to INT8 per block, with the FlashAttention block
      as the granularity, and QK^T runs as an INT8 matmul with int32
      accumulation;
  (3) P and V stay in 16-bit floating point.

The article leaves the exact constants open (its algorithm figure is an
image).  Readings taken here:
  * the mean is per channel over ALL tokens of one (batch, kv head), so the
    same vector is removed from every key row (the invariance the article
    states holds only for such a vector);
  * one scale per 128-token block x all d channels, per (batch, head);
  * symmetric absmax: scale = amax / 127, inv = 127 / amax, code =
    clamp(rint(x * inv), -127, 127), ties to even, and an all-zero block has
    scale 0 and codes 0;
  * Q is not smoothed; the softmax scale is applied after dequantisation;
  * the row term scale * q_i . mean removed from every score of row i is
    added back to lse, so lse stays the log-sum-exp of the user's scores.

Every step is IEEE binary32 / binary64 with round-to-nearest-even, in the
order written below; numpy float32 array arithmetic performs each operation
once with no fused multiply-add, which is exactly what the contract asks.
"""
from __future__ import annotations

import numpy as np

from .exact import _f64, _kv_head

QBLOCK = 128  # tokens per quantisation block and per mean partial sum


def _nblocks(N: int) -> int:
    return (N + QBLOCK - 1) // QBLOCK


def k_channel_mean(k) -> np.ndarray:
    """mean[b, g, c] over all N tokens, as float32.

    Sum order (fixed, so a parallel implementation can reproduce it bit for
    bit): within each 128-token block the tokens are added one after another
    in ascending order into a float64 partial starting at 0.0; the block
    partials are then added one after another in ascending block order into a
    float64 total starting at 0.0; mean = float32(total / float64(N)).
    """
    k = _f64(k)  # exact: every bf16/fp16 value is a float64
    B, H, N, d = k.shape
    total = np.zeros((B, H, d))
    for t in range(_nblocks(N)):
        part = np.zeros((B, H, d))
        for i in range(t * QBLOCK, min(N, (t + 1) * QBLOCK)):
            part = part + k[:, :, i, :]
        total = total + part
    return (total / np.float64(N)).astype(np.float32)


def quant_block(x32: np.ndarray):
    """Symmetric INT8 quantisation of one block of float32 values.

    Returns (codes int8 array, scale float32).  amax = max|x|; if amax is 0
    the scale is 0 and every code is 0; otherwise scale = amax/127 and
    inv = 127/amax (each one IEEE float32 division), and
    code = clamp(rint(x*inv), -127, 127) with one float32 multiply.
    """
    x32 = np.asarray(x32, dtype=np.float32)
    amax = np.float32(np.max(np.abs(x32))) if x32.size else np.float32(0)
    if amax == 0:
        return np.zeros(x32.shape, np.int8), np.float32(0)
    scale = np.float32(amax / np.float32(127.0))
    inv = np.float32(np.float32(127.0) / amax)
    prod = (x32 * inv).astype(np.float32)
    codes = np.clip(np.rint(prod), -127, 127).astype(np.int8)
    return codes, scale


def smooth_quant_k(k, mean):
    """ks = float32(k) - mean (float32 subtract), then per-block quantisation.

    Returns k8 [B, Hkv, N, d] int8 and sk [B, Hkv, ceil(N/128)] float32.
    """
    k32 = _f64(k).astype(np.float32)  # exact: 16-bit floats fit in float32
    mean = np.asarray(mean, dtype=np.float32)
    B, H, N, d = k32.shape
    ks = (k32 - mean[:, :, None, :]).astype(np.float32)
    k8 = np.zeros((B, H, N, d), np.int8)
    sk = np.zeros((B, H, _nblocks(N)), np.float32)
    for b in range(B):
        for h in range(H):
            for t in range(_nblocks(N)):
                lo, hi = t * QBLOCK, min(N, (t + 1) * QBLOCK)
                k8[b, h, lo:hi], sk[b, h, t] = quant_block(ks[b, h, lo:hi])
    return k8, sk


def quant_q(q):
    """Per-block quantisation of Q with no smoothing: q8 int8, sq float32."""
    q32 = _f64(q).astype(np.float32)
    B, H, N, d = q32.shape
    q8 = np.zeros((B, H, N, d), np.int8)
    sq = np.zeros((B, H, _nblocks(N)), np.float32)
    for b in range(B):
        for h in range(H):
            for t in range(_nblocks(N)):
                lo, hi = t * QBLOCK, min(N, (t + 1) * QBLOCK)
                q8[b, h, lo:hi], sq[b, h, t] = quant_block(q32[b, h, lo:hi])
    return q8, sq


def lse_bias(q, mean, scale) -> np.ndarray:
    """bias[b, h, i] = scale * sum_c q[b,h,i,c] * mean[b, g(h), c] in float64.

    Smoothing removes exactly this term from every score of row i, so it is
    added back to lse (softmax itself is unchanged by a per-row constant).
    """
    q = _f64(q)
    mean = np.asarray(mean, dtype=np.float64)
    B, Hq, N, d = q.shape
    Hkv = mean.shape[1]
    out = np.empty((B, Hq, N))
    for b in range(B):
        for h in range(Hq):
            out[b, h] = scale * (q[b, h] @ mean[b, _kv_head(h, Hq, Hkv)])
    return out


def prepass(q, k, scale):
    """All pre-pass outputs: (q8, sq, k8, sk, mean, bias)."""
    mean = k_channel_mean(k)
    k8, sk = smooth_quant_k(k, mean)
    q8, sq = quant_q(q)
    return q8, sq, k8, sk, mean, lse_bias(q, mean, scale)


def scores_int32(q8, k8, b, h, rows=None):
    """Exact integer scores acc[i, j] = sum_c q8[i, c] * k8[j, c] of one head.

    An int64 matmul of int8 codes is exact; |acc| <= d*127^2 < 2^31, so the
    values are those an int32 accumulator holds.
    """
    Hq, Hkv = q8.shape[1], k8.shape[1]
    g = _kv_head(h, Hq, Hkv)
    qi = q8[b, h].astype(np.int64)
    if rows is not None:
        qi = qi[np.asarray(rows)]
    return qi @ k8[b, g].astype(np.int64).T


def attention_int8(q8, sq, k8, sk, bias, v, scale, causal, rows=None):
    """Attention from the quantised scores, float64 from dequantisation on.

    s[i, j] = scale * acc[i, j] * sq[block(i)] * sk[block(j)], then O1's
    masked softmax and P V in float64.  lse = lse(s) + bias[i].
    Returns (O [B, Hq, R, d], lse [B, Hq, R]).
    """
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
            acc = scores_int32(q8, k8, b, h, rows).astype(np.float64)
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
