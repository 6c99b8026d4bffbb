"""O1: exact softmax attention in float64 (the plain definition).

Follows:
  * "注意力即一切：从 MHA 到 GQA", section 2.2 (four steps: Score = Q·K^T,
    softmax(Score/sqrt(d_k)), Output = weights·V) and section 2.3 (causal
    masking sets the scores of future positions to -inf before the softmax);
  * same page, section 3.2 (heads are independent) and section 5.1 (a group
    of query heads shares one K/V head).  The grouping is read as contiguous:
    query head h uses kv head h // (Hq / Hkv).
  * same page, section 3.4 (KV cache: the keys and values of earlier tokens are kept and each
    new token's query attends to all of them), which fixes the causal alignment of Nq < Nk
    query rows: they are the last Nq positions;
  * "FlashAttention" glossary page (aiunderstanding.org), FAQ: FlashAttention
    computes exactly the values of standard attention, only reordered, so the
    plain definition is the reference for the tiled kernel.

The scale is an argument (1/sqrt(d) for every named workload).  lse is the
natural-log log-sum-exp of the scaled, masked scores of each row.

Inputs may be torch tensors or numpy arrays of any float dtype; they are
converted exactly to float64.  No blocking, no online softmax: one full score
matrix per (batch, head), or per selected rows.
"""
from __future__ import annotations

import numpy as np


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # torch tensor, converted exactly
        import torch

        return x.detach().to(device="cpu", dtype=torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def _kv_head(h: int, Hq: int, Hkv: int) -> int:
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    return h // (Hq // Hkv)


def _scores(qh, kh, scale, causal, rows):
    """Scaled scores of the selected query rows against all keys, masked.

    With Nq query rows and Nk keys, query row i sits at position Nk - Nq + i (the queries are
    the last Nq tokens, as when a KV cache holds the earlier ones); under the causal mask it
    sees keys j <= Nk - Nq + i.  With Nq = Nk this is the usual j <= i.
    """
    S = scale * (qh[rows] @ kh.T)
    if causal:
        offset = kh.shape[0] - qh.shape[0]
        j = np.arange(kh.shape[0])[None, :]
        S = np.where(j > np.asarray(rows)[:, None] + offset, -np.inf, S)
    return S


def attention_probs(q, k, scale, causal, b=0, h=0, rows=None):
    """Softmax weights P (rows x N) of one (batch, head): exp(S - max) / sum."""
    q, k = _f64(q), _f64(k)
    Hq, Hkv, N = q.shape[1], k.shape[1], q.shape[2]
    rows = np.arange(N) if rows is None else np.asarray(rows)
    S = _scores(q[b, h], k[b, _kv_head(h, Hq, Hkv)], scale, causal, rows)
    m = S.max(axis=1, keepdims=True)
    P = np.exp(S - m)
    return P / P.sum(axis=1, keepdims=True)


def logsumexp_rows(S):
    m = S.max(axis=1)
    return m + np.log(np.exp(S - m[:, None]).sum(axis=1))


def attention(q, k, v, scale, causal, rows=None):
    """O = softmax(scale*Q K^T [+causal mask]) V and lse, in float64.

    q: [B, Hq, Nq, d]; k, v: [B, Hkv, Nk, d] (Nq = Nk for self-attention; Nq < Nk for
    queries that follow Nk - Nq cached tokens, see _scores).  ``rows`` optionally restricts the
    query rows (each row is independent, so a subset is exact for those rows).
    Returns (O [B, Hq, R, d], lse [B, Hq, R]).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    rows = np.arange(N) if rows is None else np.asarray(rows)
    O = np.empty((B, Hq, len(rows), v.shape[3]))
    L = np.empty((B, Hq, len(rows)))
    for b in range(B):
        for h in range(Hq):
            g = _kv_head(h, Hq, Hkv)
            S = _scores(q[b, h], k[b, g], scale, causal, rows)
            m = S.max(axis=1, keepdims=True)
            P = np.exp(S - m)
            l = P.sum(axis=1, keepdims=True)
            O[b, h] = (P @ v[b, g]) / l
            L[b, h] = m[:, 0] + np.log(l[:, 0])
    return O, L


def attention_prefix(q, k, v, scale, row_limit, rows=None):
    """O and lse with a per-query-row visible key prefix: query row i sees keys j < row_limit[i]
    (the same limits for every batch and head), in float64.

    This is the mask shape of the APB article ("在长文本上比Flash Attention快10倍！清华等提出APB序列
    并行推理框架", sections on the anchor block, the passing block and the computation step: a
    special FlashAttention kernel with a changed mask).  With the keys laid out as
    [anchor | passing | local] and the queries as [anchor | local], an anchor query sees the
    anchor causally and a local query sees the whole anchor and passing blocks and the local block
    causally; both are prefixes of the key sequence (``apb_row_limits`` in the tests builds them).
    Plain causal attention is row_limit[i] = i + 1.

    Limits are clamped to [0, Nk].  A row with limit 0 sees no key; its softmax is empty and it is
    reported as O = 0, lse = -inf (the same convention as the KV-cache decode path).
    q: [B, Hq, Nq, d]; k, v: [B, Hkv, Nk, d]; row_limit: [Nq] integers.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    lim = np.clip(np.asarray(row_limit, dtype=np.int64).reshape(-1), 0, Nk)
    if lim.shape[0] != Nq:
        raise ValueError("row_limit needs one entry per query row")
    rows = np.arange(Nq) if rows is None else np.asarray(rows)
    O = np.zeros((B, Hq, len(rows), v.shape[3]))
    L = np.full((B, Hq, len(rows)), -np.inf)
    visible = np.arange(Nk)[None, :] < lim[rows][:, None]
    seen = visible.any(axis=1)
    for b in range(B):
        for h in range(Hq):
            g = _kv_head(h, Hq, Hkv)
            S = np.where(visible, scale * (q[b, h][rows] @ k[b, g].T), -np.inf)[seen]
            m = S.max(axis=1, keepdims=True)
            P = np.exp(S - m)
            l = P.sum(axis=1, keepdims=True)
            O[b, h, seen] = (P @ v[b, g]) / l
            L[b, h, seen] = m[:, 0] + np.log(l[:, 0])
    return O, L

