"""Pins for the float64 oracle O1 (exact attention), independent of the oracle.

Each test checks the oracle against something it does not compute itself:
hand-worked closed forms, invariants stated on the pages, a pure-Python
brute force, and torch's own CPU scaled_dot_product_attention in float64.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle

RNG = np.random.default_rng(1234)


def _num(x):
    if isinstance(x, (int, float)):
        return float(x)
    if x.startswith("ln"):
        return math.log(float(x[2:]))
    return float(Fraction(x))


def _arr(a):
    return np.array([[_num(x) for x in row] for row in a], dtype=np.float64)


def test_hand_cases_n4(golden_dir):
    spec = json.load(open(os.path.join(golden_dir, "hand_cases_n4.json")))
    for case in spec["cases"]:
        if "q_heads" in case:
            q = np.stack([_arr(h) for h in case["q_heads"]])[None]
            k = _arr(case["k"])[None, None]
            v = _arr(case["v"])[None, None]
            o_exp = np.stack([_arr(h) for h in case["o_heads"]])[None]
            lse_exp = np.array([[_num(x) for x in h] for h in case["lse_heads"]])[None]
        else:
            q = _arr(case["q"])[None, None]
            k = _arr(case["k"])[None, None]
            v = _arr(case["v"])[None, None]
            o_exp = _arr(case["o"])[None, None]
            lse_exp = np.array([_num(x) for x in case["lse"]])[None, None]
        O, L = oracle.attention(q, k, v, case["scale"], case["causal"])
        np.testing.assert_allclose(O, o_exp, rtol=0, atol=1e-12, err_msg=case["name"])
        np.testing.assert_allclose(L, lse_exp, rtol=0, atol=1e-12, err_msg=case["name"])


def _brute(q, k, v, scale, causal):
    """Pure-Python loops with math.exp: no numpy, no matmul.  Query i of Nq is token
    Nk - Nq + i (the last Nq tokens), so causally it sees keys 0 .. Nk - Nq + i."""
    B, Hq, N, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    O = np.zeros((B, Hq, N, v.shape[3]))
    L = np.zeros((B, Hq, N))
    for b in range(B):
        for h in range(Hq):
            g = h // (Hq // Hkv)
            for i in range(N):
                js = range(Nk - N + i + 1) if causal else range(Nk)
                s = [scale * sum(float(q[b, h, i, c]) * float(k[b, g, j, c]) for c in range(d)) for j in js]
                m = max(s)
                w = [math.exp(x - m) for x in s]
                tot = math.fsum(w)
                for c in range(v.shape[3]):
                    O[b, h, i, c] = math.fsum(w[t] * float(v[b, g, j, c]) for t, j in enumerate(js)) / tot
                L[b, h, i] = m + math.log(tot)
    return O, L


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Hq,Hkv", [(2, 2), (4, 2), (3, 1)])
def test_brute_force_tiny(causal, Hq, Hkv):
    q = RNG.standard_normal((2, Hq, 7, 5))
    k = RNG.standard_normal((2, Hkv, 7, 5))
    v = RNG.standard_normal((2, Hkv, 7, 3))
    O, L = oracle.attention(q, k, v, 0.7, causal)
    Ob, Lb = _brute(q, k, v, 0.7, causal)
    np.testing.assert_allclose(O, Ob, rtol=0, atol=1e-12)
    np.testing.assert_allclose(L, Lb, rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_matches_torch_sdpa_float64(causal):
    """Library cross-check: torch's CPU SDPA in float64, GQA expanded."""
    B, Hq, Hkv, N, d = 2, 8, 2, 133, 64
    g = torch.Generator().manual_seed(7)
    q = torch.randn(B, Hq, N, d, generator=g, dtype=torch.float64)
    k = torch.randn(B, Hkv, N, d, generator=g, dtype=torch.float64)
    v = torch.randn(B, Hkv, N, d, generator=g, dtype=torch.float64)
    scale = 1 / math.sqrt(d)
    ke = k.repeat_interleave(Hq // Hkv, dim=1)
    ve = v.repeat_interleave(Hq // Hkv, dim=1)
    ref = torch.nn.functional.scaled_dot_product_attention(q, ke, ve, is_causal=causal, scale=scale)
    O, L = oracle.attention(q, k, v, scale, causal)
    np.testing.assert_allclose(O, ref.numpy(), rtol=0, atol=1e-12)
    # lse against torch.logsumexp of the masked scores
    S = torch.einsum("bhid,bhjd->bhij", q, ke) * scale
    if causal:
        S = S.masked_fill(torch.ones(N, N, dtype=torch.bool).triu(1), float("-inf"))
    np.testing.assert_allclose(L, torch.logsumexp(S, dim=-1).numpy(), rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_softmax_rows_sum_to_one(causal):
    """注意力即一切, section 2.2: softmax weights add up to 1 in every row."""
    q = RNG.standard_normal((1, 2, 50, 16))
    k = RNG.standard_normal((1, 2, 50, 16))
    P = oracle.attention_probs(q, k, 0.25, causal, b=0, h=1)
    np.testing.assert_allclose(P.sum(axis=1), 1.0, rtol=0, atol=1e-13)
    assert (P >= 0).all()
    if causal:
        assert np.all(np.triu(P, 1) == 0.0)


def test_identical_keys_give_mean_of_v():
    q = RNG.standard_normal((1, 1, 40, 8))
    k = np.repeat(RNG.standard_normal((1, 1, 1, 8)), 40, axis=2)
    v = RNG.standard_normal((1, 1, 40, 8))
    O, L = oracle.attention(q, k, v, 0.3, False)
    np.testing.assert_allclose(O[0, 0], np.broadcast_to(v[0, 0].mean(axis=0), (40, 8)), atol=1e-12)
    Oc, _ = oracle.attention(q, k, v, 0.3, True)
    prefix_mean = np.cumsum(v[0, 0], axis=0) / np.arange(1, 41)[:, None]
    np.testing.assert_allclose(Oc[0, 0], prefix_mean, atol=1e-12)


def test_dominant_score_reproduces_v_row():
    N, d = 32, 4
    k = np.zeros((1, 1, N, d))
    k[0, 0, 17, 0] = 1.0
    q = np.zeros((1, 1, N, d))
    q[0, 0, :, 0] = 200.0  # score 200 on key 17, 0 elsewhere: weights e^-200 elsewhere
    v = RNG.standard_normal((1, 1, N, d))
    O, _ = oracle.attention(q, k, v, 1.0, False)
    np.testing.assert_allclose(O[0, 0], np.broadcast_to(v[0, 0, 17], (N, d)), atol=1e-60)


def test_causal_row0_is_v0_and_no_future_dependence():
    """注意力即一切, section 2.3: row i sees keys 0..i only."""
    q = RNG.standard_normal((1, 2, 30, 8))
    k = RNG.standard_normal((1, 2, 30, 8))
    v = RNG.standard_normal((1, 2, 30, 8))
    O, _ = oracle.attention(q, k, v, 0.5, True)
    np.testing.assert_allclose(O[0, :, 0], v[0, :, 0], atol=1e-14)
    k2, v2 = k.copy(), v.copy()
    k2[:, :, 20:] += 5.0
    v2[:, :, 20:] -= 3.0
    O2, _ = oracle.attention(q, k2, v2, 0.5, True)
    np.testing.assert_array_equal(O2[:, :, :20], O[:, :, :20])
    assert not np.allclose(O2[:, :, 20:], O[:, :, 20:])


@pytest.mark.parametrize("causal", [False, True])
def test_per_channel_k_shift_invariance(causal):
    """SageAttention article, section 技术方案: softmax(QK^T) = softmax(Q(K - c)^T)
    for a vector c subtracted from every key; lse moves by scale*q.c."""
    q = RNG.standard_normal((1, 2, 60, 16))
    k = RNG.standard_normal((1, 2, 60, 16))
    v = RNG.standard_normal((1, 2, 60, 16))
    c = 3.0 * RNG.standard_normal((1, 2, 1, 16))
    O, L = oracle.attention(q, k, v, 0.25, causal)
    O2, L2 = oracle.attention(q, k + c, v, 0.25, causal)
    np.testing.assert_allclose(O2, O, atol=1e-12)
    np.testing.assert_allclose(L2 - L, 0.25 * np.einsum("bhid,bhd->bhi", q, c[:, :, 0]), atol=1e-11)


def test_gqa_equals_mha_on_expanded_kv():
    q = RNG.standard_normal((2, 8, 20, 8))
    k = RNG.standard_normal((2, 2, 20, 8))
    v = RNG.standard_normal((2, 2, 20, 8))
    O, L = oracle.attention(q, k, v, 0.4, True)
    O2, L2 = oracle.attention(q, np.repeat(k, 4, axis=1), np.repeat(v, 4, axis=1), 0.4, True)
    np.testing.assert_array_equal(O, O2)
    np.testing.assert_array_equal(L, L2)


def test_row_subset_is_exact():
    q = RNG.standard_normal((1, 2, 64, 8))
    k = RNG.standard_normal((1, 2, 64, 8))
    v = RNG.standard_normal((1, 2, 64, 8))
    O, L = oracle.attention(q, k, v, 0.3, True)
    rows = [0, 5, 63, 31]
    Os, Ls = oracle.attention(q, k, v, 0.3, True, rows=rows)
    np.testing.assert_allclose(Os, O[:, :, rows], atol=1e-14)
    np.testing.assert_allclose(Ls, L[:, :, rows], atol=1e-14)


def test_byte_and_flop_figures_from_the_pages():
    """注意力即一切, sections 3.4 and 8.1: a 128K x 128K fp16 score matrix is
    about 32 GB; LLaMA-7B's KV cache is 32 heads x 128 dims x 2 x 2 B = 16 KB
    per token.  The workload FLOP formula 4*B*Hq*N^2*d (halved when causal)
    is checked on its smallest case by counting multiply-adds."""
    from attn_workloads import attention_flops

    assert 128 * 1024 * 128 * 1024 * 2 == 32 * 2**30
    assert 32 * 128 * 2 * 2 == 16 * 1024
    # count: QK^T is N*N*d multiply-adds, PV the same; 2 FLOPs each
    B, H, N, d = 1, 2, 128, 64
    assert attention_flops(B, H, N, d, False) == 2 * (2 * B * H * N * N * d)
    assert attention_flops(B, H, N, d, True) == attention_flops(B, H, N, d, False) / 2


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Nq,Nk", [(1, 9), (3, 11), (5, 5)])
def test_brute_force_short_queries(causal, Nq, Nk):
    """Queries that follow a KV cache: Nq < Nk, bottom-right causal alignment."""
    q = RNG.standard_normal((1, 4, Nq, 6))
    k = RNG.standard_normal((1, 2, Nk, 6))
    v = RNG.standard_normal((1, 2, Nk, 3))
    O, L = oracle.attention(q, k, v, 0.5, causal)
    Ob, Lb = _brute(q, k, v, 0.5, causal)
    np.testing.assert_allclose(O, Ob, rtol=0, atol=1e-12)
    np.testing.assert_allclose(L, Lb, rtol=0, atol=1e-12)


def test_short_queries_match_torch_sdpa_with_explicit_mask():
    """Library cross-check for Nq < Nk: torch's SDPA with an explicit bottom-right causal mask
    (its own is_causal aligns top-left, so the mask is passed)."""
    g = torch.Generator().manual_seed(11)
    Nq, Nk = 7, 300
    q = torch.randn(2, 8, Nq, 64, generator=g, dtype=torch.float64)
    k = torch.randn(2, 2, Nk, 64, generator=g, dtype=torch.float64)
    v = torch.randn(2, 2, Nk, 64, generator=g, dtype=torch.float64)
    mask = torch.arange(Nk)[None, :] <= (torch.arange(Nq)[:, None] + Nk - Nq)
    ref = torch.nn.functional.scaled_dot_product_attention(
        q, k.repeat_interleave(4, dim=1), v.repeat_interleave(4, dim=1), attn_mask=mask, scale=0.125)
    O, _ = oracle.attention(q, k, v, 0.125, True)
    np.testing.assert_allclose(O, ref.numpy(), rtol=0, atol=1e-12)


def test_short_queries_equal_the_last_rows_of_full_self_attention():
    """The last Nq rows of Nk x Nk causal self-attention are the Nq-query problem over the same
    keys; a single query (Nq = 1) sees every key, with or without the mask."""
    q = RNG.standard_normal((1, 2, 40, 8))
    k = RNG.standard_normal((1, 2, 40, 8))
    v = RNG.standard_normal((1, 2, 40, 8))
    O, L = oracle.attention(q, k, v, 0.3, True)
    Os, Ls = oracle.attention(q[:, :, -6:], k, v, 0.3, True)
    np.testing.assert_array_equal(Os, O[:, :, -6:])
    np.testing.assert_array_equal(Ls, L[:, :, -6:])
    O1c, _ = oracle.attention(q[:, :, -1:], k, v, 0.3, True)
    O1n, _ = oracle.attention(q[:, :, -1:], k, v, 0.3, False)
    np.testing.assert_array_equal(O1c, O1n)


# ---------------------------------------------------------------------------------------------
# Per-row visible key prefix (the APB mask shape)
# ---------------------------------------------------------------------------------------------
def apb_mask_blockwise(A, Pb, L):
    """The APB mask written block by block from the article's description, independent of any
    limit formula: keys [anchor A | passing Pb | local L], queries [anchor A | local L].  Anchor
    queries see the anchor block causally; local queries see the anchor and passing blocks in
    full and the local block causally."""
    Nq, Nk = A + L, A + Pb + L
    M = np.zeros((Nq, Nk), dtype=bool)
    M[:A, :A] = np.tril(np.ones((A, A), dtype=bool))            # anchor x anchor: causal
    M[A:, :A] = True                                            # local x anchor: full
    M[A:, A:A + Pb] = True                                      # local x passing: full
    M[A:, A + Pb:] = np.tril(np.ones((L, L), dtype=bool))       # local x local: causal
    return M


def apb_limits(A, Pb, L):
    return np.concatenate([np.arange(1, A + 1), A + Pb + np.arange(1, L + 1)])


@pytest.mark.parametrize("A,Pb,L", [(2, 3, 4), (1, 0, 5), (3, 5, 1), (4, 4, 4)])
def test_apb_block_mask_is_a_row_prefix(A, Pb, L):
    """Every row of the block-built APB mask is a prefix of the key sequence, of the length the
    limit formula gives."""
    M = apb_mask_blockwise(A, Pb, L)
    lim = apb_limits(A, Pb, L)
    assert np.array_equal(M, np.arange(A + Pb + L)[None, :] < lim[:, None])


@pytest.mark.parametrize("A,Pb,L", [(2, 3, 4), (3, 0, 3)])
def test_prefix_brute_force_apb(A, Pb, L):
    q = RNG.standard_normal((1, 4, A + L, 5))
    k = RNG.standard_normal((1, 2, A + Pb + L, 5))
    v = RNG.standard_normal((1, 2, A + Pb + L, 3))
    M = apb_mask_blockwise(A, Pb, L)
    O, Lse = oracle.attention_prefix(q, k, v, 0.6, apb_limits(A, Pb, L))
    for h in range(4):
        g = h // 2
        for i in range(A + L):
            js = [j for j in range(A + Pb + L) if M[i, j]]
            s = [0.6 * sum(float(q[0, h, i, c]) * float(k[0, g, j, c]) for c in range(5)) for j in js]
            m = max(s)
            w = [math.exp(x - m) for x in s]
            tot = math.fsum(w)
            for c in range(3):
                ref = math.fsum(w[t] * float(v[0, g, j, c]) for t, j in enumerate(js)) / tot
                assert abs(O[0, h, i, c] - ref) <= 1e-12
            assert abs(Lse[0, h, i] - (m + math.log(tot))) <= 1e-12


def test_prefix_matches_torch_sdpa_with_block_mask():
    A, Pb, L = 48, 80, 200
    g = torch.Generator().manual_seed(21)
    q = torch.randn(2, 8, A + L, 64, generator=g, dtype=torch.float64)
    k = torch.randn(2, 2, A + Pb + L, 64, generator=g, dtype=torch.float64)
    v = torch.randn(2, 2, A + Pb + L, 64, generator=g, dtype=torch.float64)
    M = torch.from_numpy(apb_mask_blockwise(A, Pb, L))
    ref = torch.nn.functional.scaled_dot_product_attention(
        q, k.repeat_interleave(4, dim=1), v.repeat_interleave(4, dim=1), attn_mask=M, scale=0.125)
    O, _ = oracle.attention_prefix(q, k, v, 0.125, apb_limits(A, Pb, L))
    np.testing.assert_allclose(O, ref.numpy(), rtol=0, atol=1e-12)


def test_prefix_reduces_to_causal_and_full():
    q = RNG.standard_normal((1, 2, 37, 8))
    k = RNG.standard_normal((1, 2, 37, 8))
    v = RNG.standard_normal((1, 2, 37, 8))
    Oc, Lc = oracle.attention(q, k, v, 0.4, True)
    Op, Lp = oracle.attention_prefix(q, k, v, 0.4, np.arange(1, 38))
    np.testing.assert_array_equal(Op, Oc)
    np.testing.assert_array_equal(Lp, Lc)
    On, Ln = oracle.attention(q, k, v, 0.4, False)
    Of, Lf = oracle.attention_prefix(q, k, v, 0.4, np.full(37, 10 ** 6))  # clamped to Nk
    np.testing.assert_array_equal(Of, On)
    np.testing.assert_array_equal(Lf, Ln)


def test_prefix_empty_rows_and_row_subset():
    q = RNG.standard_normal((1, 1, 6, 4))
    k = RNG.standard_normal((1, 1, 9, 4))
    v = RNG.standard_normal((1, 1, 9, 4))
    lim = np.array([0, 3, 0, 9, 1, -5])
    O, L = oracle.attention_prefix(q, k, v, 1.0, lim)
    for i in (0, 2, 5):
        assert (O[0, 0, i] == 0).all() and L[0, 0, i] == -np.inf
    np.testing.assert_allclose(O[0, 0, 4], v[0, 0, 0], atol=1e-15)  # one visible key: its value
    Os, Ls = oracle.attention_prefix(q, k, v, 1.0, lim, rows=[3, 1])
    np.testing.assert_array_equal(Os[0, 0], O[0, 0, [3, 1]])
    np.testing.assert_array_equal(Ls[0, 0], L[0, 0, [3, 1]])
