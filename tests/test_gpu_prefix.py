"""GPU parity of the row-prefix-masked forward (attn_fwd_prefix_masked, through the C ABI) against
the float64 oracle (oracle.attention_prefix).

The APB layout's limits come from the library's ``apb_row_limits``; the oracle side takes limits
derived from a block-by-block construction of the APB mask (``apb_mask_blockwise``, written from
the article's description), and the two are checked equal first.  Bars: the bf16_exact bars
(tests/tolerances.py: |o - O| <= 2e-2 + h|O| with h the output type's half-ulp, mean abs error over
|O| <= 1 at most 2e-3, lse <= 1e-3); rows with no visible key must be O = 0 and lse = -inf.
"""
import numpy as np
import pytest
import torch

import oracle
from attn_workloads import APB_WORKLOADS, ApbWorkload, Workload, make_apb_inputs, make_inputs
from tolerances import BF16_LSE, BF16_MAX, BF16_MEAN, max_excess, mean_abs_small

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ta():
    from tiled_attention_22_b200 import build

    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import tiled_attention_22_b200 as ta

    ta.attn_check_status()
    return ta


def apb_mask_blockwise(A, Pb, L):
    M = np.zeros((A + L, A + Pb + L), dtype=bool)
    M[:A, :A] = np.tril(np.ones((A, A), dtype=bool))
    M[A:, :A] = True
    M[A:, A:A + Pb] = True
    M[A:, A + Pb:] = np.tril(np.ones((L, L), dtype=bool))
    return M


def limits_of(M):
    """Row limits of a mask whose rows are prefixes (asserted)."""
    lim = M.sum(axis=1)
    assert np.array_equal(M, np.arange(M.shape[1])[None, :] < lim[:, None])
    return lim


def _np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def run(ta, q, k, v, lim):
    o, l = ta.attn_fwd_prefix_masked(q.cuda(), k.cuda(), v.cuda(), torch.as_tensor(lim, dtype=torch.int32).cuda())
    torch.cuda.synchronize()
    assert ta.attn_check_status() == 0
    return _np(o), l.cpu().numpy().astype(np.float64)


def check(o, l, O, L, what, dtype="bf16"):
    seen = np.isfinite(L)
    assert np.isfinite(o).all(), what
    err, mean = max_excess(o, O, dtype), mean_abs_small(o, O)
    assert err <= BF16_MAX, f"{what}: max err {err:.3e}"
    assert mean <= BF16_MEAN, f"{what}: mean err {mean:.3e}"
    if seen.any():
        assert np.abs(l[seen] - L[seen]).max() <= BF16_LSE, f"{what}: lse err"
    if (~seen).any():
        assert (o[~seen] == 0).all() and np.isneginf(l[~seen]).all(), f"{what}: rows without keys"


def _qkv(B, Hq, Hkv, Nq, Nk, d, dtype, seed):
    q, _, _ = make_inputs(Workload("q", B, Hq, Hkv, Nq, d, False, dtype, "normal", seed))
    _, k, v = make_inputs(Workload("kv", B, Hq, Hkv, Nk, d, False, dtype, "normal", seed + 5))
    return q, k, v


@pytest.mark.parametrize("A,Pb,L,Hq,Hkv,d,dtype", [
    (64, 100, 300, 8, 2, 128, "bf16"),     # GQA, ragged tails everywhere
    (128, 0, 257, 4, 4, 64, "fp16"),       # no passing block
    (200, 333, 129, 6, 3, 128, "bf16"),    # anchor longer than a tile
    (1, 5, 1, 2, 1, 64, "bf16"),           # tiny
])
def test_apb_small(ta, A, Pb, L, Hq, Hkv, d, dtype):
    lim_lib = ta.apb_row_limits(A, Pb, L).numpy()
    lim = limits_of(apb_mask_blockwise(A, Pb, L))
    assert np.array_equal(lim_lib, lim)
    q, k, v = _qkv(1, Hq, Hkv, A + L, A + Pb + L, d, dtype, 60000 + A)
    O, Lr = oracle.attention_prefix(q, k, v, d ** -0.5, lim)
    o, l = run(ta, q, k, v, lim_lib)
    check(o, l, O, Lr, f"APB A={A} P={Pb} L={L}", dtype)


@pytest.mark.parametrize("Nq,Nk,kind", [(300, 700, "random"), (520, 400, "random_with_zeros"), (257, 257, "zeros"),
                                        (300, 900, "bottom_right")])
def test_general_limits(ta, Nq, Nk, kind):
    rng = np.random.default_rng(Nq + Nk)
    if kind == "random":
        lim = rng.integers(1, Nk + 50, size=Nq)                      # not monotone; some past Nk
    elif kind == "random_with_zeros":
        lim = rng.integers(-3, Nk + 1, size=Nq)
        lim[rng.random(Nq) < 0.3] = 0
    elif kind == "zeros":
        lim = np.zeros(Nq, dtype=np.int64)
    else:                                                           # Nq queries after a KV cache
        lim = Nk - Nq + np.arange(1, Nq + 1)
    q, k, v = _qkv(2, 4, 2, Nq, Nk, 128, "bf16", 61000 + Nq)
    O, Lr = oracle.attention_prefix(q, k, v, 128 ** -0.5, lim)
    o, l = run(ta, q, k, v, lim)
    check(o, l, O, Lr, kind)
    if kind == "bottom_right":
        O2, L2 = oracle.attention(q, k, v, 128 ** -0.5, True)
        np.testing.assert_allclose(O2, O, atol=1e-12)


def test_causal_and_full_limits_equal_the_plain_kernel(ta):
    """limit = i + 1 is the causal mask and limit >= Nk is no mask: the masked kernel must give the
    plain kernel's bytes exactly (same tiles, same masks)."""
    q, k, v = _qkv(1, 4, 2, 700, 700, 128, "bf16", 62000)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    for causal, lim in ((True, np.arange(1, 701)), (False, np.full(700, 10 ** 6))):
        o1, l1 = ta.attn_fwd(qc, kc, vc, causal=causal)
        o2, l2 = ta.attn_fwd_prefix_masked(qc, kc, vc, torch.as_tensor(lim, dtype=torch.int32).cuda())
        torch.cuda.synchronize()
        assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("cfg", sorted(APB_WORKLOADS))
def test_apb_workload_full_size(ta, cfg):
    """The APB workload at full size (the benchmark's launch), sampled rows of sampled heads,
    anchor and local rows both."""
    w = APB_WORKLOADS[cfg]
    q, k, v = make_apb_inputs(w)
    lim = limits_of(apb_mask_blockwise(w.anchor, w.passing, w.local))
    o, l = run(ta, q, k, v, ta.apb_row_limits(w.anchor, w.passing, w.local).numpy())
    rng = np.random.default_rng(cfg)
    rows = np.unique(np.concatenate([[0, w.anchor - 1, w.anchor, w.Nq - 1], rng.integers(0, w.Nq, 40)]))
    for h in (0, 13, w.Hq - 1):
        O, Lr = oracle.attention_prefix(q[:, h:h + 1], k[:, h // (w.Hq // w.Hkv):h // (w.Hq // w.Hkv) + 1],
                                        v[:, h // (w.Hq // w.Hkv):h // (w.Hq // w.Hkv) + 1], w.scale, lim, rows=rows)
        check(o[:, h:h + 1, rows], l[:, h:h + 1, rows], O, Lr, f"{w.name} head {h}")


def test_output_without_lse_equals_output_with_lse(ta):
    """lse = NULL only skips the lse write (rows with limit 0 still get O = 0)."""
    q, k, v = _qkv(1, 4, 2, 600, 900, 128, "bf16", 62500)
    lim = torch.as_tensor(np.concatenate([np.zeros(40), np.arange(1, 561) + 300]).astype(np.int32)).cuda()
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    o1, l1 = ta.attn_fwd_prefix_masked(qc, kc, vc, lim)
    o2, l2 = ta.attn_fwd_prefix_masked(qc, kc, vc, lim, lse=False)
    torch.cuda.synchronize()
    assert ta.attn_check_status() == 0
    assert l2 is None and l1 is not None
    assert torch.equal(o1, o2)
    assert (o2[:, :, :40] == 0).all()
