"""GPU parity of the lse merge (attn_merge_lse, through the C ABI) and of context-parallel (ring)
attention, against the float64 oracle.

* merge: two partial results over disjoint key sets, computed by the oracle and rounded to the
  kernel's input types (16-bit O, float32 lse), joined by the kernel; the float32 running result
  must match the float64 join of the same rounded inputs to float32 rounding, and the 16-bit
  output must match exact attention over all keys within the bf16_exact bars.
* ring: the ring of W ranks emulated on one GPU (every rank's steps in schedule order, the same
  kernels and merges as with NCCL) against exact attention over the whole sequence: the
  bf16_exact bars, and for int8_qk the int8 bars of the prefill tests (cosine >= 0.999, max
  |o - O| - h|O| <= 5e-2, max |lse - lse_ref| <= 5e-2).  The int8 ring smooths each key block by
  that block's own mean, a variant of the method; it is also held at the bf16_exact bars to an
  oracle of that variant built from oracle parts: the INT8 emulation of each step (the pre-pass of
  the rank's query block against the key block it holds, then the dequantised float64 attention),
  joined over the steps by their log-sum-exp in float64.
  (Bars: tests/tolerances.py; h is the half-ulp of the 16-bit output type.)
* ring_attention itself over a one-rank NCCL group: the same bytes as attn_fwd.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle
from attn_workloads import WORKLOADS, Workload, make_inputs
from tolerances import INT8_COS, INT8_LSE, INT8_MAX, assert_close16, cosine, max_excess

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ta():
    from tiled_attention_22_b200 import build

    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import tiled_attention_22_b200 as ta

    ta.attn_check_status()
    return ta


def _np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def assert_bf16(o, l, O, L, what, dtype="bf16"):
    assert_close16(o, l, O, L, dtype, what)


def _join64(Oa, La, Ob, Lb):
    """float64 join of two partial results by their log-sum-exp (rows with lse -inf add nothing)."""
    m = np.maximum(La, Lb)
    safe = np.where(np.isneginf(m), 0.0, m)
    wa, wb = np.exp(La - safe), np.exp(Lb - safe)
    s = wa + wb
    with np.errstate(invalid="ignore", divide="ignore"):
        O = (wa[..., None] * Oa + wb[..., None] * Ob) / s[..., None]
        L = safe + np.log(s)
    O = np.where(np.isneginf(m)[..., None], 0.0, O)
    L = np.where(np.isneginf(m), -np.inf, L)
    return O, L


@pytest.mark.parametrize("d,dt", [(128, torch.bfloat16), (64, torch.float16)])
def test_merge_two_key_halves(ta, d, dt):
    w = Workload("m", 2, 3, 3, 300, d, False, "bf16" if dt == torch.bfloat16 else "fp16", "k_offset", 97000 + d)
    q, k, v = make_inputs(w)
    a = 137
    O, L = oracle.attention(q, k, v, w.scale, False)
    Oa, La = oracle.attention(q, k[:, :, :a], v[:, :, :a], w.scale, False)
    Ob, Lb = oracle.attention(q, k[:, :, a:], v[:, :, a:], w.scale, False)
    # the kernel's inputs: 16-bit O, float32 lse
    oa = torch.from_numpy(Oa).to(dt)
    ob = torch.from_numpy(Ob).to(dt)
    la = torch.from_numpy(La).float()
    lb = torch.from_numpy(Lb).float()
    acc = torch.empty(O.shape, dtype=torch.float32, device="cuda")
    lacc = torch.empty(L.shape, dtype=torch.float32, device="cuda")
    out = torch.empty(O.shape, dtype=dt, device="cuda")
    ta.attn_merge_lse(acc, lacc, oa.cuda(), la.cuda(), first=True)
    ta.attn_merge_lse(acc, lacc, ob.cuda(), lb.cuda(), out=out)
    torch.cuda.synchronize()
    # the float32 running result against the float64 join of the same rounded inputs
    Oj, Lj = _join64(_np(oa), la.double().numpy(), _np(ob), lb.double().numpy())
    assert np.abs(_np(acc) - Oj).max() <= 4e-6 * max(1.0, np.abs(Oj).max())
    assert np.abs(lacc.cpu().double().numpy() - Lj).max() <= 2e-6 * max(1.0, np.abs(Lj).max())
    # the 16-bit output against exact attention over all keys
    assert_bf16(_np(out), lacc.cpu().double().numpy(), O, L, f"merge d={d}", "bf16" if dt == torch.bfloat16 else "fp16")
    # the 16-bit output is the float32 result rounded to nearest even
    assert torch.equal(out.cpu(), acc.cpu().to(dt))


def test_merge_rows_without_keys_and_finalise(ta):
    torch.manual_seed(5)
    rows, d = 40, 128
    oa = torch.randn(rows, d).to(torch.bfloat16)
    la = torch.randn(rows).float()
    ob = torch.randn(rows, d).to(torch.bfloat16)
    lb = torch.randn(rows).float()
    # rows 0..9: b has no keys; rows 10..19: a has no keys; rows 20..24: neither
    lb[:10] = -float("inf"); ob[:10] = 0
    la[10:25] = -float("inf"); oa[10:25] = 0
    lb[20:25] = -float("inf"); ob[20:25] = 0
    acc = torch.empty(rows, d, device="cuda")
    lacc = torch.empty(rows, device="cuda")
    ta.attn_merge_lse(acc, lacc, oa.cuda(), la.cuda(), first=True)
    ta.attn_merge_lse(acc, lacc, ob.cuda(), lb.cuda())
    out = torch.empty(rows, d, dtype=torch.bfloat16, device="cuda")
    ta.attn_merge_lse(acc, lacc, out=out)  # finalise only
    torch.cuda.synchronize()
    acc, lacc, out = acc.cpu(), lacc.cpu(), out.cpu()
    assert torch.equal(acc[:10], oa[:10].float()) and torch.equal(lacc[:10], la[:10])
    assert torch.equal(acc[10:20], ob[10:20].float()) and torch.equal(lacc[10:20], lb[10:20])
    assert (acc[20:25] == 0).all() and torch.isneginf(lacc[20:25]).all()
    assert torch.isfinite(acc).all()
    assert torch.equal(out, acc.to(torch.bfloat16))


def test_merge_argument_errors(ta):
    acc = torch.empty(4, 128, device="cuda")
    lacc = torch.empty(4, device="cuda")
    part = torch.empty(4, 128, dtype=torch.bfloat16, device="cuda")
    lp = torch.empty(4, device="cuda")
    lib = ta.load_library()
    import ctypes
    vp = ctypes.c_void_p
    p = lambda t: vp(t.data_ptr())  # noqa: E731
    assert lib.attn_merge_lse(None, p(lacc), p(part), p(lp), None, 4, 128, 0, 0, None) == ta.ATTN_ERR_ARG
    assert lib.attn_merge_lse(p(acc), p(lacc), None, None, None, 4, 128, 0, 1, None) == ta.ATTN_ERR_ARG
    assert lib.attn_merge_lse(p(acc), p(lacc), p(part), None, None, 4, 128, 0, 0, None) == ta.ATTN_ERR_ARG
    assert lib.attn_merge_lse(p(acc), p(lacc), p(part), p(lp), None, 4, 96, 0, 0, None) == ta.ATTN_ERR_UNSUPPORTED
    assert lib.attn_merge_lse(p(acc), p(lacc), p(part), p(lp), None, -1, 128, 0, 0, None) == ta.ATTN_ERR_ARG
    assert lib.attn_merge_lse(vp(acc.data_ptr() + 4), p(lacc), p(part), p(lp), None, 3, 128, 0, 0, None) \
        == ta.ATTN_ERR_ALIGN
    assert lib.attn_merge_lse(p(acc), p(lacc), p(part), p(lp), None, 0, 128, 0, 0, None) == ta.ATTN_OK


RING = [
    # B, Hq, Hkv, N, d, causal, dtype, kind, world
    (1, 4, 2, 800, 128, True, "bf16", "normal", 4),
    (1, 4, 2, 800, 128, False, "bf16", "k_offset", 2),
    (2, 2, 2, 3 * 257, 64, True, "fp16", "normal", 3),
    (1, 8, 1, 2 * 640, 128, True, "bf16", "k_offset", 2),
    (1, 2, 2, 8 * 128, 128, True, "bf16", "normal", 8),
]


@pytest.mark.parametrize("case", RING, ids=lambda c: "x".join(map(str, c)))
@pytest.mark.parametrize("mode", ["bf16_exact", "int8_qk"])
def test_ring_emulated_equals_attention_over_the_sequence(ta, case, mode):
    from tiled_attention_22_b200.ring import ring_attention_emulated

    B, Hq, Hkv, N, d, causal, dt, kind, world = case
    w = Workload("r", B, Hq, Hkv, N, d, causal, dt, kind, 98000 + RING.index(case) * 10)
    q, k, v = make_inputs(w)
    o, l = ring_attention_emulated(q.cuda(), k.cuda(), v.cuda(), world, causal=causal, mode=mode)
    torch.cuda.synchronize()
    assert ta.attn_check_status() == 0
    O, L = oracle.attention(q, k, v, w.scale, causal)
    o, l = _np(o), l.cpu().double().numpy()
    what = f"{case} {mode}"
    if mode == "bf16_exact":
        assert_bf16(o, l, O, L, what, dt)
    else:
        cos = cosine(o, O)
        assert cos >= INT8_COS, f"{what}: cosine {cos:.6f}"
        assert max_excess(o, O, dt) <= INT8_MAX, f"{what}: max err {max_excess(o, O, dt):.3e}"
        assert np.abs(l - L).max() <= INT8_LSE, f"{what}: lse err {np.abs(l - L).max():.3e}"
        Oe, Le = ring_int8_oracle(q, k, v, world, causal, w.scale)
        assert_bf16(o, l, Oe, Le, what + " vs the per-block-mean INT8 emulation", dt)


def ring_int8_oracle(q, k, v, world, causal, scale):
    """The int8 ring's method in float64, from oracle parts: rank r's query block against key block
    j (j <= r under the causal mask; every j without it) is the INT8 emulation of that pair (the
    pre-pass of q_r with k_j, which smooths k_j by its own mean, then the dequantised float64
    attention, causal on the diagonal block); the steps are joined by their log-sum-exp."""
    N = q.shape[2]
    n = N // world
    O = np.zeros(q.shape, dtype=np.float64)
    L = np.zeros(q.shape[:3], dtype=np.float64)
    for r in range(world):
        qr = q[:, :, r * n:(r + 1) * n]
        acc_o = acc_l = None
        for j in range(world):
            if causal and j > r:
                continue
            kj, vj = k[:, :, j * n:(j + 1) * n], v[:, :, j * n:(j + 1) * n]
            q8, sq, k8, sk, mean, bias = oracle.prepass(qr, kj, scale)
            Oj, Lj = oracle.attention_int8(q8, sq, k8, sk, bias, vj, scale, causal and j == r)
            acc_o, acc_l = (Oj, Lj) if acc_o is None else _join64(acc_o, acc_l, Oj, Lj)
        O[:, :, r * n:(r + 1) * n] = acc_o
        L[:, :, r * n:(r + 1) * n] = acc_l
    return O, L


def test_ring_emulated_long_sequence_sampled_rows(ta):
    """The 131K-token GQA workload split over 4 ranks (the benchmark's context-parallel case):
    sampled rows of sampled heads against exact attention."""
    from tiled_attention_22_b200.ring import ring_attention_emulated

    w = WORKLOADS[5]
    q, k, v = make_inputs(w)
    o, l = ring_attention_emulated(q.cuda(), k.cuda(), v.cuda(), 4, causal=True, mode="bf16_exact")
    torch.cuda.synchronize()
    assert ta.attn_check_status() == 0
    rng = np.random.default_rng(55)
    n = w.N // 4
    rows = sorted({0, n - 1, n, 2 * n + 5, w.N - 1} | set(rng.integers(0, w.N, 6).tolist()))
    G = w.Hq // w.Hkv
    for h in (0, w.Hq - 1):
        g = h // G
        O, L = oracle.attention(q[:, h:h + 1], k[:, g:g + 1], v[:, g:g + 1], w.scale, True, rows=rows)
        assert_bf16(_np(o[:, h:h + 1, rows]), l[:, h:h + 1, rows].cpu().double().numpy(), O, L, f"h{h}")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_ring_attention_one_rank_group_equals_attn_fwd(ta):
    """ring_attention over a one-rank NCCL group runs one step and one merge: the same bytes as
    attn_fwd (16-bit -> float32 -> 16-bit is exact)."""
    from tiled_attention_22_b200.ring import ring_attention

    w = Workload("g", 1, 4, 2, 500, 128, True, "bf16", "normal", 99000)
    q, k, v = (t.cuda() for t in make_inputs(w))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1)
    try:
        o, l = ring_attention(q, k, v, causal=True)
        o2, l2 = ta.attn_fwd(q, k, v, causal=True)
        torch.cuda.synchronize()
        assert torch.equal(o, o2) and torch.equal(l, l2)
    finally:
        dist.destroy_process_group()
