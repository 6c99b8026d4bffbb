"""GPU parity of the FP8 (E4M3) Q K^T mode (fp8_qk) against the float64 oracle.

  pre-pass: E4M3 codes (bit patterns), sq, sk, kmean bit-exact against O3; lse_bias within 1e-4.
  fused kernel: against O3 (the same codes; the GPU accumulates the exact code products in fp32)
    at the bf16_exact bars, and against exact attention O1 at the int8_qk bars (cosine >= 0.999,
    max |o - O| - h|O| <= 5e-2 with h the output type's half-ulp, lse <= 5e-2) wherever O3 itself
    meets them, else within a small margin of O3's own error (tests/tolerances.py).
"""
import numpy as np
import pytest
import torch

import oracle
from attn_workloads import WORKLOADS, Workload, make_inputs
from oracle import fp8_emulation as f8
from sampling import boundary_rows, sample_heads
from tolerances import INT8_COS as Q_COS, INT8_LSE as Q_LSE, INT8_MAX as Q_MAX, assert_close16, quant_metrics

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


def assert_fp8(o, l, O, L, Oe, Le, what, dtype="bf16"):
    assert np.isfinite(o).all(), what
    assert_close16(o, l, Oe, Le, dtype, f"{what}: vs emulation")
    g, e = quant_metrics(o, l, O, L, dtype), quant_metrics(Oe, Le, O, L, dtype)
    if e["cos"] >= Q_COS and e["err"] <= Q_MAX and e["lse"] <= Q_LSE:
        assert g["cos"] >= Q_COS and g["err"] <= Q_MAX and g["lse"] <= Q_LSE, f"{what}: {g}"
    else:
        assert g["cos"] >= e["cos"] - 1e-3 and g["err"] <= e["err"] + 2e-2 and g["lse"] <= e["lse"] + 1e-2, \
            f"{what}: gpu {g} method {e}"
    return g, e


def emulated(q, k, v, causal, scale, rows=None):
    q8, sq, k8, sk, mean, bias = f8.prepass(q, k, scale)
    return f8.attention_fp8(q8, sq, k8, sk, bias, v, scale, causal, rows=rows)


PREPASS = [
    (1, 2, 2, 128, 64, "fp16", "normal"),
    (2, 4, 2, 300, 128, "bf16", "k_offset"),
    (1, 3, 1, 1, 64, "bf16", "normal"),
    (1, 2, 2, 515, 64, "fp16", "outlier_channels"),
    (1, 4, 2, 2048, 128, "bf16", "k_offset"),
    (1, 8, 1, 16384, 128, "bf16", "k_offset"),  # 8 query heads on one kv head
    (1, 2, 2, 16385, 64, "fp16", "normal"),     # one-token ragged tail
]


@pytest.mark.parametrize("case", PREPASS, ids=lambda c: "x".join(map(str, c)))
def test_fp8_prepass_bit_exact(ta, case):
    B, Hq, Hkv, N, d, dt, kind = case
    w = Workload("t", B, Hq, Hkv, N, d, False, dt, kind, 96000 + PREPASS.index(case) * 10)
    q, k, _ = make_inputs(w)
    pre = ta.attn_quant_smooth_k_fp8(q.cuda(), k.cuda(), scale=w.scale)
    torch.cuda.synchronize()
    q8, sq, k8, sk, mean, bias = f8.prepass(q, k, w.scale)
    np.testing.assert_array_equal(pre["kmean"].cpu().numpy(), mean)
    np.testing.assert_array_equal(pre["k8"].cpu().numpy(), f8.e4m3_bits(k8))
    np.testing.assert_array_equal(pre["sk"].cpu().numpy(), sk)
    np.testing.assert_array_equal(pre["q8"].cpu().numpy(), f8.e4m3_bits(q8))
    np.testing.assert_array_equal(pre["sq"].cpu().numpy(), sq)
    np.testing.assert_allclose(pre["lse_bias"].cpu().numpy(), bias, rtol=1e-4, atol=1e-4)


SMALL = [
    (1, 2, 2, 128, 64, False, "fp16", "normal"),
    (1, 2, 2, 300, 64, True, "bf16", "normal"),
    (2, 4, 2, 257, 128, True, "bf16", "k_offset"),
    (1, 4, 1, 257, 128, True, "fp16", "normal"),
    (1, 2, 2, 1, 64, False, "bf16", "normal"),
    (1, 3, 3, 129, 64, True, "bf16", "outlier_channels"),
    (1, 8, 2, 383, 128, False, "fp16", "k_offset"),
    (1, 2, 1, 1000, 64, False, "bf16", "normal"),
]


@pytest.mark.parametrize("case", SMALL, ids=lambda c: "x".join(map(str, c)))
def test_fp8_qk_small(ta, case):
    B, Hq, Hkv, N, d, causal, dt, kind = case
    w = Workload("t", B, Hq, Hkv, N, d, causal, dt, kind, 97000 + SMALL.index(case) * 10)
    q, k, v = make_inputs(w)
    o, l = ta.attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal, mode="fp8_qk")
    torch.cuda.synchronize()
    assert ta.attn_check_status() == 0
    O, L = oracle.attention(q, k, v, w.scale, causal)
    Oe, Le = emulated(q, k, v, causal, w.scale)
    assert_fp8(_np(o), l.cpu().numpy().astype(np.float64), O, L, Oe, Le, str(case), dt)


def test_fp8_fwd_equals_prepass_plus_fused(ta):
    w = Workload("t", 2, 4, 2, 700, 128, True, "bf16", "k_offset", 98000)
    q, k, v = (t.cuda() for t in make_inputs(w))
    o1, l1 = ta.attn_fwd(q, k, v, causal=True, mode="fp8_qk")
    pre = ta.attn_quant_smooth_k_fp8(q, k)
    o2, l2 = ta.attn_fwd_fp8_quantized(pre, v, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("cfg", [2, 3, 4, 5])
def test_fp8_full_size_sampled_rows(ta, cfg):
    w = WORKLOADS[cfg]
    q, k, v = make_inputs(w)
    o, l = ta.attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=w.causal, mode="fp8_qk")
    torch.cuda.synchronize()
    assert ta.attn_check_status() == 0
    rng = np.random.default_rng(cfg + 50)
    G = w.Hq // w.Hkv
    rows = boundary_rows(w.N, rng)
    for b, h in sample_heads(w.B, w.Hq, w.Hkv, rng):
        g = h // G
        qs, ks, vs = q[b:b + 1, h:h + 1], k[b:b + 1, g:g + 1], v[b:b + 1, g:g + 1]
        og = _np(o[b, h, rows])[None, None]
        lg = l[b, h, rows].cpu().numpy().astype(np.float64)[None, None]
        O, L = oracle.attention(qs, ks, vs, w.scale, w.causal, rows=rows)
        Oe, Le = emulated(qs, ks, vs, w.causal, w.scale, rows=rows)
        gm, em = assert_fp8(og, lg, O, L, Oe, Le, f"cfg{cfg} b{b} h{h}")
        print(f"cfg{cfg} b{b} h{h} fp8_qk vs exact: gpu {gm}  method {em}")
