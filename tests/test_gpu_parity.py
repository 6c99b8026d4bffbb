"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle.

Tolerances (tests/tolerances.py; element-wise, against float64 on the same bf16/fp16 input bytes).
Each output element may differ from the oracle by the bar plus the half-ulp of the 16-bit output
type, |o - O| <= bar + h|O| with h = 2^-8 (bf16) or 2^-11 (fp16): the kernels store O in that type,
and that rounding alone is h|O|.
  bf16_exact: max excess <= 2e-2, mean abs error (elements with |O| <= 1) <= 2e-3,
              max |lse - lse_ref| <= 1e-3
  int8_qk:    the bf16_exact bounds against the INT8 emulation (same quantised scores), and
              against exact attention cosine >= 0.999, max excess <= 5e-2, max |lse - lse_ref| <= 5e-2
              wherever the method itself (the CPU emulation) meets those bars.  On inputs where
              the emulation misses them (x10 outlier channels in both Q and K: one per-block
              absmax scale cannot hold a x10 channel and the N(0,1) channels at once), the GPU
              must stay within a small margin of the emulation's own error.
  pre-pass:   q8, k8, sq, sk, kmean bit-exact; lse_bias within 1e-4 (+1e-4 relative)
  int32 Q K^T: bit-exact.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from attn_workloads import WORKLOADS, Workload, make_inputs
from sampling import boundary_rows, sample_heads
from tolerances import (BF16_LSE, BF16_MAX, INT8_COS, INT8_LSE, INT8_MAX, assert_close16, cosine, max_excess,
                        quant_metrics)

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


def gpu_fwd(ta, q, k, v, causal, mode):
    o, l = ta.attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal, mode=mode)
    torch.cuda.synchronize()
    assert ta.attn_check_status() == 0
    return _np(o), l.cpu().numpy().astype(np.float64)


def assert_bf16(o, l, O, L, what="", dtype="bf16"):
    assert_close16(o, l, O, L, dtype, what)


def assert_int8(o, l, O, L, Oe, Le, what="", dtype="bf16"):
    """GPU int8_qk output (o, l) against exact attention (O, L) and the INT8 emulation (Oe, Le)."""
    assert np.isfinite(o).all(), what
    assert_bf16(o, l, Oe, Le, "vs emulation " + what, dtype)
    g = quant_metrics(o, l, O, L, dtype)
    e = quant_metrics(Oe, Le, O, L, dtype)  # the method's own error
    if e["cos"] >= INT8_COS and e["err"] <= INT8_MAX and e["lse"] <= INT8_LSE:
        assert g["cos"] >= INT8_COS, f"{what}: cosine {g['cos']:.6f}"
        assert g["err"] <= INT8_MAX, f"{what}: max err {g['err']:.3e}"
        assert g["lse"] <= INT8_LSE, f"{what}: lse err {g['lse']:.3e}"
    else:
        assert g["cos"] >= e["cos"] - 1e-3, f"{what}: cosine {g['cos']:.6f} vs method {e['cos']:.6f}"
        assert g["err"] <= e["err"] + 2e-2, f"{what}: max err {g['err']:.3e} vs method {e['err']:.3e}"
        assert g["lse"] <= e["lse"] + 1e-2, f"{what}: lse err {g['lse']:.3e} vs method {e['lse']:.3e}"
    return g, e


def emulated(q, k, v, causal, scale, rows=None):
    q8, sq, k8, sk, mean, bias = oracle.prepass(q, k, scale)
    return oracle.attention_int8(q8, sq, k8, sk, bias, v, scale, causal, rows=rows)


SMALL = [
    # B, Hq, Hkv, N, d, causal, dtype, kind
    (1, 2, 2, 128, 64, False, "fp16", "normal"),     # the N=128 fp16 workload's shape
    (1, 2, 2, 128, 64, True, "fp16", "normal"),
    (1, 2, 2, 300, 64, True, "bf16", "normal"),
    (2, 4, 2, 515, 128, False, "bf16", "k_offset"),
    (1, 4, 1, 257, 128, True, "fp16", "normal"),     # MQA, ragged
    (1, 2, 2, 1, 64, False, "bf16", "normal"),       # N = 1
    (1, 2, 2, 2, 128, True, "bf16", "normal"),
    (1, 3, 3, 129, 64, True, "bf16", "outlier_channels"),
    (1, 2, 2, 640, 128, True, "bf16", "k_offset"),   # several 256-row blocks, no tail
    (1, 8, 2, 383, 128, False, "fp16", "k_offset"),
    (1, 2, 1, 1000, 64, False, "bf16", "normal"),
    # many work items over several SMs with a ragged tail: 8 per head, 16 heads, 4:1 GQA
    (2, 8, 2, 1999, 128, True, "bf16", "k_offset"),
    (1, 6, 3, 1537, 64, True, "fp16", "outlier_channels"),
]


def _small(case, seed):
    B, Hq, Hkv, N, d, causal, dt, kind = case
    w = Workload("t", B, Hq, Hkv, N, d, causal, dt, kind, seed)
    return w, make_inputs(w)


@pytest.mark.parametrize("case", SMALL, ids=lambda c: "x".join(map(str, c)))
def test_bf16_exact_small(ta, case):
    w, (q, k, v) = _small(case, 70000 + SMALL.index(case) * 10)
    o, l = gpu_fwd(ta, q, k, v, w.causal, "bf16_exact")
    O, L = oracle.attention(q, k, v, w.scale, w.causal)
    assert_bf16(o, l, O, L, str(case), w.dtype)


@pytest.mark.parametrize("case", SMALL, ids=lambda c: "x".join(map(str, c)))
def test_int8_qk_small(ta, case):
    w, (q, k, v) = _small(case, 80000 + SMALL.index(case) * 10)
    o, l = gpu_fwd(ta, q, k, v, w.causal, "int8_qk")
    O, L = oracle.attention(q, k, v, w.scale, w.causal)
    Oe, Le = emulated(q, k, v, w.causal, w.scale)
    assert_int8(o, l, O, L, Oe, Le, str(case), w.dtype)


PREPASS = [
    (1, 2, 2, 128, 64, "fp16", "normal"),
    (2, 4, 2, 300, 128, "bf16", "k_offset"),
    (1, 3, 1, 1, 64, "bf16", "normal"),
    (1, 2, 2, 515, 64, "fp16", "outlier_channels"),
    (1, 4, 2, 2048, 128, "bf16", "k_offset"),
    # many short units; 16 query heads on one kv head (16K tokens); a one-token ragged tail
    (8, 8, 8, 256, 128, "bf16", "normal"),
    (1, 16, 1, 16384, 128, "bf16", "k_offset"),
    (1, 2, 2, 16385, 64, "fp16", "normal"),
]


@pytest.mark.parametrize("case", PREPASS, ids=lambda c: "x".join(map(str, c)))
def test_prepass_bit_exact(ta, case):
    B, Hq, Hkv, N, d, dt, kind = case
    w = Workload("t", B, Hq, Hkv, N, d, False, dt, kind, 90000 + PREPASS.index(case) * 10)
    q, k, _ = make_inputs(w)
    pre = ta.attn_quant_smooth_k(q.cuda(), k.cuda(), scale=w.scale)
    torch.cuda.synchronize()
    q8, sq, k8, sk, mean, bias = oracle.prepass(q, k, w.scale)
    np.testing.assert_array_equal(pre["kmean"].cpu().numpy(), mean)
    np.testing.assert_array_equal(pre["k8"].cpu().numpy(), k8)
    np.testing.assert_array_equal(pre["sk"].cpu().numpy(), sk)
    np.testing.assert_array_equal(pre["q8"].cpu().numpy(), q8)
    np.testing.assert_array_equal(pre["sq"].cpu().numpy(), sq)
    np.testing.assert_allclose(pre["lse_bias"].cpu().numpy(), bias, rtol=1e-4, atol=1e-4)


@pytest.mark.parametrize("d", [64, 128])
def test_int32_scores_bit_exact(ta, d):
    w = Workload("t", 2, 4, 2, 300, d, False, "bf16", "k_offset", 95000 + d)
    q, k, _ = make_inputs(w)
    pre = ta.attn_quant_smooth_k(q.cuda(), k.cuda())
    tiles = [(0, 0, 0, 0), (1, 3, 2, 1), (0, 1, 1, 2), (1, 2, 2, 2), (0, 3, 0, 2), (5, 0, 0, 0)]  # last: invalid
    out = ta.attn_probe_qk_int32(pre["q8"], pre["k8"], tiles).cpu().numpy()
    q8, k8 = pre["q8"].cpu().numpy(), pre["k8"].cpu().numpy()
    N = w.N
    for i, (b, h, m, n) in enumerate(tiles):
        want = np.zeros((128, 128), np.int64)
        if b < w.B:
            acc = oracle.scores_int32(q8, k8, b, h)
            blk = acc[m * 128:(m + 1) * 128, n * 128:(n + 1) * 128]
            want[:blk.shape[0], :blk.shape[1]] = blk
        np.testing.assert_array_equal(out[i], want, err_msg=str((b, h, m, n)))


@pytest.mark.parametrize("cfg", [2, 3, 4, 5])
@pytest.mark.parametrize("mode", ["bf16_exact", "int8_qk"])
def test_full_size_sampled_rows(ta, cfg, mode):
    """The named workloads at full size, in the launch configuration the benchmark times; the oracle
    computes sampled rows of sampled heads (rows are independent, so this is exact for them): every
    query-tile and work-item boundary near the start, middle and end, the last rows, random rows,
    and heads on both sides of a GQA group boundary (tests/sampling.py)."""
    w = WORKLOADS[cfg]
    q, k, v = make_inputs(w)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o, l = ta.attn_fwd(qd, kd, vd, causal=w.causal, mode=mode)
    torch.cuda.synchronize()
    assert ta.attn_check_status() == 0
    rng = np.random.default_rng(cfg)
    G = w.Hq // w.Hkv
    heads = sample_heads(w.B, w.Hq, w.Hkv, rng)
    rows = boundary_rows(w.N, rng)
    o_all, O_all, Oe_all = [], [], []
    for b, h in heads:
        g = h // G
        qs, ks, vs = q[b:b + 1, h:h + 1], k[b:b + 1, g:g + 1], v[b:b + 1, g:g + 1]
        og = _np(o[b, h, rows])[None, None]
        lg = l[b, h, rows].cpu().numpy().astype(np.float64)[None, None]
        O, L = oracle.attention(qs, ks, vs, w.scale, w.causal, rows=rows)
        if mode == "bf16_exact":
            assert_bf16(og, lg, O, L, f"cfg{cfg} b{b} h{h}")
        else:
            Oe, Le = emulated(qs, ks, vs, w.causal, w.scale, rows=rows)
            g, e = assert_int8(og, lg, O, L, Oe, Le, f"cfg{cfg} b{b} h{h}")
            print(f"cfg{cfg} b{b} h{h} int8_qk vs exact: gpu {g}  method {e}")
            o_all.append(og.reshape(-1))
            O_all.append(O.reshape(-1))
            Oe_all.append(Oe.reshape(-1))
    if mode == "int8_qk":
        c_gpu = cosine(np.concatenate(o_all), np.concatenate(O_all))
        c_emu = cosine(np.concatenate(Oe_all), np.concatenate(O_all))
        assert c_gpu >= min(INT8_COS, c_emu - 1e-3), (c_gpu, c_emu)
    assert torch.isfinite(o).all()


def test_tensors_beyond_2_31_elements(ta):
    """Q and O hold more than 2^31 elements: 136 query heads (8 kv heads) of 131072 tokens at
    d = 128, 2.28 G elements each (about 12 GB on the device with K, V, lse and the INT8
    workspace).  Head 128 starts at element 2^31, so an element offset computed in 32 bits would
    wrap there.  Sampled rows of heads on both sides of that boundary, and of the last head,
    against the oracle in both modes."""
    w = Workload("t", 1, 136, 8, 131072, 128, True, "bf16", "k_offset", 99950)
    q, k, v = make_inputs(w)
    assert q.numel() > 2 ** 31
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    rng = np.random.default_rng(31)
    rows = sorted(set([0, 1, 127, 128, 255, 256, w.N // 2, w.N - 257, w.N - 129, w.N - 128, w.N - 1]
                      + [int(x) for x in rng.integers(0, w.N, 5)]))
    G = w.Hq // w.Hkv
    for mode in ("bf16_exact", "int8_qk"):
        o, l = ta.attn_fwd(qd, kd, vd, causal=True, mode=mode)
        torch.cuda.synchronize()
        assert ta.attn_check_status() == 0
        for h in (0, 127, 128, 135):
            g = h // G
            qs, ks, vs = q[:, h:h + 1], k[:, g:g + 1], v[:, g:g + 1]
            og = _np(o[0, h, rows])[None, None]
            lg = l[0, h, rows].cpu().numpy().astype(np.float64)[None, None]
            O, L = oracle.attention(qs, ks, vs, w.scale, True, rows=rows)
            if mode == "bf16_exact":
                assert_bf16(og, lg, O, L, f"head {h}")
            else:
                Oe, Le = emulated(qs, ks, vs, True, w.scale, rows=rows)
                assert_int8(og, lg, O, L, Oe, Le, f"head {h}")
        del o, l
        torch.cuda.empty_cache()


@pytest.mark.parametrize("scale", [0.02, 0.35])
@pytest.mark.parametrize("mode", ["bf16_exact", "int8_qk"])
def test_explicit_softmax_scale(ta, mode, scale):
    """A scale other than 1/sqrt(d): 0.35 makes the scores four times larger (more running-max
    moves), 0.02 flattens them; the oracle gets the same scale."""
    w = Workload("t", 1, 4, 2, 700, 128, True, "bf16", "k_offset", 99800)
    q, k, v = make_inputs(w)
    o, l = ta.attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=True, scale=scale, mode=mode)
    torch.cuda.synchronize()
    assert ta.attn_check_status() == 0
    o, l = _np(o), l.cpu().numpy().astype(np.float64)
    O, L = oracle.attention(q, k, v, scale, True)
    if mode == "bf16_exact":
        assert_bf16(o, l, O, L, f"scale {scale}")
    else:
        Oe, Le = emulated(q, k, v, True, scale)
        assert_int8(o, l, O, L, Oe, Le, f"scale {scale}")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("mode", ["bf16_exact", "int8_qk", "fp8_qk"])
def test_output_without_lse_equals_output_with_lse(ta, mode, d):
    """lse = NULL skips the lse write (and, in the 8-bit modes, the lse-bias load); O must be the
    same bytes as with lse requested (bf16 at d = 128 takes the persistent kernel)."""
    w = Workload("t", 2, 4, 2, 777, d, True, "bf16", "k_offset", 99900 + d)
    q, k, v = (t.cuda() for t in make_inputs(w))
    o1, l1 = ta.attn_fwd(q, k, v, causal=True, mode=mode)
    o2, l2 = ta.attn_fwd(q, k, v, causal=True, mode=mode, lse=False)
    torch.cuda.synchronize()
    assert ta.attn_check_status() == 0
    assert l2 is None and l1 is not None and torch.isfinite(l1).all()
    assert torch.equal(o1, o2)


@pytest.mark.parametrize("mode", ["bf16_exact", "int8_qk"])
def test_zero_inputs(ta, mode):
    z = torch.zeros((1, 2, 300, 128), dtype=torch.bfloat16)
    o, l = gpu_fwd(ta, z, z, z, True, mode)
    assert (o == 0).all()
    np.testing.assert_allclose(l[0, 0], np.log(np.arange(1, 301)), atol=1e-4)


@pytest.mark.parametrize("mode", ["bf16_exact", "int8_qk"])
def test_large_scores_exercise_rescaling(ta, mode):
    """Scores up to a few hundred: the running max grows by more than 2^8 within rows."""
    w = Workload("t", 1, 2, 2, 700, 64, False, "bf16", "normal", 96000)
    q, k, v = make_inputs(w)
    q = (q.float() * 6).to(torch.bfloat16)
    k = (k.float() * 6 + torch.linspace(0, 3, 700)[None, None, :, None]).to(torch.bfloat16)
    o, l = gpu_fwd(ta, q, k, v, False, mode)
    O, L = oracle.attention(q, k, v, w.scale, False)
    if mode == "bf16_exact":
        assert_bf16(o, l, O, L)
    else:
        Oe, Le = emulated(q, k, v, False, w.scale)
        assert max_excess(o, Oe) <= BF16_MAX and np.abs(l - Le).max() <= INT8_LSE


def test_deterministic_and_gqa_equals_expanded_mha(ta):
    w = Workload("t", 1, 8, 2, 400, 128, True, "bf16", "k_offset", 97000)
    q, k, v = (t.cuda() for t in make_inputs(w))
    for mode in ("bf16_exact", "int8_qk"):
        o1, l1 = ta.attn_fwd(q, k, v, causal=True, mode=mode)
        o2, l2 = ta.attn_fwd(q, k, v, causal=True, mode=mode)
        o3, l3 = ta.attn_fwd(q, k.repeat_interleave(4, dim=1).contiguous(), v.repeat_interleave(4, dim=1).contiguous(),
                             causal=True, mode=mode)
        torch.cuda.synchronize()
        assert torch.equal(o1, o2) and torch.equal(l1, l2), mode
        assert torch.equal(o1, o3) and torch.equal(l1, l3), mode


def test_causal_outputs_ignore_future_keys(ta):
    w = Workload("t", 1, 2, 2, 600, 64, True, "bf16", "normal", 98000)
    q, k, v = make_inputs(w)
    o1, l1 = gpu_fwd(ta, q, k, v, True, "bf16_exact")
    k2, v2 = k.clone(), v.clone()
    k2[:, :, 300:] += 4.0
    v2[:, :, 300:] -= 2.0
    o2, l2 = gpu_fwd(ta, q, k2, v2, True, "bf16_exact")
    np.testing.assert_array_equal(o1[:, :, :300], o2[:, :, :300])
    np.testing.assert_array_equal(l1[:, :, :300], l2[:, :, :300])
    np.testing.assert_allclose(o1[:, :, 0], _np(v[:, :, 0]), atol=1e-2)  # row 0 is V[0]


@pytest.mark.parametrize("mode", ["bf16_exact", "int8_qk"])
def test_canaries_around_outputs(ta, mode):
    """Outputs placed inside guard regions: nothing outside O and lse may change."""
    w = Workload("t", 1, 2, 2, 333, 128, True, "bf16", "normal", 99000)
    q, k, v = (t.cuda() for t in make_inputs(w))
    n_o, n_l, g = q.numel(), 2 * 333, 4096
    obuf = torch.full((n_o + 2 * g,), 7.0, device="cuda", dtype=torch.bfloat16)
    lbuf = torch.full((n_l + 2 * g,), -3.0, device="cuda", dtype=torch.float32)
    o = obuf[g:g + n_o].view(q.shape)
    l = lbuf[g:g + n_l].view(1, 2, 333)
    ta.attn_fwd(q, k, v, causal=True, mode=mode, out=o, lse=l)
    torch.cuda.synchronize()
    assert (obuf[:g] == 7.0).all() and (obuf[g + n_o:] == 7.0).all()
    assert (lbuf[:g] == -3.0).all() and (lbuf[g + n_l:] == -3.0).all()
    assert torch.isfinite(o).all() and torch.isfinite(l).all()


@pytest.mark.parametrize("shape", [(1, 4, 2, 500, 128), (3, 6, 3, 333, 64), (2, 8, 8, 1024, 128), (1, 4, 1, 256, 128),
                                   (2, 8, 2, 2048, 64)])
def test_host_buffer_entry_point_matches_device_call(ta, shape):
    """attn_fwd_host pipelines copies and compute over pieces of query heads (single heads at both
    ends, runs of (batch, kv head) units between, or whole units only when N % 4 != 0); its host
    outputs must equal the device call's bit for bit (odd N exercises 4-unit-aligned pieces)."""
    B, Hq, Hkv, N, d = shape
    w = Workload("t", B, Hq, Hkv, N, d, True, "bf16", "k_offset", 99500 + N)
    q, k, v = make_inputs(w)
    qh, kh, vh = (t.pin_memory() for t in (q, k, v))
    oh = torch.empty_like(qh).pin_memory()
    lh = torch.empty((B, Hq, N), dtype=torch.float32).pin_memory()
    for mode in ("bf16_exact", "int8_qk"):
        dq, dk, dv = torch.empty_like(q, device="cuda"), torch.empty_like(k, device="cuda"), torch.empty_like(v, device="cuda")
        do = torch.empty_like(dq)
        dl = torch.empty((B, Hq, N), device="cuda", dtype=torch.float32)
        ws_bytes = ta.attn_workspace_bytes(B, Hq, Hkv, N, d, mode)
        ws = torch.empty(max(ws_bytes, 1), device="cuda", dtype=torch.uint8) if ws_bytes else None
        ta.attn_fwd_host(qh, kh, vh, oh, lh, dq, dk, dv, do, dl, causal=True, mode=mode, workspace=ws)
        o_ref, l_ref = ta.attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=True, mode=mode)
        torch.cuda.synchronize()
        assert torch.equal(oh, o_ref.cpu()) and torch.equal(lh, l_ref.cpu()), mode


def test_bounded_wait_reports_timeout_and_context_survives(ta):
    ta.attn_check_status()
    ta.attn_test_wait_timeout(2000)  # 2 ms limit on a barrier nothing completes
    assert ta.attn_check_status() == ta.ATTN_ERR_TIMEOUT
    assert ta.attn_check_status() == 0  # cleared
    w = Workload("t", 1, 2, 2, 200, 64, False, "bf16", "normal", 99700)
    q, k, v = make_inputs(w)
    o, l = gpu_fwd(ta, q, k, v, False, "bf16_exact")
    O, L = oracle.attention(q, k, v, w.scale, False)
    assert_bf16(o, l, O, L)


@pytest.mark.parametrize("use_poly", [True, False])
def test_kernel_exp2_against_cuda_exp2f(ta, use_poly):
    """The softmax's exp2 routines against CUDA's exp2f on the softmax argument range.  The
    polynomial's bound is its Remez fit (7.5e-5 relative) plus float32 rounding; ex2.approx is
    documented to about 2 ulp."""
    x = torch.cat([torch.linspace(-125.0, 8.0, 1 << 20), torch.tensor([0.0, -0.5, 0.5, -1e-7, 7.999])]).cuda()
    y = ta.attn_test_exp2(x, 1 if use_poly else 0)
    ref = torch.exp2(x.double())
    rel = ((y.double() - ref).abs() / ref).max().item()
    assert rel <= (8e-5 if use_poly else 1e-6), rel
    assert torch.isfinite(y).all()
    if use_poly:
        assert torch.equal(ta.attn_test_exp2(x, 2), y)  # packed pairs: the same bits


def test_persistent_path_deterministic_and_stream_safe(ta):
    """16-bit Q K^T at d = 128 runs on persistent CTAs that take work items from a per-stream ticket
    counter: the bytes must not depend on which CTA took which item (two calls agree), and calls on
    two streams at once (two counters) must give the bytes of the same calls made one by one."""
    w1 = Workload("p1", 2, 8, 2, 1000, 128, True, "bf16", "normal", 95000)
    w2 = Workload("p2", 1, 16, 16, 777, 128, False, "bf16", "k_offset", 95010)
    ins = [[t.cuda() for t in make_inputs(w)] for w in (w1, w2)]
    ref = []
    for (q, k, v), w in zip(ins, (w1, w2)):
        ref.append(ta.attn_fwd(q, k, v, causal=w.causal))
    again = ta.attn_fwd(*ins[0], causal=w1.causal)
    torch.cuda.synchronize()
    assert torch.equal(again[0], ref[0][0]) and torch.equal(again[1], ref[0][1])
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    outs = []
    for s, (q, k, v), w in zip(streams, ins, (w1, w2)):
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            outs.append([ta.attn_fwd(q, k, v, causal=w.causal, stream=s) for _ in range(3)])
    torch.cuda.synchronize()
    assert ta.attn_check_status() == 0
    for got, (o, l) in zip(outs, ref):
        for go, gl in got:
            assert torch.equal(go, o) and torch.equal(gl, l)
    O, L = oracle.attention(ins[0][0].cpu(), ins[0][1].cpu(), ins[0][2].cpu(), w1.scale, True)
    assert_bf16(_np(ref[0][0]), ref[0][1].cpu().numpy().astype(np.float64), O, L, "persistent")


def test_persistent_counter_per_thread_stream_and_graph_capture(ta):
    """The persistent kernel's work-item counter belongs to one stream at a time.  Two host threads
    call attn_fwd (bf16, d = 128) at once, first on torch streams of their own, then on
    cudaStreamPerThread (one handle value that names a different stream in each thread); a call
    captured into a CUDA graph is replayed on a second stream while a direct call runs on the
    capturing stream.  Every output must be the bytes of the same call made alone."""
    import ctypes
    import threading

    lib = ta.load_library()
    per_thread_stream = ctypes.c_void_p(2)  # cudaStreamPerThread
    ws = [Workload("a", 2, 8, 2, 1000, 128, True, "bf16", "normal", 95200),
          Workload("b", 1, 16, 16, 777, 128, False, "bf16", "k_offset", 95210)]
    ins = [[t.cuda() for t in make_inputs(w)] for w in ws]
    ref = [ta.attn_fwd(q, k, v, causal=w.causal) for (q, k, v), w in zip(ins, ws)]
    # the one-CTA-per-item kernel used under capture: set up before any capture
    ta.attn_fwd_prefix_masked(*ins[0], torch.arange(1, 1001, dtype=torch.int32, device="cuda"))
    reps = 4
    outs = [[(torch.empty_like(ins[i][0]), torch.empty((w.B, w.Hq, w.N), device="cuda")) for _ in range(2 * reps)]
            for i, w in enumerate(ws)]
    torch.cuda.synchronize()
    errors = []

    def worker(i):
        try:
            (q, k, v), w = ins[i], ws[i]
            s = torch.cuda.Stream()
            with torch.cuda.stream(s):
                for r in range(reps):
                    ta.attn_fwd(q, k, v, causal=w.causal, out=outs[i][r][0], lse=outs[i][r][1], stream=s)
            s.synchronize()
            for r in range(reps, 2 * reps):
                o, l = outs[i][r]
                rc = lib.attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), l.data_ptr(), w.B, w.Hq,
                                  w.Hkv, w.N, w.d, int(w.causal), w.scale, 0, 0, None, 0, per_thread_stream)
                assert rc == 0, rc
            torch.cuda.synchronize()
        except Exception as e:  # reported by the main thread
            errors.append(e)

    threads = [threading.Thread(target=worker, args=(i,)) for i in range(2)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    torch.cuda.synchronize()
    assert not errors, errors
    assert ta.attn_check_status() == 0
    for i in range(2):
        for o, l in outs[i]:
            assert torch.equal(o, ref[i][0]) and torch.equal(l, ref[i][1]), f"thread {i}"

    (q, k, v), w = ins[0], ws[0]
    cap = torch.cuda.Stream()
    o_g, l_g = torch.empty_like(q), torch.empty((w.B, w.Hq, w.N), device="cuda")
    g = torch.cuda.CUDAGraph()
    cap.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(g, stream=cap):
        ta.attn_fwd(q, k, v, causal=True, out=o_g, lse=l_g)
    torch.cuda.synchronize()
    other = torch.cuda.Stream()
    direct = []
    for _ in range(3):
        o_g.zero_()
        torch.cuda.synchronize()
        with torch.cuda.stream(other):
            g.replay()
        with torch.cuda.stream(cap):
            direct.append(ta.attn_fwd(q, k, v, causal=True, stream=cap))
        torch.cuda.synchronize()
        assert torch.equal(o_g, ref[0][0]) and torch.equal(l_g, ref[0][1])
    assert ta.attn_check_status() == 0
    for o, l in direct:
        assert torch.equal(o, ref[0][0]) and torch.equal(l, ref[0][1])
    del g
