"""The allocation-free pre-pass entry point (attn_quant_smooth_k_noalloc).

Some callers cannot allocate device memory (their device memory belongs to another owner's pool,
or they cannot afford cudaMalloc's device-wide synchronisation).  For them the library offers a
pre-pass whose float64 K-mean partials live in an 8 MiB array built into the library instead of
caller scratch.  This file checks, through the C ABI, that it gives the same outputs as
attn_quant_smooth_k on two calls in a row with different inputs (the shared array keeps the
previous call's contents, which must not leak into the next call), that those outputs are the CPU
emulation's (bit for bit; the lse bias within 1e-4), and that sizes beyond the array are refused
before anything is launched.  It is named to run last.
"""
import numpy as np
import pytest
import torch

import oracle
from attn_workloads import Workload, make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ta():
    from tiled_attention_22_b200 import build

    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import tiled_attention_22_b200 as ta

    return ta


def _same(ref, got, what):
    for name in ("q8", "k8", "sq", "sk", "kmean"):
        assert torch.equal(ref[name], got[name]), f"{what}: {name} differs"
    np.testing.assert_allclose(got["lse_bias"].cpu().numpy(), ref["lse_bias"].cpu().numpy(), rtol=1e-4,
                               atol=1e-4, err_msg=what)


def test_noalloc_prepass_equals_caller_scratch_prepass_twice(ta):
    cases = [Workload("a", 2, 8, 2, 1000, 128, False, "bf16", "k_offset", 12340),
             Workload("b", 1, 4, 4, 300, 64, False, "fp16", "outlier_channels", 12350)]
    for w in cases + cases[:1]:  # a, b, then a again after b has used the array
        q, k, _ = (t.cuda() for t in make_inputs(w))
        ref = ta.attn_quant_smooth_k(q, k, scale=w.scale)
        got = ta.attn_quant_smooth_k_noalloc(q, k, scale=w.scale)
        torch.cuda.synchronize()
        assert ta.attn_check_status() == 0
        _same(ref, got, w.name)
        q8, sq, k8, sk, mean, bias = oracle.prepass(q.cpu(), k.cpu(), w.scale)
        for name, want in (("q8", q8), ("sq", sq), ("k8", k8), ("sk", sk), ("kmean", mean)):
            np.testing.assert_array_equal(got[name].cpu().numpy(), want, err_msg=f"{w.name}: {name}")
        np.testing.assert_allclose(got["lse_bias"].cpu().numpy(), bias, rtol=1e-4, atol=1e-4, err_msg=w.name)


def test_noalloc_prepass_refuses_sizes_beyond_its_array(ta):
    """One K-mean partial past the array: B*Hkv*ceil(N/128)*d = 8193 * 128 > 1 Mi.  Every pointer is
    a real device buffer of the size the call describes, so the call is in bounds on its inputs
    and outputs whatever the order of its checks; only the array would be too small."""
    from tiled_attention_22_b200 import binding

    lib = binding.load_library()
    B, Hq, Hkv, N, d = 1, 1, 1, 128 * 8193, 128
    T = N // 128
    dev = torch.device("cuda")
    q = torch.zeros((B, Hq, N, d), dtype=torch.bfloat16, device=dev)
    k = torch.zeros((B, Hkv, N, d), dtype=torch.bfloat16, device=dev)
    q8 = torch.empty((B, Hq, N, d), dtype=torch.int8, device=dev)
    k8 = torch.empty((B, Hkv, N, d), dtype=torch.int8, device=dev)
    sq = torch.empty((B, Hq, T), dtype=torch.float32, device=dev)
    sk = torch.empty((B, Hkv, T), dtype=torch.float32, device=dev)
    kmean = torch.empty((B, Hkv, d), dtype=torch.float32, device=dev)
    bias = torch.empty((B, Hq, N), dtype=torch.float32, device=dev)
    torch.cuda.synchronize()
    p = [t.data_ptr() for t in (q, k)]
    outs = [t.data_ptr() for t in (q8, sq, k8, sk, kmean, bias)]
    rc = lib.attn_quant_smooth_k_noalloc(p[0], p[1], B, Hq, Hkv, N, d, 0, 0.088, *outs, None)
    torch.cuda.synchronize()
    assert rc == binding.ATTN_ERR_WORKSPACE
    assert b"8388608" in lib.attn_last_cuda_error()
    assert ta.attn_check_status() == 0
