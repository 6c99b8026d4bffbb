"""GPU parity of the KV-cache decode path (attn_decode, through the C ABI) against the float64 oracle.

The oracle is the plain definition with Nq query rows after Nk - Nq cached tokens: for sequence b
it is called on the first kv_lens[b] cached keys, and under the causal mask query i sees keys
0 .. kv_lens[b] - Nq + i.  Rows that see no key must come out as O = 0 and lse = -inf.

Tolerances: the bf16_exact bars of the prefill path (tests/tolerances.py: |o - O| <= 2e-2 + h|O| with
h the half-ulp of the 16-bit output type, mean abs error over |O| <= 1 at most 2e-3; max
|lse - lse_ref| <= 1e-3).  Cache entries past kv_lens[b] are filled
with NaN before the call: they must not reach any output.
"""
import numpy as np
import pytest
import torch

import oracle
from attn_workloads import DECODE_WORKLOADS, DecodeWorkload, make_decode_inputs
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


def _np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def expected(q, k, v, lens, causal, scale, heads=None):
    """(O, lse, seen) from the oracle, per sequence; seen marks rows with at least one visible key.
    ``heads`` optionally restricts the query heads (a list of (b, h))."""
    B, Hq, Nq, d = q.shape
    O = np.zeros((B, Hq, Nq, d))
    L = np.full((B, Hq, Nq), -np.inf)
    seen = np.zeros((B, Hq, Nq), dtype=bool)
    G = Hq // k.shape[1]
    pairs = heads if heads is not None else [(b, h) for b in range(B) for h in range(Hq)]
    for b, h in pairs:
        n = int(lens[b])
        first = max(0, Nq - n) if causal else (0 if n > 0 else Nq)  # rows before `first` see no key
        if first >= Nq:
            continue
        g = h // G
        Ob, Lb = oracle.attention(q[b:b + 1, h:h + 1], k[b:b + 1, g:g + 1, :n], v[b:b + 1, g:g + 1, :n], scale,
                                  causal, rows=np.arange(first, Nq))
        O[b, h, first:] = Ob[0, 0]
        L[b, h, first:] = Lb[0, 0]
        seen[b, h, first:] = True
    return O, L, seen


def check(o, l, O, L, seen, what, heads=None, dtype="bf16"):
    if heads is not None:
        idx = tuple(np.array(heads).T)
        o, l, O, L, seen = o[idx], l[idx], O[idx], L[idx], seen[idx]
    assert np.isfinite(o).all(), f"{what}: non-finite output"
    err, mean = max_excess(o, O, dtype), mean_abs_small(o, O)
    assert err <= BF16_MAX, f"{what}: max err {err:.3e}"
    assert mean <= BF16_MEAN, f"{what}: mean err {mean:.3e}"
    if seen.any():
        assert np.abs(l[seen] - L[seen]).max() <= BF16_LSE, f"{what}: lse err {np.abs(l[seen] - L[seen]).max():.3e}"
    if (~seen).any():
        assert (o[~seen] == 0).all(), f"{what}: rows without keys must be 0"
        assert np.isneginf(l[~seen]).all(), f"{what}: rows without keys must have lse = -inf"


def run(ta, q, k, v, lens, causal, ctas, nan_tail=True):
    """Call attn_decode on copies of the inputs whose cache entries past kv_lens are NaN."""
    kc, vc = k, v
    if nan_tail and lens is not None:
        kc, vc = k.clone(), v.clone()
        for b, n in enumerate(lens.tolist()):
            kc[b, :, n:] = float("nan")
            vc[b, :, n:] = float("nan")
    o, l = ta.attn_decode(q.cuda(), kc.cuda(), vc.cuda(), None if lens is None else lens.cuda(), causal=causal,
                          num_ctas=ctas)
    torch.cuda.synchronize()
    assert ta.attn_check_status() == 0
    return _np(o), l.cpu().numpy().astype(np.float64)


def _inputs(B, Hq, Hkv, Nq, Nk, dtype, kind, seed, lens):
    w = DecodeWorkload("case", B, Hq, Hkv, Nq, Nk, 128, False, dtype, kind, "full", seed)
    q, k, v, _ = make_decode_inputs(w)
    return q, k, v, (None if lens is None else torch.tensor(lens, dtype=torch.int32))


# (B, Hq, Hkv, Nq, Nk, causal, kv_lens, num_ctas, dtype, kind)
CASES = [
    (2, 8, 8, 1, 300, False, [300, 1], 1, "bf16", "normal"),            # MHA, one row per kv head
    (2, 32, 8, 1, 1000, False, [1000, 513], 0, "bf16", "k_offset"),      # GQA 4:1, one CTA per SM
    (1, 32, 8, 4, 777, True, [777], 3, "fp16", "normal"),                 # 16 rows, causal drafts
    (3, 16, 2, 4, 2048, True, [2048, 129, 3], 5, "bf16", "normal"),       # 32 rows; len 3 < Nq
    (2, 8, 1, 8, 640, True, [640, 200], 2, "bf16", "k_offset"),           # 64 rows (MQA)
    (1, 4, 4, 16, 256, False, [0], 1, "bf16", "normal"),                  # empty cache
    (2, 4, 1, 16, 4096, True, [4096, 4000], 7, "fp16", "normal"),         # 64 rows, 7 CTAs
    (5, 8, 2, 1, 900, False, [0, 900, 1, 0, 129], 3, "bf16", "normal"),   # empty units between pieces
    (6, 8, 8, 1, 256, False, [256, 3, 128, 129, 0, 200], 0, "bf16", "normal"),  # more CTAs than tiles
    (1, 2, 2, 1, 128 * 40, False, None, 1, "bf16", "k_offset"),           # 40 tiles in one CTA
    (2, 24, 8, 2, 3000, True, [3000, 2999], 0, "bf16", "normal"),         # 6 rows, padded to 16
]


@pytest.mark.parametrize("case", CASES)
def test_decode_small(ta, case):
    B, Hq, Hkv, Nq, Nk, causal, lens, ctas, dtype, kind = case
    q, k, v, lt = _inputs(B, Hq, Hkv, Nq, Nk, dtype, kind, 90000 + CASES.index(case) * 10, lens)
    ll = lt.tolist() if lt is not None else [Nk] * B
    O, L, seen = expected(q, k, v, ll, causal, 128 ** -0.5)
    o, l = run(ta, q, k, v, lt, causal, ctas)
    check(o, l, O, L, seen, f"case {case}", dtype=dtype)


def test_cta_counts_agree(ta):
    """1, 2, 5, 16, 37 and 148 CTAs (different cuts of the tile sequence into pieces): each within
    the bars of the oracle, and the merged lse equal to the one-CTA lse up to float rounding."""
    q, k, v, lt = _inputs(3, 32, 8, 2, 5000, "bf16", "normal", 91000, [5000, 4321, 77])
    O, L, seen = expected(q, k, v, [5000, 4321, 77], True, 128 ** -0.5)
    ref = None
    for s in (1, 2, 5, 16, 37, 148):
        o, l = run(ta, q, k, v, lt, True, s)
        check(o, l, O, L, seen, f"{s} CTAs")
        if ref is None:
            ref = l
        else:
            assert np.abs(l - ref).max() <= 1e-4


def test_decode_deterministic_and_gqa_equals_mha(ta):
    """Same call twice: identical bytes.  GQA against the same problem with K/V expanded to one
    head per query head (each query head then its own group): same values up to rounding order."""
    q, k, v, lt = _inputs(1, 16, 4, 1, 2000, "bf16", "normal", 92000, [1999])
    a = run(ta, q, k, v, lt, False, 3)
    b = run(ta, q, k, v, lt, False, 3)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    ke, ve = k.repeat_interleave(4, dim=1).contiguous(), v.repeat_interleave(4, dim=1).contiguous()
    c = run(ta, q, ke, ve, lt, False, 3)
    assert np.abs(a[0] - c[0]).max() <= 1e-2
    assert np.abs(a[1] - c[1]).max() <= 1e-4


def test_causal_future_keys_do_not_matter(ta):
    """Under the causal mask the first drafted token must not see the later ones: changing the
    last Nq - 1 cached keys/values changes only the rows that see them."""
    q, k, v, lt = _inputs(1, 8, 2, 4, 700, "bf16", "normal", 93000, [700])
    a_o, a_l = run(ta, q, k, v, lt, True, 2)
    k2, v2 = k.clone(), v.clone()
    k2[:, :, 699] += 3.0
    v2[:, :, 699] -= 2.0
    b_o, b_l = run(ta, q, k2, v2, lt, True, 2)
    assert np.array_equal(a_o[:, :, :3], b_o[:, :, :3]) and np.array_equal(a_l[:, :, :3], b_l[:, :, :3])
    assert not np.allclose(a_o[:, :, 3], b_o[:, :, 3])


def test_unsupported_shapes_raise(ta):
    q = torch.zeros(1, 8, 16, 128, dtype=torch.bfloat16, device="cuda")  # 8 heads x 16 tokens = 128 rows
    k = torch.zeros(1, 1, 256, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ta.AttnError, match="unsupported"):
        ta.attn_decode(q, k, k)
    q64 = torch.zeros(1, 2, 1, 64, dtype=torch.bfloat16, device="cuda")
    k64 = torch.zeros(1, 2, 256, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ta.AttnError, match="unsupported"):
        ta.attn_decode(q64, k64, k64)


@pytest.mark.parametrize("cfg", sorted(DECODE_WORKLOADS))
def test_decode_workloads_full_size(ta, cfg):
    """The named decode workloads at full size, in the launch configuration the benchmark times
    (one CTA per SM), checked on 24 sampled (batch, query head) pairs."""
    w = DECODE_WORKLOADS[cfg]
    q, k, v, lt = make_decode_inputs(w)
    rng = np.random.default_rng(cfg)
    heads = sorted({(int(rng.integers(w.B)), int(rng.integers(w.Hq))) for _ in range(24)}
                   | {(w.B - 1, w.Hq - 1), (0, 0)})
    O, L, seen = expected(q, k, v, lt.tolist(), w.causal, w.scale, heads=heads)
    o, l = run(ta, q, k, v, lt, w.causal, 0, nan_tail=(w.lens != "full"))
    check(o, l, O, L, seen, w.name, heads=heads)


def test_workspace_reuse_across_calls(ta):
    """One zeroed workspace reused for several calls with different lengths and CTA counts: the
    per-unit arrival counters must come back to zero after every call."""
    q, k, v, _ = _inputs(3, 16, 4, 2, 3000, "bf16", "normal", 94000, None)
    ws = torch.zeros(ta.attn_decode_workspace_bytes(3, 16, 4, 2, 3000, 128, 148), dtype=torch.uint8, device="cuda")
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    for lens, ctas in (([3000, 2000, 1000], 148), ([17, 2999, 640], 37), ([3000, 3000, 3000], 148), ([5, 0, 2500], 9)):
        lt = torch.tensor(lens, dtype=torch.int32)
        o, l = ta.attn_decode(qc, kc, vc, lt.cuda(), causal=True, num_ctas=ctas, workspace=ws)
        torch.cuda.synchronize()
        assert ta.attn_check_status() == 0
        O, L, seen = expected(q, k, v, lens, True, 128 ** -0.5)
        check(_np(o), l.cpu().numpy().astype(np.float64), O, L, seen, f"lens {lens} ctas {ctas}")
    # the per-unit arrival counters (the first U int32 of the workspace) are back at zero
    assert not ws[:3 * 4 * 4].cpu().numpy().any()


def test_output_without_lse_equals_output_with_lse(ta):
    """lse = NULL only skips the lse write: the split-KV pieces are still merged by their own
    log-sum-exp in the workspace, so O is the same bytes (pieces over several CTAs, causal drafts,
    one sequence with an empty cache)."""
    q, k, v, lt = _inputs(3, 16, 4, 4, 3000, "bf16", "k_offset", 93000, [3000, 1777, 0])
    qc, kc, vc, lc = q.cuda(), k.cuda(), v.cuda(), lt.cuda()
    o1, l1 = ta.attn_decode(qc, kc, vc, lc, causal=True, num_ctas=9)
    o2, l2 = ta.attn_decode(qc, kc, vc, lc, causal=True, num_ctas=9, lse=False)
    torch.cuda.synchronize()
    assert ta.attn_check_status() == 0
    assert l2 is None and l1 is not None
    assert torch.equal(o1, o2)
