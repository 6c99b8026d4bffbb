"""Context-parallel (ring) attention, host side on CPU: the schedule, and the key/value exchange
over gloo ranks (2 and 3 processes) with the same ring_pass_blocks code the GPU path runs over
NCCL.  The attention arithmetic of each step is checked on the GPU (test_gpu_ring.py)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from tiled_attention_22_b200.ring import ring_pass_blocks, ring_schedule


@pytest.mark.parametrize("world", [1, 2, 3, 5, 8])
@pytest.mark.parametrize("causal", [False, True])
def test_schedule_visits_every_block_once(world, causal):
    for r in range(world):
        sched = ring_schedule(r, world, causal)
        assert [s for s, _, _ in sched] == list(range(world))
        assert sorted(j for _, j, _ in sched) == list(range(world))
        for s, j, kind in sched:
            assert j == (r - s) % world
            if not causal:
                assert kind == "full"
            else:
                # the diagonal block at step 0, earlier blocks unmasked, later blocks invisible
                assert kind == ("causal" if j == r else "full" if j < r else "skip")
        if causal:
            # rank r sees blocks 0..r: r + 1 useful steps, the last at step r
            useful = [s for s, _, kind in sched if kind != "skip"]
            assert useful == list(range(r + 1))


def test_schedule_rejects_bad_rank():
    with pytest.raises(ValueError):
        ring_schedule(3, 3, True)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _block(rank, shape):
    k = torch.arange(torch.Size(shape).numel(), dtype=torch.float32).reshape(shape) + 1000.0 * rank
    return k, -k


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        shape = (2, 3, 5, 4)
        k, v = _block(rank, shape)
        k0, v0 = k.clone(), v.clone()
        seen = []

        def on_step(s, j, kj, vj):
            seen.append((s, j, kj.clone(), vj.clone()))

        ring_pass_blocks(k, v, on_step)
        res = []
        for s, j, kj, vj in seen:
            ek, ev = _block(j, shape)
            res.append((s, j, bool(torch.equal(kj, ek)), bool(torch.equal(vj, ev))))
        out[rank] = (res, bool(torch.equal(k, k0) and torch.equal(v, v0)))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
@pytest.mark.parametrize("world", [2, 3])
def test_gloo_ring_delivers_block_r_minus_s(world):
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
    for r in range(world):
        res, untouched = out[r]
        assert untouched, f"rank {r}: its own block was overwritten"
        assert [s for s, _, _, _ in res] == list(range(world))
        for s, j, k_ok, v_ok in res:
            assert j == (r - s) % world
            assert k_ok and v_ok, f"rank {r} step {s}: block {j} arrived wrong"


def _join(Oa, La, Ob, Lb):
    """The log-sum-exp join of two partial attention results (float64)."""
    m = np.maximum(La, Lb)
    safe = np.where(np.isneginf(m), 0.0, m)
    wa, wb = np.exp(La - safe), np.exp(Lb - safe)
    s = wa + wb
    with np.errstate(invalid="ignore", divide="ignore"):
        O = (wa[..., None] * Oa + wb[..., None] * Ob) / s[..., None]
        L = safe + np.log(s)
    return np.where(np.isneginf(m)[..., None], 0.0, O), np.where(np.isneginf(m), -np.inf, L)


@pytest.mark.parametrize("split", [1, 37, 64, 99])
def test_partials_over_key_blocks_join_to_full_attention(split):
    """Ring attention's premise: attention over keys A u B is the log-sum-exp join of the attention
    over A and over B (which pins the oracle's lse as well: a wrong lse breaks the join)."""
    import oracle
    from attn_workloads import Workload, make_inputs

    w = Workload("j", 1, 4, 2, 100, 64, False, "bf16", "k_offset", 4242)
    q, k, v = make_inputs(w)
    O, L = oracle.attention(q, k, v, w.scale, False)
    Oa, La = oracle.attention(q, k[:, :, :split], v[:, :, :split], w.scale, False)
    Ob, Lb = oracle.attention(q, k[:, :, split:], v[:, :, split:], w.scale, False)
    Oj, Lj = _join(Oa, La, Ob, Lb)
    np.testing.assert_allclose(Oj, O, rtol=0, atol=1e-12)
    np.testing.assert_allclose(Lj, L, rtol=0, atol=1e-12)


def test_causal_ring_blocks_join_to_causal_attention():
    """The causal ring over 4 blocks: rank r joins its diagonal block (causal within the block) and
    the full blocks before it, and gets the rows of causal attention over the whole sequence."""
    import oracle
    from attn_workloads import Workload, make_inputs

    W, n = 4, 40
    w = Workload("c", 1, 2, 1, W * n, 64, True, "bf16", "normal", 4343)
    q, k, v = make_inputs(w)
    O, L = oracle.attention(q, k, v, w.scale, True)
    for r in range(W):
        qr = q[:, :, r * n:(r + 1) * n]
        acc = None
        for s, j, kind in ring_schedule(r, W, True):
            if kind == "skip":
                continue
            kj, vj = k[:, :, j * n:(j + 1) * n], v[:, :, j * n:(j + 1) * n]
            part = oracle.attention(qr, kj, vj, w.scale, kind == "causal")
            acc = part if acc is None else _join(acc[0], acc[1], part[0], part[1])
        np.testing.assert_allclose(acc[0], O[:, :, r * n:(r + 1) * n], rtol=0, atol=1e-12)
        np.testing.assert_allclose(acc[1], L[:, :, r * n:(r + 1) * n], rtol=0, atol=1e-12)


def test_emulated_ring_needs_a_divisible_sequence():
    from tiled_attention_22_b200.ring import ring_attention_emulated

    q = torch.zeros(1, 2, 10, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="multiple"):
        ring_attention_emulated(q, q[:, :1], q[:, :1], 3)


def test_merge_binding_validates_arguments_on_the_host():
    """attn_merge_lse checks shapes, dtypes and devices before it reaches the library."""
    from tiled_attention_22_b200 import attn_merge_lse

    acc = torch.zeros(4, 128)
    lacc = torch.zeros(4)
    part = torch.zeros(4, 128, dtype=torch.bfloat16)
    lp = torch.zeros(4)
    with pytest.raises(ValueError):  # float32 accumulator required
        attn_merge_lse(acc.double(), lacc, part, lp)
    with pytest.raises(ValueError):  # one lse per row
        attn_merge_lse(acc, torch.zeros(5), part, lp)
    with pytest.raises(ValueError):  # nothing to merge and nowhere to write
        attn_merge_lse(acc, lacc)
    with pytest.raises(ValueError):  # CUDA tensors only
        attn_merge_lse(acc, lacc, part, lp)
