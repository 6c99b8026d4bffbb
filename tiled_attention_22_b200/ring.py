"""Context-parallel (ring) attention: one query block per rank, key/value blocks passed round a ring.

The APB article ("在长文本上比Flash Attention快10倍！…", section on the baselines) names ring attention
as the exact sequence-parallel way to run attention over a context split across devices.  Its
parts here:

* the sequence of N = W * n tokens is split into W contiguous blocks; rank r holds query, key and
  value block r ([B, H, n, d] each, GQA allowed);
* at step s (0 .. W-1) rank r holds the key/value block j = (r - s) mod W.  While it computes on
  block j it sends that block to rank r + 1 and receives block j - 1 from rank r - 1, so the
  exchange of step s + 1's block overlaps step s's attention;
* under the causal mask block j is the diagonal block (j == r, the causal kernel), a block of
  earlier tokens (j < r, no mask) or a block of later tokens (j > r, no key visible: skipped);
* each step's (O, lse) from ``attn_fwd`` is joined into a float32 running result by
  ``attn_merge_lse`` (the log-sum-exp identity the "FlashAttention" glossary uses to rescale
  partial results); the last step's merge writes the 16-bit output.

The exchange uses torch.distributed point-to-point operations (NCCL on GPUs: over NVLink /
NVSwitch on a B200 node; gloo works for CPU tensors, which the tests use for the exchange
alone).  ``ring_attention_emulated`` runs every rank's steps one after another on one device
with the same kernels and the same schedule, for checking the numerics on a single GPU.

int8_qk / fp8_qk: each step quantises its query block and the key block it holds, smoothing the
key block by that block's own mean; ``attn_fwd``'s lse includes the matching bias, so the merged
result is that of the method with per-block means (softmax is unchanged by a per-block shift, so
the exact result is the same; the 8-bit codes differ from those of one whole-sequence mean).
"""
from __future__ import annotations

import contextlib
import math

import torch
import torch.distributed as dist

from .binding import attn_fwd, attn_merge_lse

__all__ = ["ring_schedule", "ring_pass_blocks", "ring_attention", "ring_rank_emulated", "ring_attention_emulated"]


def ring_schedule(rank: int, world: int, causal: bool):
    """[(step, kv_block, kind)] for ``rank``: kind is "causal" (the diagonal block), "full" or
    "skip" (a block of later tokens under the causal mask)."""
    if not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a world of {world}")
    out = []
    for s in range(world):
        j = (rank - s) % world
        if not causal:
            kind = "full"
        elif j == rank:
            kind = "causal"
        elif j < rank:
            kind = "full"
        else:
            kind = "skip"
        out.append((s, j, kind))
    return out


def _exchange(send, recv, to, frm, group):
    """Post the sends of ``send`` to rank ``to`` and the receives into ``recv`` from rank ``frm``;
    returns the requests."""
    ops = [dist.P2POp(dist.isend, t, to, group) for t in send]
    ops += [dist.P2POp(dist.irecv, t, frm, group) for t in recv]
    return dist.batch_isend_irecv(ops)


def ring_pass_blocks(k, v, on_step, group=None):
    """Pass this rank's key/value block round the ring of ``group``; ``on_step(s, j, k_j, v_j)`` is
    called with the block j = (rank - s) mod W the rank holds at step s.  The exchange for step
    s + 1 is posted before ``on_step`` runs, so it overlaps that step's work; the block this rank
    was given is never written."""
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    if world == 1:
        on_step(0, rank, k, v)
        return
    # global ranks of the ring neighbours (P2P ops take global ranks)
    to = dist.get_global_rank(group, (rank + 1) % world) if group is not None else (rank + 1) % world
    frm = dist.get_global_rank(group, (rank - 1) % world) if group is not None else (rank - 1) % world
    bufs = [(torch.empty_like(k), torch.empty_like(v)), (torch.empty_like(k), torch.empty_like(v))]
    cur = (k, v)
    for s in range(world):
        reqs = None
        if s + 1 < world:
            nxt = bufs[s % 2]
            reqs = _exchange(cur, nxt, to, frm, group)
        on_step(s, (rank - s) % world, cur[0], cur[1])
        if reqs is not None:
            for r in reqs:
                r.wait()
            cur = nxt


def _scale(d, scale):
    return 1.0 / math.sqrt(d) if scale is None else float(scale)


class _Accumulator:
    """The float32 running result of one rank and the merge of each step into it."""

    def __init__(self, q, last_step):
        B, H, n, d = q.shape
        self.o_acc = torch.empty((B, H, n, d), device=q.device, dtype=torch.float32)
        self.lse_acc = torch.empty((B, H, n), device=q.device, dtype=torch.float32)
        self.out = torch.empty_like(q)
        self.last_step = last_step
        self.first = True

    def add(self, s, o_s, lse_s):
        attn_merge_lse(self.o_acc, self.lse_acc, o_s, lse_s, out=self.out if s == self.last_step else None,
                       first=self.first)
        self.first = False


def _rank_step(q, k_j, v_j, kind, scale, mode, acc, s):
    if kind == "skip":
        return
    o_s, l_s = attn_fwd(q, k_j, v_j, causal=(kind == "causal"), scale=scale, mode=mode)
    acc.add(s, o_s, l_s)


def _on(stream):
    """Run on ``stream`` (the current stream when None): the exchange's NCCL stream waits for the
    current stream's earlier work, so compute and exchange must share it."""
    return torch.cuda.stream(stream) if stream is not None else contextlib.nullcontext()


def ring_attention(q, k, v, causal=False, scale=None, mode="bf16_exact", group=None, stream=None):
    """Attention of this rank's query block over the whole sequence held by the ranks of
    ``group`` (rank r holds tokens r*n .. (r+1)*n - 1 of q, k and v).  Returns (o, lse) for this
    rank's rows: o 16-bit [B, Hq, n, d], lse float32 [B, Hq, n] (natural log).  Every kernel and
    the exchange run on ``stream`` (default: the current stream)."""
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    scale = _scale(q.shape[-1], scale)
    sched = ring_schedule(rank, world, causal)
    last = max(s for s, _, kind in sched if kind != "skip")
    kinds = {s: kind for s, _, kind in sched}
    with _on(stream):
        acc = _Accumulator(q, last)
        ring_pass_blocks(k, v, lambda s, j, kj, vj: _rank_step(q, kj, vj, kinds[s], scale, mode, acc, s),
                         group=group)
    return acc.out, acc.lse_acc


def ring_rank_emulated(q_r, kv_blocks, rank, causal=False, scale=None, mode="bf16_exact"):
    """Rank ``rank``'s part of the ring run on one device: its steps in schedule order over the
    key/value blocks ``kv_blocks`` (a list of (k_j, v_j), one per rank), with the kernels and
    merges of ``ring_attention``.  Returns (o, lse) for the rank's rows (current stream)."""
    world = len(kv_blocks)
    scale = _scale(q_r.shape[-1], scale)
    sched = ring_schedule(rank, world, causal)
    last = max(s for s, _, kind in sched if kind != "skip")
    acc = _Accumulator(q_r, last)
    for s, j, kind in sched:
        _rank_step(q_r, kv_blocks[j][0], kv_blocks[j][1], kind, scale, mode, acc, s)
    return acc.out, acc.lse_acc


def ring_attention_emulated(q, k, v, world, causal=False, scale=None, mode="bf16_exact", stream=None):
    """The ring of ``world`` ranks run on one device, rank after rank, with the kernels, schedule
    and merge order of ``ring_attention`` (no exchange: block j is a slice).  q [B, Hq, N, d],
    k and v [B, Hkv, N, d] with N divisible by ``world``.  Returns (o, lse) for all N rows."""
    N = q.shape[2]
    if N % world:
        raise ValueError(f"sequence length {N} is not a multiple of {world} ranks")
    n = N // world
    scale = _scale(q.shape[-1], scale)
    blocks = [(k[:, :, j * n:(j + 1) * n].contiguous(), v[:, :, j * n:(j + 1) * n].contiguous()) for j in range(world)]
    outs, lses = [], []
    with _on(stream):
        for r in range(world):
            o_r, l_r = ring_rank_emulated(q[:, :, r * n:(r + 1) * n].contiguous(), blocks, r, causal, scale, mode)
            outs.append(o_r)
            lses.append(l_r)
        return torch.cat(outs, dim=2), torch.cat(lses, dim=2)
