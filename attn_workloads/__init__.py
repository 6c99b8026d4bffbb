"""Seeded synthetic inputs for the attention forward pass.

This module only draws random tensors. It holds none of the attention
arithmetic, so both the CPU oracle and the CUDA path can take their inputs
from it without sharing any of the method.

Recipe (one rule for every workload):
  * each tensor is drawn with its own ``torch.Generator`` seeded
    ``1000*cfg + {0: Q, 1: K, 2: V, 3: offsets / outlier channels}``;
  * values are drawn as float32 on the CPU and then cast to the workload's
    dtype; the oracle reads the cast values exactly;
  * ``kind="normal"``: Q, K, V i.i.d. N(0, 1);
  * ``kind="k_offset"``: as normal, plus a per-(batch, kv-head, channel)
    offset drawn from N(0, 3^2) and added to every token of K.  This models
    the channel-wise outliers of K that the SageAttention article
    ("又快又准，即插即用！清华8比特量化Attention…", section 挑战) reports
    for video and image models;
  * ``kind="outlier_channels"``: as normal, then in each of Q, K and V, for
    every (batch, head), max(1, round(0.01*d)) channels drawn at random are
    multiplied by 10 on all tokens (independent draws per tensor).
"""
from __future__ import annotations

import dataclasses
import math

import torch

__all__ = ["Workload", "WORKLOADS", "make_inputs", "attention_flops", "workload", "DecodeWorkload",
           "DECODE_WORKLOADS", "make_decode_inputs", "decode_bytes", "ApbWorkload", "APB_WORKLOADS",
           "make_apb_inputs"]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    N: int
    d: int
    causal: bool
    dtype: str          # "bf16" | "fp16"
    kind: str           # "normal" | "k_offset" | "outlier_channels"
    seed_base: int      # 1000 * cfg for the named workloads
    modes: tuple = ("bf16_exact", "int8_qk")

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def torch_dtype(self):
        return {"bf16": torch.bfloat16, "fp16": torch.float16}[self.dtype]

    def flops(self) -> float:
        return attention_flops(self.B, self.Hq, self.N, self.d, self.causal)

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


def attention_flops(B: int, Hq: int, N: int, d: int, causal: bool) -> float:
    """Algorithmic FLOPs of one forward pass: 4*B*Hq*N^2*d, halved when causal."""
    f = 4.0 * B * Hq * N * N * d
    return f / 2.0 if causal else f


# The five seeded workloads.  Workload 1 is small enough for a full-matrix
# float64 oracle in milliseconds; 5 (131072 tokens) is the largest, the
# benchmark's headline; 3, 4 and 5 are the sizes (N >= 8192) the throughput
# targets apply to.
WORKLOADS = {
    1: Workload("mha_n128_d64_fp16", 1, 2, 2, 128, 64, False, "fp16", "normal", 1000),
    2: Workload("mha_causal_b4_h32_n4096_d128", 4, 32, 32, 4096, 128, True, "bf16", "normal", 2000),
    3: Workload("gqa_causal_b2_hq32_hkv8_n8192_d128_koffset", 2, 32, 8, 8192, 128, True, "bf16",
                "k_offset", 3000),
    4: Workload("mha_b2_h24_n16384_d64_outliers", 2, 24, 24, 16384, 64, False, "bf16",
                "outlier_channels", 4000, ("int8_qk", "bf16_exact")),
    5: Workload("gqa_causal_b1_hq32_hkv8_n131072_d128_koffset", 1, 32, 8, 131072, 128, True, "bf16",
                "k_offset", 5000),
}


def workload(cfg: int) -> Workload:
    return WORKLOADS[cfg]


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def make_inputs(w: Workload):
    """Return (q, k, v) as CPU tensors of ``w.dtype`` in [B, H, N, d] layout."""
    B, Hq, Hkv, N, d = w.B, w.Hq, w.Hkv, w.N, w.d
    f32 = torch.float32
    q = torch.randn((B, Hq, N, d), generator=_gen(w.seed_base + 0), dtype=f32)
    k = torch.randn((B, Hkv, N, d), generator=_gen(w.seed_base + 1), dtype=f32)
    v = torch.randn((B, Hkv, N, d), generator=_gen(w.seed_base + 2), dtype=f32)
    if w.kind == "k_offset":
        off = torch.randn((B, Hkv, 1, d), generator=_gen(w.seed_base + 3), dtype=f32) * 3.0
        k.add_(off)
    elif w.kind == "outlier_channels":
        g = _gen(w.seed_base + 3)
        n_out = max(1, round(0.01 * d))
        for t in (q, k, v):
            for b in range(B):
                for h in range(t.shape[1]):
                    ch = torch.randperm(d, generator=g)[:n_out]
                    t[b, h][:, ch] *= 10.0
    elif w.kind != "normal":
        raise ValueError(f"unknown input kind {w.kind!r}")
    dt = w.torch_dtype
    return q.to(dt), k.to(dt), v.to(dt)


# ------------------------------------------------------------------------------------------------
# KV-cache decoding: Nq new tokens per sequence against a cache of capacity Nk.
#
# Recipe: as above (q, k, v i.i.d. N(0, 1) drawn in float32 with seeds seed_base + {0, 1, 2},
# "k_offset" adds the per-channel N(0, 3^2) offset with seed seed_base + 3, then cast), with the
# cache drawn at full capacity Nk.  Lengths: "full" gives every sequence Nk cached keys; "ragged"
# draws kv_lens[b] uniformly from [Nk/2, Nk] with seed seed_base + 4.
# ------------------------------------------------------------------------------------------------
@dataclasses.dataclass(frozen=True)
class DecodeWorkload:
    name: str
    B: int
    Hq: int
    Hkv: int
    Nq: int
    Nk: int
    d: int
    causal: bool
    dtype: str
    kind: str
    lens: str           # "full" | "ragged"
    seed_base: int

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def torch_dtype(self):
        return {"bf16": torch.bfloat16, "fp16": torch.float16}[self.dtype]

    def replace(self, **kw) -> "DecodeWorkload":
        return dataclasses.replace(self, **kw)


# 101: one decoding step of a LLaMA-3-8B-shaped GQA layer (32 query heads, 8 kv heads, d = 128)
#      for 8 sequences at 32K context: 1 GiB of cache.
# 102: the same for an MHA layer of the LLaMA-7B shape (32 heads x 128: 16 KB of K and V per token
#      and layer in 16-bit) for 16 sequences at 8K context: 2 GiB of cache.
# 103: verifying 4 drafted tokens (causal among themselves) over ragged lengths up to 16K.
DECODE_WORKLOADS = {
    101: DecodeWorkload("gqa_decode_b8_hq32_hkv8_nq1_nk32768_d128", 8, 32, 8, 1, 32768, 128, False, "bf16",
                        "normal", "full", 101000),
    102: DecodeWorkload("mha_decode_b16_h32_nq1_nk8192_d128", 16, 32, 32, 1, 8192, 128, False, "bf16",
                        "normal", "full", 102000),
    103: DecodeWorkload("gqa_verify_b4_hq32_hkv8_nq4_nk16384_ragged_causal", 4, 32, 8, 4, 16384, 128, True,
                        "bf16", "k_offset", "ragged", 103000),
}


def make_decode_inputs(w: DecodeWorkload):
    """Return (q, k_cache, v_cache, kv_lens) as CPU tensors; kv_lens is int32 [B]."""
    f32 = torch.float32
    q = torch.randn((w.B, w.Hq, w.Nq, w.d), generator=_gen(w.seed_base + 0), dtype=f32)
    k = torch.randn((w.B, w.Hkv, w.Nk, w.d), generator=_gen(w.seed_base + 1), dtype=f32)
    v = torch.randn((w.B, w.Hkv, w.Nk, w.d), generator=_gen(w.seed_base + 2), dtype=f32)
    if w.kind == "k_offset":
        k.add_(torch.randn((w.B, w.Hkv, 1, w.d), generator=_gen(w.seed_base + 3), dtype=f32) * 3.0)
    elif w.kind != "normal":
        raise ValueError(f"unknown input kind {w.kind!r}")
    if w.lens == "full":
        lens = torch.full((w.B,), w.Nk, dtype=torch.int32)
    elif w.lens == "ragged":
        lens = torch.randint(w.Nk // 2, w.Nk + 1, (w.B,), generator=_gen(w.seed_base + 4), dtype=torch.int32)
    else:
        raise ValueError(f"unknown length rule {w.lens!r}")
    dt = w.torch_dtype
    return q.to(dt), k.to(dt), v.to(dt), lens


def decode_bytes(B: int, Hq: int, Hkv: int, Nq: int, d: int, lens) -> float:
    """Algorithmic HBM bytes of one decoding call in 16-bit: the used cache (K and V, sum of the
    lengths x Hkv x d each), the queries and the outputs; every byte once."""
    total_len = float(sum(int(x) for x in lens))
    return 2.0 * 2.0 * total_len * Hkv * d + 2.0 * 2.0 * B * Hq * Nq * d


# ------------------------------------------------------------------------------------------------
# APB-shaped prefill on one device: keys [anchor A | passing P | local L], queries [anchor A |
# local L] (the APB article's layout; the anchor block is 1/4 to 1/8 of the local block).
# Recipe: q [B, Hq, A + L, d] and k, v [B, Hkv, A + P + L, d] drawn as above (seeds
# seed_base + {0, 1, 2}, float32 N(0, 1), cast).
# ------------------------------------------------------------------------------------------------
@dataclasses.dataclass(frozen=True)
class ApbWorkload:
    name: str
    B: int
    Hq: int
    Hkv: int
    anchor: int
    passing: int
    local: int
    d: int
    dtype: str
    seed_base: int

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def torch_dtype(self):
        return {"bf16": torch.bfloat16, "fp16": torch.float16}[self.dtype]

    @property
    def Nq(self) -> int:
        return self.anchor + self.local

    @property
    def Nk(self) -> int:
        return self.anchor + self.passing + self.local


# 201: a 16K-token local block with an anchor of 1/8 of it and a 4K-token passing block (the
#      compressed context of earlier devices), LLaMA-3-8B-shaped GQA heads.
APB_WORKLOADS = {
    201: ApbWorkload("apb_b1_hq32_hkv8_anchor2048_passing4096_local16384_d128", 1, 32, 8, 2048, 4096, 16384, 128,
                     "bf16", 201000),
}


def make_apb_inputs(w: ApbWorkload):
    """Return (q, k, v) as CPU tensors: q [B, Hq, anchor + local, d], k and v
    [B, Hkv, anchor + passing + local, d]."""
    f32 = torch.float32
    q = torch.randn((w.B, w.Hq, w.Nq, w.d), generator=_gen(w.seed_base + 0), dtype=f32)
    k = torch.randn((w.B, w.Hkv, w.Nk, w.d), generator=_gen(w.seed_base + 1), dtype=f32)
    v = torch.randn((w.B, w.Hkv, w.Nk, w.d), generator=_gen(w.seed_base + 2), dtype=f32)
    dt = w.torch_dtype
    return q.to(dt), k.to(dt), v.to(dt)

