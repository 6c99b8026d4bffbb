"""CPU oracle for the tiled attention forward pass.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may call it.  It shares no code with
the CUDA path (no kernels, tables, helpers or constants); the only thing the
two sides have in common is the seeded input generator in ``attn_workloads``.

Contents
  exact            O1: plain float64 softmax attention (the definition), also
                   with Nq < Nk (queries after a KV cache) and with a per-row
                   visible key prefix (the APB mask shape).
  fp8_emulation    O3: the same smoothing with per-block FP8 (E4M3) codes
                   (round to nearest even, saturating at 448) and exact
                   code-product scores.
  int8_emulation   O2: bit-exact emulation of K smoothing and per-block INT8
                   quantisation of Q and K, exact integer QK^T, and the
                   float64 attention that follows from those quantised scores.

Pins (tests/test_oracle_*.py check these against something other than the
oracle itself): invariants the pages state (softmax rows sum to one, a K shift
per channel leaves the output unchanged, causal row 0 equals V[0]), closed
forms (identical keys give the mean of V, a dominant score reproduces one row
of V), hand-worked N=4 cases in tests/golden/, brute force in pure Python on
tiny inputs, torch's CPU scaled_dot_product_attention in float64, and exact
rational arithmetic for every float32 rounding step of the quantiser.

Parity unpinned: the dequantised float64 attention of O2 (``attention_int8``)
is pinned only through its parts (the exact integer scores and O1); the pages
print no value for it.  The quantiser's constants and rounding are a reading of
the pages (they are silent on them), so O2 is pinned to that reading, not to a
number the pages print.
"""
from .exact import attention, attention_prefix, attention_probs, logsumexp_rows  # noqa: F401
from .int8_emulation import (  # noqa: F401
    QBLOCK,
    k_channel_mean,
    smooth_quant_k,
    quant_q,
    quant_block,
    lse_bias,
    scores_int32,
    attention_int8,
    prepass,
)
