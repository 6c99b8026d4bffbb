"""B200 (sm_100a) tiled attention forward: bf16_exact, SageAttention-style int8_qk and fp8_qk,
a row-prefix-masked variant (the APB mask shape), a KV-cache decode path, and context-parallel
(ring) attention over torch.distributed with log-sum-exp merges (``ring``).

The computation runs in the CUDA library built from ``csrc/`` (C ABI in
``include/tiled_attention.h``); this package only marshals arguments.
"""
from .binding import (  # noqa: F401
    ATTN_ERR_ALIGN,
    ATTN_ERR_ARG,
    ATTN_ERR_LAUNCH,
    ATTN_ERR_TIMEOUT,
    ATTN_ERR_UNSUPPORTED,
    ATTN_ERR_WORKSPACE,
    ATTN_OK,
    AttnError,
    LIB_PATH,
    apb_row_limits,
    attn_check_status,
    attn_decode,
    attn_decode_workspace_bytes,
    attn_error_string,
    attn_fwd,
    attn_fwd_host,
    attn_fwd_fp8_quantized,
    attn_fwd_int8_quantized,
    attn_fwd_prefix_masked,
    attn_merge_lse,
    attn_probe_qk_int32,
    attn_quant_scratch_bytes,
    attn_quant_smooth_k,
    attn_quant_smooth_k_fp8,
    attn_quant_smooth_k_noalloc,
    attn_test_exp2,
    attn_test_host_pieces,
    attn_test_wait_timeout,
    attn_workspace_bytes,
    exported_symbols,
    load_library,
)
