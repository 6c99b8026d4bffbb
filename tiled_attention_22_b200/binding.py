"""ctypes binding of include/tiled_attention.h (argument marshalling only).

Every function here has the name of the C entry point it calls.  torch is used
for device memory and streams: outputs are allocated with torch, pointers and
the current CUDA stream are passed to the library, and every step of the
computation runs in the library's kernels.  There is no fallback: if the built
library is missing, or no CUDA device is present, the call raises.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "_lib", "libtiled_attention.so")

ATTN_OK = 0
ATTN_ERR_ARG = -1
ATTN_ERR_UNSUPPORTED = -2
ATTN_ERR_ALIGN = -3
ATTN_ERR_WORKSPACE = -4
ATTN_ERR_LAUNCH = -5
ATTN_ERR_TIMEOUT = -6

MODES = {"bf16_exact": 0, "int8_qk": 1, "fp8_qk": 2}
DTYPES = {torch.bfloat16: 0, torch.float16: 1}

_vp, _i, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
_SIGNATURES = {
    "attn_fwd": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _i, _i, _vp, _sz, _vp]),
    "attn_workspace_bytes": (_sz, [_i, _i, _i, _i, _i, _i]),
    "attn_quant_smooth_k": (_i, [_vp, _vp, _i, _i, _i, _i, _i, _i, _f, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "attn_quant_scratch_bytes": (_sz, [_i, _i, _i, _i]),
    "attn_quant_smooth_k_fp8": (_i, [_vp, _vp, _i, _i, _i, _i, _i, _i, _f, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "attn_fwd_fp8_quantized": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _i, _vp]),
    "attn_quant_smooth_k_noalloc": (_i, [_vp, _vp, _i, _i, _i, _i, _i, _i, _f, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "attn_fwd_int8_quantized": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _i, _vp]),
    "attn_probe_qk_int32": (_i, [_vp, _vp, _i, _i, _i, _i, _i, _vp, _i, _vp, _vp]),
    "attn_fwd_host": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _i, _i,
                           _vp, _sz, _vp]),
    "attn_fwd_prefix_masked": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _f, _i, _vp]),
    "attn_decode": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _f, _i, _i, _vp, _sz, _vp]),
    "attn_decode_workspace_bytes": (_sz, [_i, _i, _i, _i, _i, _i, _i]),
    "attn_merge_lse": (_i, [_vp, _vp, _vp, _vp, _vp, ctypes.c_longlong, _i, _i, _i, _vp]),
    "attn_check_status": (_i, []),
    "attn_error_string": (ctypes.c_char_p, [_i]),
    "attn_last_cuda_error": (ctypes.c_char_p, []),
    "attn_test_host_pieces": (_i, [_i, _i, _i, _i, _i, _vp, _i]),
    "attn_test_wait_timeout": (_i, [_i, _vp]),
    "attn_test_exp2": (_i, [_vp, _vp, _i, _i, _vp]),
}

_lib = None


class AttnError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        lib = load_library()
        msg = lib.attn_error_string(code).decode()
        extra = lib.attn_last_cuda_error().decode() if code == ATTN_ERR_LAUNCH else ""
        super().__init__(f"{where}: {msg} ({code}){' - ' + extra if extra else ''}")


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the built library (raises if it is missing: there is no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise RuntimeError(f"CUDA library not built: {path} (run python -m tiled_attention_22_b200.build)")
        lib = ctypes.CDLL(path)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def exported_symbols():
    return list(_SIGNATURES)


def _check(rc: int, where: str):
    if rc != ATTN_OK:
        raise AttnError(rc, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _device_of(*tensors) -> int:
    """The one CUDA device of a call's tensors (None entries are skipped).  The library resolves the
    device of every launch, and of its per-device state, from the current device, so each call is
    made with this device current; tensors on different devices are refused."""
    dev = None
    for t in tensors:
        if t is None:
            continue
        d = t.device
        if d.type != "cuda" or d.index is None:
            raise ValueError("every device tensor of the call must be a CUDA tensor")
        if dev is None:
            dev = d.index
        elif d.index != dev:
            raise ValueError(f"tensors on cuda:{dev} and cuda:{d.index}: one call runs on one device")
    if dev is None:
        raise ValueError("the call has no CUDA tensor")
    return dev


def _stream(stream, dev=None):
    """The cudaStream_t to pass: ``stream`` (a torch.cuda.Stream on the call's device), else the
    current stream of that device."""
    if stream is None:
        stream = torch.cuda.current_stream(dev)
    elif dev is not None and stream.device.index != dev:
        raise ValueError(f"stream of cuda:{stream.device.index} for tensors on cuda:{dev}")
    return ctypes.c_void_p(stream.cuda_stream)


def _lse_arg(lse, shape, device):
    """lse=True: allocate; None/False: skip; a tensor: write into it."""
    if lse is True:
        return torch.empty(shape, device=device, dtype=torch.float32)
    if lse is None or lse is False:
        return None
    return lse


def _shape(q, k, v):
    if q.dim() != 4 or k.dim() != 4 or v.dim() != 4:
        raise ValueError("q, k, v must be [B, H, N, d]")
    B, Hq, N, d = q.shape
    if k.shape != v.shape or k.shape[0] != B or k.shape[2] != N or k.shape[3] != d:
        raise ValueError(f"shape mismatch: q {tuple(q.shape)} k {tuple(k.shape)} v {tuple(v.shape)}")
    for t in (q, k, v):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous CUDA tensors")
    if q.dtype not in DTYPES or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k, v must share one dtype: bfloat16 or float16")
    return B, Hq, k.shape[1], N, d


def attn_workspace_bytes(B, Hq, Hkv, N, d, mode="int8_qk") -> int:
    return int(load_library().attn_workspace_bytes(B, Hq, Hkv, N, d, MODES[mode]))


def attn_quant_scratch_bytes(B, Hkv, N, d) -> int:
    return int(load_library().attn_quant_scratch_bytes(B, Hkv, N, d))


def attn_fwd(q, k, v, causal=False, scale=None, mode="bf16_exact", out=None, lse=True, workspace=None,
             stream=None):
    """O = softmax(scale Q K^T [+causal]) V on the GPU.  Returns (o, lse or None)."""
    lib = load_library()
    B, Hq, Hkv, N, d = _shape(q, k, v)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    o = torch.empty_like(q) if out is None else out
    l = _lse_arg(lse, (B, Hq, N), q.device)
    ws_bytes = attn_workspace_bytes(B, Hq, Hkv, N, d, mode)
    if ws_bytes and workspace is None:
        workspace = torch.empty(ws_bytes, device=q.device, dtype=torch.uint8)
    dev = _device_of(q, k, v, o, l, workspace)
    with torch.cuda.device(dev):
        rc = lib.attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(l), B, Hq, Hkv, N, d, int(bool(causal)), scale,
                          MODES[mode], DTYPES[q.dtype], _ptr(workspace),
                          0 if workspace is None else workspace.numel() * workspace.element_size(),
                          _stream(stream, dev))
    _check(rc, "attn_fwd")
    return o, l


def apb_row_limits(anchor: int, passing: int, local: int, device=None):
    """Row limits of the APB layout: keys [anchor | passing | local], queries [anchor | local];
    anchor row i sees keys < i + 1, local row i sees keys < anchor + passing + i + 1."""
    a = torch.arange(1, anchor + 1, dtype=torch.int32)
    l = anchor + passing + torch.arange(1, local + 1, dtype=torch.int32)
    return torch.cat([a, l]).to(device) if device is not None else torch.cat([a, l])


def attn_fwd_prefix_masked(q, k, v, row_kv_limit, scale=None, out=None, lse=True, stream=None):
    """Attention where query row i sees keys j < row_kv_limit[i] (int32 CUDA tensor [Nq]).
    q [B, Hq, Nq, d]; k, v [B, Hkv, Nk, d].  Returns (o, lse or None)."""
    lib = load_library()
    if q.dim() != 4 or k.dim() != 4 or v.dim() != 4 or k.shape != v.shape:
        raise ValueError("q, k, v must be [B, H, N, d] with k and v of one shape")
    B, Hq, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    if k.shape[0] != B or k.shape[3] != d:
        raise ValueError(f"shape mismatch: q {tuple(q.shape)} k {tuple(k.shape)}")
    for t in (q, k, v):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous CUDA tensors")
    if q.dtype not in DTYPES or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k, v must share one dtype: bfloat16 or float16")
    if (row_kv_limit.dtype != torch.int32 or not row_kv_limit.is_cuda or row_kv_limit.numel() != Nq
            or not row_kv_limit.is_contiguous()):
        raise ValueError("row_kv_limit must be a contiguous int32 CUDA tensor of Nq entries")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    o = torch.empty_like(q) if out is None else out
    l = _lse_arg(lse, (B, Hq, Nq), q.device)
    dev = _device_of(q, k, v, o, l, row_kv_limit)
    with torch.cuda.device(dev):
        rc = lib.attn_fwd_prefix_masked(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(l), B, Hq, Hkv, Nq, Nk, d,
                                        _ptr(row_kv_limit), scale, DTYPES[q.dtype], _stream(stream, dev))
    _check(rc, "attn_fwd_prefix_masked")
    return o, l


def attn_decode_workspace_bytes(B, Hq, Hkv, Nq, Nk, d, num_ctas=0) -> int:
    return int(load_library().attn_decode_workspace_bytes(B, Hq, Hkv, Nq, Nk, d, num_ctas))


def attn_decode(q, k_cache, v_cache, kv_lens=None, causal=False, scale=None, num_ctas=0, out=None, lse=True,
                workspace=None, stream=None):
    """Attention of q [B, Hq, Nq, d] against the first kv_lens[b] keys of k_cache / v_cache
    [B, Hkv, Nk, d] (kv_lens: int32 CUDA tensor [B] or None for all Nk).  Returns (o, lse or None)."""
    lib = load_library()
    if q.dim() != 4 or k_cache.dim() != 4 or v_cache.dim() != 4:
        raise ValueError("q, k_cache, v_cache must be [B, H, N, d]")
    B, Hq, Nq, d = q.shape
    if k_cache.shape != v_cache.shape or k_cache.shape[0] != B or k_cache.shape[3] != d:
        raise ValueError(f"shape mismatch: q {tuple(q.shape)} k {tuple(k_cache.shape)} v {tuple(v_cache.shape)}")
    Hkv, Nk = k_cache.shape[1], k_cache.shape[2]
    for t in (q, k_cache, v_cache):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("q, k_cache, v_cache must be contiguous CUDA tensors")
    if q.dtype not in DTYPES or k_cache.dtype != q.dtype or v_cache.dtype != q.dtype:
        raise ValueError("q, k_cache, v_cache must share one dtype: bfloat16 or float16")
    if kv_lens is not None and (kv_lens.dtype != torch.int32 or not kv_lens.is_cuda or kv_lens.numel() != B
                                or not kv_lens.is_contiguous()):
        raise ValueError("kv_lens must be a contiguous int32 CUDA tensor of B entries")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    o = torch.empty_like(q) if out is None else out
    l = _lse_arg(lse, (B, Hq, Nq), q.device)
    ws_bytes = attn_decode_workspace_bytes(B, Hq, Hkv, Nq, Nk, d, num_ctas)
    if ws_bytes and workspace is None:  # (a reused workspace must have been zeroed once)
        workspace = torch.zeros(ws_bytes, device=q.device, dtype=torch.uint8)
    dev = _device_of(q, k_cache, v_cache, kv_lens, o, l, workspace)
    with torch.cuda.device(dev):
        rc = lib.attn_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(kv_lens), _ptr(o), _ptr(l), B, Hq, Hkv,
                             Nq, Nk, d, int(bool(causal)), scale, DTYPES[q.dtype], int(num_ctas), _ptr(workspace),
                             0 if workspace is None else workspace.numel() * workspace.element_size(),
                             _stream(stream, dev))
    _check(rc, "attn_decode")
    return o, l


def attn_quant_smooth_k(q, k, scale=None, scratch=None, stream=None, out=None):
    """The INT8 pre-pass alone.  Returns dict(q8, sq, k8, sk, kmean, lse_bias) (``out`` if given)."""
    lib = load_library()
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    _shape(q, k, k)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    T = (N + 127) // 128
    dev = q.device
    out = out or dict(
        q8=torch.empty((B, Hq, N, d), device=dev, dtype=torch.int8),
        sq=torch.empty((B, Hq, T), device=dev, dtype=torch.float32),
        k8=torch.empty((B, Hkv, N, d), device=dev, dtype=torch.int8),
        sk=torch.empty((B, Hkv, T), device=dev, dtype=torch.float32),
        kmean=torch.empty((B, Hkv, d), device=dev, dtype=torch.float32),
        lse_bias=torch.empty((B, Hq, N), device=dev, dtype=torch.float32),
    )
    nbytes = attn_quant_scratch_bytes(B, Hkv, N, d)
    if scratch is None:
        scratch = torch.empty(nbytes, device=dev, dtype=torch.uint8)
    dev = _device_of(q, k, scratch, *out.values())
    with torch.cuda.device(dev):
        rc = lib.attn_quant_smooth_k(_ptr(q), _ptr(k), B, Hq, Hkv, N, d, DTYPES[q.dtype], scale, _ptr(out["q8"]),
                                     _ptr(out["sq"]), _ptr(out["k8"]), _ptr(out["sk"]), _ptr(out["kmean"]),
                                     _ptr(out["lse_bias"]), _ptr(scratch), scratch.numel(), _stream(stream, dev))
    _check(rc, "attn_quant_smooth_k")
    return out


def attn_quant_smooth_k_noalloc(q, k, scale=None, out=None, stream=None):
    """The pre-pass without caller scratch: its float64 K-mean partials use the library's built-in
    8 MiB array (for callers that cannot allocate device memory).  Output buffers are still the
    caller's; ``out`` may supply them (else they are allocated here with torch)."""
    lib = load_library()
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    _shape(q, k, k)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    T = (N + 127) // 128
    dev = q.device
    out = out or dict(
        q8=torch.empty((B, Hq, N, d), device=dev, dtype=torch.int8),
        sq=torch.empty((B, Hq, T), device=dev, dtype=torch.float32),
        k8=torch.empty((B, Hkv, N, d), device=dev, dtype=torch.int8),
        sk=torch.empty((B, Hkv, T), device=dev, dtype=torch.float32),
        kmean=torch.empty((B, Hkv, d), device=dev, dtype=torch.float32),
        lse_bias=torch.empty((B, Hq, N), device=dev, dtype=torch.float32),
    )
    dev = _device_of(q, k, *out.values())
    with torch.cuda.device(dev):
        rc = lib.attn_quant_smooth_k_noalloc(_ptr(q), _ptr(k), B, Hq, Hkv, N, d, DTYPES[q.dtype], scale,
                                             _ptr(out["q8"]), _ptr(out["sq"]), _ptr(out["k8"]), _ptr(out["sk"]),
                                             _ptr(out["kmean"]), _ptr(out["lse_bias"]), _stream(stream, dev))
    _check(rc, "attn_quant_smooth_k_noalloc")
    return out


def attn_fwd_int8_quantized(pre, v, causal=False, scale=None, out=None, lse=True, stream=None):
    """The fused INT8 kernel on the outputs of attn_quant_smooth_k (``pre``)."""
    lib = load_library()
    q8, k8 = pre["q8"], pre["k8"]
    B, Hq, N, d = q8.shape
    Hkv = k8.shape[1]
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    o = torch.empty((B, Hq, N, d), device=v.device, dtype=v.dtype) if out is None else out
    l = _lse_arg(lse, (B, Hq, N), v.device)
    dev = _device_of(q8, k8, pre["sq"], pre["sk"], pre["lse_bias"], v, o, l)
    with torch.cuda.device(dev):
        rc = lib.attn_fwd_int8_quantized(_ptr(q8), _ptr(pre["sq"]), _ptr(k8), _ptr(pre["sk"]),
                                         _ptr(pre["lse_bias"]), _ptr(v), _ptr(o), _ptr(l), B, Hq, Hkv, N, d,
                                         int(bool(causal)), scale, DTYPES[v.dtype], _stream(stream, dev))
    _check(rc, "attn_fwd_int8_quantized")
    return o, l


def attn_quant_smooth_k_fp8(q, k, scale=None, scratch=None, stream=None, out=None):
    """The FP8 pre-pass alone: E4M3 codes (uint8 bit patterns) and per-block scales.  Returns
    dict(q8, sq, k8, sk, kmean, lse_bias) (``out`` if given)."""
    lib = load_library()
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    _shape(q, k, k)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    T = (N + 127) // 128
    dev = q.device
    out = out or dict(
        q8=torch.empty((B, Hq, N, d), device=dev, dtype=torch.uint8),
        sq=torch.empty((B, Hq, T), device=dev, dtype=torch.float32),
        k8=torch.empty((B, Hkv, N, d), device=dev, dtype=torch.uint8),
        sk=torch.empty((B, Hkv, T), device=dev, dtype=torch.float32),
        kmean=torch.empty((B, Hkv, d), device=dev, dtype=torch.float32),
        lse_bias=torch.empty((B, Hq, N), device=dev, dtype=torch.float32),
    )
    if scratch is None:
        scratch = torch.empty(attn_quant_scratch_bytes(B, Hkv, N, d), device=dev, dtype=torch.uint8)
    dev = _device_of(q, k, scratch, *out.values())
    with torch.cuda.device(dev):
        rc = lib.attn_quant_smooth_k_fp8(_ptr(q), _ptr(k), B, Hq, Hkv, N, d, DTYPES[q.dtype], scale,
                                         _ptr(out["q8"]), _ptr(out["sq"]), _ptr(out["k8"]), _ptr(out["sk"]),
                                         _ptr(out["kmean"]), _ptr(out["lse_bias"]), _ptr(scratch), scratch.numel(),
                                         _stream(stream, dev))
    _check(rc, "attn_quant_smooth_k_fp8")
    return out


def attn_fwd_fp8_quantized(pre, v, causal=False, scale=None, out=None, lse=True, stream=None):
    """The fused FP8 kernel on the outputs of attn_quant_smooth_k_fp8 (``pre``)."""
    lib = load_library()
    q8, k8 = pre["q8"], pre["k8"]
    B, Hq, N, d = q8.shape
    Hkv = k8.shape[1]
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    o = torch.empty((B, Hq, N, d), device=v.device, dtype=v.dtype) if out is None else out
    l = _lse_arg(lse, (B, Hq, N), v.device)
    dev = _device_of(q8, k8, pre["sq"], pre["sk"], pre["lse_bias"], v, o, l)
    with torch.cuda.device(dev):
        rc = lib.attn_fwd_fp8_quantized(_ptr(q8), _ptr(pre["sq"]), _ptr(k8), _ptr(pre["sk"]),
                                        _ptr(pre["lse_bias"]), _ptr(v), _ptr(o), _ptr(l), B, Hq, Hkv, N, d,
                                        int(bool(causal)), scale, DTYPES[v.dtype], _stream(stream, dev))
    _check(rc, "attn_fwd_fp8_quantized")
    return o, l


def attn_probe_qk_int32(q8, k8, tiles, stream=None):
    """int32 scores of 128x128 tiles; ``tiles`` is a list of (b, h, m_tile, n_tile)."""
    lib = load_library()
    B, Hq, N, d = q8.shape
    Hkv = k8.shape[1]
    t = torch.tensor(tiles, dtype=torch.int32).reshape(-1, 4).to(q8.device)
    out = torch.empty((t.shape[0], 128, 128), device=q8.device, dtype=torch.int32)
    dev = _device_of(q8, k8, t, out)
    with torch.cuda.device(dev):
        rc = lib.attn_probe_qk_int32(_ptr(q8), _ptr(k8), B, Hq, Hkv, N, d, _ptr(t), t.shape[0], _ptr(out),
                                     _stream(stream, dev))
    _check(rc, "attn_probe_qk_int32")
    return out


def attn_fwd_host(q_host, k_host, v_host, o_host, lse_host, dq, dk, dv, do_, dlse, causal=False, scale=None,
                  mode="bf16_exact", workspace=None, stream=None):
    """attn_fwd with host buffers: H2D of q, k, v, the forward pass, D2H of o (and lse); synchronises."""
    lib = load_library()
    B, Hq, N, d = q_host.shape
    Hkv = k_host.shape[1]
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    dev = _device_of(dq, dk, dv, do_, dlse, workspace)
    with torch.cuda.device(dev):
        rc = lib.attn_fwd_host(_ptr(q_host), _ptr(k_host), _ptr(v_host), _ptr(o_host), _ptr(lse_host), _ptr(dq),
                               _ptr(dk), _ptr(dv), _ptr(do_), _ptr(dlse), B, Hq, Hkv, N, d, int(bool(causal)),
                               scale, MODES[mode], DTYPES[q_host.dtype], _ptr(workspace),
                               0 if workspace is None else workspace.numel(), _stream(stream, dev))
    _check(rc, "attn_fwd_host")


def attn_merge_lse(o_acc, lse_acc, o_part=None, lse_part=None, out=None, first=False, stream=None):
    """Join a partial attention result (o_part 16-bit [..., d], lse_part float32 [...]) into the
    running result (o_acc float32 [..., d], lse_acc float32 [...]) by their log-sum-exp, in place;
    ``first`` sets the running result to the part; ``out`` (16-bit, like o_part) receives the
    merged O.  Returns ``out``."""
    lib = load_library()
    if o_acc.dtype != torch.float32 or lse_acc.dtype != torch.float32:
        raise ValueError("o_acc and lse_acc must be float32")
    d = o_acc.shape[-1]
    rows = o_acc.numel() // d
    if lse_acc.numel() != rows:
        raise ValueError("lse_acc must hold one value per row of o_acc")
    ref = o_part if o_part is not None else out
    if ref is None:
        raise ValueError("nothing to do: give o_part/lse_part, out, or both")
    for t in (o_acc, lse_acc, o_part, lse_part, out):
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("every tensor must be a contiguous CUDA tensor")
    for t in (o_part, out):
        if t is not None and (t.dtype not in DTYPES or t.dtype != ref.dtype or t.numel() != rows * d):
            raise ValueError("o_part and out must be 16-bit tensors of o_acc's size and one dtype")
    if lse_part is not None and (lse_part.dtype != torch.float32 or lse_part.numel() != rows):
        raise ValueError("lse_part must be float32 with one value per row")
    dev = _device_of(o_acc, lse_acc, o_part, lse_part, out)
    with torch.cuda.device(dev):
        rc = lib.attn_merge_lse(_ptr(o_acc), _ptr(lse_acc), _ptr(o_part), _ptr(lse_part), _ptr(out), rows, d,
                                DTYPES[ref.dtype], int(bool(first)), _stream(stream, dev))
    _check(rc, "attn_merge_lse")
    return out


def attn_check_status() -> int:
    """Synchronise and return (and clear) the device status: 0 or ATTN_ERR_TIMEOUT."""
    return int(load_library().attn_check_status())


def attn_error_string(code: int) -> str:
    return load_library().attn_error_string(code).decode()


def attn_test_host_pieces(B, Hq, Hkv, N, d):
    """The query-head cut points attn_fwd_host uses for this shape (a list of ints)."""
    buf = (ctypes.c_int * 17)()
    n = load_library().attn_test_host_pieces(B, Hq, Hkv, N, d, ctypes.cast(buf, ctypes.c_void_p), 17)
    if n < 0:
        raise AttnError(n, "attn_test_host_pieces")
    return list(buf[:n + 1])


def attn_test_wait_timeout(limit_us: int, stream=None) -> None:
    _check(load_library().attn_test_wait_timeout(int(limit_us), _stream(stream)), "attn_test_wait_timeout")


def attn_test_exp2(x, use_poly, stream=None):
    """Apply the kernel's exp2 routine to a float32 CUDA tensor: use_poly 0 = MUFU ex2.approx,
    1 = FMA-pipe polynomial, 2 = the polynomial on packed pairs."""
    y = torch.empty_like(x)
    dev = _device_of(x, y)
    with torch.cuda.device(dev):
        _check(load_library().attn_test_exp2(_ptr(x), _ptr(y), x.numel(), int(use_poly), _stream(stream, dev)),
               "attn_test_exp2")
    return y
