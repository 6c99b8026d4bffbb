"""CPU-side checks of the C ABI: the library loads, exports every symbol the
header declares, and rejects bad arguments on the host before any launch.
No kernel runs here (there is no GPU); every call below returns during
argument validation."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tiled_attention.h")


@pytest.fixture(scope="module")
def lib():
    from tiled_attention_22_b200 import build, binding

    build.build()
    return binding.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*(attn_[a-z0-9_]+)\s*\(", text, flags=re.M)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("attn_fwd", "attn_quant_smooth_k", "attn_workspace_bytes", "attn_error_string",
                 "attn_probe_qk_int32", "attn_check_status", "attn_fwd_host", "attn_fwd_int8_quantized"):
        assert must in names


def test_library_exports_every_declared_symbol(lib):
    from tiled_attention_22_b200 import binding

    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in the header but not exported"
    assert set(declared_functions()) == set(binding.exported_symbols())


def test_error_strings(lib):
    for code in range(0, -7, -1):
        assert lib.attn_error_string(code)
    assert b"unknown" in lib.attn_error_string(-99)


def test_workspace_sizes(lib):
    # bf16_exact needs none; int8 holds q8, k8 (1 byte/elt), scales, mean, bias and float64 partials
    assert lib.attn_workspace_bytes(4, 32, 32, 4096, 128, 0) == 0
    B, Hq, Hkv, N, d = 2, 32, 8, 8192, 128
    T = N // 128
    need = B * Hq * N * d + B * Hkv * N * d + 4 * (B * Hq * T + B * Hkv * T + B * Hkv * d + B * Hq * N) \
        + 8 * B * Hkv * T * d
    got = lib.attn_workspace_bytes(B, Hq, Hkv, N, d, 1)
    assert need <= got <= need + 7 * 256
    assert lib.attn_quant_scratch_bytes(1, 8, 131072, 128) == 8 * 1024 * 128 * 8
    assert lib.attn_workspace_bytes(1, 3, 2, 128, 128, 1) == 0  # Hq % Hkv != 0


FAKE = 1 << 20  # a 16-byte aligned non-null value; never dereferenced (validation fails first)


def _fwd(lib, q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=None, B=1, Hq=2, Hkv=2, N=128, d=64, causal=0, scale=0.125,
         mode=0, dtype=0, ws=None, ws_bytes=0):
    return lib.attn_fwd(q, k, v, o, lse, B, Hq, Hkv, N, d, causal, scale, mode, dtype, ws, ws_bytes, None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), -1), (dict(o=None), -1), (dict(N=0), -1), (dict(B=0), -1), (dict(Hq=3, Hkv=2), -1),
    (dict(scale=float("nan")), -1), (dict(scale=float("inf")), -1), (dict(scale=-1.0), -1), (dict(mode=7), -1),
    (dict(dtype=5), -1), (dict(causal=2), -1), (dict(d=96), -2), (dict(d=256), -2),
    (dict(q=FAKE + 8), -3), (dict(v=FAKE + 2), -3), (dict(lse=FAKE + 4), -3),
    (dict(mode=1, ws=None), -4), (dict(mode=1, ws=FAKE, ws_bytes=16), -4),
])
def test_attn_fwd_rejects_bad_arguments(lib, kw, code):
    assert _fwd(lib, **kw) == code


def test_quant_and_probe_reject_bad_arguments(lib):
    f = lib.attn_quant_smooth_k
    args = [FAKE, FAKE, 1, 2, 2, 128, 64, 0, 0.125, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 20, None]
    bad = list(args); bad[0] = None
    assert f(*bad) == -1
    bad = list(args); bad[6] = 80
    assert f(*bad) == -2
    bad = list(args); bad[9] = FAKE + 1
    assert f(*bad) == -3
    bad = list(args); bad[16] = 8
    assert f(*bad) == -4
    p = lib.attn_probe_qk_int32
    assert p(FAKE, FAKE, 1, 2, 2, 128, 64, FAKE, 0, FAKE, None) == -1
    assert p(FAKE, FAKE, 1, 2, 2, 128, 48, FAKE, 1, FAKE, None) == -2
    assert lib.attn_test_wait_timeout(0, None) == -1
    assert lib.attn_fwd_int8_quantized(FAKE, None, FAKE, FAKE, FAKE, FAKE, FAKE, None, 1, 2, 2, 128, 64, 0, 0.1, 0,
                                       None) == -1


def test_product_path_fails_loudly_without_library(tmp_path):
    from tiled_attention_22_b200 import binding

    saved = binding._lib
    try:
        binding._lib = None
        with pytest.raises(RuntimeError, match="not built"):
            binding.load_library(str(tmp_path / "missing.so"))
    finally:
        binding._lib = saved


def test_product_package_does_not_import_the_oracle():
    pkg = os.path.join(ROOT, "tiled_attention_22_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, fn), encoding="utf-8").read()
                assert not re.search(r"^\s*(from|import)\s+oracle", text, flags=re.M), fn


def _dec(lib, q=FAKE, k=FAKE, v=FAKE, lens=None, o=FAKE, lse=None, B=1, Hq=8, Hkv=2, Nq=1, Nk=1024, d=128,
         causal=0, scale=0.125, dtype=0, ctas=1, ws=None, ws_bytes=0):
    return lib.attn_decode(q, k, v, lens, o, lse, B, Hq, Hkv, Nq, Nk, d, causal, scale, dtype, ctas, ws, ws_bytes,
                           None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), -1), (dict(o=None), -1), (dict(Nq=0), -1), (dict(Nq=2000), -1), (dict(Hq=3), -1),
    (dict(scale=0.0), -1), (dict(causal=-1), -1), (dict(dtype=2), -1), (dict(ctas=-1), -1),
    (dict(d=64), -2), (dict(Hq=128, Hkv=1), -2), (dict(Hq=8, Hkv=1, Nq=9), -2),
    (dict(q=FAKE + 2), -3), (dict(lens=FAKE + 2), -3), (dict(lse=FAKE + 8), -3),
    (dict(ctas=4), -4), (dict(ws=FAKE, ws_bytes=64), -4),
])
def test_attn_decode_rejects_bad_arguments(lib, kw, code):
    assert _dec(lib, **kw) == code


def test_decode_workspace_sizes(lib):
    # U + P - 1 slots of fp32 partial outputs (R x 128) and lse (R), one arrival counter per unit
    B, Hq, Hkv, Nq, Nk, P = 8, 32, 8, 1, 32768, 148
    U, R = B * Hkv, (Hq // Hkv) * Nq
    slots = U + P - 1
    need = slots * R * 128 * 4 + slots * R * 4 + U * 4
    got = lib.attn_decode_workspace_bytes(B, Hq, Hkv, Nq, Nk, 128, P)
    assert need <= got <= need + 3 * 256
    # the CTA count is capped at the number of key tiles of the largest problem (here 2)
    assert lib.attn_decode_workspace_bytes(1, 2, 2, 1, 256, 128, 50) == \
        lib.attn_decode_workspace_bytes(1, 2, 2, 1, 256, 128, 4)
    assert lib.attn_decode_workspace_bytes(1, 2, 2, 1, 256, 64, 2) == 0  # d = 64 unsupported


class _FakeTensor:
    """Stands in for a tensor in the binding's device check (only .device is read)."""

    def __init__(self, kind, index=None):
        import torch

        self.device = torch.device(kind, index) if index is not None else torch.device(kind)


def test_binding_refuses_tensors_on_two_devices():
    """Every launch and the library's per-device state follow the current device, so a binding call
    runs with its tensors' device current and refuses tensors spread over several devices."""
    from tiled_attention_22_b200 import binding

    a0, b0, a1 = _FakeTensor("cuda", 0), _FakeTensor("cuda", 0), _FakeTensor("cuda", 1)
    assert binding._device_of(a0, None, b0) == 0
    assert binding._device_of(None, a1) == 1
    with pytest.raises(ValueError, match="one device"):
        binding._device_of(a0, a1)
    with pytest.raises(ValueError, match="CUDA tensor"):
        binding._device_of(a0, _FakeTensor("cpu"))
    with pytest.raises(ValueError, match="no CUDA tensor"):
        binding._device_of(None, None)


def test_plain_c_consumer_builds_and_runs(lib, tmp_path):
    """The header is usable from C99 on its own: tests/c_consumer.c includes only it, links the
    shared library, and checks the host-side calls (no device work)."""
    import shutil
    import subprocess

    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    from tiled_attention_22_b200 import binding

    libdir = os.path.dirname(binding.LIB_PATH)
    exe = str(tmp_path / "c_consumer")
    subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c_consumer.c"), "-L", libdir, "-ltiled_attention",
                    "-Wl,-rpath," + libdir, "-lm", "-o", exe], check=True, capture_output=True, text=True)
    run = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0 and run.stdout.strip().endswith("OK"), run.stdout + run.stderr


@pytest.mark.parametrize("shape", [
    (1, 32, 8, 131072), (2, 32, 8, 8192), (4, 32, 32, 4096), (2, 24, 24, 16384),  # the named workloads
    (1, 4, 2, 500), (3, 6, 3, 333), (2, 8, 8, 1024), (1, 4, 1, 256), (2, 8, 2, 2048),  # the GPU test shapes
    (1, 1, 1, 1), (1, 2, 1, 4), (1, 3, 3, 334), (5, 8, 1, 12), (64, 16, 4, 100), (1, 128, 2, 96),
])
def test_host_buffer_pieces(lib, shape):
    """The query-head pieces of attn_fwd_host: contiguous cover of all B*Hq heads; each piece
    whole (batch, kv head) units or heads inside one unit (so one kernel call can do it); every
    piece's lse slice 16-byte aligned; at most 10 pieces; single heads (or single units when
    Hq == Hkv) at both ends whenever N % 4 == 0."""
    from tiled_attention_22_b200 import binding

    B, Hq, Hkv, N = shape
    cuts = binding.attn_test_host_pieces(B, Hq, Hkv, N, 128)
    heads, G = B * Hq, Hq // Hkv
    assert cuts[0] == 0 and cuts[-1] == heads
    assert all(a < b for a, b in zip(cuts, cuts[1:]))
    assert len(cuts) - 1 <= 10
    for a, b in zip(cuts, cuts[1:]):
        whole = a % G == 0 and (b - a) % G == 0
        assert whole or a // G == (b - 1) // G, (a, b)
        assert (a * N * 4) % 16 == 0, (a, "lse slice not 16-byte aligned")
    if N % 4 == 0 and heads > 1:
        first, last = cuts[1] - cuts[0], cuts[-1] - cuts[-2]
        assert first == (1 if G > 1 else G) and last == (1 if G > 1 else G)


def test_host_buffer_pieces_reject_bad_shapes(lib):
    from tiled_attention_22_b200 import binding

    for args, code in (((1, 3, 2, 128, 128), -1), ((1, 2, 2, 128, 96), -2), ((0, 2, 2, 128, 64), -1)):
        with pytest.raises(binding.AttnError) as e:
            binding.attn_test_host_pieces(*args)
        assert e.value.code == code
    assert lib.attn_test_host_pieces(1, 2, 2, 128, 64, None, 17) == -1
