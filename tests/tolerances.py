"""Output tolerances shared by the GPU parity suites.

The bars come from the method's accuracy targets: bf16_exact output max-abs error <= 2e-2 and
mean-abs error <= 2e-3 against float64; int8_qk output cosine similarity >= 0.999 and max-abs error
<= 5e-2.  They are absolute errors.  The kernels return O in the input's 16-bit type, and rounding
a float64 value to that type alone moves it by up to half a unit in the last place: 2^-8 |O| for
bf16 (8 significant bits), 2^-11 |O| for fp16 (11).  Each element is therefore allowed the bar plus
that half-ulp and nothing more:

    |o - O| <= bar + h |O|,   h = 2^-8 (bf16 output) or 2^-11 (fp16 output).

``excess`` returns |o - O| - h |O| per element, which is compared with the bar.  The mean bar is
applied to the plain absolute error of the elements with |O| <= 1 (where the half-ulp term is at
most h and the bar is meaningful on its own).
"""
import numpy as np

BF16_MAX, BF16_MEAN, BF16_LSE = 2e-2, 2e-3, 1e-3
INT8_COS, INT8_MAX, INT8_LSE = 0.999, 5e-2, 5e-2

HALF_ULP = {"bf16": 2.0 ** -8, "fp16": 2.0 ** -11}


def half_ulp(dtype) -> float:
    """Relative half-ulp of the 16-bit output type (a workload dtype name or a torch dtype)."""
    name = str(dtype)
    if "bfloat16" in name or name == "bf16":
        return HALF_ULP["bf16"]
    if "float16" in name or name in ("fp16", "half"):
        return HALF_ULP["fp16"]
    raise ValueError(f"no 16-bit output type for {dtype!r}")


def excess(o, O, dtype="bf16"):
    """|o - O| minus the output type's rounding allowance h |O|, element by element."""
    return np.abs(o - O) - half_ulp(dtype) * np.abs(O)


def max_excess(o, O, dtype="bf16") -> float:
    return float(np.max(excess(o, O, dtype))) if np.size(O) else 0.0


def mean_abs_small(o, O) -> float:
    """Mean plain absolute error over the elements with |O| <= 1 (0 if there are none)."""
    sel = np.abs(O) <= 1.0
    return float(np.mean(np.abs(o - O)[sel])) if sel.any() else 0.0


def cosine(a, b) -> float:
    a, b = np.reshape(a, -1), np.reshape(b, -1)
    return float(a @ b / (np.linalg.norm(a) * np.linalg.norm(b) + 1e-300))


def assert_close16(o, l, O, L, dtype="bf16", what="", bar=BF16_MAX, mean_bar=BF16_MEAN, lse_bar=BF16_LSE):
    """The bf16_exact bars: max excess <= bar, mean abs (|O| <= 1) <= mean_bar, lse max-abs <= lse_bar."""
    assert np.isfinite(o).all(), what
    e = max_excess(o, O, dtype)
    m = mean_abs_small(o, O)
    assert e <= bar, f"{what}: max |o - O| - h|O| = {e:.3e} > {bar}"
    assert m <= mean_bar, f"{what}: mean abs err {m:.3e} > {mean_bar}"
    if l is not None:
        fin = np.isfinite(L)
        assert np.array_equal(fin, np.isfinite(l)), f"{what}: lse finiteness differs"
        if fin.any():
            le = float(np.abs(l - L)[fin].max())
            assert le <= lse_bar, f"{what}: lse err {le:.3e} > {lse_bar}"
            return e, m, le
    return e, m, 0.0


def quant_metrics(o, l, O, L, dtype="bf16"):
    """Accuracy of an 8-bit-Q K^T output against exact attention: cosine, max excess, lse error."""
    return {"cos": cosine(o, O), "err": max_excess(o, O, dtype), "lse": float(np.abs(l - L).max())}
