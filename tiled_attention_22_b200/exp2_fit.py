"""Fit the polynomial used by the kernels' FMA-pipe exp2 (run: python -m tiled_attention_22_b200.exp2_fit).

Method: Cody-Waite style range reduction, 2^x = 2^n * 2^f with n = rint(x) and f = x - n in
[-1/2, 1/2] (W. J. Cody and W. Waite, "Software Manual for the Elementary Functions", 1980),
and a minimax polynomial for 2^f on that interval found with the Remez exchange algorithm
(E. Remez, 1934), minimising the maximum RELATIVE error |p(f) / 2^f - 1|.

The coefficients are rounded to float32 and the error is re-measured in float32 Horner
arithmetic with fused multiply-adds, which is how the kernel evaluates them.  The kernel's
copy of the coefficients (attn_fwd_kernels.cuh, exp2_poly) must equal the printed values.
"""
from __future__ import annotations

import numpy as np


def remez_relative(degree: int, lo: float = -0.5, hi: float = 0.5, iters: int = 40):
    f = lambda x: np.exp2(x)  # noqa: E731
    n = degree + 2
    # Chebyshev points as the first reference set
    k = np.arange(n)
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * (n - 1 - k) / (n - 1))
    grid = np.linspace(lo, hi, 200001)
    c = None
    for _ in range(iters):
        # solve sum_j c_j x_i^j - f(x_i) = (-1)^i E f(x_i)
        A = np.zeros((n, n))
        for j in range(degree + 1):
            A[:, j] = x ** j
        A[:, degree + 1] = -((-1.0) ** np.arange(n)) * f(x)
        sol = np.linalg.solve(A, f(x))
        c = sol[: degree + 1]
        err = np.polyval(c[::-1], grid) / f(grid) - 1.0
        # new reference: extrema of the error between sign changes
        idx = [0]
        for i in range(1, len(grid) - 1):
            if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0:
                idx.append(i)
        idx.append(len(grid) - 1)
        idx = np.array(sorted(set(idx)))
        # keep n alternating extrema with the largest magnitude
        cand = idx[np.argsort(-np.abs(err[idx]))]
        chosen = []
        for i in sorted(cand[: max(n * 4, n)]):
            chosen.append(i)
        chosen = sorted(chosen)
        alt = [chosen[0]]
        for i in chosen[1:]:
            if np.sign(err[i]) == np.sign(err[alt[-1]]):
                if abs(err[i]) > abs(err[alt[-1]]):
                    alt[-1] = i
            else:
                alt.append(i)
        while len(alt) > n:
            # drop the smaller end
            if abs(err[alt[0]]) < abs(err[alt[-1]]):
                alt.pop(0)
            else:
                alt.pop()
        if len(alt) < n:
            break
        x = grid[np.array(alt)]
    return c


def float32_horner_error(c32, lo=-0.5, hi=0.5):
    f = np.linspace(lo, hi, 400001).astype(np.float32)
    acc = np.full_like(f, c32[-1])
    for cj in c32[-2::-1]:
        acc = (acc.astype(np.float64) * f + np.float64(cj)).astype(np.float32)  # one rounding = fma
    ref = np.exp2(f.astype(np.float64))
    return float(np.max(np.abs(acc / ref - 1.0)))


def main():
    for deg in (3, 4):
        c = remez_relative(deg)
        c32 = c.astype(np.float32)
        print(f"degree {deg}: coefficients c0..c{deg} (float32):")
        for j, v in enumerate(c32):
            print(f"  c{j} = {float(v):.9e}f  (hex {np.float32(v).view(np.uint32):#010x})")
        print(f"  max relative error in float32 Horner/FMA: {float32_horner_error(c32):.3e}")


if __name__ == "__main__":
    main()
