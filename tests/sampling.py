"""Row and head samples for the full-size parity tests (the oracle computes selected rows only;
rows are independent, so the comparison is exact for them).

Rows: the first rows, every boundary of a 128-row query tile and of a 256-row work item in the
first and last 1024 rows and around the middle, the last rows (including the ragged tail's last
full tile), and random rows.  Heads: the first and last (batch, head), both sides of a GQA group
boundary, and random ones."""
import numpy as np


def boundary_rows(N, rng, n_random=12):
    rows = {0, 1, 2, N - 1, N // 2}
    for base in (0, max(0, N // 2 - 512), max(0, N - 1024)):
        for r in range(base, min(N, base + 1024), 128):
            rows |= {r, r - 1, r + 127}
    for off in (1, 2, 127, 128, 129, 255, 256, 257):
        rows.add(N - off)
    rows |= set(rng.integers(0, N, n_random).tolist())
    return sorted(r for r in rows if 0 <= r < N)


def sample_heads(B, Hq, Hkv, rng, n_random=2):
    G = Hq // Hkv
    heads = {(0, 0), (B - 1, Hq - 1)}
    if G > 1:
        heads |= {(0, G - 1), (0, G)} if Hq > G else {(0, G - 1)}
    for _ in range(n_random):
        heads.add((int(rng.integers(B)), int(rng.integers(Hq))))
    return sorted(heads)
