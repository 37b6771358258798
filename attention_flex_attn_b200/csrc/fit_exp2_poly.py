"""Fits the polynomial the forward kernel uses to evaluate 2^f on the FMA pipe.

The kernel splits x = n + f with n = round(x) (an fp32 add of 1.5 * 2^23 and its
subtraction) and f in [-1/2, 1/2], evaluates p(f) ~ 2^f with Horner's rule, and adds
n to the exponent field of p(f).  This script finds p of a given degree that minimises
the maximum RELATIVE error of p(f) / 2^f on [-1/2, 1/2]: a least-squares start on
Chebyshev nodes, then Remez exchange iterations on the weighted error
e(f) = (p(f) - 2^f) / 2^f.  The printed coefficients are what the kernel stores
(rounded to fp32); the reported error is re-measured with the fp32-rounded values.

    python attention_flex_attn_b200/csrc/fit_exp2_poly.py [degree]
"""
from __future__ import annotations

import sys

import numpy as np


def _weighted_fit(x, deg):
    """Least squares of p(x)/2^x ~ 1, i.e. rows x^k / 2^x against ones."""
    A = np.vander(x, deg + 1, increasing=True) / np.exp2(x)[:, None]
    c, *_ = np.linalg.lstsq(A, np.ones_like(x), rcond=None)
    return c


def _rel_err(c, x):
    return np.polynomial.polynomial.polyval(x, c) / np.exp2(x) - 1.0


def remez(deg: int, lo: float = -0.5, hi: float = 0.5, iters: int = 30):
    k = np.arange(4 * deg + 8)
    nodes = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * (k + 0.5) / k.size)
    c = _weighted_fit(np.sort(nodes), deg)
    grid = np.linspace(lo, hi, 200001)
    # reference points: deg + 2 alternation points
    ref = np.linspace(lo, hi, deg + 2)
    for _ in range(iters):
        # solve p(x_i) / 2^x_i - 1 = (-1)^i E at the reference
        A = np.zeros((deg + 2, deg + 2))
        for i, x in enumerate(ref):
            A[i, : deg + 1] = x ** np.arange(deg + 1) / np.exp2(x)
            A[i, deg + 1] = (-1) ** i
        sol = np.linalg.solve(A, np.ones(deg + 2))
        c = sol[: deg + 1]
        e = _rel_err(c, grid)
        # new reference: extrema of e between sign changes
        idx = [0]
        for i in range(1, grid.size - 1):
            if (e[i] - e[i - 1]) * (e[i + 1] - e[i]) <= 0:
                idx.append(i)
        idx.append(grid.size - 1)
        idx = np.array(sorted(set(idx)))
        # keep the deg+2 largest alternating extrema
        pts = grid[idx]
        vals = e[idx]
        chosen = [0]
        for i in range(1, len(pts)):
            if np.sign(vals[i]) != np.sign(vals[chosen[-1]]):
                chosen.append(i)
            elif abs(vals[i]) > abs(vals[chosen[-1]]):
                chosen[-1] = i
        if len(chosen) >= deg + 2:
            best = max(range(len(chosen) - deg - 1),
                       key=lambda s: min(abs(vals[chosen[s + t]]) for t in range(deg + 2)))
            ref = pts[[chosen[best + t] for t in range(deg + 2)]]
    return c


def main():
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c = remez(deg)
    c32 = c.astype(np.float32).astype(np.float64)
    grid = np.linspace(-0.5, 0.5, 400001)
    print(f"degree {deg}: max relative error {np.abs(_rel_err(c, grid)).max():.3e} "
          f"(fp32 coefficients {np.abs(_rel_err(c32, grid)).max():.3e})")
    for i, v in enumerate(c.astype(np.float32)):
        print(f"  c{i} = {float(v)!r}f")


if __name__ == "__main__":
    main()
