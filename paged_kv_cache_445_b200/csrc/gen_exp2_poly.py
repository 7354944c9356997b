"""Coefficients of the polynomial 2^f ~ p(f) on f in [0, 1) that the chunk
kernel evaluates on the FMA pipe for part of its softmax exponentials.

Method: Cody-Waite range reduction (W. J. Cody and W. Waite, "Software Manual
for the Elementary Functions", 1980): 2^x = 2^n * 2^f with n = floor(x) and
f = x - n in [0, 1); then a polynomial of degree N for 2^f with p(0) = 1,
whose other coefficients minimise the maximum RELATIVE error on [0, 1]
(minimax, found with the Remez exchange algorithm: alternate between solving
for the coefficients that equioscillate on N + 1 reference points and moving
the points to the error's extrema).  The kernel adds n to the exponent field
of p(f).

    python -m paged_kv_cache_445_b200.csrc.gen_exp2_poly [degree]

prints the coefficients c1 .. cN (c0 = 1) as binary32 values and the maximum
relative error of the binary32 evaluation.
"""
from __future__ import annotations

import sys

import numpy as np


def remez_exp2(degree: int, iters: int = 30):
    """p(f) = 1 + c1 f + ... + cN f^N minimising max |p(f) / 2^f - 1| on [0, 1]."""
    n = degree  # unknowns c1..cN and the level E: N + 1 equations on N + 1 points
    # start: Chebyshev extrema mapped to (0, 1]
    k = np.arange(n + 1)
    pts = 0.5 - 0.5 * np.cos(np.pi * (k + 1) / (n + 1))
    grid = np.linspace(0.0, 1.0, 200001)
    c = None
    for _ in range(iters):
        # (p(x_i) - 2^x_i) / 2^x_i = (-1)^i E  ->  sum_j c_j x_i^j - (-1)^i E 2^x_i = 2^x_i - 1
        a = np.zeros((n + 1, n + 1))
        for i, x in enumerate(pts):
            for j in range(1, n + 1):
                a[i, j - 1] = x ** j
            a[i, n] = -((-1) ** i) * 2.0 ** x
        b = 2.0 ** pts - 1.0
        sol = np.linalg.solve(a, b)
        c = sol[:n]
        err = (1.0 + sum(c[j - 1] * grid ** j for j in range(1, n + 1))) / 2.0 ** grid - 1.0
        # new reference: the extremum of each sign run
        sign = np.sign(err)
        sign[sign == 0] = 1
        bounds = np.flatnonzero(np.diff(sign)) + 1
        runs = np.split(np.arange(len(grid)), bounds)
        ext = [r[np.argmax(np.abs(err[r]))] for r in runs]
        if len(ext) > n + 1:  # keep the n + 1 largest while alternating: drop the smallest at the ends
            while len(ext) > n + 1:
                if abs(err[ext[0]]) < abs(err[ext[-1]]):
                    ext = ext[1:]
                else:
                    ext = ext[:-1]
        if len(ext) == n + 1:
            pts = grid[ext]
    return c


def eval_f32(c, f):
    """Horner in binary32 with fused multiply-adds, as the kernel does it."""
    f = np.asarray(f, dtype=np.float32)
    acc = np.full_like(f, np.float32(c[-1]))
    for cj in list(c[:-1])[::-1]:
        acc = (acc.astype(np.float64) * f + np.float64(np.float32(cj))).astype(np.float32)
    return (acc.astype(np.float64) * f + 1.0).astype(np.float32)


def main(argv=None) -> int:
    argv = sys.argv[1:] if argv is None else argv
    degree = int(argv[0]) if argv else 3
    c = [float(np.float32(x)) for x in remez_exp2(degree)]
    f = np.linspace(0.0, 1.0, 1 << 20, dtype=np.float32)
    rel = np.abs(eval_f32(c, f).astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0).max()
    for j, cj in enumerate(c, start=1):
        print(f"c{j} = {cj!r}  ({np.float32(cj).view(np.uint32):#010x})")
    print(f"max relative error of the binary32 evaluation on [0, 1): {rel:.3e}")
    return 0


if __name__ == "__main__":
    sys.exit(main())
