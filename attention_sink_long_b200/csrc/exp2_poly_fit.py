"""Fit the polynomial that the attention kernels use for part of their 2^x.

The softmax evaluates most exponentials on the special-function unit and a
fixed share on the FMA pipe, as 2^x = 2^n * 2^f with n = round(x) (Cody and
Waite's additive range reduction, done with the 1.5 * 2^23 rounding trick)
and f in [-1/2, 1/2]; 2^f is a degree-4 polynomial whose coefficients are the
minimax fit of the RELATIVE error on [-1/2, 1/2], computed here with the
Remez exchange algorithm in float64, then rounded to float32.

    python attention_sink_long_b200/csrc/exp2_poly_fit.py

prints the coefficients (to paste into lg_common.cuh) and the worst relative
error of the float32 evaluation.
"""

from __future__ import annotations

import numpy as np

DEGREE = 4
LO, HI = -0.5, 0.5


def remez_relative(degree: int, iters: int = 30):
    """Minimax polynomial p of the given degree minimising max |p(f)/2^f - 1| on [LO, HI]."""
    n = degree + 2
    # Chebyshev extrema as the initial reference.
    k = np.arange(n)
    ref = (LO + HI) / 2 + (HI - LO) / 2 * np.cos(np.pi * k / (n - 1))[::-1]
    grid = np.linspace(LO, HI, 200001)
    for _ in range(iters):
        # Solve p(x_i) - (-1)^i * E * 2^{x_i} = 2^{x_i}  (relative equioscillation).
        A = np.zeros((n, n))
        for i, x in enumerate(ref):
            A[i, :degree + 1] = x ** np.arange(degree + 1)
            A[i, degree + 1] = (-1) ** i * 2.0 ** x
        sol = np.linalg.solve(A, 2.0 ** ref)
        c = sol[:degree + 1]
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
        # New reference: the extrema of the error, one per sign change interval.
        idx = [0]
        for j in range(1, len(grid) - 1):
            if (err[j] - err[j - 1]) * (err[j + 1] - err[j]) <= 0:
                idx.append(j)
        idx.append(len(grid) - 1)
        cand = sorted(idx, key=lambda j: -abs(err[j]))
        # keep n alternating extrema
        pts = sorted(cand[: 4 * n])
        chosen = []
        for j in pts:
            if chosen and np.sign(err[j]) == np.sign(err[chosen[-1]]):
                if abs(err[j]) > abs(err[chosen[-1]]):
                    chosen[-1] = j
            else:
                chosen.append(j)
        while len(chosen) > n:
            if abs(err[chosen[0]]) < abs(err[chosen[-1]]):
                chosen.pop(0)
            else:
                chosen.pop()
        if len(chosen) < n:
            break
        ref = grid[chosen]
    return c


def eval_f32(c32, x):
    """Mirror of the device evaluation in float32: clamp, round, Horner, exponent add."""
    x = np.maximum(np.float32(x), np.float32(-127.0)).astype(np.float32)
    y = (x + np.float32(12582912.0)).astype(np.float32)
    n = (y - np.float32(12582912.0)).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = np.full_like(f, c32[-1])
    for ck in c32[-2::-1]:
        p = (p * f + ck).astype(np.float32)  # fmaf rounding differs by < 1 ulp
    bits = p.view(np.uint32) + (y.view(np.uint32) << np.uint32(23))
    out = bits.view(np.float32)
    return np.where(x <= np.float32(-127.0), np.float32(0.0), out)


def main():
    c = remez_relative(DEGREE)
    c32 = c.astype(np.float32)
    xs = np.linspace(-126.0, 64.0, 2_000_001, dtype=np.float64)
    got = eval_f32(c32, xs.astype(np.float32)).astype(np.float64)
    rel = np.abs(got / np.exp2(xs.astype(np.float32).astype(np.float64)) - 1.0)
    for k, v in enumerate(c32):
        print(f"C{k} = {float(v)!r}  ({v.view(np.uint32):#010x})")
    print(f"max relative error on [-126, 64]: {rel.max():.3e}")


if __name__ == "__main__":
    main()
