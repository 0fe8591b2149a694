"""Fit the polynomial the prefill softmax uses to evaluate 2^f on the FMA pipe.

Method: Cody-Waite style range reduction, x = n + f with n = round(x) and
f in [-1/2, 1/2], so 2^x = 2^n * 2^f, where 2^n is built by adding n to the
exponent field and 2^f comes from a degree-3 polynomial.  The coefficients are
a minimax fit of the relative error on [-1/2, 1/2], obtained here with the
Remez exchange algorithm (Remez, 1934), rounded to float32.

    python -m sliding_window_sparse_b200.fit_exp2_poly

prints the coefficients (lowest order first) and the maximum relative error
of the float32 Horner evaluation; the values are copied into csrc/sm100.cuh.
"""

from __future__ import annotations

import numpy as np

DEGREE = 3
LO, HI = -0.5, 0.5


def _solve(nodes):
    # p(x_i) - 2^x_i = (-1)^i * E * 2^x_i   (equioscillating relative error)
    n = DEGREE + 2
    A = np.zeros((n, n))
    b = np.exp2(nodes)
    for i, x in enumerate(nodes):
        A[i, :DEGREE + 1] = x ** np.arange(DEGREE + 1)
        A[i, DEGREE + 1] = -((-1) ** i) * np.exp2(x)
    sol = np.linalg.solve(A, b)
    return sol[:DEGREE + 1], sol[DEGREE + 1]


def remez(iters: int = 30):
    k = np.arange(DEGREE + 2)
    nodes = (LO + HI) / 2 + (HI - LO) / 2 * np.cos(np.pi * (DEGREE + 1 - k) / (DEGREE + 1))
    grid = np.linspace(LO, HI, 200001)
    for _ in range(iters):
        c, _ = _solve(nodes)
        err = (np.polyval(c[::-1], grid) - np.exp2(grid)) / np.exp2(grid)
        # new nodes: the extrema of err between sign changes
        idx = [0]
        for i in range(1, len(grid) - 1):
            if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0:
                idx.append(i)
        idx.append(len(grid) - 1)
        idx = sorted(set(idx), key=lambda i: -abs(err[i]))[:DEGREE + 2]
        nodes = np.sort(grid[idx])
    return c


def horner_f32(c32, f):
    f = np.asarray(f, dtype=np.float32)
    acc = np.full_like(f, c32[-1])
    for ci in c32[-2::-1]:
        acc = (acc * f + ci).astype(np.float32)
    return acc


def max_rel_error(c32):
    f = np.linspace(LO, HI, 1000001, dtype=np.float32)
    p = horner_f32(c32, f).astype(np.float64)
    return float(np.max(np.abs(p - np.exp2(f.astype(np.float64))) / np.exp2(f.astype(np.float64))))


def main():
    c = remez()
    c32 = np.array(c, dtype=np.float32)
    for i, v in enumerate(c32):
        print(f"c{i} = {float(v)!r:>24}  ({float(v).hex()})")
    print(f"max relative error (float32 Horner) = {max_rel_error(c32):.3e}")


if __name__ == "__main__":
    main()
