"""Reproduce the cubic used for 2^f in the prefill softmax (prefill_tc.cu, exp2_poly).

A Remez exchange for the best minimax *relative* error of a degree-3 polynomial to
2^f on f in [-1/2, 1/2]. Run ``python -m block_sparse_long_06_b200.exp2_poly_fit``
to print the coefficients (float32) and the achieved error.
"""
from __future__ import annotations

import numpy as np


def remez_exp2(deg: int = 3, a: float = -0.5, b: float = 0.5, iters: int = 40):
    n = deg + 2
    x = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    xs = np.linspace(a, b, 200001)
    for _ in range(iters):
        A = np.zeros((n, n))
        for i, xi in enumerate(x):
            A[i, :deg + 1] = xi ** np.arange(deg + 1) / 2.0 ** xi
            A[i, deg + 1] = (-1) ** i
        sol = np.linalg.solve(A, np.ones(n))
        c = sol[:deg + 1]
        err = np.polyval(c[::-1], xs) / 2.0 ** xs - 1.0
        # alternating extrema of the error become the next reference points
        ext = [0] + [k for k in range(1, len(xs) - 1)
                     if (err[k] - err[k - 1]) * (err[k + 1] - err[k]) <= 0] + [len(xs) - 1]
        pts = []
        for k in ext:
            if pts and np.sign(err[k]) == np.sign(err[pts[-1]]):
                if abs(err[k]) > abs(err[pts[-1]]):
                    pts[-1] = k
            else:
                pts.append(k)
        while len(pts) > n:
            pts.pop(0 if abs(err[pts[0]]) < abs(err[pts[-1]]) else -1)
        x = xs[pts]
    return c, float(np.max(np.abs(err)))


def emulate_exp2_f32(x: np.ndarray, coeffs) -> np.ndarray:
    """The kernel's arithmetic in float32: clamp, round-to-nearest split via 1.5*2^23,
    Horner cubic, exponent insertion."""
    c0, c1, c2, c3 = (np.float32(v) for v in coeffs)
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    shift = np.float32(12582912.0)
    r = (x + shift).astype(np.float32)
    nn = (shift - r).astype(np.float32)
    f = (x + nn).astype(np.float32)
    p = ((c3 * f + c2) * f + c1) * f + c0
    p = p.astype(np.float32)
    bits = p.view(np.uint32).astype(np.uint64) + (r.view(np.uint32).astype(np.uint64) << np.uint64(23))
    return (bits & np.uint64(0xFFFFFFFF)).astype(np.uint32).view(np.float32)


if __name__ == "__main__":
    c, e = remez_exp2()
    print("coefficients c0..c3 (float32):", [float(np.float32(v)) for v in c])
    print("max relative error:", e)
