"""Fits the polynomial the prefill kernel uses to evaluate part of its exponentials on the FMA pipe.

Method (Cody-Waite range reduction, then a minimax polynomial):
    2^x = 2^j * 2^f,  j = round-to-nearest(x),  f = x - j in [-1/2, 1/2]
    2^f ~ p(f) = c0 + c1 f + c2 f^2 + c3 f^3
and 2^j is applied by adding j to the IEEE exponent field of p(f).  The coefficients minimise the maximum
relative error |p(f) / 2^f - 1| over [-1/2, 1/2]; they are found with Lawson's iteratively re-weighted
least squares (which converges to the minimax solution) on a dense grid, then rounded to float32.

Run:  python exact_tiled_attention_43_b200/csrc/fit_exp2_poly.py    (prints the float32 constants that
exp2_poly.cuh holds; the CPU test checks that they match this fit and the error bound).
"""
from __future__ import annotations

import numpy as np

DEGREE = 3


def fit(degree: int = DEGREE, n: int = 20001, iters: int = 200) -> np.ndarray:
    f = np.linspace(-0.5, 0.5, n)
    y = np.exp2(f)
    A = np.vander(f, degree + 1, increasing=True) / y[:, None]  # relative-error rows
    b = np.ones_like(f)
    w = np.full(n, 1.0 / n)
    c = None
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A * sw[:, None], b * sw, rcond=None)
        err = np.abs(A @ c - b)
        w = w * err
        w /= w.sum()
    return c.astype(np.float32)


def eval_f32(x: np.ndarray, c: np.ndarray) -> np.ndarray:
    """The kernel's evaluation, step by step in float32 (clamp, round via the 1.5*2^23 shifter, Horner,
    exponent add)."""
    x = np.maximum(np.asarray(x, np.float32), np.float32(-125.0))
    shifter = np.float32(12582912.0)
    t = (x + shifter).astype(np.float32)
    r = (t - shifter).astype(np.float32)
    fr = (x - r).astype(np.float32)
    p = np.float32(c[3])
    for k in (2, 1, 0):
        p = (p * fr + np.float32(c[k])).astype(np.float32)
    bits = p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << np.uint64(23))
    return (bits & np.uint64(0xFFFFFFFF)).astype(np.uint32).view(np.float32)


def max_rel_error(c: np.ndarray, lo: float = -125.0, hi: float = 8.0, n: int = 2_000_001) -> float:
    x = np.linspace(lo, hi, n, dtype=np.float64).astype(np.float32)
    got = eval_f32(x, c).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    return float(np.max(np.abs(got / ref - 1.0)))


if __name__ == "__main__":
    c = fit()
    for k, v in enumerate(c):
        print(f"c{k} = {float(v)!r}f  /* 0x{np.float32(v).view(np.uint32):08x} */")
    print("max relative error over [-125, 8]:", max_rel_error(c))
