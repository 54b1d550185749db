"""Fits the polynomial the prefill kernel uses to evaluate part of HSTU's tanh on the FMA pipe.

Method: tanh is odd, so on [-1, 1] it is approximated as
    tanh(y) ~ y * (c0 + c1 y^2 + c2 y^4 + c3 y^6)
with the coefficients chosen to minimise the maximum absolute error, found with Lawson's iteratively
re-weighted least squares (which converges to the minimax solution) on a dense grid of [0, 1], then rounded
to float32.  The kernel applies it only to arguments it has checked lie in [-1, 1]; elsewhere it uses the
MUFU's tanh.

Run:  python exact_tiled_attention_43_b200/csrc/fit_tanh_poly.py   (prints the float32 constants prefill.cuh
holds; the CPU test checks that they match this fit and its error bound).
"""
from __future__ import annotations

import numpy as np

TERMS = 4


def fit(terms: int = TERMS, n: int = 40000, iters: int = 300) -> np.ndarray:
    y = np.linspace(0.0, 1.0, n + 1)[1:]
    t = np.tanh(y)
    A = np.vstack([y ** (2 * k + 1) for k in range(terms)]).T
    w = np.full(y.size, 1.0 / y.size)
    c = None
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A * sw[:, None], t * sw, rcond=None)
        err = np.abs(A @ c - t)
        w = w * err
        w /= w.sum()
    return c.astype(np.float32)


def eval_f32(y: np.ndarray, c: np.ndarray) -> np.ndarray:
    """The kernel's evaluation, step by step in float32: y2 = y*y, Horner in y2, times y."""
    y = np.asarray(y, np.float32)
    y2 = (y * y).astype(np.float32)
    p = np.float32(c[-1])
    for k in range(len(c) - 2, -1, -1):
        p = (p * y2 + np.float32(c[k])).astype(np.float32)
    return (p * y).astype(np.float32)


def max_abs_error(c: np.ndarray, n: int = 2_000_001) -> float:
    y = np.linspace(-1.0, 1.0, n, dtype=np.float64).astype(np.float32)
    return float(np.max(np.abs(eval_f32(y, c).astype(np.float64) - np.tanh(y.astype(np.float64)))))


if __name__ == "__main__":
    c = fit()
    for k, v in enumerate(c):
        print(f"c{k} = {float(v)!r}f")
    print("max abs error on [-1, 1]:", max_abs_error(c))
