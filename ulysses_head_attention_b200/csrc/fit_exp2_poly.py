"""Fit the polynomial the kernels use for 2^f on f in [-1/2, 1/2].

Method: exponent/fraction range reduction (2^x = 2^n * 2^f, n = round(x)),
then a polynomial p(f) ~ 2^f whose maximum *relative* error on [-1/2, 1/2]
is minimised by iteratively reweighted least squares (Lawson's algorithm,
which converges to the minimax solution).  Prints the coefficients
(c0 + c1 f + c2 f^2 + c3 f^3) in float32 and the achieved max relative
error evaluated in float32 Horner arithmetic.

    python ulysses_head_attention_b200/csrc/fit_exp2_poly.py [degree]
"""
import sys

import numpy as np


def fit(degree: int, iters: int = 200):
    f = np.cos(np.linspace(0, np.pi, 4001))[::-1] * 0.5        # Chebyshev-spaced points on [-1/2, 1/2]
    target = np.exp2(f)
    V = np.vander(f, degree + 1, increasing=True) / target[:, None]   # relative-error system
    w = np.ones_like(f) / len(f)
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(V * sw[:, None], sw, rcond=None)
        err = np.abs(V @ c - 1.0)
        w = w * err
        w /= w.sum()
    return c


def horner_f32(c, f):
    c = [np.float32(x) for x in c]
    acc = np.full_like(f, c[-1], dtype=np.float32)
    for ck in reversed(c[:-1]):
        acc = (acc * f + ck).astype(np.float32)
    return acc


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c = fit(deg)
    f = np.linspace(-0.5, 0.5, 2_000_001, dtype=np.float32)
    rel = np.abs(horner_f32(c, f).astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0)
    print("coefficients (float32):", ", ".join(f"{np.float32(x)!r}" for x in c))
    print("hex:", ", ".join(hex(np.float32(x).view(np.uint32)) for x in c))
    print(f"max relative error (float32 Horner): {rel.max():.3e}")
