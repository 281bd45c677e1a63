"""Fit the polynomial behind the FMA-pipe base-2 exponential used by the attention kernel.

Method (Cody and Waite's argument reduction, then a minimax polynomial):
    2^x = 2^n * 2^f,   n = round-to-nearest(x),  f = x - n in [-1/2, 1/2],
    2^f ~ c0 + f*(c1 + f*(c2 + f*c3)),
with 2^n applied by adding n to the IEEE-754 exponent field.  The coefficients minimise the
maximum *relative* error on [-1/2, 1/2]; they are found here with Lawson's iteratively
re-weighted least-squares algorithm on a dense grid (no tabulated constants are used).

    python sequence_partition_attn_b200/csrc/fit_exp2_poly.py

prints the coefficients (as float32 hex and decimal) and the maximum relative error of the
float32 Horner evaluation, which the kernel's exponent-field trick leaves unchanged.
"""
import numpy as np


def fit(degree=3, n=20001, iters=400):
    f = np.linspace(-0.5, 0.5, n)
    y = np.exp2(f)
    A = np.vander(f, degree + 1, increasing=True) / y[:, None]   # relative error basis
    b = np.ones_like(f)
    w = np.full(n, 1.0 / n)
    c = None
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A * sw[:, None], b * sw, rcond=None)
        r = np.abs(A @ c - b)
        w = w * r
        w /= w.sum()
    return c


def horner_f32(c, f):
    c = c.astype(np.float32)
    f = f.astype(np.float32)
    p = c[-1]
    for k in range(len(c) - 2, -1, -1):
        p = (p * f + c[k]).astype(np.float32)
    return p


if __name__ == "__main__":
    c = fit().astype(np.float32)
    f = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
    err = np.max(np.abs(horner_f32(c, f).astype(np.float64) / np.exp2(f.astype(np.float64)) - 1))
    for k, v in enumerate(c):
        print(f"c{k} = {float(v)!r:>24}  ({np.float32(v).view(np.uint32):#010x})")
    print(f"max relative error (fp32 Horner) = {err:.3e}")
