"""Fits the polynomial the forward kernel uses for part of its exponentials.

    python block_sparse_paged_gbsa_b200/csrc/fit_exp2_poly.py

Method: the classical minimax (Chebyshev) approximation, solved as a linear
program on a dense grid: choose c1..c3 of p(f) = 1 + c1 f + c2 f^2 + c3 f^3
minimising max |p(f) - 2^f| / 2^f over f in [-1/2, 1/2].  The constant term is
pinned to 1 so that p(0) = 1 exactly: with the kernel's clamp of the
argument at -127, 2^-127 is then built as exactly +0.  The range reduction
that brings any x to f in [-1/2, 1/2] (x = n + f, n the nearest integer) is
the textbook one; 2^n is applied by adding n to the exponent field.

Prints the coefficients as float32 hex/decimal and the achieved relative
error; the values are pasted into gbsa_fwd.cu (kExp2C1..kExp2C3).
"""
import numpy as np
from scipy.optimize import linprog


def fit(degree=3, n=4001):
    f = np.linspace(-0.5, 0.5, n)
    target = np.exp2(f)
    # variables: c1..cd, t ; minimise t
    powers = np.stack([f ** k for k in range(1, degree + 1)], 1)
    w = 1.0 / target
    # (1 + P c - target) * w <= t  and  -(1 + P c - target) * w <= t
    A1 = np.hstack([powers * w[:, None], -np.ones((n, 1))])
    b1 = (target - 1.0) * w
    A2 = np.hstack([-powers * w[:, None], -np.ones((n, 1))])
    b2 = -(target - 1.0) * w
    res = linprog(np.r_[np.zeros(degree), 1.0], A_ub=np.vstack([A1, A2]), b_ub=np.r_[b1, b2],
                  bounds=[(None, None)] * degree + [(0, None)], method="highs")
    return res.x[:degree], res.x[degree]


def fp32_eval(c, f):
    c = [np.float32(x) for x in c]
    f = f.astype(np.float32)
    p = np.float32(c[2]) * f + np.float32(c[1])
    p = p.astype(np.float32) * f + np.float32(c[0])
    p = p.astype(np.float32) * f + np.float32(1.0)
    return p.astype(np.float32)


if __name__ == "__main__":
    c, err = fit()
    c32 = [np.float32(x) for x in c]
    f = np.linspace(-0.5, 0.5, 200001)
    rel = np.abs(fp32_eval(c32, f).astype(np.float64) - np.exp2(f)) / np.exp2(f)
    for k, x in enumerate(c32, 1):
        print(f"c{k} = {float(x)!r}  (0x{np.float32(x).view(np.uint32):08x})")
    print(f"minimax relative error {err:.3e}; with fp32 coefficients and Horner {rel.max():.3e}")
