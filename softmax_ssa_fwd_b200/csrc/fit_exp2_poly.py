"""Derive the polynomial the kernel uses to evaluate part of its exp2 calls on
the FMA pipe instead of the MUFU unit.

Method (Cody-Waite style range reduction, then a minimax polynomial):
  x = n + f with n = round-to-nearest(x) and f in [-1/2, 1/2];
  2^x = 2^n * p(f), p a degree-3 polynomial minimising the maximum relative
  error of p(f) / 2^f over [-1/2, 1/2] (solved as a linear program on a dense
  grid); 2^n is applied by adding n to the float's exponent field.
Prints the coefficients (fp32) and the achieved relative error.
"""
import numpy as np
from scipy.optimize import linprog


def fit(deg=3, npts=4001):
    f = np.linspace(-0.5, 0.5, npts)
    y = np.exp2(f)
    V = np.stack([f ** i for i in range(deg + 1)], 1) / y[:, None]  # p(f)/2^f
    # minimise t subject to -t <= V c - 1 <= t
    nc = deg + 1
    c_obj = np.zeros(nc + 1)
    c_obj[-1] = 1.0
    A = np.block([[V, -np.ones((npts, 1))], [-V, -np.ones((npts, 1))]])
    b = np.concatenate([np.ones(npts), -np.ones(npts)])
    res = linprog(c_obj, A_ub=A, b_ub=b, bounds=[(None, None)] * nc + [(0, None)], method="highs")
    c = res.x[:nc].astype(np.float32)
    ff = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
    p = np.zeros_like(ff)
    for ci in c[::-1]:
        p = p * ff + ci
    err = np.max(np.abs(p.astype(np.float64) / np.exp2(ff.astype(np.float64)) - 1))
    return c, err


if __name__ == "__main__":
    c, err = fit()
    print("coefficients c0..c3 (fp32):", [float(x).hex() for x in c], [repr(float(x)) for x in c])
    print("max relative error:", err)
