"""Fits the polynomial of the software exp2 used by the attention kernel.

2^x is split as 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2]
(Cody and Waite's argument reduction); 2^f is approximated by a degree-4
polynomial 1 + c1 f + c2 f^2 + c3 f^3 + c4 f^4.  The constant term is held at
exactly 1 so that integer arguments give exact powers of two; c1..c4 minimise
the maximum relative error on a dense grid of [-1/2, 1/2], solved as the
linear program of discrete Chebyshev approximation

    minimise E  subject to  -E <= (p(f_i) - 2^f_i) / 2^f_i <= E  for all i.

The coefficients are rounded to fp32 and the fp32 Horner evaluation (one
rounding per fused multiply-add) is checked against float64 2^f.

    python pair_biased_attention_b200/csrc/fit_exp2_poly.py

prints the coefficients written into pba_ptx.cuh and the achieved maximum
relative error.
"""
import numpy as np
from scipy.optimize import linprog

DEG = 4
LO, HI = -0.5, 0.5


def fit(deg=DEG, npts=4001):
    f = np.linspace(LO, HI, npts)
    w = 1.0 / 2.0 ** f                      # relative-error weight
    V = np.stack([f ** j for j in range(1, deg + 1)], axis=1) * w[:, None]
    r = (2.0 ** f - 1.0) * w                # target of sum_j c_j f^j, weighted
    # variables: c1..c_deg, E ; minimise E
    cost = np.zeros(deg + 1)
    cost[-1] = 1.0
    A = np.vstack([np.hstack([V, -np.ones((npts, 1))]), np.hstack([-V, -np.ones((npts, 1))])])
    b = np.concatenate([r, -r])
    res = linprog(cost, A_ub=A, b_ub=b, bounds=[(None, None)] * deg + [(0, None)], method="highs")
    assert res.success, res.message
    return np.concatenate([[1.0], res.x[:deg]])


def fp32_horner(c32, f):
    """Horner evaluation with one fp32 rounding per fused multiply-add."""
    f = f.astype(np.float32)
    acc = np.float32(c32[-1])
    for cj in c32[-2::-1]:
        acc = (acc.astype(np.float64) * f.astype(np.float64) + np.float64(cj)).astype(np.float32)
    return acc


if __name__ == "__main__":
    c = fit()
    c32 = np.array(c, dtype=np.float32)
    f = np.linspace(LO, HI, 1000001)
    rel = np.abs(fp32_horner(c32, f).astype(np.float64) / 2.0 ** f - 1.0)
    for j, cj in enumerate(c32):
        print(f"c{j} = {float(cj):.9e}f  ({np.float32(cj).view(np.uint32):#010x})")
    print(f"max relative error of the fp32 evaluation on [-1/2, 1/2]: {rel.max():.3e}")
