"""Coefficients of the polynomial 2^f ~ 1 + c1 f + c2 f^2 + c3 f^3 on [-1/2, 1/2].

The softmax kernels evaluate part of their exponentials without the SFU:
x = n + f with n = round(x) (the classic 1.5 * 2^23 rounding constant) and
2^x = 2^n * p(f), the 2^n factor added into the exponent field.  This script
finds p by minimax fit of the relative error, posed as a linear program over
a dense grid, with the constant term fixed at exactly 1 so that p(0) = 1 and a
clamped input of -127 yields the bit pattern of +0.0.  It prints the float32
coefficients and the relative error of the float32 evaluation (Horner form,
each step rounded to float32), the figure the kernels' accuracy test checks.

Run: python exp2_poly_fit.py
"""
import numpy as np
from scipy.optimize import linprog


def fit(degree=3, n=20001):
    f = np.linspace(-0.5, 0.5, n)
    w = np.exp2(-f)  # relative error = (1 + sum c_k f^k) * 2^-f - 1
    k = np.arange(1, degree + 1)
    A = (f[:, None] ** k[None, :]) * w[:, None]  # n x degree
    b = 1.0 - w
    # minimise t subject to |A c - b| <= t
    A_ub = np.block([[A, -np.ones((n, 1))], [-A, -np.ones((n, 1))]])
    b_ub = np.concatenate([b, -b])
    cost = np.zeros(degree + 1)
    cost[-1] = 1.0
    res = linprog(cost, A_ub=A_ub, b_ub=b_ub, bounds=[(None, None)] * (degree + 1), method="highs")
    assert res.success, res.message
    return res.x[:degree], res.x[-1]


def eval_f32(c, f):
    f = f.astype(np.float32)
    p = np.float32(c[-1])
    for ck in list(c[:-1])[::-1]:
        p = (p * f + np.float32(ck)).astype(np.float32)
    return (p * f + np.float32(1.0)).astype(np.float32)


if __name__ == "__main__":
    c, t = fit()
    c32 = [np.float32(x) for x in c]
    g = np.linspace(-0.5, 0.5, 2000001)
    rel = eval_f32(c32, g).astype(np.float64) / np.exp2(g) - 1.0
    print("minimax relative error (exact arithmetic): %.3e" % t)
    print("relative error of the float32 evaluation: %.3e" % np.abs(rel).max())
    for i, x in enumerate(c32, start=1):
        print("c%d = %.9ef  (0x%08x)" % (i, float(x), int(np.float32(x).view(np.uint32))))
