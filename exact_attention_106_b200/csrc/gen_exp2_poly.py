"""Fit the polynomial behind the kernels' FMA-pipe exp2.

The forward evaluates part of its exponentials as 2^x = 2^n * p(f), with
n = floor(x) and f = x - n in [0, 1), so that they run on the FMA pipe instead
of the special-function unit.  p is the degree-3 polynomial that minimises the
maximum relative error |p(f) / 2^f - 1| on [0, 1] subject to p(0) = 1 and
p(1) = 2 (so the approximation is continuous across integers), found here as
a linear program on a dense grid (scipy.optimize.linprog), then rounded to
fp32.  Running this script prints the coefficients pasted into fwd.cuh and the
fp32 relative error of the whole evaluation.
"""
import numpy as np
from scipy.optimize import linprog

DEGREE = 3


def fit(degree: int = DEGREE, grid: int = 20001):
    f = np.linspace(0.0, 1.0, grid)
    t = np.exp2(f)
    # variables: c_0..c_deg, e ; minimise e
    V = np.vander(f, degree + 1, increasing=True) / t[:, None]  # p(f)/2^f
    ones = np.ones((grid, 1))
    A_ub = np.vstack([np.hstack([V, -ones]), np.hstack([-V, -ones])])
    b_ub = np.concatenate([np.ones(grid), -np.ones(grid)])
    A_eq = np.zeros((2, degree + 2))
    A_eq[0, 0] = 1.0                     # p(0) = 1
    A_eq[1, :degree + 1] = 1.0           # p(1) = 2
    b_eq = np.array([1.0, 2.0])
    c = np.zeros(degree + 2)
    c[-1] = 1.0
    res = linprog(c, A_ub=A_ub, b_ub=b_ub, A_eq=A_eq, b_eq=b_eq, bounds=[(None, None)] * (degree + 2),
                  method="highs")
    assert res.success, res.message
    return res.x[:degree + 1], res.x[-1]


def emulate_fp32(x, coeffs):
    """The kernel's arithmetic in float32: clamp, floor, Horner, exponent add."""
    x = np.maximum(np.asarray(x, np.float32), np.float32(-127.0))
    n = np.floor(x).astype(np.float32)
    f = (x - n).astype(np.float32)
    c = [np.float32(v) for v in coeffs]
    p = np.float32(c[-1])
    for ck in reversed(c[:-1]):
        p = (p * f + ck).astype(np.float32)
    bits = p.view(np.int32) + (n.astype(np.int32) << 23)
    return bits.view(np.float32)


if __name__ == "__main__":
    coeffs, err = fit()
    c32 = [float(np.float32(v)) for v in coeffs]
    x = np.linspace(-100.0, 8.0, 2_000_001, dtype=np.float64).astype(np.float32)
    y = emulate_fp32(x, c32).astype(np.float64)
    rel = np.max(np.abs(y / np.exp2(x.astype(np.float64)) - 1.0))
    print(f"minimax relative error (real arithmetic): {err:.3e}")
    print(f"fp32 evaluation, max relative error on [-100, 8]: {rel:.3e}")
    for i, v in enumerate(c32):
        print(f"  c{i} = {v!r}f  ({np.float32(v).view(np.uint32):#010x})")
