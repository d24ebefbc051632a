"""Fit the cubic used by exp2_poly2 (ptx.cuh): p(f) = 1 + f (c1 + f (c2 + f c3)) ~ 2^f on
[-1/2, 1/2], minimising the maximum relative error |p(f) / 2^f - 1| as a linear program over a
dense grid, then reporting the error of the fp32-rounded coefficients evaluated in fp32 the
way the kernel does (Horner with fused multiply-adds).

    python query_union_paged_b200/csrc/fit_exp2_poly.py
"""
import numpy as np
from scipy.optimize import linprog


def fit(deg=3, n=4001):
    f = np.linspace(-0.5, 0.5, n)
    e = np.exp2(f)
    # variables: c1..c_deg, err ; minimise err s.t. |1 + sum c_k f^k - e| <= err * e
    A = np.stack([f ** k for k in range(1, deg + 1)], axis=1)
    ones = e[:, None]
    A_ub = np.vstack([np.hstack([A, -ones]), np.hstack([-A, -ones])])
    b_ub = np.concatenate([e - 1.0, 1.0 - e])
    c = np.zeros(deg + 1)
    c[-1] = 1.0
    res = linprog(c, A_ub=A_ub, b_ub=b_ub, bounds=[(None, None)] * (deg + 1), method="highs")
    assert res.success, res.message
    return res.x[:deg], res.x[deg]


def fp32_error(coef, n=200001):
    c = np.asarray(coef, np.float32)
    f = np.linspace(-0.5, 0.5, n).astype(np.float32)
    p = np.full_like(f, c[-1])
    for k in range(len(c) - 2, -1, -1):
        p = (p * f + c[k]).astype(np.float32)
    p = (p * f + np.float32(1.0)).astype(np.float32)
    return float(np.max(np.abs(p.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0)))


if __name__ == "__main__":
    coef, err = fit()
    print("c1..c3 =", ", ".join(f"{np.float32(c)!r}" for c in coef))
    print(f"LP max relative error {err:.3e}; fp32 evaluation {fp32_error(coef):.3e}")
