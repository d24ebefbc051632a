"""The softmax's polynomial exponential on the CPU: the constants in ptx.cuh are the fp32 output of
the committed fitting script (fit_exp2_poly.py), and the kernel's evaluation, emulated step by step
in fp32 (round to nearest by adding 1.5 * 2^23, cubic in the remainder, exponent-field add), stays
within the fit's relative error bound over the range the softmax uses."""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "query_union_paged_b200", "csrc")


def _kernel_coefficients():
    src = open(os.path.join(CSRC, "ptx.cuh")).read()
    m = re.search(r"kExp2C1 = ([0-9.e+-]+)f, kExp2C2 = ([0-9.e+-]+)f, kExp2C3 = ([0-9.e+-]+)f", src)
    assert m, "coefficients not found in ptx.cuh"
    return [np.float32(float(x)) for x in m.groups()]


def _fit_module():
    spec = importlib.util.spec_from_file_location("fit_exp2_poly", os.path.join(CSRC, "fit_exp2_poly.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _emulate(y, c1, c2, c3):
    """The kernel's steps in fp32 (exp2_poly2)."""
    y = np.maximum(y.astype(np.float32), np.float32(-127.0))
    magic = np.float32(12582912.0)
    t = (y + magic).astype(np.float32)
    n = (t - magic).astype(np.float32)
    f = (y - n).astype(np.float32)
    p = (f * c3 + c2).astype(np.float32)
    p = (p * f + c1).astype(np.float32)
    p = (p * f + np.float32(1.0)).astype(np.float32)
    bits = (p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_kernel_constants_are_the_fitted_ones():
    coef, err = _fit_module().fit()
    assert err < 1.05e-4
    assert [np.float32(c) for c in coef] == _kernel_coefficients()


def test_emulated_evaluation_meets_the_bound():
    c1, c2, c3 = _kernel_coefficients()
    y = np.linspace(-125.0, 16.0, 1_000_001, dtype=np.float32)
    got = _emulate(y, c1, c2, c3).astype(np.float64)
    rel = np.abs(got / np.exp2(y.astype(np.float64)) - 1.0)
    assert rel.max() <= 1.05e-4, rel.max()
    # the clamp: at and below -127 the result is exactly +0
    z = _emulate(np.array([-127.0, -130.0, -np.inf], np.float32), c1, c2, c3)
    assert np.all(z == 0.0)
