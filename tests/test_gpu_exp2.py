"""The softmax's polynomial 2^x (Cody-Waite reduction + a cubic fitted by
query_union_paged_b200/csrc/fit_exp2_poly.py), called through the C ABI's test
hook and checked against the exact exponential: relative error within the fit's
bound on the range the kernel uses, exact zeros at and below the clamp."""
import math

import numpy as np
import pytest

import query_union_paged_b200 as qup

pytestmark = pytest.mark.gpu

REL_BOUND = 1.05e-4  # the fitted cubic's max relative error in fp32 is 1.014e-4


def test_poly_exp2_relative_error_on_the_softmax_range():
    import torch
    x = torch.linspace(-125.0, 16.0, 2_000_001, dtype=torch.float32, device="cuda")
    # plus every fp32 in a few unit intervals (the reduction's ties sit at half-integers)
    fine = np.concatenate([np.arange(k, k + 1, 2.0 ** -16, dtype=np.float32) for k in (-3, -1, 0, 7)])
    x = torch.cat([x, torch.from_numpy(fine).cuda()])
    y = qup.exp2_poly(x)
    torch.cuda.synchronize()
    exact = torch.exp2(x.double())
    rel = ((y.double() - exact).abs() / exact).max().item()
    assert rel <= REL_BOUND, rel


def test_poly_exp2_is_zero_at_the_clamp_and_for_masked_scores():
    import torch
    x = torch.tensor([-127.0, -127.4, -200.0, -1e30, -math.inf, float("nan")], device="cuda")
    y = qup.exp2_poly(x)
    torch.cuda.synchronize()
    assert torch.equal(y.cpu(), torch.zeros(6))
    # just above the clamp the result is tiny and non-negative (subnormal range)
    z = qup.exp2_poly(torch.tensor([-126.9, -126.5, -126.0], device="cuda")).cpu()
    assert torch.all(z >= 0) and torch.all(z < 2.0 ** -125)


def test_poly_exp2_odd_length_and_empty():
    import torch
    x = torch.tensor([0.0, 1.0, -1.0, 0.5, 3.25], device="cuda")
    y = qup.exp2_poly(x).cpu().double()
    assert torch.allclose(y, torch.exp2(x.cpu().double()), rtol=REL_BOUND, atol=0)
    qup.exp2_poly(torch.empty(0, device="cuda"))
