"""The forward kernel's FMA-pipe exponential (exp2_poly_pair in csrc/fwd_sm100.cuh).

One exponential pair in four of the softmax's full tiles is computed on the FMA pipe
instead of the MUFU unit: x = n + f with n = round(x), |f| <= 1/2, 2^n through the
exponent field and 2^f by a cubic.  The cubic's coefficients come from the fit below
(weighted least squares for minimum relative error on [-1/2, 1/2], the weights reset
Lawson-style towards the points of largest error until the error equi-oscillates); the
CPU test refits them and compares with the constants compiled into the kernel, and checks
the fitted cubic's error.  The GPU test runs the kernel's own code (sa_diag_exp2_poly)
over [-125, 8.5] against 2^x in float64: relative error at most 8e-5 (the cubic's 7.6e-5
plus the float32 rounding of the evaluation); arguments below -125 give 2^-125.  (With
n = -126 the cubic's values just under 1 would meet the subnormal range through the
exponent-field addition, which is why the kernel clamps at -125.)"""
import os
import re

import numpy as np
import pytest
import torch

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "online_softmax_attention_sm_b200",
                   "csrc", "fwd_sm100.cuh")


def fit_exp2_cubic(iterations=60, points=20001):
    """Near-minimax relative-error cubic for 2^f on [-1/2, 1/2], lowest power first."""
    f = np.linspace(-0.5, 0.5, points)
    y = 2.0 ** f
    w = 1.0 / y
    for _ in range(iterations):
        A = np.vander(f, 4, increasing=True) * w[:, None]
        c, *_ = np.linalg.lstsq(A, y * w, rcond=None)
        rel = (np.polyval(c[::-1], f) - y) / y
        w = w * (1.0 + 50.0 * np.abs(rel) / np.abs(rel).max())
    return c


def kernel_coefficients():
    """The cubic's constants as compiled into exp2_poly_pair, lowest power first."""
    body = open(SRC).read()
    fn = body[body.index("void exp2_poly_pair"):]
    fn = fn[:fn.index("\n}\n")]
    consts = [float(x) for x in re.findall(r"pack_f2\(([0-9.]+)f, \1f\)", fn) if float(x) < 2.0]
    # the Horner chain names them highest power first: c3, c2, c1, c0
    assert len(consts) == 4, consts
    return np.array(consts[::-1])


def test_kernel_constants_are_the_fitted_cubic():
    c = fit_exp2_cubic().astype(np.float32).astype(np.float64)
    k = kernel_coefficients()
    np.testing.assert_allclose(k, c, rtol=2e-7, atol=0)


def test_fitted_cubic_relative_error():
    k = kernel_coefficients()
    f = np.linspace(-0.5, 0.5, 100001)
    rel = np.abs(np.polyval(k[::-1], f) / 2.0 ** f - 1.0)
    assert rel.max() <= 7.6e-5
    # equi-oscillation: the error reaches its maximum at both ends of the interval
    assert rel[0] > 0.9 * rel.max() and rel[-1] > 0.9 * rel.max()


@pytest.mark.gpu
def test_kernel_exp2_poly_against_exact():
    from online_softmax_attention_sm_b200 import sa_diag_exp2_poly, sa_check_status
    g = torch.Generator().manual_seed(3)
    grid = torch.linspace(-125.0, 8.5, 400001, dtype=torch.float32)
    rnd = torch.rand(200000, generator=g, dtype=torch.float32) * 133.5 - 125.0
    # integers, half-integers and their neighbours: where the rounding of n changes
    half = torch.arange(-125, 9, dtype=torch.float32) + 0.5
    ints = torch.arange(-125, 9, dtype=torch.float32)
    edges = torch.cat([half, ints] + [torch.nextafter(t, torch.full_like(t, d)) for t in (half, ints)
                                      for d in (1e9, -1e9)])
    x = torch.cat([grid, rnd, edges]).clamp(-125.0, 8.5).contiguous()
    y = sa_diag_exp2_poly(x.cuda())
    sa_check_status()
    exact = np.exp2(x.double().numpy())
    rel = np.abs(y.double().cpu().numpy() / exact - 1.0)
    worst = int(rel.argmax())
    assert rel.max() <= 8e-5, f"relative error {rel.max():.3e} at x = {float(x[worst])!r}"


@pytest.mark.gpu
def test_kernel_exp2_poly_clamps_below_the_normal_range():
    from online_softmax_attention_sm_b200 import sa_diag_exp2_poly, sa_check_status
    x = torch.tensor([-125.0, -125.5, -126.0, -127.0, -150.0, -1e4, -3.0e38], dtype=torch.float32)
    y = sa_diag_exp2_poly(x.cuda()).cpu().double().numpy()
    sa_check_status()
    # arguments below -125 give 2^-125 (within the cubic's error), a normal float: never a
    # subnormal or non-finite value
    assert np.all(np.isfinite(y)) and np.all(y >= 2.0 ** -126)
    np.testing.assert_allclose(y, 2.0 ** -125, rtol=8e-5)
