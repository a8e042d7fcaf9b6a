"""The prefill kernel's FMA-pipe exponential (csrc/exp2_poly.cuh).

2^x = 2^n * p(f) with n the integer nearest to x (ties to even), f = x - n
and p a cubic fitted by Lawson's algorithm to minimise the relative error on
[-1/2, 1/2]. Pins, without a GPU:

* the fit script reproduces the four float32 constants compiled into the
  kernel, bit for bit;
* a float32 model of the kernel's instruction sequence (range reduction by
  the 1.5 * 2^23 trick, three FMAs, the integer exponent add) stays within the
  fit's relative-error bound against exact 2^x over [-125, 127], on a dense
  grid, on every half-integer (the ties of the range reduction, f = +-1/2) and
  on every integer (f = 0, where p(0) = C0);
* the clamp: every input at or below -126 (-inf included) gives a finite,
  non-negative result below 2^-125;
* the exponent add equals ldexp wherever the result is a normal number.

On a B200 the device function itself, run through the library's diagnostic
entry point, must agree with that model (bit for bit almost everywhere, one
ulp at most), with exact 2^x within the same bound, and with the MUFU
ex2.approx instruction within the bound plus that instruction's own error.
"""
import os
import re

import numpy as np
import pytest

from attention_tiled_exact_b200 import exp2_poly_fit

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "attention_tiled_exact_b200", "csrc", "exp2_poly.cuh")

# The fit's maximum relative error is 7.48e-5; the float32 evaluation adds a
# few roundings of 2^-24 relative each.
REL_BOUND = 7.5e-5


def _kernel_coefficients():
    src = open(HEADER).read()
    vals = {}
    for i in range(4):
        m = re.search(rf"constexpr float EXP2_C{i} = ([0-9.eE+-]+)f;", src)
        assert m, f"EXP2_C{i} not found in {HEADER}"
        vals[i] = np.float32(float(m.group(1)))
    return np.array([vals[i] for i in range(4)], dtype=np.float32)


def _fma32(a, b, c):
    """float32 fused multiply-add: the float32 product is exact in float64."""
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def exp2_poly_model(x, coeffs):
    """The kernel's instruction sequence on float32 inputs, in NumPy."""
    c0, c1, c2, c3 = (np.float32(c) for c in coeffs)
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-126.0))
    t = (x + np.float32(12582912.0)).astype(np.float32)          # 1.5 * 2^23: n in the low mantissa bits
    n = (t - np.float32(12582912.0)).astype(np.float32)
    f = _fma32(n, np.full_like(n, -1.0), x)
    p = _fma32(np.full_like(f, c3), f, np.full_like(f, c2))
    p = _fma32(p, f, np.full_like(f, c1))
    p = _fma32(p, f, np.full_like(f, c0))
    bits = p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))  # n added to the exponent field (mod 2^32)
    return bits.astype(np.uint32).view(np.float32), n, p


def _rel_err(y, x):
    exact = np.exp2(np.asarray(x, dtype=np.float64))
    return np.abs(y.astype(np.float64) / exact - 1.0)


def test_fit_reproduces_the_kernel_constants():
    fitted = exp2_poly_fit.fit()
    kernel = _kernel_coefficients()
    assert np.array_equal(fitted.view(np.uint32), kernel.view(np.uint32)), (fitted, kernel)
    err = exp2_poly_fit.max_relative_error(fitted)
    assert 7.4e-5 < err < 7.49e-5, err


def test_fit_is_equioscillating():
    """A minimax cubic's error alternates in sign at 5 points with equal size
    (Chebyshev's alternation theorem): check that the fitted error reaches
    its maximum, with alternating signs, near both ends and three inner points."""
    c = exp2_poly_fit.fit().astype(np.float64)
    f = np.linspace(-0.5, 0.5, 200001)
    e = ((c[3] * f + c[2]) * f + c[1]) * f + c[0]
    e = e / np.exp2(f) - 1.0
    emax = np.abs(e).max()
    # local extrema of e at the ends and where its slope changes sign
    idx = [0] + [i for i in range(1, f.size - 1) if (e[i] - e[i - 1]) * (e[i + 1] - e[i]) <= 0] + [f.size - 1]
    peaks = [e[i] for i in idx if abs(e[i]) > 0.98 * emax]
    signs = np.sign(peaks)
    assert len(peaks) >= 5
    assert all(signs[i] != signs[i + 1] for i in range(len(signs) - 1))


def test_model_within_bound_on_a_dense_grid():
    c = _kernel_coefficients()
    x = np.linspace(-125.0, 127.0, 2_000_001, dtype=np.float64).astype(np.float32)
    y, _, _ = exp2_poly_model(x, c)
    assert np.isfinite(y).all()
    err = _rel_err(y, x)
    assert err.max() <= REL_BOUND, (err.max(), x[err.argmax()])


def test_model_at_half_integers_and_integers():
    """Half-integers are the ties of the range reduction: n is the even
    neighbour, so f = +1/2 or -1/2, the two ends of the fitted interval.
    At integers f = 0 and the result is exactly C0 * 2^n."""
    c = _kernel_coefficients()
    k = np.arange(-125, 127, dtype=np.float32)
    xh = (k + np.float32(0.5)).astype(np.float32)
    y, n, _ = exp2_poly_model(xh, c)
    assert np.all(n.astype(np.int64) % 2 == 0), "ties must round to the even integer"
    assert set(np.unique(xh - n)) <= {np.float32(0.5), np.float32(-0.5)}
    assert _rel_err(y, xh).max() <= REL_BOUND
    yi, ni, _ = exp2_poly_model(k, c)
    assert np.array_equal(ni, k)
    assert np.array_equal(yi.astype(np.float64), np.ldexp(np.float64(c[0]), k.astype(np.int64)))


def test_clamp_at_minus_126():
    c = _kernel_coefficients()
    x = np.array([-126.0, -126.25, -127.0, -150.0, -1e30, -np.inf, -125.9999], dtype=np.float32)
    y, _, _ = exp2_poly_model(x, c)
    assert np.isfinite(y).all() and (y >= 0).all()
    assert (y.astype(np.float64) < 2.0 ** -125).all(), y
    # everything at or below the clamp gives one and the same value
    assert len(set(y[:6].view(np.uint32).tolist())) == 1


def test_exponent_add_matches_ldexp_for_normal_results():
    c = _kernel_coefficients()
    rng = np.random.default_rng(0)
    x = rng.uniform(-125.0, 127.0, 200_000).astype(np.float32)
    y, n, p = exp2_poly_model(x, c)
    ref = np.ldexp(p.astype(np.float64), n.astype(np.int64)).astype(np.float32)
    assert np.array_equal(y.view(np.uint32), ref.view(np.uint32))


def test_model_catches_a_planted_coefficient_error():
    """A coefficient off by 1e-4 (or a dropped cubic term) breaks the bound."""
    c = _kernel_coefficients()
    x = np.linspace(-3.0, 3.0, 100_001, dtype=np.float32)
    for bad in (c + np.array([0, 0, 1e-4, 0], dtype=np.float32), c * np.array([1, 1, 1, 0], dtype=np.float32)):
        y, _, _ = exp2_poly_model(x, bad)
        assert _rel_err(y, x).max() > REL_BOUND


@pytest.mark.gpu
def test_device_polynomial_matches_model_exp2_and_mufu(lib):
    import torch
    c = _kernel_coefficients()
    rng = np.random.default_rng(1)
    k = np.arange(-125, 127, dtype=np.float32)
    x = np.concatenate([
        np.linspace(-125.0, 127.0, 1_000_001, dtype=np.float64).astype(np.float32),
        rng.uniform(-20.0, 8.0, 1_000_000).astype(np.float32),  # the range the softmax uses
        k, k + np.float32(0.5),
        np.array([-126.0, -127.0, -200.0, -np.inf], dtype=np.float32),
    ])
    y_poly, y_mufu = lib.selftest_exp2(torch.from_numpy(x).cuda())
    torch.cuda.synchronize()
    yp, ym = y_poly.cpu().numpy(), y_mufu.cpu().numpy()
    model, _, _ = exp2_poly_model(x, c)
    ulps = np.abs(yp.view(np.int32).astype(np.int64) - model.view(np.int32).astype(np.int64))
    assert ulps.max() <= 1 and (ulps == 0).mean() > 0.999, (ulps.max(), (ulps == 0).mean())
    main = x >= -125.0
    assert _rel_err(yp[main], x[main]).max() <= REL_BOUND
    assert (yp[~main] >= 0).all() and (yp[~main].astype(np.float64) < 2.0 ** -125).all()
    # against the hardware instruction: within the bound plus ex2.approx's own error (2^-22 relative)
    rel = np.abs(yp[main].astype(np.float64) / ym[main].astype(np.float64) - 1.0)
    assert rel.max() <= REL_BOUND + 2.0 ** -21, rel.max()
