"""Where the FMA-pipe polynomials of csrc/common.cuh come from.

Two kernels' worth of transcendental work runs as polynomials on the FMA pipe
instead of the special-function unit:

* exp2_fma2: 2^f for f in [-0.5, 0.5] (after the Cody-Waite split x = n + f),
  a degree-5 polynomial in f;
* softplus_fast / softplus2: log1p(e) = 2 atanh(s) with s = e / (2 + e) in
  (0, 1/3], written as s * q(s^2) with q a degree-4 polynomial approximating
  2 atanh(s) / s on s^2 in [0, 1/9].

Both were fitted for the smallest maximum RELATIVE error on their interval and
their coefficients rounded to fp32. This test re-derives both fits with
Lawson's iteratively reweighted least squares (which converges to the minimax,
equioscillating polynomial), rounds the result to fp32, and checks that the
coefficients in the source agree with the fit to 1e-5 relative (a Taylor
polynomial or another fit of the same degree differs by far more in its top
coefficients) and that their error is the minimax error up to fp32 rounding.
"""

import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
COMMON = os.path.join(ROOT, "selective_state_space_causal_b200", "csrc", "common.cuh")


def lawson_minimax(x, f, degree, iters=500):
    """Coefficients (lowest degree first) of the polynomial p minimising
    max |p(x) / f(x) - 1| over the grid x."""
    V = np.vander(x, degree + 1, increasing=True) / f[:, None]
    target = np.ones_like(f)
    w = np.full(x.shape, 1.0 / x.size)
    c = None
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(V * sw[:, None], target * sw, rcond=None)
        err = np.abs(V @ c - target)
        w = w * err
        w /= w.sum()
    return c


def rel_err(coeffs, x, f):
    return float(np.max(np.abs(np.polyval(np.asarray(coeffs)[::-1], x) / f - 1.0)))


def body(name):
    text = open(COMMON).read()
    start = text.index(name + "(")
    end = text.index("\n}\n", start)
    return text[start:end]


def literals(src):
    """Floating literals of a function body; a packed pair pk2(c, c) counts once."""
    vals = [float(v) for v in re.findall(r"(-?\d+\.\d+(?:e-?\d+)?)f", src)]
    return [v for i, v in enumerate(vals) if i == 0 or v != vals[i - 1]]


def exp2_coeffs():
    vals = [v for v in literals(body("exp2_fma2"))
            if abs(v) not in (126.0, 12582912.0, 1.0)]
    return vals[::-1]  # the source evaluates Horner from the highest degree


def softplus_coeffs(name):
    vals = [v for v in literals(body(name)) if v not in (0.0, 2.0)]
    return vals[::-1]


EXP2_X = np.linspace(-0.5, 0.5, 20001)
EXP2_F = 2.0 ** EXP2_X
S2 = np.linspace(0.0, 1.0 / 9.0, 20001)
_S = np.sqrt(S2)
ATANH_F = np.where(_S > 0, 2.0 * np.arctanh(_S) / np.where(_S > 0, _S, 1.0), 2.0)


def _rel(a, b):
    return abs(float(a) - float(b)) / abs(float(a))


def test_exp2_polynomial_is_the_rounded_minimax_fit():
    src = exp2_coeffs()
    assert len(src) == 6
    fit = lawson_minimax(EXP2_X, EXP2_F, 5)
    minimax = rel_err(fit, EXP2_X, EXP2_F)
    assert minimax < 1e-7
    for i, (a, b) in enumerate(zip(fit, src)):
        assert _rel(a, b) <= 1e-5, f"degree {i}: fitted {a!r}, source {b!r}"
    # fp32 rounding of the constant term alone adds up to half an ulp of 1
    assert rel_err(src, EXP2_X, EXP2_F) <= minimax + 2.0 ** -23


@pytest.mark.parametrize("name", ["softplus_fast", "softplus2"])
def test_softplus_polynomial_is_the_rounded_minimax_fit(name):
    src = softplus_coeffs(name)
    assert len(src) == 5
    fit = lawson_minimax(S2, ATANH_F, 4)
    minimax = rel_err(fit, S2, ATANH_F)
    assert minimax < 1e-8
    for i, (a, b) in enumerate(zip(fit, src)):
        assert _rel(a, b) <= 1e-5, f"degree {i}: fitted {a!r}, source {b!r}"
    assert rel_err(src, S2, ATANH_F) <= 1.05 * minimax


def test_fit_catches_a_wrong_coefficient():
    """A planted change of one coefficient by 1e-4 relative fails the check."""
    src = exp2_coeffs()
    bad = list(src)
    bad[3] *= 1.0 + 1e-4
    fit = lawson_minimax(EXP2_X, EXP2_F, 5)
    minimax = rel_err(fit, EXP2_X, EXP2_F)
    assert _rel(fit[3], bad[3]) > 1e-5
    assert rel_err(bad, EXP2_X, EXP2_F) > minimax + 2.0 ** -23


def test_fit_tells_the_taylor_polynomial_apart():
    """The degree-5 Taylor polynomial of 2^f is a plausible wrong source: its
    top coefficients differ from the fit's by far more than the tolerance."""
    from math import factorial, log

    taylor = [log(2.0) ** k / factorial(k) for k in range(6)]
    fit = lawson_minimax(EXP2_X, EXP2_F, 5)
    assert max(_rel(a, b) for a, b in zip(fit, taylor)) > 1e-3
