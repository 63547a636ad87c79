"""The device GELU takes erf from Abramowitz & Stegun, Handbook of
Mathematical Functions, formula 7.1.26: erf(x) = 1 - t (a1 + t (a2 + t (a3 +
t (a4 + t a5)))) exp(-x^2), t = 1 / (1 + p x), x >= 0, |error| <= 1.5e-7. This
pins the formula and its coefficients against math.erf (fp64 evaluation, so
the published bound applies); the GPU GEMM tests compare the GELU and GELU'
epilogues that use it with the oracle's exact erf."""
import math

import numpy as np

P = 0.3275911
A = (0.254829592, -0.284496736, 1.421413741, -1.453152027, 1.061405429)


def erf_as(x):
    ax = abs(x)
    t = 1.0 / (1.0 + P * ax)
    poly = t * (A[0] + t * (A[1] + t * (A[2] + t * (A[3] + t * A[4]))))
    return math.copysign(1.0 - poly * math.exp(-ax * ax), x)


def test_erf_as_within_published_bound():
    xs = np.concatenate([np.linspace(-6, 6, 20001), [0.0, 1e-6, -1e-6, 10.0, -10.0]])
    err = max(abs(erf_as(float(x)) - math.erf(float(x))) for x in xs)
    assert err <= 1.5e-7, err


def test_gelu_and_derivative_from_erf_as():
    # GELU(z) = z (1 + erf(z / sqrt 2)) / 2 and GELU'(z) = Phi(z) + z phi(z), with the shared exponential
    for z in np.linspace(-8, 8, 4001):
        x = z / math.sqrt(2.0)
        e = math.exp(-x * x)
        g = 0.5 * z * (1.0 + erf_as(x))
        gp = 0.5 * (1.0 + erf_as(x)) + z * e / math.sqrt(2.0 * math.pi)
        assert abs(g - 0.5 * z * (1.0 + math.erf(x))) <= 1.5e-7 * abs(z) * 0.5 + 1e-15
        gp_ref = 0.5 * (1.0 + math.erf(x)) + z * math.exp(-0.5 * z * z) / math.sqrt(2.0 * math.pi)
        assert abs(gp - gp_ref) <= 1e-7
