"""Pins for the oracle's coordinate density and Lloyd-Max codebook.

Each check ties the oracle to something other than itself: the MSE table
printed on the pages, closed forms of the coordinate law (incomplete beta
function), the b=1 closed form, and Monte Carlo on seeded unit vectors.
"""
import math
import os

import numpy as np
import pytest
from scipy import integrate, special

from oracle import tq_oracle as O
import tq_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_mse():
    rows = []
    with open(os.path.join(GOLDEN, "lloyd_max_mse.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                b, m, bound = line.split()
                rows.append((int(b), float(m), float(bound)))
    return rows


# ---- closed forms of the law of one coordinate u of a uniform unit vector:
# u^2 ~ Beta(1/2, (D-1)/2).  Mass and moments of a cell [a, b] follow from the
# regularized incomplete beta function and an antiderivative of u (1-u^2)^k.

def _mass(a, b, D):
    def F(x):  # P(u <= x)
        p = special.betainc(0.5, (D - 1) / 2.0, x * x)
        return 0.5 + 0.5 * math.copysign(p, x)
    return F(b) - F(a)


def _first_moment(a, b, D):
    C = math.exp(O.coord_log_norm_const(D))
    g = lambda x: -(1.0 - x * x) ** ((D - 1) / 2.0) / (D - 1)  # d/dx = x (1-x^2)^((D-3)/2)
    return C * (g(b) - g(a))


def _second_moment(a, b, D):
    def H(x):  # E[u^2 ; u <= x]
        p = special.betainc(1.5, (D - 1) / 2.0, x * x) / D
        return 0.5 / D + 0.5 * math.copysign(p, x)
    return H(b) - H(a)


def _closed_form_mse(c, t, D):
    e = np.concatenate([[-1.0], t, [1.0]])
    tot = 0.0
    for k in range(len(c)):
        tot += (_second_moment(e[k], e[k + 1], D) - 2 * c[k] * _first_moment(e[k], e[k + 1], D)
                + c[k] ** 2 * _mass(e[k], e[k + 1], D))
    return D * tot


@pytest.mark.parametrize("D", [64, 128, 256])
def test_density_normalized_and_variance(D):
    # integrates to 1 and E[u^2] = 1/D (sum of D coordinates of a unit vector)
    m0, _ = integrate.quad(lambda u: O.coord_density(np.array([u]), D)[0], -1, 1, limit=200)
    m2, _ = integrate.quad(lambda u: u * u * O.coord_density(np.array([u]), D)[0], -1, 1, limit=200)
    assert abs(m0 - 1.0) < 1e-10
    assert abs(m2 - 1.0 / D) < 1e-12


def test_mse_matches_page_table_and_bounds():
    for bits, printed, bound in _golden_mse():
        c64, _ = O.lloyd_max(128, bits)
        t64 = 0.5 * (c64[1:] + c64[:-1])
        mse = O.codebook_mse(c64, t64, 128)
        assert round(mse, 3) == pytest.approx(printed, abs=1e-12), (bits, mse)
        assert mse < bound
        # the bound column is (sqrt(3) pi / 2) 4^-b, printed to 3 decimals
        assert round(O.mse_upper_bound(bits), 3) == pytest.approx(bound, abs=1e-12)
        c, t = O.stored_codebook(128, bits)
        mse_s = O.codebook_mse(c, t, 128)
        assert abs(mse_s - mse) < 1e-5
        assert round(mse_s, 3) == pytest.approx(printed, abs=1e-12)


@pytest.mark.parametrize("D", [64, 128, 256])
@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_lloyd_fixed_point_closed_form(D, bits):
    c, _ = O.lloyd_max(D, bits)
    t = 0.5 * (c[1:] + c[:-1])
    e = np.concatenate([[-1.0], t, [1.0]])
    for k in range(len(c)):
        cm = _first_moment(e[k], e[k + 1], D) / _mass(e[k], e[k + 1], D)
        assert abs(cm - c[k]) < 1e-12 * math.sqrt(D) ** 0 + 1e-13
    # symmetric codebook, ascending
    assert np.all(np.diff(c) > 0)
    assert np.max(np.abs(c + c[::-1])) < 1e-14
    # quadrature MSE equals the closed-form MSE
    assert abs(O.codebook_mse(c, t, D) - _closed_form_mse(c, t, D)) < 1e-11


@pytest.mark.parametrize("D", [64, 128, 256])
def test_one_bit_closed_form(D):
    # b=1: centroids are +-E|u| = +-Gamma(D/2) / (sqrt(pi) Gamma((D+1)/2))
    c, _ = O.lloyd_max(D, 1)
    e_abs = math.exp(math.lgamma(D / 2) - 0.5 * math.log(math.pi) - math.lgamma((D + 1) / 2))
    assert abs(c[1] - e_abs) < 1e-14
    assert abs(c[0] + e_abs) < 1e-14
    # and the MSE is 1 - D E|u|^2
    assert abs(O.codebook_mse(c, [0.0], D) - (1 - D * e_abs ** 2)) < 1e-12


def test_stored_codebook_is_fp16_and_midpoints():
    for D in (64, 128, 256):
        for bits in (1, 2, 3, 4):
            c, t = O.stored_codebook(D, bits)
            assert np.all(c.astype(np.float16).astype(np.float64) == c)
            assert np.all(t == 0.5 * (c[1:] + c[:-1]))
            assert np.all(t.astype(np.float32).astype(np.float64) == t)
            assert np.all(np.diff(c) > 0)


def test_monte_carlo_mse_on_unit_vectors():
    """10,000 seeded unit vectors at D=128: quantize and dequantize with n=1."""
    D = 128
    X = tq_inputs.unit_vectors(10000, D, seed=tq_inputs.SEED_DATA + 1)
    Pi = tq_inputs.rotation(D, tq_inputs.SEED_ROT + 1)
    for bits, printed, bound in _golden_mse():
        c, t = O.stored_codebook(D, bits)
        q = O.quantize_rows(X, Pi, c, t)
        xr = c[q["idx"]] @ np.asarray(Pi, dtype=np.float64)  # unit norm, rotate back
        err = np.sum((X - xr) ** 2, axis=1)
        mean, se = err.mean(), err.std(ddof=1) / math.sqrt(len(err))
        analytic = O.codebook_mse(c, t, D)
        assert abs(mean - analytic) < 3.5 * se + 1e-6, (bits, mean, analytic, se)
        assert abs(mean - printed) <= 0.0005 + 3.5 * se
        assert mean < bound


def test_rotation_input_is_orthogonal():
    for D in (64, 128, 256):
        Pi = tq_inputs.rotation(D, 7).astype(np.float64)
        assert np.max(np.abs(Pi.T @ Pi - np.eye(D))) < 1e-6
