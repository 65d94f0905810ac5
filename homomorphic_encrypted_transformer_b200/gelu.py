"""GELU coefficients for the degree-15 polynomial engine (he_poly_eval_ps15),
fitted with the input distribution in mind.

The Nimbus page (the two-party Transformer inference summary among the AEGIS
pages) observes that activation inputs are far from uniform: about 85% of
GELU's inputs are negative.  A polynomial fitted to weigh each input by how
often it occurs reaches a lower expected error, for the same degree, than one
fitted uniformly over the interval.  The page gives no density or degree.
This module takes the following reading:
  - inputs ~ N(mean, 1) with mean = -z_0.85 (so that P(x < 0) = 0.85),
    truncated to [-4, 4];
  - a weighted least-squares fit of degree 8 in the monomial basis, weights
    = that density on a uniform grid of the interval;
  - the engine's 16 coefficients are the fit's, then zeros.
The engine's constants need |c_k| < 2 (they are c_k T q / S < 2^63 at
T = 2^62); the fit's coefficients are far below that.
Host arithmetic only (numpy); the encrypted evaluation is he_poly_eval_ps15.
"""
import math

import numpy as np

NEG_SHARE = 0.85
LO, HI = -4.0, 4.0
DEGREE = 8


def gelu(x):
    """x Phi(x) with the standard normal CDF Phi (the exact GELU)."""
    x = np.asarray(x, dtype=np.float64)
    return 0.5 * x * (1.0 + np.vectorize(math.erf)(x / math.sqrt(2.0)))


def _normal_quantile(p):
    """Phi^-1(p) by bisection on math.erf (p in (0, 1))."""
    lo, hi = -10.0, 10.0
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        if 0.5 * (1.0 + math.erf(mid / math.sqrt(2.0))) < p:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def input_mean(neg_share=NEG_SHARE):
    """Mean of a unit-variance normal with P(x < 0) = neg_share."""
    return -_normal_quantile(neg_share)


def input_density(x, neg_share=NEG_SHARE):
    """Unnormalised N(input_mean, 1) density."""
    m = input_mean(neg_share)
    return np.exp(-0.5 * (np.asarray(x, dtype=np.float64) - m) ** 2)


def fit(degree=DEGREE, lo=LO, hi=HI, weighted=True, neg_share=NEG_SHARE, n_grid=4001):
    """Least-squares monomial coefficients c_0..c_degree of GELU on [lo, hi]:
    minimises sum_x w(x) (p(x) - GELU(x))^2 over a uniform grid, w the input
    density (weighted) or 1.  Returns 16 coefficients (zeros above degree)."""
    if not 0 <= degree <= 15:
        raise ValueError("degree must be in [0, 15]")
    x = np.linspace(lo, hi, n_grid)
    w = input_density(x, neg_share) if weighted else np.ones_like(x)
    V = np.vander(x, degree + 1, increasing=True)
    sw = np.sqrt(w)
    c, *_ = np.linalg.lstsq(V * sw[:, None], gelu(x) * sw, rcond=None)
    out = np.zeros(16)
    out[: degree + 1] = c
    return out


def expected_sq_error(coeffs, lo=LO, hi=HI, neg_share=NEG_SHARE, n_grid=4001):
    """E[(p(x) - GELU(x))^2] under the truncated input density (grid average)."""
    x = np.linspace(lo, hi, n_grid)
    w = input_density(x, neg_share)
    p = np.polynomial.polynomial.polyval(x, coeffs)
    return float(np.sum(w * (p - gelu(x)) ** 2) / np.sum(w))
