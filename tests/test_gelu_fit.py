"""GELU coefficients for the degree-15 engine, fitted by input distribution:
the fit against GELU's definition and identities, least-squares optimality
under the input density, and an encrypted evaluation through the oracle's
Paterson-Stockmeyer schedule (CPU)."""
import math

import numpy as np

from homomorphic_encrypted_transformer_b200 import gelu as G
from oracle import ckks as C
import seeded_inputs as S


def test_gelu_definition_and_identities():
    x = np.linspace(-5, 5, 101)
    g = G.gelu(x)
    assert G.gelu(0.0) == 0.0
    assert np.allclose(g - G.gelu(-x), x, atol=1e-14)  # x Phi(x) + x Phi(-x) = x
    assert abs(G.gelu(1.0) - 0.5 * (1 + math.erf(1 / math.sqrt(2)))) < 1e-15


def test_input_density_puts_the_stated_share_below_zero():
    m = G.input_mean()
    assert abs(0.5 * (1 + math.erf((0 - m) / math.sqrt(2))) - G.NEG_SHARE) < 1e-12


def test_weighted_fit_minimises_the_expected_error():
    """Weighted least squares is optimal for the weighted objective: lower
    expected squared error than the uniform fit of the same degree, and than
    small perturbations of its own coefficients."""
    cw, cu = G.fit(), G.fit(weighted=False)
    ew = G.expected_sq_error(cw)
    assert ew < G.expected_sq_error(cu)
    rng = np.random.default_rng(0)
    for _ in range(5):
        d = np.zeros(16)
        d[: G.DEGREE + 1] = rng.normal(0, 1e-4, G.DEGREE + 1)
        assert ew <= G.expected_sq_error(cw + d)
    assert np.all(cw[G.DEGREE + 1:] == 0) and np.max(np.abs(cw)) < 2  # engine constants stay below 2^63


def test_fit_is_close_where_the_inputs_are():
    x = np.linspace(-3, 1, 401)  # about 95% of the input mass
    p = np.polynomial.polynomial.polyval(x, G.fit())
    assert np.max(np.abs(p - G.gelu(x))) < 0.01


def test_encrypted_gelu_by_the_degree15_schedule():
    """The fitted coefficients through the oracle's Paterson-Stockmeyer
    evaluation (N = 2^12, 8 limbs): within 1e-6 of the plain polynomial on
    the decrypted input, and within the fit error of GELU on the slots."""
    P = C.Params(12, 8, 3, 3)
    seed = 33
    z = S.normal_slots(seed, P.n_slots, G.input_mean(), 1.0, G.LO, G.HI)
    coeffs = G.fit()
    s = S.secret(seed, P.N)
    pa, pe = S.public_key_draws(seed, P.q, P.N)
    pk = C.public_key(s, pa, pe, P)
    v, e0, e1 = S.encryption_draws(seed, 0, P.N)
    ct = C.make_ct(C.encrypt(pk, C.encode(z, 2.0 ** 40, 8, P), v, e0, e1, 8, P), 8, 2.0 ** 40)
    a, e = S.key_draws(seed, 2, P.mods, P.N, P.dnum)
    out = C.ps_eval_deg15(ct, coeffs, C.relin_key(s, a, e, P), P)
    got = C.decrypt_decode(out, s, P).real
    x_dec = C.decrypt_decode(ct, s, P)
    assert np.max(np.abs(got - C.ps_eval_plain(x_dec, coeffs).real)) < 1e-6
    fit_err = np.abs(np.polynomial.polynomial.polyval(z.real, coeffs) - G.gelu(z.real))
    assert np.all(np.abs(got - G.gelu(z.real)) <= fit_err + 1e-5)
