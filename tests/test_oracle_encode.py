"""Pins for the oracle's encoding (canonical embedding) and slot semantics."""
import numpy as np
import pytest

from oracle import ckks as C
import seeded_inputs as S


@pytest.mark.parametrize("log_n", [3, 6, 10])
def test_encode_fft_matches_definition(log_n):
    P = C.Params(log_n, 2, 1, 2)
    z = S.complex_slots(1, P.n_slots, -1, 1)
    scale = 2.0 ** 20
    a = C.encode_coeffs(z, scale, P)
    b = C.encode_coeffs_direct(z, scale, P)
    assert np.max(np.abs(a - b)) <= 1.0
    assert np.mean(a == b) > 0.99


@pytest.mark.parametrize("log_n", [3, 6, 10])
def test_decode_fft_matches_definition(log_n):
    P = C.Params(log_n, 2, 1, 2)
    m = np.random.default_rng(log_n).integers(-(1 << 30), 1 << 30, size=P.N).astype(np.float64)
    a = C.decode_coeffs(m, 2.0 ** 30, P)
    b = C.decode_coeffs_direct(m, 2.0 ** 30, P)
    assert np.max(np.abs(a - b)) < 1e-9 * max(1.0, np.max(np.abs(b)))


@pytest.mark.parametrize("log_n", [4, 12, 16])
def test_decode_encode_roundtrip(log_n):
    P = C.Params(log_n, 2, 1, 2)
    z = S.complex_slots(2, P.n_slots, -1, 1)
    assert np.max(np.abs(C.decode_coeffs(C.encode_coeffs(z, 2.0 ** 40, P), 2.0 ** 40, P) - z)) < 1e-9


def test_constant_slots_are_constant_polynomial():
    """Every slot equal to the real c <=> m(X) = c * scale (only the constant term)."""
    P = C.Params(8, 2, 1, 2)
    m = C.encode_coeffs(np.full(P.n_slots, 0.75 + 0j), 2.0 ** 30, P)
    assert m[0] == round(0.75 * 2 ** 30) and np.all(m[1:] == 0)


@pytest.mark.parametrize("step", [1, 2, 7, -1])
def test_galois_element_rotates_slots_left(step):
    """X -> X^(5^r) moves slot j + r to slot j (the rotation direction)."""
    P = C.Params(6, 2, 1, 2)
    z = S.complex_slots(3, P.n_slots, -1, 1)
    m = C.encode_coeffs(z, 2.0 ** 30, P).astype(np.int64)
    k = P.galois_elt(step)
    mk = np.zeros(P.N, dtype=np.int64)
    for i in range(P.N):
        e = i * k % (2 * P.N)
        if e < P.N:
            mk[e] += m[i]
        else:
            mk[e - P.N] -= m[i]
    out = C.decode_coeffs(mk.astype(np.float64), 2.0 ** 30, P)
    assert np.max(np.abs(out - np.roll(z, -step))) < 1e-6


def test_conjugation_element():
    P = C.Params(6, 2, 1, 2)
    z = S.complex_slots(4, P.n_slots, -1, 1)
    m = C.encode_coeffs(z, 2.0 ** 30, P).astype(np.int64)
    mk = np.zeros(P.N, dtype=np.int64)
    k = 2 * P.N - 1
    for i in range(P.N):
        e = i * k % (2 * P.N)
        if e < P.N:
            mk[e] += m[i]
        else:
            mk[e - P.N] -= m[i]
    out = C.decode_coeffs(mk.astype(np.float64), 2.0 ** 30, P)
    assert np.max(np.abs(out - np.conj(z))) < 1e-6


def test_encode_rns_decode_roundtrip():
    P = C.Params(12, 3, 1, 3)
    z = S.complex_slots(5, P.n_slots, -1, 1)
    pt = C.encode(z, 2.0 ** 40, 3, P)
    assert np.max(np.abs(C.decode(pt, 3, 2.0 ** 40, P) - z)) < 1e-9
