"""Pins of the oracle's seeded sampler (oracle/sampler.py): SplitMix64
against its published known-answer outputs, the Gaussian threshold table
against closed forms, and the three samplers against their distributions."""
import math
import os

import numpy as np
import pytest

from oracle import sampler as R

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_splitmix64_known_answer_from_state_zero():
    vals = []
    for line in open(os.path.join(GOLDEN, "splitmix64_state0.txt")):
        if line.startswith("outputs"):
            vals = [int(v, 16) for v in line.split()[1:]]
    assert len(vals) == 4
    assert [int(x) for x in R.outputs(0, 0, 4)] == vals
    # counter form: outputs 3..4 alone equal the tail
    assert [int(x) for x in R.outputs(0, 2, 2)] == vals[2:]


def _sequential(s0, n):
    """The generator stepped one state at a time (Python integers)."""
    out, s = [], s0
    for _ in range(n):
        s = (s + R.GAMMA) & R.M64
        z = s
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & R.M64
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & R.M64
        out.append(z ^ (z >> 31))
    return out


def test_rejection_keeps_stream_order():
    # q = 5 rejects the draws 5..7 of the top three bits; the kept values are
    # the stream's accepted draws in order
    seed, obj = 99, R.obj_id(R.TAG_KEY_A, 5, 1, 2)
    raw = _sequential(R.stream_start(seed, obj), 400)
    want = [x >> 61 for x in raw if (x >> 61) < 5][:200]
    assert R.uniform(seed, obj, 5, 200).tolist() == want


def test_cdt_symmetry_and_float_agreement():
    T = R.gaussian_cdt()
    assert len(T) == 38 and all(a < b for a, b in zip(T, T[1:]))
    # P(-k) = P(k): C_i + C_{37-i} = 1, so the floors add up to 2^64 - 1
    for i in range(38):
        assert T[i] + T[37 - i] == (1 << 64) - 1
    rho = np.exp(-np.arange(-19, 20, dtype=np.float64) ** 2 / (2 * 3.2 ** 2))
    cdf = np.cumsum(rho)[:38] / rho.sum()
    assert np.max(np.abs(np.array(T, dtype=np.float64) / 2.0 ** 64 - cdf)) < 2.0 ** -40


def test_cdt_variance_is_sigma_squared():
    # Poisson summation: a discrete Gaussian of sigma 3.2 has variance sigma^2
    # up to exp(-2 pi^2 sigma^2); the cut at +-19 removes mass below 1e-7
    T = [0] + R.gaussian_cdt() + [1 << 64]
    p = np.array([(T[i + 1] - T[i]) / 2.0 ** 64 for i in range(39)])
    k = np.arange(-19, 20)
    assert abs(p.sum() - 1) < 1e-15 and abs(p @ k) < 1e-12
    assert p @ k ** 2 == pytest.approx(3.2 ** 2, rel=1e-6)


def test_planted_wrong_sigma_fails_the_variance_pin(monkeypatch):
    # exp(-k^2 / sigma^2) instead of exp(-k^2 / (2 sigma^2)) halves the variance
    from decimal import Decimal, getcontext

    def wrong():
        getcontext().prec = 60
        rho = [(Decimal(-25 * k * k) / Decimal(256)).exp() for k in range(-19, 20)]
        tot, acc, out = sum(rho, Decimal(0)), Decimal(0), []
        for i in range(38):
            acc += rho[i]
            out.append(int((Decimal(2) ** 64 * acc / tot).to_integral_value(rounding="ROUND_FLOOR")))
        return out

    monkeypatch.setattr(R, "gaussian_cdt", wrong)
    with pytest.raises(AssertionError):
        test_cdt_variance_is_sigma_squared()


def test_samplers_ranges_and_frequencies():
    n = 1 << 16
    s = R.secret(7, n)
    assert set(np.unique(s).tolist()) <= {-1, 0, 1}
    freq = np.bincount(s.astype(np.int64) + 1, minlength=3) / n
    assert np.all(np.abs(freq - 1 / 3) < 0.01)
    q = 0xffffe80001  # a 40-bit prime of the chain
    a = R.uniform(7, R.obj_id(R.TAG_KEY_A, 3, 0, 0), q, n)
    assert a.max() < q
    h = np.bincount((a.astype(np.float64) / q * 16).astype(np.int64), minlength=16)
    chi2 = ((h - n / 16) ** 2 / (n / 16)).sum()
    assert chi2 < 40  # 15 degrees of freedom: p ~ 5e-4
    e = R.gaussian(7, R.obj_id(R.TAG_KEY_E, 3, 0, 0), n)
    assert np.abs(e).max() <= 19
    assert abs(e.mean()) < 0.05 and e.var() == pytest.approx(10.24, rel=0.03)


def test_streams_differ_by_object_and_seed():
    a = R.uniform(1, R.obj_id(R.TAG_KEY_A, 5, 0, 0), 97, 64)
    b = R.uniform(1, R.obj_id(R.TAG_KEY_A, 5, 0, 1), 97, 64)
    c = R.uniform(2, R.obj_id(R.TAG_KEY_A, 5, 0, 0), 97, 64)
    assert not np.array_equal(a, b) and not np.array_equal(a, c)
    assert math.isclose(np.mean(a), 48, abs_tol=15)


def _a_seeded_brute(seed, obj, q, n, tries):
    """Coefficient i from the generator stepped one state at a time: output
    number 1 + i + t n is raw[i + t n]."""
    sh = 64 - q.bit_length()
    raw = _sequential(R.stream_start(seed, obj), tries * n)
    out = []
    for i in range(n):
        for t in range(tries):
            x = raw[i + t * n] >> sh
            if x < q:
                out.append(x)
                break
        else:
            out.append(x - q)
    return out


def test_seeded_a_row_against_the_stepped_generator():
    # q = 5 keeps 5 of the 8 values of the top three bits: many coefficients
    # need a second or third try
    seed, obj = 0xA5EED, R.obj_id(R.TAG_KEY_A_SEEDED, 7, 2, 3)
    want = _a_seeded_brute(seed, obj, 5, 24, R.A_SEEDED_TRIES)
    assert R.a_seeded_row(seed, obj, 5, 24).tolist() == want
    assert max(want) < 5


def test_seeded_a_row_fallback_after_the_last_try():
    # two tries only: about 14% of the coefficients reject both and take the
    # last draw minus q
    seed, obj = 11, R.obj_id(R.TAG_KEY_A_SEEDED, 3, 0, 1)
    sh = 61
    raw = _sequential(R.stream_start(seed, obj), 2 * 64)
    fell = [i for i in range(64) if (raw[i] >> sh) >= 5 and (raw[i + 64] >> sh) >= 5]
    assert fell, "the seed must exercise the fallback"
    got = R.a_seeded_row(seed, obj, 5, 64, tries=2).tolist()
    assert got == _a_seeded_brute(seed, obj, 5, 64, 2)
    assert all(got[i] == (raw[i + 64] >> sh) - 5 for i in fell)


def test_seeded_a_ranges_frequencies_and_streams():
    n = 1 << 16
    q = 0xffffe80001  # a 40-bit prime of the chain
    a = R.a_seeded_row(5, R.obj_id(R.TAG_KEY_A_SEEDED, 9, 1, 4), q, n)
    assert a.max() < q
    h = np.bincount((a.astype(np.float64) / q * 16).astype(np.int64), minlength=16)
    assert ((h - n / 16) ** 2 / (n / 16)).sum() < 40
    # distinct from the stored-key stream of the same key, digit and prime
    b = R.uniform(5, R.obj_id(R.TAG_KEY_A, 9, 1, 4), q, n)
    assert np.mean(a == b) < 1e-3
    A = R.key_a_seeded(5, 9, [97, q], 256, 2)
    assert A.shape == (2, 2, 256) and A[:, 0].max() < 97
    assert np.array_equal(A[1, 1], R.a_seeded_row(5, R.obj_id(R.TAG_KEY_A_SEEDED, 9, 1, 1), q, 256))
    assert np.array_equal(R.key_errors(5, 9, 256, 2), R.key_draws(5, 9, [97], 256, 2)[1])
