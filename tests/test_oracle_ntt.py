"""Pins for the oracle's negacyclic NTT and automorphism.

References: direct evaluation at the odd powers of psi in Python integers,
the schoolbook negacyclic product, and the evaluation identity of X -> X^k.
"""
import numpy as np
import pytest

from oracle import ckks as C


def _brev(j, bits):
    return int(format(j, "0%db" % bits)[::-1], 2) if bits else 0


def _small_params(log_n):
    return C.Params(log_n, 2, 1, 2, q0_bits=60, q_bits=40, p_bits=60)


def _rand_rows(rng, mods, n):
    return np.stack([rng.integers(0, m, size=n, dtype=np.uint64) for m in mods])


def check_ntt_direct(P, a, mods):
    """A[j] = sum_i a_i psi^((2 brev(j) + 1) i) mod q."""
    A = C.ntt_rows(a, mods, P)
    for r, q in enumerate(mods):
        psi = P.psi_of(q)
        for j in range(P.N):
            x = pow(psi, 2 * _brev(j, P.log_n) + 1, q)
            want = sum(int(a[r, i]) * pow(x, i, q) for i in range(P.N)) % q
            assert int(A[r, j]) == want, (q, j)


@pytest.mark.parametrize("log_n", [1, 2, 3, 4, 5, 6, 7, 8])
def test_ntt_equals_direct_evaluation(log_n):
    P = _small_params(log_n)
    rng = np.random.default_rng(log_n)
    check_ntt_direct(P, _rand_rows(rng, P.mods, P.N), P.mods)


@pytest.mark.parametrize("log_n", [4, 10, 12, 16])
def test_ntt_roundtrip(log_n):
    P = _small_params(log_n)
    rng = np.random.default_rng(100 + log_n)
    a = _rand_rows(rng, P.mods, P.N)
    assert np.array_equal(C.intt_rows(C.ntt_rows(a, P.mods, P), P.mods, P), a)
    assert np.array_equal(C.ntt_rows(C.intt_rows(a, P.mods, P), P.mods, P), a)


def _schoolbook_negacyclic(a, b, q):
    n = len(a)
    out = [0] * n
    for i in range(n):
        ai = int(a[i])
        for j in range(n):
            k = i + j
            if k < n:
                out[k] += ai * int(b[j])
            else:
                out[k - n] -= ai * int(b[j])
    return [v % q for v in out]


@pytest.mark.parametrize("log_n", [3, 6, 9])
def test_ntt_convolution_is_negacyclic_product(log_n):
    P = _small_params(log_n)
    rng = np.random.default_rng(200 + log_n)
    a = _rand_rows(rng, P.mods, P.N)
    b = _rand_rows(rng, P.mods, P.N)
    c = C.intt_rows(C.mul_rows(C.ntt_rows(a, P.mods, P), C.ntt_rows(b, P.mods, P), P.mods), P.mods, P)
    for r, q in enumerate(P.mods):
        assert [int(v) for v in c[r]] == _schoolbook_negacyclic(a[r], b[r], q)


def check_automorph_evaluation(P, a, k, mods):
    """sigma_k(a)(x) = a(x^k) at every primitive 2N-th root x = psi^e (e odd)."""
    s = C.automorph_coeff_rows(a, k, mods, P)
    for r, q in enumerate(mods):
        psi = P.psi_of(q)
        for e in range(1, 2 * P.N, 2):
            x = pow(psi, e, q)
            lhs = sum(int(s[r, i]) * pow(x, i, q) for i in range(P.N)) % q
            xk = pow(x, k, q)
            rhs = sum(int(a[r, i]) * pow(xk, i, q) for i in range(P.N)) % q
            assert lhs == rhs


@pytest.mark.parametrize("log_n,k", [(3, 5), (4, 25 % 32), (5, 3), (6, 127)])
def test_automorphism_evaluation_identity(log_n, k):
    P = _small_params(log_n)
    rng = np.random.default_rng(300 + log_n)
    check_automorph_evaluation(P, _rand_rows(rng, P.mods, P.N), k, P.mods)


def test_automorphism_is_index_permutation_in_ntt_domain():
    """In the evaluation domain sigma_k permutes values: storage j (point
    psi^(2 brev(j)+1)) takes the value stored at the point psi^((2 brev(j)+1) k)."""
    P = _small_params(8)
    rng = np.random.default_rng(5)
    a = _rand_rows(rng, P.mods, P.N)
    A = C.ntt_rows(a, P.mods, P)
    for k in (5, 25, 2 * P.N - 1):
        S = C.automorph_ntt_rows(A, k, P.mods, P)
        for j in range(P.N):
            e = (2 * _brev(j, P.log_n) + 1) * k % (2 * P.N)
            jj = _brev((e - 1) // 2, P.log_n)
            assert np.array_equal(S[:, j], A[:, jj])


def test_mutation_ntt_wrong_root_is_caught():
    """A plausible mistake planted in the oracle (a wrong root) fails the direct pin."""
    P = _small_params(4)
    rng = np.random.default_rng(9)
    a = _rand_rows(rng, P.mods, P.N)
    good = list(P.psi)
    P.psi = [pow(x, 3, m) for x, m in zip(good, P.mods)]  # another primitive root
    with pytest.raises(AssertionError):
        # expected values computed with the stated root, transform with the planted one
        A = C.ntt_rows(a, P.mods, P)
        P.psi = good
        for r, q in enumerate(P.mods):
            psi = P.psi_of(q)
            for j in range(P.N):
                x = pow(psi, 2 * _brev(j, P.log_n) + 1, q)
                assert int(A[r, j]) == sum(int(a[r, i]) * pow(x, i, q) for i in range(P.N)) % q
