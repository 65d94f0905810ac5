"""Pins for the oracle's number theory: primes, roots of unity, CRT.

Independent references: sympy's primality test and n-th root solver, and
brute-force enumeration for small moduli.
"""
import math
import random

import numpy as np
import pytest
import sympy

from oracle import ckks as C


def test_miller_rabin_matches_sympy():
    rnd = random.Random(7)
    # strong pseudoprimes to several small bases, Carmichael numbers, and random odds
    special = [3215031751, 2152302898747, 3474749660383, 341550071728321, 561, 1105, 1729, 2465, 2821, 6601]
    cands = special + [rnd.randrange(3, 1 << 62) | 1 for _ in range(2000)] + list(range(2, 3000))
    for n in cands:
        assert C.is_prime(n) == sympy.isprime(n), n


@pytest.mark.parametrize("log_n,L,K", [(12, 3, 1), (16, 24, 8)])
def test_prime_rule(log_n, L, K):
    """Primes = 1 mod 2N, of the stated sizes, distinct, prime by sympy, and
    consecutive in the downward scan (every skipped candidate is composite)."""
    P = C.Params(log_n, L, K, 3)
    two_n = 2 * P.N
    for m in P.mods:
        assert m % two_n == 1 and sympy.isprime(m)
    assert len(set(P.mods)) == L + K
    assert P.q[0].bit_length() == 60 and all(x.bit_length() == 60 for x in P.p)
    assert all(x.bit_length() == 40 for x in P.q[1:])
    # 60-bit scan: q0, p0, ..., p_{K-1} are the K+1 largest
    scan60 = [P.q[0]] + P.p
    top = ((1 << 60) - 2) // two_n * two_n + 1
    cand = top
    found = []
    while len(found) < K + 1:
        if sympy.isprime(cand):
            found.append(cand)
        cand -= two_n
    assert found == scan60
    top = ((1 << 40) - 2) // two_n * two_n + 1
    cand, found = top, []
    while len(found) < L - 1:
        if sympy.isprime(cand):
            found.append(cand)
        cand -= two_n
    assert found == P.q[1:]


def test_smallest_primitive_root_bruteforce_small():
    """Against enumeration of every residue, for small primes and orders."""
    for order in (4, 8, 16, 32):
        for q in [p for p in range(order + 1, 3000, order) if sympy.isprime(p)][:6]:
            roots = [z for z in range(1, q) if pow(z, order // 2, q) == q - 1]
            assert C.smallest_primitive_root(q, order) == min(roots)


def test_smallest_primitive_root_sympy_n4096():
    P = C.Params(12, 3, 1, 3)
    for q, psi in zip(P.mods, P.psi):
        roots = sympy.ntheory.residue_ntheory.nthroot_mod(q - 1, P.N, q, all_roots=True)
        assert len(roots) == P.N
        assert psi == min(roots)


def test_crt_and_centered():
    rnd = random.Random(3)
    mods = [97, 193, 257, 65537]
    Q = math.prod(mods)
    xs = [rnd.randrange(Q) for _ in range(50)]
    res = np.array([[x % m for x in xs] for m in mods], dtype=np.uint64)
    assert list(C.crt(res, mods)) == xs
    cen = C.centered(np.array(xs, dtype=object), Q)
    for x, c in zip(xs, cen):
        assert (c - x) % Q == 0 and -Q // 2 < c <= Q // 2
