"""GPU parity: batched NTT / inverse NTT through the C ABI vs the oracle, bit-exact."""
import numpy as np
import pytest

from oracle import ckks as C
from tests.helpers import Setup, dev, host, lib, random_rows

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("log_n,L,K,n_polys", [(12, 3, 1, 3), (11, 3, 1, 2), (13, 4, 2, 1), (14, 3, 1, 1),
                                               (15, 3, 1, 1), (10, 7, 3, 2), (16, 24, 8, 2)])
def test_ntt_fwd_inv_bit_exact(log_n, L, K, n_polys):
    he = lib()
    st = Setup(log_n, L, K, min(3, L), seed=100 + log_n)
    P = st.P
    mods = P.mods
    a = random_rows(st.seed, mods, n_polys, P.N)
    d = dev(a)
    he.he_ntt_fwd(st.ctx, d, n_polys, len(mods), 0)
    he.he_sync(st.ctx)
    got = host(d, a.shape)
    for i in range(n_polys):
        assert np.array_equal(got[i], C.ntt_rows(a[i], mods, P))
    he.he_ntt_inv(st.ctx, d, n_polys, len(mods), 0)
    he.he_sync(st.ctx)
    assert np.array_equal(host(d, a.shape), a)
    # inverse on its own against the oracle
    d2 = dev(a)
    he.he_ntt_inv(st.ctx, d2, n_polys, len(mods), 0)
    he.he_sync(st.ctx)
    got = host(d2, a.shape)
    for i in range(n_polys):
        assert np.array_equal(got[i], C.intt_rows(a[i], mods, P))


def test_ntt_sub_range_of_primes():
    """first_prime selects the primes: the special primes alone."""
    he = lib()
    st = Setup(12, 3, 2, 2, seed=7)
    P = st.P
    mods = P.p
    a = random_rows(st.seed, mods, 1, P.N)
    d = dev(a)
    he.he_ntt_fwd(st.ctx, d, 1, len(mods), P.L)
    he.he_sync(st.ctx)
    assert np.array_equal(host(d, a.shape)[0], C.ntt_rows(a[0], mods, P))


def test_ntt_edge_values():
    """All-zero, all q-1 and a single spike survive the lazy reductions."""
    he = lib()
    st = Setup(16, 2, 1, 2, seed=8)
    P = st.P
    mods = P.mods
    a = np.zeros((3, len(mods), P.N), dtype=np.uint64)
    for r, q in enumerate(mods):
        a[1, r, :] = q - 1
        a[2, r, P.N - 1] = q - 1
    d = dev(a)
    he.he_ntt_fwd(st.ctx, d, 3, len(mods), 0)
    he.he_sync(st.ctx)
    got = host(d, a.shape)
    for i in range(3):
        assert np.array_equal(got[i], C.ntt_rows(a[i], mods, P))


def test_ntt_bad_arguments_rejected():
    he = lib()
    st = Setup(12, 3, 1, 3, seed=9)
    d = dev(np.zeros((4, st.P.N), dtype=np.uint64))
    with pytest.raises(he.HEError) as ei:
        he.he_ntt_fwd(st.ctx, d, 1, 5, 0)
    assert ei.value.code == he.HE_EINVAL


@pytest.mark.parametrize("q_bits", [41, 42, 30])
def test_ntt_prime_size_edges(q_bits):
    """The FP64 butterflies serve primes below 2^41: the largest such primes
    (the bound analysis at its limit), 42-bit primes (integer path) and small
    primes, forward and inverse, bit-exact."""
    he = lib()
    log_n, L, K = 16, 3, 1
    P = C.Params(log_n, L, K, 3, q_bits=q_bits)
    ctx = he.he_ctx_create(log_n, L, K, 3, q_bits=q_bits)
    assert ctx.primes == P.mods
    mods = P.mods
    a = random_rows(31 + q_bits, mods, 2, P.N)
    for r, q in enumerate(mods):  # extremes in the first polynomial
        a[0, r, :16] = q - 1
        a[0, r, 16:32] = 0
    d = dev(a)
    he.he_ntt_fwd(ctx, d, 2, len(mods), 0)
    he.he_sync(ctx)
    got = host(d, a.shape)
    for i in range(2):
        assert np.array_equal(got[i], C.ntt_rows(a[i], mods, P))
    d2 = dev(a)
    he.he_ntt_inv(ctx, d2, 2, len(mods), 0)
    he.he_sync(ctx)
    got = host(d2, a.shape)
    for i in range(2):
        assert np.array_equal(got[i], C.intt_rows(a[i], mods, P))
    he.he_ctx_destroy(ctx)
