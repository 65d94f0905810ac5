"""The C ABI (include/he.h): library loads, exports every declared symbol,
derives the same parameters as the oracle, and rejects bad arguments on the
host.  No device work."""
import ctypes
import os
import re

import pytest

from oracle import ckks as C

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def he():
    import __graft_entry__

    __graft_entry__.build()
    from homomorphic_encrypted_transformer_b200 import he as mod

    return mod


def declared_functions():
    src = open(os.path.join(ROOT, "include", "he.h")).read()
    return re.findall(r"^\s*(?:int|const char\*|long long)\s+(he_\w+)\(", src, re.M)


def test_header_declares_the_hot_path_calls():
    names = set(declared_functions())
    for n in ["he_keygen_upload", "he_ntt_fwd", "he_ntt_inv", "he_rotate", "he_hmult_relin_rescale",
              "he_pmult_accum_bsgs", "he_rescale", "he_rotate_hoisted", "he_rotate_sum",
              "he_rotate_sum_hoisted", "he_attention_scores", "he_attention_output"]:
        assert n in names


def test_library_exports_every_declared_symbol(he):
    lib = ctypes.CDLL(he.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert hasattr(he, name), "binding lacks " + name


@pytest.mark.parametrize("log_n,L,K,dnum", [(12, 3, 1, 3), (16, 24, 8, 3), (11, 3, 1, 3), (12, 8, 3, 3),
                                            (10, 7, 3, 3)])
def test_library_derives_oracle_primes_and_roots(he, log_n, L, K, dnum):
    P = C.Params(log_n, L, K, dnum)
    primes, psi = he.he_derive_primes(log_n, L, K, dnum)
    assert primes == P.mods
    assert psi == P.psi


@pytest.mark.parametrize("args", [(9, 3, 1, 3), (17, 3, 1, 3), (12, 0, 1, 1), (12, 3, 0, 3), (12, 3, 1, 4),
                                  (12, 24, 4, 3), (12, 40, 30, 3)])
def test_invalid_parameters_rejected_on_host(he, args):
    with pytest.raises(he.HEError) as ei:
        he.he_derive_primes(*args)
    assert ei.value.code == he.HE_EINVAL
    with pytest.raises(he.HEError) as ei:
        he.he_ctx_create(*args)
    assert ei.value.code == he.HE_EINVAL


def test_explicit_primes_checked(he):
    P = C.Params(12, 3, 1, 3)
    primes, _ = he.he_derive_primes(12, 3, 1, 3, q=P.q, p=P.p)
    assert primes == P.mods
    with pytest.raises(he.HEError):  # not = 1 mod 2N
        he.he_derive_primes(12, 3, 1, 3, q=[P.q[0], P.q[1], 1000003], p=P.p)
    with pytest.raises(he.HEError):  # repeated prime
        he.he_derive_primes(12, 3, 1, 3, q=[P.q[0], P.q[1], P.q[1]], p=P.p)


def test_bindings_check_list_lengths_before_calling(he):
    """The list-taking bindings reject mismatched lengths on the host, before
    any call into the library (no context needed)."""
    import torch

    x = he.Ciphertext(torch.zeros(16, dtype=torch.int64), 1, 1.0)
    with pytest.raises(ValueError):
        he.he_rotate_hoisted(None, [x, x], [1, 2], [x, x, x])  # needs 2 x 2 outputs
    with pytest.raises(ValueError):
        he.he_rotate_sum(None, [x, x, x], [1, 2], None, [x, x])  # needs 2 x 2 terms
    with pytest.raises(ValueError):
        he.he_rotate_sum(None, [x, x], [1, 2], [x, x], [x])  # one base per output
    with pytest.raises(ValueError):
        he.he_rotate_sum_hoisted(None, [x, x], [1], [x])  # one output per input
    with pytest.raises(ValueError):
        he.he_attention_scores(None, x, x, 32, 16, [0, 1], [x])  # one output per offset
    with pytest.raises(ValueError):
        he.he_attention_output(None, [x], x, 32, [0, 1], x)  # one weight per offset


def test_library_sampler_matches_the_oracle_sampler(he):
    """The host sampler of he_keygen_seeded against the oracle's independent
    implementation of the same rule: threshold table, secret, key draws."""
    from oracle import sampler as R

    assert he.he_gaussian_cdt() == R.gaussian_cdt()
    for seed in (0, 0xAE615000, (1 << 64) - 5):
        assert (he.he_sample_secret(seed, 12) == R.secret(seed, 1 << 12)).all()
    P = C.Params(11, 4, 2, 2)
    for key_id in (2, P.galois_elt(3), P.galois_elt(-1)):
        a, e = he.he_sample_key_draws(77, key_id, 11, P.mods, 2)
        ra, re_ = R.key_draws(77, key_id, P.mods, P.N, 2)
        assert (a == ra).all() and (e == re_).all()
    with pytest.raises(he.HEError):
        he.he_sample_key_draws(1, 1 << 32, 11, P.mods, 2)  # key id beyond 32 bits


def test_library_seeded_a_matches_the_oracle(he):
    """The seeded a-halves (HE_KEYGEN_SEEDED_A) of the library's host sampler
    against the oracle's counter rule, including a modulus that forces
    rejections (5 of the 8 values of its top three bits kept)."""
    from oracle import sampler as R

    P = C.Params(11, 4, 2, 2)
    for key_id in (2, P.galois_elt(5)):
        a = he.he_sample_key_a_seeded(0xC0FFEE, key_id, 11, P.mods, 2)
        assert (a == R.key_a_seeded(0xC0FFEE, key_id, P.mods, P.N, 2)).all()
    a = he.he_sample_key_a_seeded(9, 4, 8, [5, 97], 3)
    assert (a == R.key_a_seeded(9, 4, [5, 97], 256, 3)).all()
    with pytest.raises(he.HEError):
        he.he_sample_key_a_seeded(1, 1 << 32, 11, P.mods, 2)
