"""The packed wire format of ciphertexts (he_ct_pack / he_ct_unpack /
he_ct_wire_bytes, host only): byte for byte against an independent numpy
encoding (each residue's first b_r little-endian bytes, b_r = ceil(bitlen(q_r)
/ 8)), round trips, the size formula and the argument checks."""
import numpy as np
import pytest

from oracle import ckks as C
import seeded_inputs as S


@pytest.fixture(scope="module")
def he():
    from homomorphic_encrypted_transformer_b200 import he as h

    return h


def _numpy_wire(cts, primes):
    """[n][2][level][N] uint64 -> bytes: per ciphertext, poly, limb, the
    first b_r bytes of every residue's little-endian 8-byte form."""
    n, _, level, N = cts.shape
    parts = []
    for i in range(n):
        for poly in range(2):
            for r in range(level):
                b = (int(primes[r]).bit_length() + 7) // 8
                le = np.ascontiguousarray(cts[i, poly, r].astype("<u8")).view(np.uint8).reshape(N, 8)
                parts.append(le[:, :b].reshape(-1))
    return np.concatenate(parts)


@pytest.mark.parametrize("log_n,L,K,level", [(11, 4, 2, 4), (11, 4, 2, 2), (12, 3, 1, 3)])
def test_pack_matches_numpy_encoding_and_round_trips(he, log_n, L, K, level):
    P = C.Params(log_n, L, K, 2)
    q = P.q[:level]
    cts = S.uniform_residues(S.master_seed(0) + level, "ct_residues", q, P.N, lead=(3, 2))
    packed = he.he_ct_pack(P.q, level, log_n, cts)
    assert packed.size == 3 * he.he_ct_wire_bytes(P.q, level, log_n)
    assert np.array_equal(packed, _numpy_wire(cts, q))
    assert np.array_equal(he.he_ct_unpack(P.q, level, log_n, packed, 3), cts)
    # extreme residues: 0 and q - 1 on every limb
    ext = np.zeros((1, 2, level, P.N), dtype=np.uint64)
    ext[..., 1::2] = np.array(q, dtype=np.uint64)[None, None, :, None] - 1
    assert np.array_equal(he.he_ct_unpack(P.q, level, log_n, he.he_ct_pack(P.q, level, log_n, ext), 1), ext)


def test_wire_size_of_the_rotation_batch_ciphertext(he):
    """N = 2^16, level 24: q_0 60-bit (8 bytes), q_1..q_23 40-bit (5 bytes)."""
    P = C.Params(16, 24, 8, 3)
    assert int(P.q[0]).bit_length() == 60 and all(int(v).bit_length() == 40 for v in P.q[1:24])
    got = he.he_ct_wire_bytes(P.q, 24, 16)
    assert got == 2 * (1 << 16) * (8 + 23 * 5)
    assert abs(got / (2 * 24 * (1 << 16) * 8) - 0.6406) < 1e-3


def test_wire_argument_checks(he):
    P = C.Params(11, 4, 2, 2)
    cts = np.zeros((1, 2, 4, P.N), dtype=np.uint64)
    cts[0, 1, 2, 5] = P.q[2]  # not a canonical residue
    with pytest.raises(he.HEError):
        he.he_ct_pack(P.q, 4, 11, cts)
    with pytest.raises(he.HEError):
        he.he_ct_wire_bytes(P.q, 0, 11)
    with pytest.raises(ValueError):  # more limbs than primes given
        he.he_ct_wire_bytes(P.q[:2], 3, 11)
    with pytest.raises(ValueError):
        he.he_ct_unpack(P.q, 4, 11, np.zeros(10, dtype=np.uint8), 1)
