"""GPU parity of keys with seeded a-halves (he_keygen_seeded_ex with
HE_KEYGEN_SEEDED_A): the key stores only b, and the key-switching kernels
regenerate a from its stream starts.  Keys, rotations (plain, hoisted,
summed, rotate-and-sum) and relinearisation against the oracle, residue for
residue; at full size, every output against a context that holds the same
keys in stored form."""
import numpy as np
import pytest

from oracle import ckks as C
import seeded_inputs as S
from tests.helpers import SeededASetup, Setup, lib
from tests.test_gpu_rotate import _hoisted_case, _rotation_batch_inputs, _sum_case, _sum_hoisted_case

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("shape", [(12, 3, 1, 3), (11, 7, 3, 3)])
def test_seeded_a_keys_match_oracle(shape):
    he = lib()
    st = SeededASetup(*shape, seed=0x5EEDA + shape[1])
    for step in (1, -3):
        st.upload_rot(step)
        got = he.he_key_download(st.ctx, he.HE_KEY_ROTATION, step)
        b, a = st.oracle_rot_key(step)
        assert np.array_equal(got[:, 0], b) and np.array_equal(got[:, 1], a)
    st.upload_relin()
    got = he.he_key_download(st.ctx, he.HE_KEY_RELIN, 0)
    b, a = st.oracle_relin_key()
    assert np.array_equal(got[:, 0], b) and np.array_equal(got[:, 1], a)


def test_seeded_a_rotation_tiny():
    he = lib()
    st = SeededASetup(12, 3, 1, 3, seed=S.master_seed(0))
    P = st.P
    z = S.complex_slots(st.seed, P.n_slots, -1, 1)
    ct = st.encrypt(z, 3)
    x = st.to_gpu(ct)
    for step in (1, 2, -1):
        st.upload_rot(step)
        y = st.empty_gpu(3)
        he.he_rotate(st.ctx, x, step, y)
        he.he_sync(st.ctx)
        want = C.rotate(ct, step, st.oracle_rot_key(step), P)
        assert np.array_equal(st.from_gpu(y), want["c"])
        assert np.max(np.abs(C.decrypt_decode(want, st.s, P) - np.roll(z, -step))) < 1e-5


@pytest.mark.parametrize("level", [7, 4, 1])
def test_seeded_a_rotation_mid_levels(level):
    """alpha = 3 (60-bit and 40-bit rows in a digit), partial digits, level 1."""
    he = lib()
    st = SeededASetup(11, 7, 3, 3, seed=144)
    P = st.P
    ct = st.encrypt(S.complex_slots(st.seed, P.n_slots, -1, 1), level)
    st.upload_rot(5)
    y = st.empty_gpu(level)
    he.he_rotate(st.ctx, st.to_gpu(ct), 5, y)
    he.he_sync(st.ctx)
    assert np.array_equal(st.from_gpu(y), C.rotate(ct, 5, st.oracle_rot_key(5), P)["c"])


@pytest.mark.parametrize("level", [7, 4])
def test_seeded_a_hoisted_and_summed(level):
    st = SeededASetup(11, 7, 3, 3, seed=145)
    _hoisted_case(st, level, 3, [5, -3, 17, 0])
    _sum_case(st, level, 2, [5, -3, 17])
    _sum_hoisted_case(st, level, 2, [5, -3, 17])


def test_seeded_a_hmult():
    he = lib()
    st = SeededASetup(12, 3, 1, 3, seed=161)
    P = st.P
    z1 = S.complex_slots(st.seed, P.n_slots, -1, 1, 1)
    z2 = S.complex_slots(st.seed, P.n_slots, -1, 1, 2)
    a, b = st.encrypt(z1, 3, ct_id=1), st.encrypt(z2, 3, ct_id=2)
    st.upload_relin()
    out = st.empty_gpu(3)
    he.he_hmult_relin_rescale(st.ctx, st.to_gpu(a), st.to_gpu(b), out)
    he.he_sync(st.ctx)
    want = C.hmult_relin_rescale(a, b, st.oracle_relin_key(), P)
    assert np.array_equal(st.from_gpu(out), want["c"])
    assert np.max(np.abs(C.decrypt_decode(want, st.s, P) - z1 * z2)) < 1e-5


def test_seeded_a_key_forms_do_not_mix():
    he = lib()
    st = SeededASetup(11, 3, 1, 3, seed=170)
    st.upload_rot(1)
    with pytest.raises(he.HEError) as ei:  # stored-a key into a seeded-a context
        a, e = st.key_draws(st.P.galois_elt(2))
        he.he_keygen_upload(st.ctx, he.HE_KEY_ROTATION, 2, st.s, a, e)
    assert ei.value.code == he.HE_EINVAL
    plain = Setup(11, 3, 1, 3, seed=171)
    plain.upload_rot(1)
    with pytest.raises(he.HEError) as ei:  # seeded-a key into a stored-a context
        he.he_keygen_seeded_ex(plain.ctx, 1, [2], False, he.HE_KEYGEN_SEEDED_A)
    assert ei.value.code == he.HE_EINVAL
    with pytest.raises(he.HEError) as ei:  # unknown flag
        he.he_keygen_seeded_ex(st.ctx, 1, [2], False, 6)
    assert ei.value.code == he.HE_EINVAL


def _full_size_pair(n_keys):
    """N = 2^16, L = 24, K = 8, dnum = 3: seeded-a keys for the rotation
    batch's steps, and a twin context with the same keys stored whole."""
    st = SeededASetup(16, 24, 8, 3, seed=S.master_seed(1))
    steps = S.rotation_steps(st.seed, n_keys, 1, st.P.n_slots - 1)
    lib().he_keygen_seeded_ex(st.ctx, st.seed, steps, False, lib().HE_KEYGEN_SEEDED_A)
    twin = st.stored_twin()
    for s_ in steps:
        st.upload_rot_stored(twin, s_)
    return st, twin, steps


def test_seeded_a_full_size():
    """The rotation batch (64 ciphertexts, 16 keys), hoisted rotations (4 x
    16 steps) and rotate-and-sum (4 x 16 steps) at N = 2^16, level 24, in the
    benchmark's launch configurations: every output equals the stored-key
    twin's; one key and one batch output against the oracle."""
    he = lib()
    st, twin, steps = _full_size_pair(16)
    P = st.P
    got = he.he_key_download(st.ctx, he.HE_KEY_ROTATION, steps[3])
    b, a = st.oracle_rot_key(steps[3])
    assert np.array_equal(got[:, 0], b) and np.array_equal(got[:, 1], a)

    n_cts = 64
    _, ct_steps = _rotation_batch_inputs(st, n_cts, 16)
    uni = S.uniform_residues(st.seed, "ct_residues", P.q, P.N, lead=(n_cts, 2))
    (k,) = S.choose_groups(st.seed + 5, n_cts, 1)
    z = S.complex_slots(st.seed, P.n_slots, -1, 1, k)
    ct_k = st.encrypt(z, 24, ct_id=k)
    cts = [ct_k if i == k else C.make_ct(uni[i], 24, 2.0 ** 40) for i in range(n_cts)]
    xs = [st.to_gpu(c) for c in cts]
    ys = [st.empty_gpu(24) for _ in range(n_cts)]
    ws = [st.empty_gpu(24) for _ in range(n_cts)]
    he.he_rotate_batch(st.ctx, xs, ct_steps, ys)
    he.he_rotate_batch(twin.ctx, xs, ct_steps, ws)
    he.he_sync(st.ctx)
    he.he_sync(twin.ctx)
    for i in range(n_cts):
        assert np.array_equal(st.from_gpu(ys[i]), st.from_gpu(ws[i])), i
    want = C.rotate(ct_k, ct_steps[k], st.oracle_rot_key(ct_steps[k]), P)
    assert np.array_equal(st.from_gpu(ys[k]), want["c"])
    assert np.max(np.abs(C.decrypt_decode(want, st.s, P) - np.roll(z, -ct_steps[k]))) < 1e-5

    hin = [st.to_gpu(cts[i]) for i in range(4)]
    ys = [st.empty_gpu(24) for _ in range(4 * len(steps))]
    ws = [st.empty_gpu(24) for _ in range(4 * len(steps))]
    he.he_rotate_hoisted(st.ctx, hin, steps, ys)
    he.he_rotate_hoisted(twin.ctx, hin, steps, ws)
    he.he_sync(st.ctx)
    he.he_sync(twin.ctx)
    for o in range(len(ys)):
        assert np.array_equal(st.from_gpu(ys[o]), st.from_gpu(ws[o])), o
    ys = [st.empty_gpu(24) for _ in range(4)]
    ws = [st.empty_gpu(24) for _ in range(4)]
    he.he_rotate_sum_hoisted(st.ctx, hin, steps, ys)
    he.he_rotate_sum_hoisted(twin.ctx, hin, steps, ws)
    he.he_sync(st.ctx)
    he.he_sync(twin.ctx)
    for o in range(4):
        assert np.array_equal(st.from_gpu(ys[o]), st.from_gpu(ws[o])), o
