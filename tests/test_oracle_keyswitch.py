"""Pins for the oracle's base conversion, keys and key switching.

Big-integer identities on small N: fast base conversion gives X + u Q with
0 <= u < #src (|u| <= #src/2 in the centred form); ModDown gives
round(X / P) - v with |v| <= K/2; a switching
key minus its gadget term is exactly the sampled error; key switching
preserves decryption up to small noise.
"""
import math

import numpy as np
import pytest

from oracle import ckks as C
import seeded_inputs as S


def _tiny():
    return C.Params(12, 3, 1, 3)


def _mid():
    # several primes per digit (alpha = 3), two special primes... K = alpha
    return C.Params(10, 7, 3, 3)


def check_base_conv(x, src, dst):
    out = C.base_conv(x, src, dst)
    Q = math.prod(src)
    X = C.crt(x, src)
    Y = C.crt(out, dst)
    D = math.prod(dst)
    assert D > len(src) * Q
    for xv, yv in zip(X, Y):
        diff = yv - xv
        assert diff % Q == 0 and 0 <= diff // Q < len(src)


def test_base_conv_crt_identity():
    P = _mid()
    rng = np.random.default_rng(1)
    src = P.q[1:4]
    dst = [P.q[0]] + P.q[4:] + P.p
    x = np.stack([rng.integers(0, m, size=P.N, dtype=np.uint64) for m in src])
    check_base_conv(x, src, dst)


def test_mutation_base_conv_dropped_term_is_caught(monkeypatch):
    P = _mid()
    rng = np.random.default_rng(2)
    src = P.q[1:4]
    dst = [P.q[0]] + P.q[4:] + P.p
    x = np.stack([rng.integers(0, m, size=P.N, dtype=np.uint64) for m in src])
    real = C.base_conv

    def broken(xx, s, d):  # plant: forget the last source limb
        return real(xx[:-1], s[:-1], d)

    monkeypatch.setattr(C, "base_conv", broken)
    with pytest.raises(AssertionError):
        check_base_conv(x, src, dst)


@pytest.mark.parametrize("level", [7, 5, 4])
def test_modup_crt_identity(level):
    """Every digit's raised polynomial CRT-reconstructs (over Q_level and P) to
    X + u Q~_j, 0 <= u < |D_j|, with X the digit's value in [0, Q~_j)."""
    P = _mid()
    rng = np.random.default_rng(level)
    qm = P.q[:level]
    d_coeff = np.stack([rng.integers(0, m, size=P.N, dtype=np.uint64) for m in qm])
    d_ntt = C.ntt_rows(d_coeff, qm, P)
    ext_mods = qm + P.p
    for D in P.digits(level):
        ext = C.modup(d_coeff, d_ntt, D, level, P)
        ext_c = C.intt_rows(ext, ext_mods, P)
        src = [P.q[i] for i in D]
        Qt = math.prod(src)
        X = C.crt(d_coeff[D], src)
        Y = C.crt(ext_c, ext_mods)
        for xv, yv in zip(X[:64], Y[:64]):
            diff = yv - xv
            assert diff % Qt == 0 and 0 <= diff // Qt < len(D)


@pytest.mark.parametrize("level", [7, 3])
def test_moddown_round_identity(level):
    """ModDown(x) = round(X / P) - v (mod Q_level) with |v| <= K/2, X the CRT
    value of x over Q_level and P."""
    P = _mid()
    rng = np.random.default_rng(10 + level)
    ext_mods = P.q[:level] + P.p
    xc = np.stack([rng.integers(0, m, size=P.N, dtype=np.uint64) for m in ext_mods])
    out = C.moddown(C.ntt_rows(xc, ext_mods, P), level, P)
    oc = C.intt_rows(out, P.q[:level], P)
    X = C.crt(xc, ext_mods)
    Ql = math.prod(P.q[:level])
    Y = C.crt(oc, P.q[:level])
    vs = []
    for xv, yv in zip(X, Y):
        rounded = (2 * xv + P.P) // (2 * P.P)
        v = int(C.centered(np.array([rounded - yv], dtype=object), Ql)[0])
        assert abs(v) <= P.K // 2
        vs.append(v)
    assert abs(np.mean(vs)) < 0.1  # no systematic offset


def test_base_conv_centred_identity():
    P = _mid()
    rng = np.random.default_rng(4)
    src = P.p
    dst = P.q
    x = np.stack([rng.integers(0, m, size=P.N, dtype=np.uint64) for m in src])
    out = C.base_conv(x, src, dst, centred=True)
    Q = math.prod(src)
    D = math.prod(dst)
    Xc = C.centered(C.crt(x, src), Q)
    Y = C.centered(C.crt(out, dst), D)
    for xv, yv in zip(Xc, Y):
        diff = yv - xv
        assert diff % Q == 0 and abs(diff // Q) <= len(src) // 2


def _keys(P, seed):
    s = S.secret(seed, P.N)
    return s


@pytest.mark.parametrize("mk", ["tiny", "mid"])
def test_switching_key_error_is_exact(mk):
    """b_j + a_j s - g_j s' = e_j exactly (coefficients, centred)."""
    P = _tiny() if mk == "tiny" else _mid()
    seed = 11
    s = S.secret(seed, P.N)
    step = 3
    k = P.galois_elt(step)
    a, e = S.key_draws(seed, k, P.mods, P.N, P.dnum)
    b, a2 = C.rotation_key(s, step, a, e, P)
    mods = P.mods
    s_n = C.secret_ntt(s, mods, P)
    s_rot = C.ntt_rows(C.automorph_coeff_rows(C.to_residues(s, mods), k, mods, P), mods, P)
    for j, D in enumerate(P.digits(P.L)):
        t = C.add_rows(b[j], C.mul_rows(a2[j], s_n, mods), mods)
        g = [(P.P % m) if r in D else 0 for r, m in enumerate(mods)]
        t = C.sub_rows(t, C.scale_rows(s_rot, g, mods), mods)
        tc = C.intt_rows(t, mods, P)
        for r, m in enumerate(mods):
            cen = np.where(tc[r] > m // 2, tc[r].astype(object) - m, tc[r].astype(object))
            assert np.array_equal(cen.astype(np.int64), e[j].astype(np.int64))


@pytest.mark.parametrize("mk,level", [("tiny", 3), ("tiny", 2), ("mid", 7), ("mid", 5)])
def test_key_switch_preserves_decryption(mk, level):
    """u0 + u1 s - d s' is small for every coefficient."""
    P = _tiny() if mk == "tiny" else _mid()
    seed = 12
    s = S.secret(seed, P.N)
    a, e = S.key_draws(seed, 2, P.mods, P.N, P.dnum)
    evk = C.relin_key(s, a, e, P)
    qm = P.q[:level]
    rng = np.random.default_rng(level)
    d = np.stack([rng.integers(0, m, size=P.N, dtype=np.uint64) for m in qm])
    u0, u1 = C.key_switch(d, level, evk, P)
    s_n = C.secret_ntt(s, qm, P)
    lhs = C.add_rows(u0, C.mul_rows(u1, s_n, qm), qm)
    rhs = C.mul_rows(d, C.mul_rows(s_n, s_n, qm), qm)
    noise = C.intt_rows(C.sub_rows(lhs, rhs, qm), qm, P)
    Q = math.prod(qm)
    cen = C.centered(C.crt(noise, qm), Q)
    assert max(abs(int(v)) for v in cen) < 2 ** 30


def test_rotation_decrypts_to_rolled_slots():
    P = _tiny()
    seed = S.master_seed(0)
    s = S.secret(seed, P.N)
    pa, pe = S.public_key_draws(seed, P.q, P.N)
    pk = C.public_key(s, pa, pe, P)
    z = S.complex_slots(seed, P.n_slots, -1, 1)
    v, e0, e1 = S.encryption_draws(seed, 0, P.N)
    ct = C.make_ct(C.encrypt(pk, C.encode(z, 2.0 ** 40, 3, P), v, e0, e1, 3, P), 3, 2.0 ** 40)
    for step in (1, 2, -1):
        a, e = S.key_draws(seed, P.galois_elt(step), P.mods, P.N, P.dnum)
        evk = C.rotation_key(s, step, a, e, P)
        r = C.rotate(ct, step, evk, P)
        assert np.max(np.abs(C.decrypt_decode(r, s, P) - np.roll(z, -step))) < 1e-5


def test_mutation_rotation_direction_is_caught():
    """Planting the opposite rotation direction in the oracle fails the slot pin."""
    P = _tiny()
    seed = 5
    s = S.secret(seed, P.N)
    pa, pe = S.public_key_draws(seed, P.q, P.N)
    pk = C.public_key(s, pa, pe, P)
    z = S.complex_slots(seed, P.n_slots, -1, 1)
    v, e0, e1 = S.encryption_draws(seed, 0, P.N)
    ct = C.make_ct(C.encrypt(pk, C.encode(z, 2.0 ** 40, 3, P), v, e0, e1, 3, P), 3, 2.0 ** 40)
    step = 1
    bad = -step  # planted mistake: key and automorphism for the other direction
    a, e = S.key_draws(seed, P.galois_elt(bad), P.mods, P.N, P.dnum)
    r = C.rotate(ct, bad, C.rotation_key(s, bad, a, e, P), P)
    assert np.max(np.abs(C.decrypt_decode(r, s, P) - np.roll(z, -step))) > 1e-2


def _encrypted(P, seed, level):
    s = S.secret(seed, P.N)
    pa, pe = S.public_key_draws(seed, P.q, P.N)
    pk = C.public_key(s, pa, pe, P)
    z = S.complex_slots(seed, P.n_slots, -1, 1)
    v, e0, e1 = S.encryption_draws(seed, 0, P.N)
    ct = C.make_ct(C.encrypt(pk, C.encode(z, 2.0 ** 40, level, P), v, e0, e1, level, P), level, 2.0 ** 40)
    return s, z, ct


def _rot_keys(P, seed, s, steps):
    keys = {}
    for st in steps:
        a, e = S.key_draws(seed, P.galois_elt(st), P.mods, P.N, P.dnum)
        keys[st] = C.rotation_key(s, st, a, e, P)
    return keys


@pytest.mark.parametrize("mk,level", [("tiny", 3), ("mid", 7), ("mid", 5)])
def test_hoisted_rotations_decrypt_to_rolled_slots(mk, level):
    """Every hoisted rotation of one ciphertext decrypts to the input's
    slots rolled left by its step."""
    P = _tiny() if mk == "tiny" else _mid()
    seed = S.master_seed(7)
    s, z, ct = _encrypted(P, seed, level)
    steps = [1, 2, -1, 5, 37]
    keys = _rot_keys(P, seed, s, steps)
    for st, r in zip(steps, C.rotate_hoisted(ct, steps, keys, P)):
        assert r["level"] == level and r["scale"] == ct["scale"]
        assert np.max(np.abs(C.decrypt_decode(r, s, P) - np.roll(z, -st))) < 1e-5


@pytest.mark.parametrize("mk,level", [("tiny", 3), ("mid", 6)])
def test_hoisted_rotation_by_identity_is_the_plain_rotation(mk, level):
    """sigma_1 is the identity, so hoisting changes nothing: a hoisted
    rotation by step 0 (Galois element 1) equals rotate() residue for residue."""
    P = _tiny() if mk == "tiny" else _mid()
    seed = S.master_seed(8)
    s, _, ct = _encrypted(P, seed, level)
    assert P.galois_elt(0) == 1
    keys = _rot_keys(P, seed, s, [0])
    got = C.rotate_hoisted(ct, [0], keys, P)[0]
    want = C.rotate(ct, 0, keys[0], P)
    assert np.array_equal(got["c"], want["c"])


def test_hoisted_raised_digits_differ_by_multiples_of_the_digit_modulus():
    """sigma_k(ModUp_j(d)) and ModUp_j(sigma_k(d)): equal on the digit's own
    rows; elsewhere every coefficient differs by m Q_{D_j}, one integer m with
    |m| <= |D_j| for all the target rows of that coefficient."""
    P = _mid()
    level = 7
    qm = P.q[:level]
    ext_mods = qm + P.p
    rng = np.random.default_rng(3)
    d = np.stack([rng.integers(0, m, size=P.N, dtype=np.uint64) for m in qm])
    d_coeff = C.intt_rows(d, qm, P)
    k = P.galois_elt(3)
    d_rot = C.automorph_ntt_rows(d, k, qm, P)
    d_rot_coeff = C.intt_rows(d_rot, qm, P)
    for D in P.digits(level):
        hoisted = C.intt_rows(C.automorph_ntt_rows(C.modup(d_coeff, d, D, level, P), k, ext_mods, P), ext_mods, P)
        plain = C.intt_rows(C.modup(d_rot_coeff, d_rot, D, level, P), ext_mods, P)
        QD = math.prod(qm[i] for i in D)
        m_ref = None
        for r, mod in enumerate(ext_mods):
            diff = (hoisted[r].astype(object) - plain[r].astype(object)) % mod
            if r in D:
                assert not diff.any()
                continue
            m = C.centered(diff * pow(QD, -1, mod), mod)
            assert max(abs(int(v)) for v in m) <= len(D)
            if m_ref is None:
                m_ref = m
                assert any(int(v) != 0 for v in m)  # the two lifts do differ
            else:
                assert np.array_equal(m, m_ref)


def test_mutation_hoisted_digits_left_unpermuted_is_caught(monkeypatch):
    """Planting a hoisted rotation that permutes c0 but not the raised digits
    fails the slot pin."""
    P = _tiny()
    seed = S.master_seed(9)
    s, z, ct = _encrypted(P, seed, 3)
    keys = _rot_keys(P, seed, s, [1])
    real = C.automorph_ntt_rows
    n_ext = 3 + P.K

    def planted(a, k, mods, params):
        return np.array(a, copy=True) if len(mods) == n_ext else real(a, k, mods, params)

    monkeypatch.setattr(C, "automorph_ntt_rows", planted)
    r = C.rotate_hoisted(ct, [1], keys, P)[0]
    assert np.max(np.abs(C.decrypt_decode(r, s, P) - np.roll(z, -1))) > 1e-2


def _several(P, seed, level, n):
    s = S.secret(seed, P.N)
    pa, pe = S.public_key_draws(seed, P.q, P.N)
    pk = C.public_key(s, pa, pe, P)
    zs, cts = [], []
    for i in range(n):
        z = S.complex_slots(seed, P.n_slots, -1, 1, i)
        v, e0, e1 = S.encryption_draws(seed, i, P.N)
        zs.append(z)
        cts.append(C.make_ct(C.encrypt(pk, C.encode(z, 2.0 ** 40, level, P), v, e0, e1, level, P), level, 2.0 ** 40))
    return s, zs, cts


@pytest.mark.parametrize("mk,level", [("tiny", 3), ("mid", 7), ("mid", 4)])
def test_rotate_sum_decrypts_to_sum_of_rolled_slots(mk, level):
    P = _tiny() if mk == "tiny" else _mid()
    seed = S.master_seed(10)
    steps = [3, -7, 64, 1]
    s, zs, cts = _several(P, seed, level, len(steps))
    keys = _rot_keys(P, seed, s, steps)
    r = C.rotate_sum(cts, steps, keys, P)
    want = sum(np.roll(z, -st) for z, st in zip(zs, steps))
    assert r["level"] == level and r["scale"] == cts[0]["scale"]
    assert np.max(np.abs(C.decrypt_decode(r, s, P) - want)) < 1e-5


@pytest.mark.parametrize("mk,level", [("tiny", 3), ("mid", 5)])
def test_rotate_sum_of_one_rotation_is_the_rotation(mk, level):
    """With one term there is nothing to share: rotate_sum == rotate, residue
    for residue."""
    P = _tiny() if mk == "tiny" else _mid()
    seed = S.master_seed(11)
    s, _, cts = _several(P, seed, level, 1)
    keys = _rot_keys(P, seed, s, [5])
    assert np.array_equal(C.rotate_sum(cts, [5], keys, P)["c"], C.rotate(cts[0], 5, keys[5], P)["c"])


def test_rotate_sum_differs_from_summed_rotations_by_moddown_rounding_only():
    """ModDown(x) = (x - [x]_P)/P - v with [x]_P centred and |v| <= K/2, so
    ModDown(sum_g u_g) - sum_g ModDown(u_g) is an integer polynomial with
    coefficients of magnitude at most (G+1)(K+1)/2, for both polynomials."""
    P = _mid()
    level = 6
    seed = S.master_seed(12)
    steps = [1, 2, 3, -4, 9]
    s, _, cts = _several(P, seed, level, len(steps))
    keys = _rot_keys(P, seed, s, steps)
    lazy = C.rotate_sum(cts, steps, keys, P)["c"]
    qm = P.q[:level]
    summed = None
    for ct, st in zip(cts, steps):
        r = C.rotate(ct, st, keys[st], P)["c"]
        summed = r if summed is None else np.stack([C.add_rows(summed[c], r[c], qm) for c in range(2)])
    bound = (len(steps) + 1) * (P.K + 1) / 2
    Q = math.prod(qm)
    worst = 0
    for c in range(2):
        diff = C.intt_rows(C.sub_rows(lazy[c], summed[c], qm), qm, P)
        cen = C.centered(C.crt(diff, qm), Q)
        worst = max(worst, max(abs(int(v)) for v in cen))
    assert 0 < worst <= bound


def test_mutation_rotate_sum_one_key_for_all_is_caught():
    """Planting the first rotation's key and automorphism for every term fails
    the slot pin."""
    P = _tiny()
    seed = S.master_seed(13)
    steps = [1, 2]
    s, zs, cts = _several(P, seed, 3, 2)
    keys = _rot_keys(P, seed, s, steps)
    r = C.rotate_sum(cts, [1, 1], keys, P)  # planted: step 1 for both terms
    want = sum(np.roll(z, -st) for z, st in zip(zs, steps))
    assert np.max(np.abs(C.decrypt_decode(r, s, P) - want)) > 1e-2


@pytest.mark.parametrize("mk,level", [("tiny", 3), ("mid", 7), ("mid", 4)])
def test_rotate_sum_hoisted_decrypts_to_sum_of_rolled_slots(mk, level):
    P = _tiny() if mk == "tiny" else _mid()
    seed = S.master_seed(14)
    s, z, ct = _encrypted(P, seed, level)
    steps = [1, 2, 4, -8, 64]
    keys = _rot_keys(P, seed, s, steps)
    r = C.rotate_sum_hoisted(ct, steps, keys, P)
    want = sum(np.roll(z, -st) for st in steps)
    assert r["level"] == level and r["scale"] == ct["scale"]
    assert np.max(np.abs(C.decrypt_decode(r, s, P) - want)) < 1e-5


@pytest.mark.parametrize("mk,level", [("tiny", 3), ("mid", 5)])
def test_rotate_sum_hoisted_of_one_step_is_the_hoisted_rotation(mk, level):
    P = _tiny() if mk == "tiny" else _mid()
    seed = S.master_seed(15)
    s, _, ct = _encrypted(P, seed, level)
    keys = _rot_keys(P, seed, s, [3])
    want = C.rotate_hoisted(ct, [3], keys, P)[0]["c"]
    assert np.array_equal(C.rotate_sum_hoisted(ct, [3], keys, P)["c"], want)


def test_rotate_sum_hoisted_differs_from_summed_hoisted_rotations_by_moddown_rounding_only():
    """Against the sum of rotate_hoisted results (one ModDown each): an
    integer polynomial of magnitude at most (G+1)(K+1)/2 per coefficient, in
    both polynomials."""
    P = _mid()
    level = 6
    seed = S.master_seed(16)
    s, _, ct = _encrypted(P, seed, level)
    steps = [1, 2, 3, -4, 9]
    keys = _rot_keys(P, seed, s, steps)
    lazy = C.rotate_sum_hoisted(ct, steps, keys, P)["c"]
    qm = P.q[:level]
    summed = None
    for r in C.rotate_hoisted(ct, steps, keys, P):
        summed = r["c"] if summed is None else np.stack([C.add_rows(summed[c], r["c"][c], qm) for c in range(2)])
    Q = math.prod(qm)
    worst = 0
    for c in range(2):
        cen = C.centered(C.crt(C.intt_rows(C.sub_rows(lazy[c], summed[c], qm), qm, P), qm), Q)
        worst = max(worst, max(abs(int(v)) for v in cen))
    assert 0 < worst <= (len(steps) + 1) * (P.K + 1) / 2


def test_mutation_rotate_sum_hoisted_dropped_step_is_caught():
    """Planting a sum that skips its last step fails the slot pin."""
    P = _tiny()
    seed = S.master_seed(17)
    s, z, ct = _encrypted(P, seed, 3)
    steps = [1, 2, 4]
    keys = _rot_keys(P, seed, s, steps)
    r = C.rotate_sum_hoisted(ct, steps[:-1], keys, P)  # planted: last step dropped
    want = sum(np.roll(z, -st) for st in steps)
    assert np.max(np.abs(C.decrypt_decode(r, s, P) - want)) > 1e-2
