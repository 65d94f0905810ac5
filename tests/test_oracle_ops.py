"""Pins for the oracle's rescale, multiplication, helpers, BSGS product and
Paterson-Stockmeyer evaluation."""
import math

import numpy as np
import pytest

from oracle import ckks as C
import seeded_inputs as S


def _setup(P, seed, z, level, scale=2.0 ** 40, ct_id=0):
    s = S.secret(seed, P.N)
    pa, pe = S.public_key_draws(seed, P.q, P.N)
    pk = C.public_key(s, pa, pe, P)
    v, e0, e1 = S.encryption_draws(seed, ct_id, P.N)
    ct = C.make_ct(C.encrypt(pk, C.encode(z, scale, level, P), v, e0, e1, level, P), level, scale)
    return s, pk, ct


def test_rescale_is_rounded_division_by_last_prime():
    """CRT(rescaled) = round(C / q_last) mod Q_{l-1}, C the CRT value of the input."""
    P = C.Params(10, 5, 2, 3)
    rng = np.random.default_rng(1)
    level = 5
    qm = P.q[:level]
    cc = np.stack([np.stack([rng.integers(0, m, size=P.N, dtype=np.uint64) for m in qm]) for _ in range(2)])
    ct = C.make_ct(np.stack([C.ntt_rows(cc[k], qm, P) for k in range(2)]), level, 2.0 ** 80)
    r = C.rescale(ct, P)
    assert r["level"] == level - 1 and r["scale"] == 2.0 ** 80 / qm[-1]
    Qn = math.prod(qm[:-1])
    ql = qm[-1]
    for k in range(2):
        X = C.crt(cc[k], qm)
        Y = C.crt(C.intt_rows(r["c"][k], qm[:-1], P), qm[:-1])
        for xv, yv in zip(X, Y):
            assert ((2 * xv + ql) // (2 * ql)) % Qn == yv


def test_tensor_is_exact_product_of_decryptions():
    P = C.Params(10, 4, 2, 2)
    seed = 3
    z1 = S.complex_slots(seed, P.n_slots, -1, 1, 1)
    z2 = S.complex_slots(seed, P.n_slots, -1, 1, 2)
    s, pk, a = _setup(P, seed, z1, 4)
    v, e0, e1 = S.encryption_draws(seed, 1, P.N)
    b = C.make_ct(C.encrypt(pk, C.encode(z2, 2.0 ** 40, 4, P), v, e0, e1, 4, P), 4, 2.0 ** 40)
    d0, d1, d2 = C.tensor(a, b, P)
    qm = P.q[:4]
    s_n = C.secret_ntt(s, qm, P)
    lhs = C.add_rows(C.add_rows(d0, C.mul_rows(d1, s_n, qm), qm), C.mul_rows(d2, C.mul_rows(s_n, s_n, qm), qm), qm)
    rhs = C.mul_rows(C.decrypt(a, s, P), C.decrypt(b, s, P), qm)
    assert np.array_equal(lhs, rhs)


def test_hmult_relin_rescale_tiny():
    P = C.Params(12, 3, 1, 3)
    seed = S.master_seed(0)
    z = S.complex_slots(seed, P.n_slots, -1, 1)
    s, pk, ct = _setup(P, seed, z, 3)
    a, e = S.key_draws(seed, 2, P.mods, P.N, P.dnum)
    rlk = C.relin_key(s, a, e, P)
    m = C.hmult_relin_rescale(ct, ct, rlk, P)
    assert m["level"] == 2
    assert m["scale"] == (2.0 ** 40 * 2.0 ** 40) / P.q[2]
    assert np.max(np.abs(C.decrypt_decode(m, s, P) - z * z)) < 1e-5


def test_helpers():
    P = C.Params(10, 4, 2, 2)
    seed = 4
    z = S.complex_slots(seed, P.n_slots, -1, 1)
    s, pk, ct = _setup(P, seed, z, 4)
    out = C.decrypt_decode(C.mul_const(ct, -3, P), s, P)
    assert np.max(np.abs(out + 3 * z)) < 1e-5
    out = C.decrypt_decode(C.add_const(ct, int(0.5 * 2 ** 40), P), s, P)
    assert np.max(np.abs(out - (z + 0.5))) < 1e-5
    out = C.decrypt_decode(C.add(ct, ct, P), s, P)
    assert np.max(np.abs(out - 2 * z)) < 1e-5
    d = C.drop_level(ct, 2)
    assert d["level"] == 2
    assert np.max(np.abs(C.decrypt_decode(d, s, P) - z)) < 1e-5


@pytest.mark.parametrize("hoisted,one_moddown", [(False, False), (True, False), (True, True)])
def test_bsgs_matvec_small(hoisted, one_moddown):
    """Feature-major packed block product y = W x by diagonals with BSGS:
    n_feat = 16 features x 64 tokens on N = 2^11, 4 baby x 4 giant steps,
    two input blocks and two output blocks; baby steps as plain or hoisted
    rotations, giant steps summed with one ModDown per rotation or per output."""
    P = C.Params(11, 3, 1, 3)
    seed = 21
    n_feat, n_tok, bs, gs = 16, 64, 4, 4
    n_in, n_out = 2, 2
    W = S.weights(seed, (n_out * n_feat, n_in * n_feat), -0.05, 0.05)
    X = S.weights(seed, (n_in * n_feat, n_tok), -1, 1, 1)
    s = S.secret(seed, P.N)
    pa, pe = S.public_key_draws(seed, P.q, P.N)
    pk = C.public_key(s, pa, pe, P)
    level = 3
    cts = []
    for j in range(n_in):
        z = X[j * n_feat:(j + 1) * n_feat].reshape(-1).astype(np.complex128)  # slot f*n_tok + t
        v, e0, e1 = S.encryption_draws(seed, j, P.N)
        cts.append(C.make_ct(C.encrypt(pk, C.encode(z, 2.0 ** 40, level, P), v, e0, e1, level, P), level, 2.0 ** 40))
    steps = sorted({n_tok * b for b in range(1, bs)} | {n_tok * bs * g for g in range(1, gs)})
    keys = {}
    for st in steps:
        a, e = S.key_draws(seed, P.galois_elt(st), P.mods, P.N, P.dnum)
        keys[st] = C.rotation_key(s, st, a, e, P)
    slots = {}
    for i in range(n_out):
        for j in range(n_in):
            Wij = W[i * n_feat:(i + 1) * n_feat, j * n_feat:(j + 1) * n_feat]
            slots[(i, j)] = C.bsgs_plaintext_slots(Wij, n_feat, n_tok, bs, gs)
    pt = lambda i, j, g, b: C.encode(slots[(i, j)][g, b], 2.0 ** 40, level, P)
    Y = C.bsgs_matvec(cts, pt, bs, gs, n_tok, keys, P, list(range(n_out)), 2.0 ** 40, hoisted=hoisted,
                      one_moddown=one_moddown)
    want = W @ X
    for i in range(n_out):
        y = C.rescale(Y[i], P)
        got = C.decrypt_decode(y, s, P).real.reshape(n_feat, n_tok)
        assert np.max(np.abs(got - want[i * n_feat:(i + 1) * n_feat])) < 1e-5


def test_bsgs_plaintext_slots_reproduce_block_product():
    """Plain slot-vector arithmetic of the BSGS identity (no encryption)."""
    n_feat, n_tok, bs, gs = 16, 4, 4, 4
    rng = np.random.default_rng(0)
    W = rng.uniform(-1, 1, (n_feat, n_feat))
    x = rng.uniform(-1, 1, (n_feat, n_tok))
    xs = x.reshape(-1)
    pts = C.bsgs_plaintext_slots(W, n_feat, n_tok, bs, gs)
    rot = lambda v, r: np.roll(v, -r)
    y = np.zeros_like(xs)
    for g in range(gs):
        inner = sum(pts[g, b] * rot(xs, n_tok * b) for b in range(bs))
        y = y + rot(inner, n_tok * bs * g)
    assert np.allclose(y.reshape(n_feat, n_tok), W @ x)


def test_ps_degree15_small():
    """Degree-15 polynomial by Paterson-Stockmeyer on N = 2^12 with 8 limbs
    (6 are consumed), slots uniform in [-4, 0]."""
    P = C.Params(12, 8, 3, 3)
    seed = 31
    z = S.real_slots(seed, P.n_slots, -4.0, 0.0)
    coeffs = S.poly_coeffs(seed, 15)
    s, pk, ct = _setup(P, seed, z, 8)
    a, e = S.key_draws(seed, 2, P.mods, P.N, P.dnum)
    rlk = C.relin_key(s, a, e, P)
    out = C.ps_eval_deg15(ct, coeffs, rlk, P)
    assert out["level"] == 2
    got = C.decrypt_decode(out, s, P)
    x_dec = C.decrypt_decode(ct, s, P)
    # homomorphic evaluation error alone (same input slots as the ciphertext holds)
    assert np.max(np.abs(got - C.ps_eval_plain(x_dec, coeffs))) < 1e-6
    # against the plaintext slots (includes the encryption noise, amplified by p')
    assert np.max(np.abs(got - C.ps_eval_plain(z, coeffs))) < 1e-5


def test_ps_plain_horner_matches_power_sum():
    coeffs = S.poly_coeffs(1, 15)
    x = np.linspace(-4, 0, 101)
    want = sum(c * x ** k for k, c in enumerate(coeffs))
    assert np.allclose(C.ps_eval_plain(x, coeffs).real, want, rtol=0, atol=1e-12)


def test_ps_schedule_matches_term_by_term_rescales():
    """The degree-15 schedule (one rescale per Horner block and per step, the
    block's products added before the step's rescale) decrypts to the same
    slots as the plain schedule that rescales every constant-multiplied
    power on its own and adds the blocks after each HMult-relin-rescale:
    the two differ only in rounding."""
    P = C.Params(12, 8, 3, 3)
    seed = 31
    z = S.real_slots(seed, P.n_slots, -4.0, 0.0)
    coeffs = S.poly_coeffs(seed, 15)
    s, pk, ct = _setup(P, seed, z, 8)
    a, e = S.key_draws(seed, 2, P.mods, P.N, P.dnum)
    rlk = C.relin_key(s, a, e, P)
    fast = C.ps_eval_deg15(ct, coeffs, rlk, P)

    hm = lambda u, v: C.hmult_relin_rescale(u, v, rlk, P)
    l0 = ct["level"]
    x2 = hm(ct, ct)
    x3 = hm(x2, C.drop_level(ct, l0 - 1))
    x4 = hm(x2, x2)
    pw = {1: ct, 2: x2, 3: x3}

    def block(i, lam, T):
        acc = None
        for j in (1, 2, 3):
            xj = C.drop_level(pw[j], lam + 1)
            K = C.ps_const(float(coeffs[4 * i + j]), T, P.q[lam], xj["scale"])
            t = C.rescale(C.mul_const(xj, K, P), P)
            acc = t if acc is None else C.make_ct(C.add(acc, t, P)["c"], lam, T)
        acc = C.add_const(acc, int(C.round_half_away(np.float64(float(coeffs[4 * i]) * T))), P)
        return C.make_ct(acc["c"], lam, T)

    acc = block(3, l0 - 3, C.PS_TOP_SCALE)
    for i in (2, 1, 0):
        acc = hm(acc, C.drop_level(x4, acc["level"]))
        acc = C.make_ct(C.add(acc, block(i, acc["level"], acc["scale"]), P)["c"], acc["level"], acc["scale"])
    assert acc["level"] == fast["level"] and acc["scale"] == fast["scale"]
    got, want = C.decrypt_decode(fast, s, P), C.decrypt_decode(acc, s, P)
    assert np.max(np.abs(got - want)) < 1e-7
    assert not np.array_equal(fast["c"], acc["c"])  # the residues do differ
