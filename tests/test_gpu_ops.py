"""GPU parity: HMult+relinearise+rescale, rescale, helpers, the degree-15
Paterson-Stockmeyer evaluation and the BSGS plaintext x ciphertext product
vs the oracle (bit-exact residues; slots within 1e-5 of fp64)."""
import numpy as np
import pytest
import torch

from oracle import ckks as C
import seeded_inputs as S
from tests.helpers import Setup, dev, host, lib

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("log_n,L,K,level", [(12, 3, 1, 3), (11, 7, 3, 7), (11, 7, 3, 4), (11, 7, 3, 2)])
def test_hmult_relin_rescale(log_n, L, K, level):
    he = lib()
    st = Setup(log_n, L, K, 3, seed=60 + level)
    P = st.P
    z1 = S.complex_slots(st.seed, P.n_slots, -1, 1, 1)
    z2 = S.complex_slots(st.seed, P.n_slots, -1, 1, 2)
    a = st.encrypt(z1, level, ct_id=1)
    b = st.encrypt(z2, level, ct_id=2)
    st.upload_relin()
    out = st.empty_gpu(level)
    he.he_hmult_relin_rescale(st.ctx, st.to_gpu(a), st.to_gpu(b), out)
    he.he_sync(st.ctx)
    want = C.hmult_relin_rescale(a, b, st.oracle_relin_key(), P)
    assert out.level == level - 1 and out.scale == want["scale"]
    assert np.array_equal(st.from_gpu(out), want["c"])
    assert np.max(np.abs(C.decrypt_decode(want, st.s, P) - z1 * z2)) < 1e-5


def test_hmult_full_size():
    he = lib()
    st = Setup(16, 24, 8, 3, seed=S.master_seed(4))
    P = st.P
    z = S.real_slots(st.seed, P.n_slots, -4.0, 0.0, 0)
    a = st.encrypt(z, 24)
    st.upload_relin()
    out = st.empty_gpu(24)
    he.he_hmult_relin_rescale(st.ctx, st.to_gpu(a), st.to_gpu(a), out)
    he.he_sync(st.ctx)
    want = C.hmult_relin_rescale(a, a, st.oracle_relin_key(), P)
    assert np.array_equal(st.from_gpu(out), want["c"])


@pytest.mark.parametrize("level", [3, 2])
def test_rescale_in_place(level):
    he = lib()
    st = Setup(12, 3, 1, 3, seed=70)
    P = st.P
    rng = np.random.default_rng(level)
    c = np.stack([np.stack([rng.integers(0, q, P.N, dtype=np.uint64) for q in P.q[:level]]) for _ in range(2)])
    ct = C.make_ct(c, level, 2.0 ** 80)
    g = st.to_gpu(ct)
    he.he_rescale(st.ctx, g)
    he.he_sync(st.ctx)
    want = C.rescale(ct, P)
    assert g.level == level - 1 and g.scale == want["scale"]
    assert np.array_equal(st.from_gpu(g), want["c"])


def test_rescale_level1_rejected():
    he = lib()
    st = Setup(12, 3, 1, 3, seed=71)
    g = st.to_gpu(C.make_ct(np.zeros((2, 1, st.P.N), dtype=np.uint64), 1, 1.0))
    with pytest.raises(he.HEError) as ei:
        he.he_rescale(st.ctx, g)
    assert ei.value.code == he.HE_ELEVEL


def test_helpers():
    he = lib()
    st = Setup(12, 4, 2, 2, seed=72)
    P = st.P
    z = S.complex_slots(st.seed, P.n_slots, -1, 1)
    ct = st.encrypt(z, 4)
    g = st.to_gpu(ct)
    for K in (-3, 5, -(2 ** 62) + 7, 2 ** 62 + 11):
        o = st.empty_gpu(4)
        he.he_mul_const(st.ctx, g, K, o)
        he.he_sync(st.ctx)
        assert np.array_equal(st.from_gpu(o), C.mul_const(ct, K, P)["c"])
    o = st.empty_gpu(4)
    he.he_add(st.ctx, g, g, o)
    he.he_sync(st.ctx)
    assert np.array_equal(st.from_gpu(o), C.add(ct, ct, P)["c"])
    for K in (12345, -99999, -(2 ** 63)):
        o = st.to_gpu(ct)
        he.he_add_const(st.ctx, o, K)
        he.he_sync(st.ctx)
        assert np.array_equal(st.from_gpu(o), C.add_const(ct, K, P)["c"])
    for lev in (4, 3, 1):
        o = st.empty_gpu(4)
        he.he_drop_level(st.ctx, g, lev, o)
        he.he_sync(st.ctx)
        assert o.level == lev
        assert np.array_equal(st.from_gpu(o), C.drop_level(ct, lev)["c"])
    o = st.to_gpu(ct)  # in place
    he.he_drop_level(st.ctx, o, 2, o)
    he.he_sync(st.ctx)
    assert np.array_equal(st.from_gpu(o), C.drop_level(ct, 2)["c"])


def test_ps15_small():
    """Degree-15 Paterson-Stockmeyer on N=2^12 with 8 limbs, 3 ciphertexts."""
    he = lib()
    st = Setup(12, 8, 3, 3, seed=31)
    P = st.P
    coeffs = S.poly_coeffs(st.seed, 15)
    st.upload_relin()
    cts = [st.encrypt(S.real_slots(st.seed, P.n_slots, -4.0, 0.0, i), 8, ct_id=i) for i in range(3)]
    xs = [st.to_gpu(c) for c in cts]
    outs = [st.empty_gpu(8) for _ in cts]
    he.he_poly_eval_ps15(st.ctx, xs, coeffs, C.PS_TOP_SCALE, outs)
    he.he_sync(st.ctx)
    for i, c in enumerate(cts):
        want = C.ps_eval_deg15(c, coeffs, st.oracle_relin_key(), P)
        assert outs[i].level == want["level"] and outs[i].scale == want["scale"]
        assert np.array_equal(st.from_gpu(outs[i]), want["c"])


def test_ps15_gelu_coefficients():
    """The distribution-fitted GELU coefficients (zeros above degree 8) on the
    same engine: 3 ciphertexts of normal inputs, residue for residue."""
    from homomorphic_encrypted_transformer_b200 import gelu as G

    he = lib()
    st = Setup(12, 8, 3, 3, seed=34)
    P = st.P
    coeffs = G.fit()
    st.upload_relin()
    cts = [st.encrypt(S.normal_slots(st.seed, P.n_slots, G.input_mean(), 1.0, G.LO, G.HI, i), 8, ct_id=i)
           for i in range(3)]
    xs = [st.to_gpu(c) for c in cts]
    outs = [st.empty_gpu(8) for _ in cts]
    he.he_poly_eval_ps15(st.ctx, xs, coeffs, C.PS_TOP_SCALE, outs)
    he.he_sync(st.ctx)
    for i, c in enumerate(cts):
        want = C.ps_eval_deg15(c, coeffs, st.oracle_relin_key(), P)
        assert outs[i].level == want["level"] and outs[i].scale == want["scale"]
        assert np.array_equal(st.from_gpu(outs[i]), want["c"])


BSGS_SMALL = [(4, 4, 2, 2), (4, 4, 2, 3), (8, 2, 13, 2)]


@pytest.mark.parametrize("bs,gs,n_in,n_grp", BSGS_SMALL, ids=["-".join(map(str, c)) for c in BSGS_SMALL])
def test_bsgs_small(bs, gs, n_in, n_grp):
    """y = W x by diagonals with BSGS on N=2^11: 16 features x 64 tokens,
    bs baby x gs giant steps, n_in input / 2 output blocks, n_grp token
    groups: two groups per staged pass, an odd group count (a last pass of
    one group), and 104 (input, baby step) terms per output."""
    he = lib()
    st = Setup(11, 3, 1, 3, seed=21)
    P = st.P
    n_feat, n_tok, n_out = 16, 64, 2
    level = 3
    W = S.weights(st.seed, (n_out * n_feat, n_in * n_feat), -0.05, 0.05)
    steps = sorted({n_tok * b for b in range(1, bs)} | {n_tok * bs * g for g in range(1, gs)})
    for s_ in steps:
        st.upload_rot(s_)
    keys = {s_: st.oracle_rot_key(s_) for s_ in steps}
    pt_slots = {}
    pts = np.zeros((n_out, n_in, gs, bs, level, P.N), dtype=np.uint64)
    for i in range(n_out):
        for j in range(n_in):
            blk = W[i * n_feat:(i + 1) * n_feat, j * n_feat:(j + 1) * n_feat]
            sl = C.bsgs_plaintext_slots(blk, n_feat, n_tok, bs, gs)
            for g in range(gs):
                for b in range(bs):
                    pts[i, j, g, b] = C.encode(sl[g, b], 2.0 ** 40, level, P)
    X, cts = [], []
    for t in range(n_grp):
        Xt = S.weights(st.seed, (n_in * n_feat, n_tok), -1, 1, 1 + t)
        X.append(Xt)
        for j in range(n_in):
            z = Xt[j * n_feat:(j + 1) * n_feat].reshape(-1).astype(np.complex128)
            cts.append(st.encrypt(z, level, ct_id=t * n_in + j))
    xs = [st.to_gpu(c) for c in cts]
    ys = [st.empty_gpu(level) for _ in range(n_grp * n_out)]
    he.he_pmult_accum_bsgs(st.ctx, xs, n_in, dev(pts), 2.0 ** 40, n_out, bs, gs, n_tok, n_grp, ys)
    he.he_sync(st.ctx)
    pt = lambda i, j, g, b: pts[i, j, g, b]
    for t in range(n_grp):
        Y = C.bsgs_matvec(cts[t * n_in:(t + 1) * n_in], pt, bs, gs, n_tok, keys, P, list(range(n_out)), 2.0 ** 40,
                          hoisted=True, one_moddown=True)
        want_plain = W @ X[t]
        for i in range(n_out):
            want = C.rescale(Y[i], P)
            got = ys[t * n_out + i]
            assert got.level == want["level"] and got.scale == want["scale"]
            assert np.array_equal(st.from_gpu(got), want["c"])
            dec = C.decrypt_decode(want, st.s, P).real.reshape(n_feat, n_tok)
            assert np.max(np.abs(dec - want_plain[i * n_feat:(i + 1) * n_feat])) < 1e-5
