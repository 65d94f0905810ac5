"""GPU parity of one encrypted attention head against the oracle, residue
for residue: the scores of 4 token offsets, their shifted exponentials by the
degree-15 engine, and A x V (N = 2^11, 16 features x 32 tokens)."""
import math

import numpy as np
import pytest

from oracle import ckks as C
import seeded_inputs as S
from tests.helpers import Setup, lib

pytestmark = pytest.mark.gpu

D, NT = 16, 32
EXP = [1.0 / math.factorial(k) for k in range(16)]


def test_attention_head_small():
    he = lib()
    st = Setup(11, 10, 4, 3, seed=S.master_seed(5))
    P = st.P
    Q = S.weights(st.seed, (D, NT), -0.25, 0.25, 1)
    K = S.weights(st.seed, (D, NT), -0.25, 0.25, 2)
    V = S.weights(st.seed, (D, NT), -0.25, 0.25, 3)
    q = st.encrypt(C.attention_pack(Q, False), P.L, ct_id=0)
    k = st.encrypt(C.attention_pack(K, True), P.L, ct_id=1)
    v = st.encrypt(C.attention_pack(V, True), P.L, ct_id=2)
    offsets = [0, 1, 5, 31]
    steps = sorted({o for o in offsets if o} | {x for st_ in C.attention_sum_steps(NT, D) for x in st_ if x})
    for s_ in steps:
        st.upload_rot(s_)
    st.upload_relin()
    keys = {s_: st.oracle_rot_key(s_) for s_ in steps}
    rlk = st.oracle_relin_key()
    gq, gk, gv = st.to_gpu(q), st.to_gpu(k), st.to_gpu(v)

    # scores
    sc = [st.empty_gpu(P.L) for _ in offsets]
    he.he_attention_scores(st.ctx, gq, gk, NT, D, offsets, sc)
    he.he_sync(st.ctx)
    want_s = C.attention_scores(q, k, NT, D, offsets, keys, rlk, P)
    for g, w in zip(sc, want_s):
        assert g.level == w["level"] == P.L - 1 and g.scale == w["scale"]
        assert np.array_equal(st.from_gpu(g), w["c"])

    # Softmax's exponential on scores shifted by -1 (|scores| <= 1 here)
    Ks = [int(C.round_half_away(np.float64(-1.0 * w["scale"]))) for w in want_s]
    for g, kk in zip(sc, Ks):
        he.he_add_const(st.ctx, g, kk)
    A = [st.empty_gpu(P.L) for _ in offsets]
    he.he_poly_eval_ps15(st.ctx, sc, EXP, C.PS_TOP_SCALE, A)
    he.he_sync(st.ctx)
    want_a = [C.ps_eval_deg15(C.add_const(w, kk, P), EXP, rlk, P) for w, kk in zip(want_s, Ks)]
    for g, w in zip(A, want_a):
        assert g.level == w["level"] and g.scale == w["scale"]
        assert np.array_equal(st.from_gpu(g), w["c"])

    # A x V
    out = st.empty_gpu(P.L)
    he.he_attention_output(st.ctx, A, gv, NT, offsets, out)
    he.he_sync(st.ctx)
    want_o = C.attention_av(want_a, v, offsets, keys, rlk, P)
    assert out.level == want_o["level"] and out.scale == want_o["scale"]
    assert np.array_equal(st.from_gpu(out), want_o["c"])
    # and the slots: sum over the 4 offsets of exp(score - 1) V
    got = C.decrypt_decode(want_o, st.s, P).real.reshape(D, 2 * NT)[:, :NT]
    Sc = Q.T @ K
    want = np.zeros((D, NT))
    for o in offsets:
        for t in range(NT):
            want[:, t] += np.exp(Sc[t, (t + o) % NT] - 1.0) * V[:, (t + o) % NT]
    assert np.max(np.abs(got - want)) < 1e-4


def test_attention_output_many_offsets():
    """A x V over 70 offsets (d = 4 features x 128 tokens at N = 2^11): the
    tensor sum runs in two launches, the second accumulating onto the first;
    every output residue equals the oracle's.  The weights are encryptions
    of seeded slots at level 3, v sits at level 4 (its rotations are read at
    the weights' level)."""
    he = lib()
    d, n_tok = 4, 128
    st = Setup(11, 6, 2, 3, seed=S.master_seed(5) + 1)
    P = st.P
    assert d * 2 * n_tok == P.n_slots
    offsets = list(range(70))
    for s_ in offsets[1:]:
        st.upload_rot(s_)
    st.upload_relin()
    keys = {s_: st.oracle_rot_key(s_) for s_ in offsets[1:]}
    rlk = st.oracle_relin_key()
    V = S.weights(st.seed, (d, n_tok), -0.5, 0.5, 3)
    v = st.encrypt(C.attention_pack(V, True), 4, ct_id=0)
    a = [st.encrypt(S.complex_slots(st.seed, P.n_slots, -1, 1, 10 + i), 3, ct_id=10 + i) for i in offsets]
    out = st.empty_gpu(3)
    he.he_attention_output(st.ctx, [st.to_gpu(x) for x in a], st.to_gpu(v), n_tok, offsets, out)
    he.he_sync(st.ctx)
    want = C.attention_av(a, v, offsets, keys, rlk, P)
    assert out.level == want["level"] == 2 and out.scale == want["scale"]
    assert np.array_equal(st.from_gpu(out), want["c"])


def test_attention_scores_two_features():
    """Scores with d = 2 features x 256 tokens at N = 2^11: the feature sum is
    one hoisted rotate-and-sum (d = 2 x 1), which ends in the scratch set
    and is copied to the outputs; residues equal the oracle's."""
    he = lib()
    d, n_tok = 2, 256
    st = Setup(11, 4, 2, 3, seed=S.master_seed(5) + 2)
    P = st.P
    assert d * 2 * n_tok == P.n_slots
    inner, outer = C.attention_sum_steps(n_tok, d)
    assert inner == [0, 2 * n_tok] and outer == [0]
    offsets = [0, 7, 255]
    steps = sorted({o for o in offsets if o} | {2 * n_tok})
    for s_ in steps:
        st.upload_rot(s_)
    st.upload_relin()
    keys = {s_: st.oracle_rot_key(s_) for s_ in steps}
    Q = S.weights(st.seed, (d, n_tok), -0.25, 0.25, 1)
    K = S.weights(st.seed, (d, n_tok), -0.25, 0.25, 2)
    q = st.encrypt(C.attention_pack(Q, False), P.L, ct_id=0)
    k = st.encrypt(C.attention_pack(K, True), P.L, ct_id=1)
    sc = [st.empty_gpu(P.L) for _ in offsets]
    he.he_attention_scores(st.ctx, st.to_gpu(q), st.to_gpu(k), n_tok, d, offsets, sc)
    he.he_sync(st.ctx)
    want = C.attention_scores(q, k, n_tok, d, offsets, keys, st.oracle_relin_key(), P)
    for g, w in zip(sc, want):
        assert g.level == w["level"] == P.L - 1 and g.scale == w["scale"]
        assert np.array_equal(st.from_gpu(g), w["c"])


def test_attention_errors():
    he = lib()
    st = Setup(11, 10, 4, 3, seed=68)
    P = st.P
    z = S.complex_slots(st.seed, P.n_slots, -1, 1)
    x = st.to_gpu(st.encrypt(z, P.L))
    y = st.to_gpu(st.encrypt(z, P.L, ct_id=1))
    out = [st.empty_gpu(P.L)]
    with pytest.raises(he.HEError) as ei:  # d * 2 * n_tok must be N/2
        he.he_attention_scores(st.ctx, x, y, 32, 8, [0], out)
    assert ei.value.code == he.HE_EINVAL
    with pytest.raises(he.HEError) as ei:  # no relinearisation key yet
        he.he_attention_scores(st.ctx, x, y, 32, 16, [0], out)
    assert ei.value.code == he.HE_ENOKEY
    st.upload_relin()
    with pytest.raises(he.HEError) as ei:  # offset outside [0, n_tok)
        he.he_attention_scores(st.ctx, x, y, 32, 16, [32], out)
    assert ei.value.code == he.HE_EINVAL
    with pytest.raises(he.HEError) as ei:  # no key for offset 3 nor the feature-sum steps
        he.he_attention_scores(st.ctx, x, y, 32, 16, [3], out)
    assert ei.value.code == he.HE_ENOKEY
    with pytest.raises(he.HEError) as ei:  # output aliases an input
        he.he_attention_output(st.ctx, [x], y, 32, [0], x)
    assert ei.value.code == he.HE_EINVAL
    # outputs that share storage only in part: views into one buffer (keys of
    # the feature sum present, so that only the overlap is wrong)
    for s_ in sorted({x for st_ in C.attention_sum_steps(32, 16) for x in st_ if x}):
        st.upload_rot(s_)
    big = st.empty_gpu(2 * P.L)
    half = (P.L - 1) * P.N  # less than one output's [2][L-1][N] words
    s0 = he.Ciphertext(big.data[:2 * P.L * P.N], P.L, 1.0)
    s1 = he.Ciphertext(big.data[half:half + 2 * P.L * P.N], P.L, 1.0)
    with pytest.raises(he.HEError) as ei:  # two score outputs overlap
        he.he_attention_scores(st.ctx, x, y, 32, 16, [0, 0], [s0, s1])
    assert ei.value.code == he.HE_EINVAL
    xin = he.Ciphertext(big.data[:2 * P.L * P.N], P.L, 2.0 ** 40)
    xin.data[:2 * P.L * P.N].copy_(x.data[:2 * P.L * P.N])
    part = he.Ciphertext(big.data[2 * P.L * P.N - 2 * P.N:], P.L, 1.0)  # tail of the input
    with pytest.raises(he.HEError) as ei:  # a score output overlaps the tail of q
        he.he_attention_scores(st.ctx, xin, y, 32, 16, [0], [part])
    assert ei.value.code == he.HE_EINVAL
    with pytest.raises(he.HEError) as ei:  # the output overlaps the tail of v
        he.he_attention_output(st.ctx, [y], xin, 32, [0], part)
    assert ei.value.code == he.HE_EINVAL


def test_attention_head_full_size_sampled():
    """One head in the launch configuration of the attention benchmark case:
    N = 2^16, level 24, d = 64 features x 256 tokens, all 256 token offsets
    (255 hoisted key rotations, 6 feature-sum rotations per offset, 256
    exponentials, A x V over every offset).  Two offsets chosen by seed are
    recomputed by the oracle: their scores and exponentials residue for
    residue.  The head's output sums all 256 offsets, more than the oracle
    recomputes in a test, so it is checked by its slots: within 1e-4 of fp64
    arithmetic on the plaintext matrices (the encryption noise of Q, K and V
    enters through the 64-feature sums and the 256-term output sum, about
    1e-5; the degree-15 Taylor exponential on [-2, 0] is within 1e-7)."""
    he = lib()
    d, n_tok = 64, 256
    st = Setup(16, 24, 8, 3, seed=S.master_seed(5))
    P = st.P
    assert d * 2 * n_tok == P.n_slots
    Q = S.weights(st.seed, (d, n_tok), -0.25, 0.25, 1)
    K = S.weights(st.seed, (d, n_tok), -0.25, 0.25, 2)
    V = S.weights(st.seed, (d, n_tok), -0.25, 0.25, 3)
    q = st.encrypt(C.attention_pack(Q, False), P.L, ct_id=0)
    k = st.encrypt(C.attention_pack(K, True), P.L, ct_id=1)
    v = st.encrypt(C.attention_pack(V, True), P.L, ct_id=2)
    offsets = list(range(n_tok))
    sum_steps = sorted({x for st_ in C.attention_sum_steps(n_tok, d) for x in st_ if x})
    for s_ in sorted(set(offsets[1:]) | set(sum_steps)):
        st.upload_rot(s_)
    st.upload_relin()
    gq, gk, gv = st.to_gpu(q), st.to_gpu(k), st.to_gpu(v)
    sc = [st.empty_gpu(P.L) for _ in offsets]
    he.he_attention_scores(st.ctx, gq, gk, n_tok, d, offsets, sc)
    he.he_sync(st.ctx)
    shift = [int(C.round_half_away(np.float64(-1.0 * x.scale))) for x in sc]
    for g, kk in zip(sc, shift):
        he.he_add_const(st.ctx, g, kk)
    A = [st.empty_gpu(P.L) for _ in offsets]
    he.he_poly_eval_ps15(st.ctx, sc, EXP, C.PS_TOP_SCALE, A)
    out = st.empty_gpu(P.L)
    he.he_attention_output(st.ctx, A, gv, n_tok, offsets, out)
    he.he_sync(st.ctx)

    rlk = st.oracle_relin_key()
    for o in S.choose_groups(st.seed + 13, n_tok, 2):
        keys = {s_: st.oracle_rot_key(s_) for s_ in ([o] if o else []) + sum_steps}
        (ws,) = C.attention_scores(q, k, n_tok, d, [o], keys, rlk, P)
        kk = int(C.round_half_away(np.float64(-1.0 * ws["scale"])))
        assert kk == shift[o]
        ws = C.add_const(ws, kk, P)
        assert sc[o].level == ws["level"] and sc[o].scale == ws["scale"]
        assert np.array_equal(st.from_gpu(sc[o]), ws["c"]), o
        wa = C.ps_eval_deg15(ws, EXP, rlk, P)
        assert A[o].level == wa["level"] and A[o].scale == wa["scale"]
        assert np.array_equal(st.from_gpu(A[o]), wa["c"]), o
        plain = np.array([Q[:, t] @ K[:, (t + o) % n_tok] for t in range(n_tok)])
        dec = C.decrypt_decode(wa, st.s, P).real.reshape(d, 2 * n_tok)[:, :n_tok]
        assert np.max(np.abs(dec - np.exp(plain - 1.0)[None, :])) < 1e-4

    got = C.decrypt_decode(C.make_ct(st.from_gpu(out), out.level, out.scale), st.s, P)
    got = got.real.reshape(d, 2 * n_tok)[:, :n_tok]
    Sc = Q.T @ K
    want = np.zeros((d, n_tok))
    for o in offsets:
        idx = (np.arange(n_tok) + o) % n_tok
        want += np.exp(Sc[np.arange(n_tok), idx] - 1.0)[None, :] * V[:, idx]
    assert np.max(np.abs(got - want)) < 1e-4
