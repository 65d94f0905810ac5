"""Pins for the oracle's encrypted attention head: scores by token offset,
the degree-15 exponential, and A x V, decrypted against plaintext fp64
arithmetic on N = 2^11 (d = 16 features x n = 32 tokens, all 32 offsets)."""
import math

import numpy as np
import pytest

from oracle import ckks as C
import seeded_inputs as S

D, NT = 16, 32
EXP = [1.0 / math.factorial(k) for k in range(16)]


def _head(seed):
    P = C.Params(11, 10, 4, 3)
    assert D * 2 * NT == P.n_slots
    Q = S.weights(seed, (D, NT), -0.25, 0.25, 1)
    K = S.weights(seed, (D, NT), -0.25, 0.25, 2)
    V = S.weights(seed, (D, NT), -0.25, 0.25, 3)
    s = S.secret(seed, P.N)
    pa, pe = S.public_key_draws(seed, P.q, P.N)
    pk = C.public_key(s, pa, pe, P)

    def enc(z, i):
        v, e0, e1 = S.encryption_draws(seed, i, P.N)
        return C.make_ct(C.encrypt(pk, C.encode(z, 2.0 ** 40, P.L, P), v, e0, e1, P.L, P), P.L, 2.0 ** 40)

    q = enc(C.attention_pack(Q, False), 0)
    k = enc(C.attention_pack(K, True), 1)
    v = enc(C.attention_pack(V, True), 2)
    offsets = list(range(NT))
    steps = sorted({o for o in offsets if o} | {x for st in C.attention_sum_steps(NT, D) for x in st if x})
    keys = {}
    for st in steps:
        a, e = S.key_draws(seed, P.galois_elt(st), P.mods, P.N, P.dnum)
        keys[st] = C.rotation_key(s, st, a, e, P)
    a, e = S.key_draws(seed, 2, P.mods, P.N, P.dnum)
    rlk = C.relin_key(s, a, e, P)
    return P, s, Q, K, V, q, k, v, offsets, keys, rlk


@pytest.fixture(scope="module")
def head():
    P, s, Q, K, V, q, k, v, offsets, keys, rlk = _head(S.master_seed(5))
    scores = C.attention_scores(q, k, NT, D, offsets, keys, rlk, P)
    shifted = [C.add_const(x, int(C.round_half_away(np.float64(-1.0 * x["scale"]))), P) for x in scores]
    A = [C.ps_eval_deg15(x, EXP, rlk, P) for x in shifted]
    O = C.attention_av(A, v, offsets, keys, rlk, P)
    return dict(P=P, s=s, Q=Q, K=K, V=V, offsets=offsets, scores=scores, A=A, O=O, keys=keys, rlk=rlk, q=q, k=k, v=v)


def _scores_plain(Q, K, delta):
    return np.array([sum(Q[f, t] * K[f, (t + delta) % NT] for f in range(D)) for t in range(NT)])


def test_scores_by_offset_in_every_feature_block(head):
    P, s = head["P"], head["s"]
    for delta, sc in zip(head["offsets"], head["scores"]):
        got = C.decrypt_decode(sc, s, P).real.reshape(D, 2 * NT)
        want = _scores_plain(head["Q"], head["K"], delta)
        assert np.max(np.abs(got[:, :NT] - want[None, :])) < 1e-5
        assert np.max(np.abs(got[:, NT:])) < 1e-5


def test_softmax_exponential_by_the_degree15_polynomial(head):
    P, s = head["P"], head["s"]
    for delta, a in zip(head["offsets"], head["A"]):
        got = C.decrypt_decode(a, s, P).real.reshape(D, 2 * NT)
        want = np.exp(_scores_plain(head["Q"], head["K"], delta) - 1.0)
        assert np.max(np.abs(got[:, :NT] - want[None, :])) < 1e-5


def test_attention_output(head):
    P, s, Q, K, V = head["P"], head["s"], head["Q"], head["K"], head["V"]
    got = C.decrypt_decode(head["O"], s, P).real.reshape(D, 2 * NT)[:, :NT]
    Sc = Q.T @ K  # Sc[t][t'] = sum_f Q[f][t] K[f][t']
    want = V @ np.exp(Sc - 1.0).T  # O[f][t] = sum_t' exp(Sc[t][t'] - 1) V[f][t']
    assert head["O"]["level"] == 2
    assert np.max(np.abs(got - want)) < 1e-4


def test_mutation_unduplicated_keys_are_caught(head):
    """Planting K without the duplicated token axis loses the wrap-around
    of the token shift: the scores pin fails."""
    P, s = head["P"], head["s"]
    v, e0, e1 = S.encryption_draws(S.master_seed(5), 7, P.N)
    pa, pe = S.public_key_draws(S.master_seed(5), P.q, P.N)
    pk = C.public_key(s, pa, pe, P)
    k_bad = C.make_ct(C.encrypt(pk, C.encode(C.attention_pack(head["K"], False), 2.0 ** 40, P.L, P), v, e0, e1,
                                P.L, P), P.L, 2.0 ** 40)
    delta = 5
    sc = C.attention_scores(head["q"], k_bad, NT, D, [delta], head["keys"], head["rlk"], P)[0]
    got = C.decrypt_decode(sc, s, P).real.reshape(D, 2 * NT)[:, :NT]
    assert np.max(np.abs(got - _scores_plain(head["Q"], head["K"], delta)[None, :])) > 1e-2


def test_feature_sum_schedule_matches_doubling_rotations(head):
    """The feature sum as two hoisted rotate-and-sums (d = 4 x 4 here) and
    as log2(d) doubling rotations S <- S + rot_{2n 2^i}(S) decrypt to the
    same slots: the two schedules differ only in key-switching noise."""
    P, s, keys, rlk = head["P"], head["s"], head["keys"], head["rlk"]
    inner, outer = C.attention_sum_steps(NT, D)
    assert inner == [0, 64, 128, 192] and outer == [0, 256, 512, 768]
    delta = 3
    hoisted = C.attention_scores(head["q"], head["k"], NT, D, [delta], keys, rlk, P)[0]
    acc = C.hmult_relin_rescale(head["q"], C.rotate(head["k"], delta, keys[delta], P), rlk, P)
    for i in range(D.bit_length() - 1):
        st = 2 * NT * (1 << i)
        acc = C.add(acc, C.rotate(acc, st, keys[st], P), P)
    a = C.decrypt_decode(hoisted, s, P)
    b = C.decrypt_decode(acc, s, P)
    assert np.max(np.abs(a - b)) < 1e-6
    assert not np.array_equal(hoisted["c"], acc["c"])  # the residues do differ


def test_output_schedule_matches_per_offset_products(head):
    """A x V with the products' tensors summed and relinearised and rescaled
    once decrypts to the same slots as the sum of per-offset
    HMult-relinearise-rescale products: the two differ only in noise and
    rounding."""
    P, s, A, v, keys, rlk = head["P"], head["s"], head["A"], head["v"], head["keys"], head["rlk"]
    offsets = head["offsets"]
    nz = [o for o in offsets if o]
    rot = dict(zip(nz, C.rotate_hoisted(v, nz, keys, P)))
    plain = None
    for ad, o in zip(A, offsets):
        vv = C.drop_level(rot[o] if o in rot else v, ad["level"])
        t = C.hmult_relin_rescale(ad, vv, rlk, P)
        plain = t if plain is None else C.add(plain, t, P)
    O = head["O"]
    assert plain["level"] == O["level"] and plain["scale"] == O["scale"]
    got, want = C.decrypt_decode(O, s, P), C.decrypt_decode(plain, s, P)
    assert np.max(np.abs(got - want)) < 1e-6
    assert not np.array_equal(O["c"], plain["c"])
