"""GPU parity at the full workload sizes (N = 2^16, L = 24, K = 8, dnum = 3),
in the launch configuration of the workload, on outputs sampled by seed that
the oracle recomputes one by one:

  * degree-15 Paterson-Stockmeyer on 64 ciphertexts from level 24, slots in [-4, 0];
  * the FFN1 BSGS product, 768 -> 3072, 256 features x 128 tokens per
    ciphertext, 16 baby x 16 giant steps, level 12: one token group (128
    tokens), and sixteen token groups (2048 tokens) sharing the weights.

For the FFN the library call covers one output block, chosen by seed, for all
groups at once: every output block is an independent launch sequence of the
same shape, so this is the per-block configuration of the full product."""
import numpy as np
import pytest
import torch

from oracle import ckks as C
import seeded_inputs as S
from tests.helpers import Setup, dev, host, lib

pytestmark = pytest.mark.gpu


def test_ps15_full_size_sampled():
    he = lib()
    st = Setup(16, 24, 8, 3, seed=S.master_seed(4))
    P = st.P
    n = 64
    coeffs = S.poly_coeffs(st.seed, 15)
    st.upload_relin()
    sample = S.choose_groups(st.seed, n, 2)
    uni = S.uniform_residues(st.seed, "ct_residues", P.q, P.N, lead=(n, 2))
    cts, xs = {}, []
    for i in range(n):
        if i in sample:
            z = S.real_slots(st.seed, P.n_slots, -4.0, 0.0, i)
            cts[i] = (st.encrypt(z, 24, ct_id=i), z)
            xs.append(st.to_gpu(cts[i][0]))
        else:
            xs.append(st.to_gpu(C.make_ct(uni[i], 24, 2.0 ** 40)))
    outs = [st.empty_gpu(24) for _ in range(n)]
    he.he_poly_eval_ps15(st.ctx, xs, coeffs, C.PS_TOP_SCALE, outs)
    he.he_sync(st.ctx)
    rlk = st.oracle_relin_key()
    for i in sample:
        ct, z = cts[i]
        want = C.ps_eval_deg15(ct, coeffs, rlk, P)
        assert outs[i].level == 18 and outs[i].scale == want["scale"]
        assert np.array_equal(st.from_gpu(outs[i]), want["c"])
        got = C.decrypt_decode(want, st.s, P)
        assert np.max(np.abs(got - C.ps_eval_plain(z, coeffs))) < 1e-5


N_FEAT, N_TOK, BS, GS, N_IN, N_OUT, LEVEL = 256, 128, 16, 16, 3, 12, 12


def _ffn_case(n_groups, check_groups, workload_index):
    he = lib()
    st = Setup(16, 24, 8, 3, seed=S.master_seed(workload_index))
    P = st.P
    W = S.weights(st.seed, (N_OUT * N_FEAT, N_IN * N_FEAT), -0.05, 0.05)
    blk = S.choose_groups(st.seed + 1, N_OUT, 1)[0]  # sampled output block
    steps = sorted({N_TOK * b for b in range(1, BS)} | {N_TOK * BS * g for g in range(1, GS)})
    for s_ in steps:
        st.upload_rot(s_)
    # plaintext diagonals of block `blk`: coefficient residues to the device,
    # forward NTT there; the oracle transforms its own copy when it needs it
    d_pt = torch.empty((1, N_IN, GS, BS, LEVEL, P.N), dtype=torch.int64, device="cuda")
    slots = {}
    for j in range(N_IN):
        Wij = W[blk * N_FEAT:(blk + 1) * N_FEAT, j * N_FEAT:(j + 1) * N_FEAT]
        slots[j] = C.bsgs_plaintext_slots(Wij, N_FEAT, N_TOK, BS, GS)
        for g in range(GS):
            for b in range(BS):
                m = C.encode_coeffs(slots[j][g, b], 2.0 ** 40, P).astype(np.int64)
                d_pt[0, j, g, b] = dev(C.to_residues(m, P.q[:LEVEL]))
    he.he_ntt_fwd(st.ctx, d_pt, N_IN * GS * BS, LEVEL, 0)

    def pt(i, j, g, b):
        m = C.encode_coeffs(slots[j][g, b], 2.0 ** 40, P).astype(np.int64)
        return C.ntt_rows(C.to_residues(m, P.q[:LEVEL]), P.q[:LEVEL], P)

    X, cts = [], []
    for t in range(n_groups):
        Xt = S.weights(st.seed, (N_IN * N_FEAT, N_TOK), -1, 1, 1 + t)
        X.append(Xt)
        for j in range(N_IN):
            z = Xt[j * N_FEAT:(j + 1) * N_FEAT].reshape(-1).astype(np.complex128)
            cts.append(st.encrypt(z, LEVEL, ct_id=t * N_IN + j))
    xs = [st.to_gpu(c) for c in cts]
    ys = [st.empty_gpu(LEVEL) for _ in range(n_groups)]
    he.he_pmult_accum_bsgs(st.ctx, xs, N_IN, d_pt, 2.0 ** 40, 1, BS, GS, N_TOK, n_groups, ys)
    he.he_sync(st.ctx)
    keys = {s_: st.oracle_rot_key(s_) for s_ in steps}
    for t in check_groups:
        Y = C.bsgs_matvec(cts[t * N_IN:(t + 1) * N_IN], pt, BS, GS, N_TOK, keys, P, [0], 2.0 ** 40, hoisted=True,
                          one_moddown=True)
        want = C.rescale(Y[0], P)
        got = ys[t]
        assert got.level == LEVEL - 1 and got.scale == want["scale"]
        assert np.array_equal(st.from_gpu(got), want["c"])
        dec = C.decrypt_decode(want, st.s, P).real.reshape(N_FEAT, N_TOK)
        assert np.max(np.abs(dec - (W @ X[t])[blk * N_FEAT:(blk + 1) * N_FEAT])) < 1e-5


def test_bsgs_ffn1_128_tokens_full_size():
    _ffn_case(1, [0], 2)


def test_bsgs_ffn1_2048_tokens_sampled_groups():
    groups = S.choose_groups(S.master_seed(3), 16, 2)
    _ffn_case(16, groups, 3)
