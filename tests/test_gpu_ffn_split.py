"""The FFN1 product split by output group on a GPU: each rank's group is
computed by the library (he_pmult_accum_bsgs on that group's weight slice)
and the groups are put back in order as the AllGather does; the result must
equal the unsplit library product and the oracle's, residue for residue.
One GPU runs both ranks' products one after the other (their kernels never
wait on each other); the collective itself is covered on the host with gloo
(tests/test_ffn_split.py)."""
import numpy as np
import pytest
import torch

from homomorphic_encrypted_transformer_b200 import ffn_split as F
from oracle import ckks as C
import seeded_inputs as S
from tests.helpers import Setup, dev, lib

pytestmark = pytest.mark.gpu

N_FEAT, N_TOK, BS, GS, N_IN, N_OUT, N_GRP, LEVEL = 16, 64, 4, 4, 2, 3, 2, 3


def test_split_ffn_groups_equal_the_unsplit_product():
    he = lib()
    st = Setup(11, 3, 1, 3, seed=31)
    P = st.P
    W = S.weights(st.seed, (N_OUT * N_FEAT, N_IN * N_FEAT), -0.05, 0.05)
    steps = sorted({N_TOK * b for b in range(1, BS)} | {N_TOK * BS * g for g in range(1, GS)})
    for s_ in steps:
        st.upload_rot(s_)
    pts = np.zeros((N_OUT, N_IN, GS, BS, LEVEL, P.N), dtype=np.uint64)
    for i in range(N_OUT):
        for j in range(N_IN):
            sl = C.bsgs_plaintext_slots(W[i * N_FEAT:(i + 1) * N_FEAT, j * N_FEAT:(j + 1) * N_FEAT], N_FEAT, N_TOK,
                                        BS, GS)
            for g in range(GS):
                for b in range(BS):
                    pts[i, j, g, b] = C.encode(sl[g, b], 2.0 ** 40, LEVEL, P)
    cts = []
    for t in range(N_GRP):
        X = S.weights(st.seed, (N_IN * N_FEAT, N_TOK), -1, 1, 1 + t)
        for j in range(N_IN):
            z = X[j * N_FEAT:(j + 1) * N_FEAT].reshape(-1).astype(np.complex128)
            cts.append(st.encrypt(z, LEVEL, ct_id=t * N_IN + j))
    xs = [st.to_gpu(c) for c in cts]
    d_pt = dev(pts).reshape(N_OUT, N_IN, GS, BS, LEVEL, P.N)

    # unsplit product
    ys = [st.empty_gpu(LEVEL) for _ in range(N_GRP * N_OUT)]
    he.he_pmult_accum_bsgs(st.ctx, xs, N_IN, d_pt, 2.0 ** 40, N_OUT, BS, GS, N_TOK, N_GRP, ys)
    he.he_sync(st.ctx)
    whole = np.stack([st.from_gpu(y) for y in ys]).reshape(N_GRP, N_OUT, 2, LEVEL - 1, P.N)

    for world in (1, 2, 3):
        m = F.max_group(N_OUT, world)
        blocks = torch.zeros((world, N_GRP, m, 2, LEVEL - 1, P.N), dtype=torch.int64, device="cuda")
        for r in range(world):
            i0, i1 = F.output_group(N_OUT, world, r)
            local, lev, scale = F.ffn1_output_group(he, st.ctx, xs, N_IN, d_pt[i0:i1].contiguous(), 2.0 ** 40,
                                                    N_OUT, BS, GS, N_TOK, N_GRP, world, r)
            assert lev == LEVEL - 1 and scale == ys[0].scale
            blocks[r, :, :i1 - i0] = local
        got = F.assemble(blocks, N_OUT, world).cpu().numpy().view(np.uint64)
        assert np.array_equal(got, whole), world

    keys = {s_: st.oracle_rot_key(s_) for s_ in steps}
    for t in range(N_GRP):
        Y = C.bsgs_matvec(cts[t * N_IN:(t + 1) * N_IN], lambda i, j, g, b: pts[i, j, g, b], BS, GS, N_TOK, keys, P,
                          list(range(N_OUT)), 2.0 ** 40, hoisted=True, one_moddown=True)
        for i in range(N_OUT):
            assert np.array_equal(whole[t, i], C.rescale(Y[i], P)["c"]), (t, i)
