"""The FFN1 product split by output group across ranks (AEGIS summary,
section 2.2: each device keeps one output group's weights, one AllGather of
the output ciphertexts): the partition of the output blocks, and the
AllGather over two gloo ranks on the host, whose gathered outputs must equal
the unsplit product residue for residue and in the unsplit order.  Each
rank's local product here is the oracle's; on a GPU it is the library's
he_pmult_accum_bsgs (tests/test_gpu_ffn_split.py)."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from homomorphic_encrypted_transformer_b200.ffn_split import (  # noqa: E402
    assemble, gather_output_groups, max_group, output_group)

N_FEAT, N_TOK, BS, GS, N_IN, N_OUT, N_GRP, LEVEL = 16, 64, 4, 4, 2, 3, 2, 3


def test_output_groups_partition_the_blocks():
    for n_out in (0, 1, 3, 12, 13, 192):
        for world in range(1, 9):
            got = [output_group(n_out, world, r) for r in range(world)]
            assert got[0][0] == 0 and got[-1][1] == n_out
            for (a0, a1), (b0, b1) in zip(got, got[1:]):
                assert a1 == b0  # contiguous, in rank order
            sizes = [i1 - i0 for i0, i1 in got]
            assert max(sizes) - min(sizes) <= 1 and max(sizes) == max_group(n_out, world)
            assert sizes == sorted(sizes, reverse=True)  # the larger groups first
    with pytest.raises(ValueError):
        output_group(12, 2, 2)


def test_assemble_drops_padding_and_restores_order():
    # 5 blocks over 3 ranks: groups of 2, 2, 1; rank r's block b tagged 10 r + b
    n_out, world = 5, 3
    m = max_group(n_out, world)
    blocks = torch.full((world, 2, m, 4), -1, dtype=torch.int64)
    for r in range(world):
        i0, i1 = output_group(n_out, world, r)
        for b in range(i1 - i0):
            blocks[r, :, b] = i0 + b
    out = assemble(blocks, n_out, world)
    assert out.shape == (2, n_out, 4)
    assert torch.equal(out[:, :, 0], torch.arange(n_out).expand(2, n_out))


def _case():
    """Small FFN product on N = 2^11 (16 features x 64 tokens per ciphertext,
    4 baby x 4 giant steps, 2 input and 3 output blocks, 2 token groups)."""
    from oracle import ckks as C
    import seeded_inputs as S

    seed = 31
    P = C.Params(11, 3, 1, 3)
    s = S.secret(seed, P.N)
    pa, pe = S.public_key_draws(seed, P.q, P.N)
    pk = C.public_key(s, pa, pe, P)
    W = S.weights(seed, (N_OUT * N_FEAT, N_IN * N_FEAT), -0.05, 0.05)
    steps = sorted({N_TOK * b for b in range(1, BS)} | {N_TOK * BS * g for g in range(1, GS)})
    keys = {}
    for st in steps:
        a, e = S.key_draws(seed, P.galois_elt(st), P.mods, P.N, P.dnum)
        keys[st] = C.rotation_key(s, st, a, e, P)
    pts = {}
    for i in range(N_OUT):
        for j in range(N_IN):
            sl = C.bsgs_plaintext_slots(W[i * N_FEAT:(i + 1) * N_FEAT, j * N_FEAT:(j + 1) * N_FEAT], N_FEAT, N_TOK,
                                        BS, GS)
            for g in range(GS):
                for b in range(BS):
                    pts[i, j, g, b] = C.encode(sl[g, b], 2.0 ** 40, LEVEL, P)
    cts = []
    for t in range(N_GRP):
        X = S.weights(seed, (N_IN * N_FEAT, N_TOK), -1, 1, 1 + t)
        for j in range(N_IN):
            v, e0, e1 = S.encryption_draws(seed, t * N_IN + j, P.N)
            z = X[j * N_FEAT:(j + 1) * N_FEAT].reshape(-1).astype(np.complex128)
            cts.append(C.make_ct(C.encrypt(pk, C.encode(z, 2.0 ** 40, LEVEL, P), v, e0, e1, LEVEL, P), LEVEL,
                                 2.0 ** 40))
    return C, P, keys, pts, cts


def _group_product(case, i0, i1):
    """Output blocks [i0, i1) of every token group: [N_GRP][i1-i0][2][LEVEL-1][N] as int64."""
    C, P, keys, pts, cts = case
    out = np.zeros((N_GRP, i1 - i0, 2, LEVEL - 1, P.N), dtype=np.uint64)
    for t in range(N_GRP):
        Y = C.bsgs_matvec(cts[t * N_IN:(t + 1) * N_IN], lambda i, j, g, b: pts[i, j, g, b], BS, GS, N_TOK, keys, P,
                          list(range(i0, i1)), 2.0 ** 40, hoisted=True, one_moddown=True)
        for i in range(i0, i1):
            out[t, i - i0] = C.rescale(Y[i], P)["c"]
    return torch.from_numpy(out.view(np.int64))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import datetime

    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        local = _group_product(_case(), *output_group(N_OUT, world, rank))
        full = gather_output_groups(local, N_OUT, world, rank)
        q.put((rank, full.numpy()))
    finally:
        dist.destroy_process_group()


def test_split_product_gathered_over_two_ranks_equals_unsplit_product():
    """3 output blocks over 2 gloo ranks (groups of 2 and 1: the gather pads
    rank 1's group): both ranks end with the unsplit product, bit-exact."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=600) for _ in procs)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    want = _group_product(_case(), 0, N_OUT).numpy()
    assert got[0].shape == want.shape
    assert np.array_equal(got[0], want) and np.array_equal(got[1], want)


def test_gather_with_one_rank_is_the_local_product():
    local = torch.arange(2 * 3 * 4, dtype=torch.int64).reshape(2, 3, 4)
    assert gather_output_groups(local, 3, 1, 0) is local
    with pytest.raises(ValueError):
        gather_output_groups(local[:, :2], 3, 1, 0)
