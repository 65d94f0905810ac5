"""A seeded sweep of small parameter sets against the oracle, residue for
residue: ring dimensions 2^10 to 2^13, chains of 2 to 16 primes, 1 to 5
special primes (some more than a digit needs), 1 to 4 digits (full and
partial), levels drawn per set.
Each set runs a rotation batch (unsorted, repeated, negative and identity
steps; more ciphertexts than one key group holds), hoisted rotations, sums
of rotations with and without hoisting (output counts that do and do not
fill blocks of four), an HMult-relinearise-rescale batch and an in-place
rescale.  The point is the boundaries of the launch plans (key groups, sum
blocks, digit splits, chunks), not the workloads."""
import numpy as np
import pytest

from oracle import ckks as C
import seeded_inputs as S
from tests.helpers import Setup, lib
from tests.test_gpu_rotate import _hoisted_case, _sum_case, _sum_hoisted_case

pytestmark = pytest.mark.gpu

SETS = [(10, 2, 1, 2), (10, 5, 2, 3), (11, 6, 3, 2), (11, 9, 3, 3), (10, 7, 4, 2), (12, 4, 4, 1), (10, 8, 2, 4),
        (10, 12, 3, 4), (13, 3, 2, 2), (10, 16, 4, 4), (11, 10, 5, 2), (10, 3, 3, 3)]


@pytest.mark.parametrize("shape", SETS, ids=["-".join(map(str, s)) for s in SETS])
def test_sweep(shape):
    he = lib()
    log_n, L, K, dnum = shape
    seed = 900 + 31 * log_n + 7 * L + K + dnum
    rng = np.random.default_rng(seed)
    st = Setup(log_n, L, K, dnum, seed=seed)
    P = st.P
    level = int(rng.integers(2, L + 1)) if L > 1 else 1

    # rotation batch: 20 ciphertexts, 5 steps (one the identity), 18 of them
    # on one step so that the key group exceeds 16 entries
    steps_set = [1, -3, 5, 2 * P.n_slots - 1, P.n_slots]
    for s_ in steps_set[:4]:
        st.upload_rot(s_)
    n = 20
    steps = [steps_set[0]] * 18 + [steps_set[1], steps_set[4]]
    rng.shuffle(steps)
    cts = [st.encrypt(S.complex_slots(seed, P.n_slots, -1, 1, i), level, ct_id=i) for i in range(n)]
    xs = [st.to_gpu(c) for c in cts]
    ys = [st.empty_gpu(level) for _ in range(n)]
    he.he_rotate_batch(st.ctx, xs, [int(s_) for s_ in steps], ys)
    he.he_sync(st.ctx)
    for i in range(n):
        if P.galois_elt(int(steps[i])) == 1:
            assert np.array_equal(st.from_gpu(ys[i]), cts[i]["c"]), i
        else:
            want = C.rotate(cts[i], int(steps[i]), st.oracle_rot_key(int(steps[i])), P)
            assert np.array_equal(st.from_gpu(ys[i]), want["c"]), i

    # hoisted rotations, sums with and without hoisting
    _hoisted_case(st, level, 3, [5, -3, P.n_slots, 1])
    _sum_case(st, level, 2, [1, 5, -3])
    _sum_case(st, level, 1, [5, P.n_slots], with_base=False)
    _sum_hoisted_case(st, level, 4, [1, -3, 5])
    _sum_hoisted_case(st, level, 5, [5, P.n_slots, 1])

    # HMult-relinearise-rescale and an in-place rescale
    if level >= 2:
        st.upload_relin()
        a = [st.encrypt(S.complex_slots(seed, P.n_slots, -1, 1, 100 + i), level, ct_id=100 + i) for i in range(3)]
        for i in range(3):
            out = st.empty_gpu(level)
            he.he_hmult_relin_rescale(st.ctx, st.to_gpu(a[i]), st.to_gpu(a[(i + 1) % 3]), out)
            he.he_sync(st.ctx)
            want = C.hmult_relin_rescale(a[i], a[(i + 1) % 3], st.oracle_relin_key(), P)
            assert np.array_equal(st.from_gpu(out), want["c"]), i
        g = st.to_gpu(a[0])
        he.he_rescale(st.ctx, g)
        he.he_sync(st.ctx)
        assert g.level == level - 1
        assert np.array_equal(st.from_gpu(g), C.rescale(a[0], P)["c"])
