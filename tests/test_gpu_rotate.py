"""GPU parity: switching keys and key-switched rotation vs the oracle, bit-exact
on every residue, plus decrypted slots within 1e-5 of the rolled plaintext."""
import numpy as np
import pytest
import torch

from oracle import ckks as C
import seeded_inputs as S
from tests.helpers import Setup, host, lib

pytestmark = pytest.mark.gpu


def test_keygen_matches_oracle_tiny():
    he = lib()
    st = Setup(12, 3, 1, 3, seed=S.master_seed(0))
    for step in (1, 2, -1):
        st.upload_rot(step)
        got = he.he_key_download(st.ctx, he.HE_KEY_ROTATION, step)
        b, a = st.oracle_rot_key(step)
        assert np.array_equal(got[:, 0], b) and np.array_equal(got[:, 1], a)
    st.upload_relin()
    got = he.he_key_download(st.ctx, he.HE_KEY_RELIN, 0)
    b, a = st.oracle_relin_key()
    assert np.array_equal(got[:, 0], b) and np.array_equal(got[:, 1], a)


def test_keygen_matches_oracle_full_size():
    he = lib()
    st = Setup(16, 24, 8, 3, seed=S.master_seed(1))
    st.upload_rot(12345)
    got = he.he_key_download(st.ctx, he.HE_KEY_ROTATION, 12345)
    b, a = st.oracle_rot_key(12345)
    assert np.array_equal(got[:, 0], b) and np.array_equal(got[:, 1], a)


def test_rotation_tiny_config():
    """N=2^12, 3+1 primes, steps {1, 2, -1}."""
    he = lib()
    st = Setup(12, 3, 1, 3, seed=S.master_seed(0))
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
        assert y.level == 3 and y.scale == ct["scale"]
        assert np.array_equal(st.from_gpu(y), want["c"])
        assert np.max(np.abs(C.decrypt_decode(want, st.s, P) - np.roll(z, -step))) < 1e-5


@pytest.mark.parametrize("level", [7, 5, 4, 1])
def test_rotation_mid_levels(level):
    """Several primes per digit (alpha = 3), partial last digits, level 1."""
    he = lib()
    st = Setup(11, 7, 3, 3, seed=44)
    P = st.P
    z = S.complex_slots(st.seed, P.n_slots, -1, 1)
    ct = st.encrypt(z, level)
    step = 5
    st.upload_rot(step)
    x = st.to_gpu(ct)
    y = st.empty_gpu(level)
    he.he_rotate(st.ctx, x, step, y)
    he.he_sync(st.ctx)
    want = C.rotate(ct, step, st.oracle_rot_key(step), P)
    assert np.array_equal(st.from_gpu(y), want["c"])


def test_rotation_errors():
    he = lib()
    st = Setup(12, 3, 1, 3, seed=3)
    z = S.complex_slots(st.seed, st.P.n_slots, -1, 1)
    x = st.to_gpu(st.encrypt(z, 3))
    y = st.empty_gpu(3)
    with pytest.raises(he.HEError) as ei:
        he.he_rotate(st.ctx, x, 7, y)
    assert ei.value.code == he.HE_ENOKEY
    with pytest.raises(he.HEError) as ei:
        he.he_rotate(st.ctx, x, 7, x)
    assert ei.value.code == he.HE_EINVAL
    x.is_ntt = False
    st.upload_rot(7)
    with pytest.raises(he.HEError) as ei:
        he.he_rotate(st.ctx, x, 7, y)
    assert ei.value.code == he.HE_EDOMAIN


def _rotation_batch_inputs(st, n_cts, n_keys):
    P = st.P
    steps = S.rotation_steps(st.seed, n_keys, 1, P.n_slots - 1)
    assign = S.step_assignment(st.seed, n_cts, n_keys)
    return steps, [steps[u] for u in assign]


def test_rotation_batch_full_size_sampled():
    """The rotation-batch workload (N=2^16, L=24, K=8, dnum=3, 64 ciphertexts,
    16 seeded keys) in the launch configuration the benchmark times; three
    ciphertexts chosen by seed are recomputed by the oracle."""
    he = lib()
    st = Setup(16, 24, 8, 3, seed=S.master_seed(1))
    P = st.P
    n_cts, n_keys = 64, 16
    steps, ct_steps = _rotation_batch_inputs(st, n_cts, n_keys)
    for s_ in steps:
        st.upload_rot(s_)
    sample = S.choose_groups(st.seed, n_cts, 3)
    # real encryptions at the sampled positions, uniform residues elsewhere
    # (a fresh encryption is computationally indistinguishable from uniform)
    xs, cts = [], {}
    uni = S.uniform_residues(st.seed, "ct_residues", P.q, P.N, lead=(n_cts, 2))
    for i in range(n_cts):
        if i in sample:
            z = S.complex_slots(st.seed, P.n_slots, -1, 1, i)
            cts[i] = (st.encrypt(z, 24, ct_id=i), z)
            xs.append(st.to_gpu(cts[i][0]))
        else:
            xs.append(st.to_gpu(C.make_ct(uni[i], 24, 2.0 ** 40)))
    ys = [st.empty_gpu(24) for _ in range(n_cts)]
    he.he_rotate_batch(st.ctx, xs, ct_steps, ys)
    he.he_sync(st.ctx)
    for i in sample:
        ct, z = cts[i]
        want = C.rotate(ct, ct_steps[i], st.oracle_rot_key(ct_steps[i]), P)
        assert np.array_equal(st.from_gpu(ys[i]), want["c"]), i
        assert np.max(np.abs(C.decrypt_decode(want, st.s, P) - np.roll(z, -ct_steps[i]))) < 1e-5
    # the uniform-residue ciphertexts: outputs canonical
    for i in range(n_cts):
        out = st.from_gpu(ys[i])
        assert np.all(out < np.array(P.q, dtype=np.uint64)[None, :, None])


def test_rotation_batch_host_buffers():
    """The host-buffer entry point gives the same residues as the device one."""
    he = lib()
    st = Setup(12, 3, 1, 3, seed=5)
    P = st.P
    n = 5
    steps = [1, 2, 1, 3, 2]
    for s_ in set(steps):
        st.upload_rot(s_)
    cts = [st.encrypt(S.complex_slots(st.seed, P.n_slots, -1, 1, i), 3, ct_id=i) for i in range(n)]
    h_in = np.stack([c["c"] for c in cts])
    h_out = np.zeros_like(h_in)
    he.he_rotate_batch_host(st.ctx, h_in, 3, steps, h_out)
    for i in range(n):
        want = C.rotate(cts[i], steps[i], st.oracle_rot_key(steps[i]), P)
        assert np.array_equal(h_out[i], want["c"])


def test_rotation_batch_host_buffers_pipelined():
    """21 ciphertexts pass the host-buffer entry in six chunks (2, 4, 5, 4,
    4, 2: both staging buffers reused, chunks of every size the plan makes);
    steps unsorted, repeated, and one identity rotation (step N/2, Galois
    element 1)."""
    he = lib()
    st = Setup(12, 3, 1, 3, seed=6)
    P = st.P
    n = 21
    steps = [3, 1, 2, 1, 7, 3, 2, P.n_slots, 1, 7, 2, 3, 1, 1, 2, 7, 3, 2, 1, 7, 3]
    for s_ in set(steps):
        if s_ != P.n_slots:
            st.upload_rot(s_)
    cts = [st.encrypt(S.complex_slots(st.seed, P.n_slots, -1, 1, i), 3, ct_id=i) for i in range(n)]
    h_in = np.stack([c["c"] for c in cts])
    h_out = np.zeros_like(h_in)
    he.he_rotate_batch_host(st.ctx, h_in, 3, steps, h_out)
    for i in range(n):
        if steps[i] == P.n_slots:
            assert np.array_equal(h_out[i], h_in[i])
            continue
        want = C.rotate(cts[i], steps[i], st.oracle_rot_key(steps[i]), P)
        assert np.array_equal(h_out[i], want["c"]), i
    # a second call reuses the staging buffers and the copy streams
    h_out2 = np.zeros_like(h_in)
    he.he_rotate_batch_host(st.ctx, h_in, 3, steps, h_out2)
    assert np.array_equal(h_out2, h_out)


def test_rotation_batch_host_buffers_full_size():
    """The host-buffer entry on the rotation batch (64 ciphertexts at
    N=2^16, level 24, 16 keys; chunks of 2 to 8 ordered by step) gives the device
    entry's residues, ciphertext for ciphertext."""
    he = lib()
    st = Setup(16, 24, 8, 3, seed=S.master_seed(1))
    P = st.P
    steps, ct_steps = _rotation_batch_inputs(st, 64, 16)
    for s_ in steps:
        st.upload_rot(s_)
    h_in = S.uniform_residues(st.seed, "ct_residues", P.q, P.N, lead=(64, 2))
    x = torch.from_numpy(h_in.view(np.int64)).cuda()
    y = torch.empty_like(x)
    he.he_rotate_batch(st.ctx, [he.Ciphertext(x[i], 24, 2.0 ** 40) for i in range(64)], ct_steps,
                       [he.Ciphertext(y[i], 24, 2.0 ** 40) for i in range(64)])
    he.he_sync(st.ctx)
    h_out = np.zeros_like(h_in)
    he.he_rotate_batch_host(st.ctx, h_in, 24, ct_steps, h_out)
    assert np.array_equal(h_out, host(y).reshape(h_in.shape))


def test_rotation_batch_host_wire():
    """The packed wire entry (he_rotate_batch_host_wire): 21 packed
    ciphertexts in six chunks, steps unsorted and repeated and one identity
    rotation; unpacked, the outputs equal the oracle's rotations, and the
    packed output equals the host packing of the unpacked entry's output."""
    he = lib()
    st = Setup(12, 3, 1, 3, seed=7)
    P = st.P
    n = 21
    steps = [3, 1, 2, 1, 7, 3, 2, P.n_slots, 1, 7, 2, 3, 1, 1, 2, 7, 3, 2, 1, 7, 3]
    for s_ in set(steps):
        if s_ != P.n_slots:
            st.upload_rot(s_)
    cts = [st.encrypt(S.complex_slots(st.seed, P.n_slots, -1, 1, i), 3, ct_id=i) for i in range(n)]
    h_in = np.stack([c["c"] for c in cts])
    w_in = he.he_ct_pack(P.q, 3, P.log_n, h_in)
    w_out = np.zeros_like(w_in)
    he.he_rotate_batch_host_wire(st.ctx, w_in, 3, steps, w_out)
    got = he.he_ct_unpack(P.q, 3, P.log_n, w_out, n)
    for i in range(n):
        if steps[i] == P.n_slots:
            assert np.array_equal(got[i], h_in[i])
            continue
        want = C.rotate(cts[i], steps[i], st.oracle_rot_key(steps[i]), P)
        assert np.array_equal(got[i], want["c"]), i
    h_out = np.zeros_like(h_in)
    he.he_rotate_batch_host(st.ctx, h_in, 3, steps, h_out)
    assert np.array_equal(w_out, he.he_ct_pack(P.q, 3, P.log_n, h_out))


def test_rotation_batch_host_wire_full_size():
    """The packed wire entry on the rotation batch (64 ciphertexts at
    N = 2^16, level 24, 16 keys): 64% of the bytes cross the host link, and
    the unpacked outputs equal the device entry's, ciphertext for ciphertext."""
    he = lib()
    st = Setup(16, 24, 8, 3, seed=S.master_seed(1))
    P = st.P
    steps, ct_steps = _rotation_batch_inputs(st, 64, 16)
    for s_ in steps:
        st.upload_rot(s_)
    h_in = S.uniform_residues(st.seed, "ct_residues", P.q, P.N, lead=(64, 2))
    x = torch.from_numpy(h_in.view(np.int64)).cuda()
    y = torch.empty_like(x)
    he.he_rotate_batch(st.ctx, [he.Ciphertext(x[i], 24, 2.0 ** 40) for i in range(64)], ct_steps,
                       [he.Ciphertext(y[i], 24, 2.0 ** 40) for i in range(64)])
    he.he_sync(st.ctx)
    w_in = he.he_ct_pack(P.q, 24, 16, h_in)
    assert w_in.nbytes == 64 * 2 * (1 << 16) * (8 + 23 * 5)
    w_out = np.zeros_like(w_in)
    he.he_rotate_batch_host_wire(st.ctx, w_in, 24, ct_steps, w_out)
    assert np.array_equal(he.he_ct_unpack(P.q, 24, 16, w_out, 64), host(y).reshape(h_in.shape))


def _hoisted_case(st, level, n_in, steps):
    """he_rotate_hoisted of n_in encrypted inputs by `steps` against the
    oracle's rotate_hoisted, residue for residue; Galois element 1 copies."""
    he = lib()
    P = st.P
    eff = [s for s in steps if P.galois_elt(s) != 1]
    for s in sorted(set(eff)):
        st.upload_rot(s)
    keys = {s: st.oracle_rot_key(s) for s in eff}
    cts = [st.encrypt(S.complex_slots(st.seed, P.n_slots, -1, 1, i), level, ct_id=i) for i in range(n_in)]
    xs = [st.to_gpu(ct) for ct in cts]
    ys = [st.empty_gpu(level) for _ in range(n_in * len(steps))]
    he.he_rotate_hoisted(st.ctx, xs, steps, ys)
    he.he_sync(st.ctx)
    for i, ct in enumerate(cts):
        want = dict(zip(eff, C.rotate_hoisted(ct, eff, keys, P)))
        for k, s in enumerate(steps):
            y = ys[i * len(steps) + k]
            assert y.level == level and y.scale == ct["scale"]
            got = st.from_gpu(y)
            if P.galois_elt(s) == 1:
                assert np.array_equal(got, ct["c"])
            else:
                assert np.array_equal(got, want[s]["c"]), (i, s)
    return cts, ys


def test_rotation_hoisted_tiny():
    """Two inputs, steps {1, 2, -1, 0}: step 0 (Galois element 1) copies;
    every output also decrypts to the rolled slots."""
    st = Setup(12, 3, 1, 3, seed=S.master_seed(0))
    steps = [1, 2, -1, 0]
    cts, ys = _hoisted_case(st, 3, 2, steps)
    for i, ct in enumerate(cts):
        z = S.complex_slots(st.seed, st.P.n_slots, -1, 1, i)
        for k, s in enumerate(steps):
            got = C.make_ct(st.from_gpu(ys[i * len(steps) + k]), 3, ct["scale"])
            assert np.max(np.abs(C.decrypt_decode(got, st.s, st.P) - np.roll(z, -s))) < 1e-5


@pytest.mark.parametrize("level", [7, 5, 1])
def test_rotation_hoisted_mid_levels(level):
    """Several primes per digit (alpha = 3, 60-bit and 40-bit rows), partial
    last digits, level 1."""
    st = Setup(11, 7, 3, 3, seed=45)
    _hoisted_case(st, level, 3, [5, -3, 17])


def test_rotation_hoisted_chunks():
    """More outputs than one launch holds: 5 inputs x 20 steps (chunks of
    3 and 2 inputs), and 1 input x 70 steps (chunks of 64 and 6 steps)."""
    st = Setup(11, 3, 1, 3, seed=46)
    _hoisted_case(st, 3, 5, list(range(1, 21)))
    _hoisted_case(st, 2, 1, list(range(-35, 0)) + list(range(1, 36)))


def _sum_case(st, level, n_out, steps, with_base=True):
    """he_rotate_sum against the oracle: base + identity terms + rotate_sum of
    the key-switched terms, residue for residue."""
    he = lib()
    P = st.P
    G = len(steps)
    eff = [s for s in steps if P.galois_elt(s) != 1]
    for s in sorted(set(eff)):
        st.upload_rot(s)
    keys = {s: st.oracle_rot_key(s) for s in eff}
    slots = lambda i: S.complex_slots(st.seed, P.n_slots, -1, 1, i)
    zs = [st.encrypt(slots(100 + i), level, ct_id=100 + i) for i in range(n_out * G)]
    bs = [st.encrypt(slots(300 + o), level, ct_id=300 + o) for o in range(n_out)] if with_base else None
    ys = [st.empty_gpu(level) for _ in range(n_out)]
    he.he_rotate_sum(st.ctx, [st.to_gpu(z) for z in zs], steps, [st.to_gpu(b) for b in bs] if with_base else None,
                     ys)
    he.he_sync(st.ctx)
    qm = P.q[:level]
    for o in range(n_out):
        terms = zs[o * G:(o + 1) * G]
        ks = [(z, s) for z, s in zip(terms, steps) if P.galois_elt(s) != 1]
        parts = [z for z, s in zip(terms, steps) if P.galois_elt(s) == 1]
        if ks:
            parts.append(C.rotate_sum([z for z, _ in ks], [s for _, s in ks], keys, P))
        if with_base:
            parts.append(bs[o])
        want = parts[0]["c"]
        for p_ in parts[1:]:
            want = np.stack([C.add_rows(want[c], p_["c"][c], qm) for c in range(2)])
        assert ys[o].level == level and ys[o].scale == zs[0]["scale"]
        assert np.array_equal(st.from_gpu(ys[o]), want), o
    return zs, bs, ys


def test_rotation_sum_tiny():
    """Two sums of 3 rotations plus a base; the sums decrypt to the base plus
    the rolled slots.  Then an identity term (step 0) without a base."""
    st = Setup(12, 3, 1, 3, seed=S.master_seed(0))
    steps = [1, 2, -1]
    zs, bs, ys = _sum_case(st, 3, 2, steps)
    for o in range(2):
        want = S.complex_slots(st.seed, st.P.n_slots, -1, 1, 300 + o)
        for g, s in enumerate(steps):
            want = want + np.roll(S.complex_slots(st.seed, st.P.n_slots, -1, 1, 100 + o * 3 + g), -s)
        got = C.make_ct(st.from_gpu(ys[o]), 3, 2.0 ** 40)
        assert np.max(np.abs(C.decrypt_decode(got, st.s, st.P) - want)) < 1e-5
    _sum_case(st, 3, 2, [3, 0], with_base=False)


@pytest.mark.parametrize("level", [7, 4, 1])
def test_rotation_sum_mid_levels(level):
    st = Setup(11, 7, 3, 3, seed=47)
    _sum_case(st, level, 2, [5, -3, 17, 2])


def test_rotation_sum_chunks():
    """5 sums of 20 rotations: chunks of 3 and 2 outputs (60 and 40 key
    switches in summed mode)."""
    st = Setup(11, 3, 1, 3, seed=48)
    _sum_case(st, 3, 5, list(range(1, 21)))


def _sum_hoisted_case(st, level, n_in, steps):
    """he_rotate_sum_hoisted against the oracle: identity steps add the input,
    the others go through rotate_sum_hoisted; residue for residue."""
    he = lib()
    P = st.P
    eff = [s for s in steps if P.galois_elt(s) != 1]
    for s in sorted(set(eff)):
        st.upload_rot(s)
    keys = {s: st.oracle_rot_key(s) for s in eff}
    cts = [st.encrypt(S.complex_slots(st.seed, P.n_slots, -1, 1, 500 + i), level, ct_id=500 + i)
           for i in range(n_in)]
    ys = [st.empty_gpu(level) for _ in range(n_in)]
    he.he_rotate_sum_hoisted(st.ctx, [st.to_gpu(c) for c in cts], steps, ys)
    he.he_sync(st.ctx)
    qm = P.q[:level]
    for i, ct in enumerate(cts):
        parts = [ct] * (len(steps) - len(eff))
        if eff:
            parts.append(C.rotate_sum_hoisted(ct, eff, keys, P))
        want = parts[0]["c"]
        for p_ in parts[1:]:
            want = np.stack([C.add_rows(want[c], p_["c"][c], qm) for c in range(2)])
        assert ys[i].level == level and ys[i].scale == ct["scale"]
        assert np.array_equal(st.from_gpu(ys[i]), want), i
    return cts, ys


def test_rotation_sum_hoisted_tiny():
    """Rotate-and-sum of two ciphertexts over {1, 2, -1, 4}: bit-exact and
    decrypting to the summed rolled slots; then an identity step."""
    st = Setup(12, 3, 1, 3, seed=S.master_seed(0))
    steps = [1, 2, -1, 4]
    cts, ys = _sum_hoisted_case(st, 3, 2, steps)
    for i in range(2):
        z = S.complex_slots(st.seed, st.P.n_slots, -1, 1, 500 + i)
        got = C.make_ct(st.from_gpu(ys[i]), 3, 2.0 ** 40)
        assert np.max(np.abs(C.decrypt_decode(got, st.s, st.P) - sum(np.roll(z, -s) for s in steps))) < 1e-5
    _sum_hoisted_case(st, 3, 1, [0, 3])


@pytest.mark.parametrize("level", [7, 4, 1])
def test_rotation_sum_hoisted_mid_levels(level):
    st = Setup(11, 7, 3, 3, seed=49)
    _sum_hoisted_case(st, level, 2, [5, -3, 17])


@pytest.mark.parametrize("level,n_in", [(7, 4), (4, 8), (1, 4)])
def test_rotation_sum_hoisted_four_outputs_per_thread(level, n_in):
    """Rotate-and-sum of 4 or 8 ciphertexts over one step list: outputs in
    blocks of four share each key word (k_ks_inner_sum_mo), with 60-bit and
    40-bit rows, partial digits and level 1; residue for residue."""
    st = Setup(11, 7, 3, 3, seed=51)
    _sum_hoisted_case(st, level, n_in, [5, -3, 17, 0, 9])


def test_rotation_sum_hoisted_chunks():
    """5 ciphertexts x 20 steps: chunks of 3 and 2 inputs."""
    st = Setup(11, 3, 1, 3, seed=50)
    _sum_hoisted_case(st, 3, 5, list(range(1, 21)))


def _full_size_inputs(n_in):
    """The hoisted and rotate-and-sum cases of the benchmark: N = 2^16,
    level 24, K = 8, dnum = 3; n_in encrypted inputs and the rotation batch's
    16 seeded steps, with their keys uploaded."""
    st = Setup(16, 24, 8, 3, seed=S.master_seed(1))
    P = st.P
    steps = S.rotation_steps(st.seed, 16, 1, P.n_slots - 1)
    for s_ in steps:
        st.upload_rot(s_)
    zs = [S.complex_slots(st.seed, P.n_slots, -1, 1, 700 + i) for i in range(n_in)]
    cts = [st.encrypt(z, 24, ct_id=700 + i) for i, z in enumerate(zs)]
    return st, steps, zs, cts


def test_rotation_hoisted_full_size_sampled():
    """he_rotate_hoisted in the launch configuration of the hoisted benchmark
    case (4 ciphertexts x the 16 steps of the rotation batch: one chunk of 64
    outputs, 4 raised inputs, 3 digits); two (ciphertext, step) outputs chosen
    by seed are recomputed by the oracle, residue for residue, and decrypt to
    the rolled slots."""
    he = lib()
    n_in = 4
    st, steps, zs, cts = _full_size_inputs(n_in)
    P = st.P
    xs = [st.to_gpu(c) for c in cts]
    ys = [st.empty_gpu(24) for _ in range(n_in * len(steps))]
    he.he_rotate_hoisted(st.ctx, xs, steps, ys)
    he.he_sync(st.ctx)
    for o in S.choose_groups(st.seed + 11, n_in * len(steps), 2):
        i, k = divmod(o, len(steps))
        s_ = steps[k]
        want = C.rotate_hoisted(cts[i], [s_], {s_: st.oracle_rot_key(s_)}, P)[0]
        assert ys[o].level == 24 and ys[o].scale == cts[i]["scale"]
        assert np.array_equal(st.from_gpu(ys[o]), want["c"]), (i, s_)
        assert np.max(np.abs(C.decrypt_decode(want, st.s, P) - np.roll(zs[i], -s_))) < 1e-5
    q = np.array(P.q, dtype=np.uint64)[None, :, None]
    for y in ys:
        assert np.all(st.from_gpu(y) < q)


def test_rotation_sum_hoisted_full_size_sampled():
    """he_rotate_sum_hoisted in the launch configuration of the rotate-and-sum
    benchmark case (4 ciphertexts, each summed over the 16 steps of the
    rotation batch: 64 key switches in summed and hoisted mode); one output
    chosen by seed is recomputed by the oracle residue for residue.  Its slots
    are within 1e-5 of the summed rolled slots of the decrypted input (the
    key-switching noise of one ModDown); against the encoded plaintext the
    fresh-encryption noise of the input enters 16 times, so that comparison
    takes 1e-4."""
    he = lib()
    n_in = 4
    st, steps, zs, cts = _full_size_inputs(n_in)
    P = st.P
    ys = [st.empty_gpu(24) for _ in range(n_in)]
    he.he_rotate_sum_hoisted(st.ctx, [st.to_gpu(c) for c in cts], steps, ys)
    he.he_sync(st.ctx)
    (i,) = S.choose_groups(st.seed + 12, n_in, 1)
    keys = {s_: st.oracle_rot_key(s_) for s_ in steps}
    want = C.rotate_sum_hoisted(cts[i], steps, keys, P)
    assert ys[i].level == 24 and ys[i].scale == cts[i]["scale"]
    assert np.array_equal(st.from_gpu(ys[i]), want["c"])
    got = C.decrypt_decode(want, st.s, P)
    dec_in = C.decrypt_decode(cts[i], st.s, P)
    assert np.max(np.abs(got - sum(np.roll(dec_in, -s_) for s_ in steps))) < 1e-5
    assert np.max(np.abs(got - sum(np.roll(zs[i], -s_) for s_ in steps))) < 1e-4
    q = np.array(P.q, dtype=np.uint64)[None, :, None]
    for y in ys:
        assert np.all(st.from_gpu(y) < q)


def test_seeded_keygen_matches_oracle():
    """he_keygen_seeded: the library samples the secret and every key's
    random parts from the seed on the host; the keys equal the oracle's keys
    built from the oracle sampler's draws of the same seed, residue for
    residue, and a rotation with them decrypts under the seed's secret."""
    from oracle import sampler as R

    he = lib()
    P = C.Params(12, 3, 1, 3)
    ctx = he.he_ctx_create(12, 3, 1, 3)
    seed = 0x5EED0001
    steps = [1, 2, -1]
    he.he_keygen_seeded(ctx, seed, steps, True)
    s = R.secret(seed, P.N)
    assert (he.he_sample_secret(seed, 12) == s).all()
    for st in steps:
        a, e = R.key_draws(seed, P.galois_elt(st), P.mods, P.N, P.dnum)
        b_, a_ = C.rotation_key(s, st, a, e, P)
        got = he.he_key_download(ctx, he.HE_KEY_ROTATION, st)
        assert np.array_equal(got[:, 0], b_) and np.array_equal(got[:, 1], a_)
    a, e = R.key_draws(seed, 2, P.mods, P.N, P.dnum)
    b_, a_ = C.relin_key(s, a, e, P)
    got = he.he_key_download(ctx, he.HE_KEY_RELIN, 0)
    assert np.array_equal(got[:, 0], b_) and np.array_equal(got[:, 1], a_)
    # a ciphertext under the seed's secret rotates correctly with these keys
    pa, pe = S.public_key_draws(seed, P.q, P.N)
    pk = C.public_key(s, pa, pe, P)
    z = S.complex_slots(seed, P.n_slots, -1, 1)
    v, e0, e1 = S.encryption_draws(seed, 0, P.N)
    ct = C.make_ct(C.encrypt(pk, C.encode(z, 2.0 ** 40, 3, P), v, e0, e1, 3, P), 3, 2.0 ** 40)
    x = he.Ciphertext(torch.from_numpy(ct["c"].view(np.int64).copy()).cuda(), 3, 2.0 ** 40)
    y = he.Ciphertext(torch.empty_like(x.data), 3, 1.0)
    he.he_rotate(ctx, x, 2, y)
    he.he_sync(ctx)
    got = C.make_ct(host(y.data, (2, 3, P.N)), 3, y.scale)
    assert np.max(np.abs(C.decrypt_decode(got, s, P) - np.roll(z, -2))) < 1e-5
    with pytest.raises(he.HEError) as ei:  # the identity rotation has no key
        he.he_keygen_seeded(ctx, seed, [P.n_slots], False)
    assert ei.value.code == he.HE_EINVAL


def test_seeded_keygen_full_size():
    """One seeded rotation key and the relinearisation key at N = 2^16,
    L = 24, K = 8, dnum = 3 against the oracle."""
    from oracle import sampler as R

    he = lib()
    P = C.Params(16, 24, 8, 3)
    ctx = he.he_ctx_create(16, 24, 8, 3)
    seed = S.master_seed(1)
    he.he_keygen_seeded(ctx, seed, [12345], True)
    s = R.secret(seed, P.N)
    a, e = R.key_draws(seed, P.galois_elt(12345), P.mods, P.N, P.dnum)
    b_, a_ = C.rotation_key(s, 12345, a, e, P)
    got = he.he_key_download(ctx, he.HE_KEY_ROTATION, 12345)
    assert np.array_equal(got[:, 0], b_) and np.array_equal(got[:, 1], a_)
    a, e = R.key_draws(seed, 2, P.mods, P.N, P.dnum)
    b_, a_ = C.relin_key(s, a, e, P)
    got = he.he_key_download(ctx, he.HE_KEY_RELIN, 0)
    assert np.array_equal(got[:, 0], b_) and np.array_equal(got[:, 1], a_)
