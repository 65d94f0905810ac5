"""GPU: argument and state errors of the C ABI come back as codes (nothing is
launched), and the context stays usable after each of them."""
import os

import numpy as np
import pytest
import torch

from oracle import ckks as C
import seeded_inputs as S
from tests.helpers import Setup, lib

pytestmark = pytest.mark.gpu


def _code(fn, *args):
    he = lib()
    with pytest.raises(he.HEError) as ei:
        fn(*args)
    return ei.value.code


def test_forced_allocation_failure_is_enomem():
    """HE_FAIL_ALLOC=1 makes every device allocation of the library fail:
    context creation reports HE_ENOMEM and leaks nothing observable."""
    he = lib()
    os.environ["HE_FAIL_ALLOC"] = "1"
    try:
        with pytest.raises(he.HEError) as ei:
            he.he_ctx_create(12, 3, 1, 3)
        assert ei.value.code == he.HE_ENOMEM
    finally:
        del os.environ["HE_FAIL_ALLOC"]
    ctx = he.he_ctx_create(12, 3, 1, 3)  # and works again without it
    he.he_ctx_destroy(ctx)


def test_unaligned_ciphertexts_are_rejected():
    he = lib()
    st = Setup(12, 3, 1, 3, seed=61)
    st.upload_rot(1)
    st.upload_relin()
    z = S.complex_slots(st.seed, st.P.n_slots, -1, 1)
    x = st.to_gpu(st.encrypt(z, 3))
    raw = torch.zeros(2 * 3 * st.P.N + 2, dtype=torch.int64, device="cuda")
    y = st.empty_gpu(3)
    # 8 bytes past a 16-byte boundary, and 16 bytes past a 32-byte one (the
    # transform passes move four residues per 256-bit access)
    for off in (1, 2):
        bad = he.Ciphertext(raw[off:off + 2 * 3 * st.P.N], 3, 1.0)
        assert _code(he.he_rotate, st.ctx, bad, 1, y) == he.HE_EINVAL
        assert _code(he.he_rotate, st.ctx, x, 1, bad) == he.HE_EINVAL
        assert _code(he.he_hmult_relin_rescale, st.ctx, x, x, bad) == he.HE_EINVAL
        assert _code(he.he_rescale, st.ctx, bad) == he.HE_EINVAL
        assert _code(he.he_ntt_fwd, st.ctx, raw[off:off + 3 * st.P.N], 1, 3, 0) == he.HE_EINVAL
    # the context still rotates correctly
    he.he_rotate(st.ctx, x, 1, y)
    he.he_sync(st.ctx)
    want = C.rotate(st.encrypt(z, 3), 1, st.oracle_rot_key(1), st.P)
    assert np.array_equal(st.from_gpu(y), want["c"])


def test_host_buffer_entry_errors():
    he = lib()
    st = Setup(12, 3, 1, 3, seed=62)
    st.upload_rot(1)
    h = np.zeros((2, 2, 3, st.P.N), dtype=np.uint64)
    out = np.zeros_like(h)
    assert _code(he.he_rotate_batch_host, st.ctx, h, 3, [1, 5], out) == he.HE_ENOKEY
    assert _code(he.he_rotate_batch_host, st.ctx, h, 9, [1, 1], out) == he.HE_EINVAL
    he.he_rotate_batch_host(st.ctx, h, 3, [1, 1], out)  # zero ciphertexts rotate to zero
    assert not out.any()
    # the packed wire entry: the same checks, and zero packs to zero
    w = he.he_ct_pack(st.P.q, 3, st.P.log_n, h)
    wout = np.full_like(w, 7)
    assert _code(he.he_rotate_batch_host_wire, st.ctx, w, 3, [1, 5], wout) == he.HE_ENOKEY
    with pytest.raises(ValueError):  # level beyond the chain: no wire size
        he.he_rotate_batch_host_wire(st.ctx, w, 9, [1, 1], wout)
    with pytest.raises(ValueError):  # buffers shorter than the ciphertexts
        he.he_rotate_batch_host_wire(st.ctx, w[:-1], 3, [1, 1], wout)
    he.he_rotate_batch_host_wire(st.ctx, w, 3, [1, 1], wout)
    assert not wout.any()
    he.he_rotate_batch_host_wire(st.ctx, w, 3, [], wout)  # no ciphertexts: nothing to do


def test_seeded_keygen_edge_cases():
    he = lib()
    st = Setup(11, 3, 1, 3, seed=66)
    he.he_keygen_seeded_ex(st.ctx, 5, [], False, he.HE_KEYGEN_SEEDED_A)  # no keys asked for: nothing made
    with pytest.raises(he.HEError) as ei:
        he.he_key_download(st.ctx, he.HE_KEY_RELIN, 0)
    assert ei.value.code == he.HE_ENOKEY
    assert _code(he.he_keygen_seeded_ex, st.ctx, 5, [st.P.n_slots], False, he.HE_KEYGEN_SEEDED_A) == he.HE_EINVAL


def test_bsgs_and_polynomial_errors():
    he = lib()
    st = Setup(12, 3, 1, 3, seed=63)
    z = S.complex_slots(st.seed, st.P.n_slots, -1, 1)
    x3 = st.to_gpu(st.encrypt(z, 3))
    ys = [st.empty_gpu(3)]
    pt = torch.zeros((1, 1, 2, 2, 3, st.P.N), dtype=torch.int64, device="cuda")
    # keys for the baby step (stride 1) and the giant step (stride 2) missing
    assert _code(he.he_pmult_accum_bsgs, st.ctx, [x3], 1, pt, 2.0 ** 40, 1, 2, 2, 1, 1, ys) == he.HE_ENOKEY
    # n_in * bs above 255
    assert _code(he.he_pmult_accum_bsgs, st.ctx, [x3], 1, pt, 2.0 ** 40, 1, 256, 1, 1, 1, ys) == he.HE_EINVAL
    # outputs and plaintexts 16 bytes past a 32-byte boundary
    raw = torch.zeros(2 * 3 * st.P.N + 2, dtype=torch.int64, device="cuda")
    bad = [he.Ciphertext(raw[2:], 3, 1.0)]
    assert _code(he.he_pmult_accum_bsgs, st.ctx, [x3], 1, pt, 2.0 ** 40, 1, 2, 2, 1, 1, bad) == he.HE_EINVAL
    pt_raw = torch.zeros(pt.numel() + 2, dtype=torch.int64, device="cuda")
    assert _code(he.he_pmult_accum_bsgs, st.ctx, [x3], 1, pt_raw[2:], 2.0 ** 40, 1, 2, 2, 1, 1, ys) == he.HE_EINVAL
    # mixed input levels
    x2 = st.to_gpu(st.encrypt(z, 2), room=3)
    st.upload_rot(1)
    assert _code(he.he_pmult_accum_bsgs, st.ctx, [x3, x2], 2, pt, 2.0 ** 40, 1, 2, 1, 1, 1, ys) == he.HE_ELEVEL
    # the polynomial needs level 7 and the relinearisation key
    coeffs = S.poly_coeffs(st.seed, 15)
    assert _code(he.he_poly_eval_ps15, st.ctx, [x3], coeffs, 2.0 ** 62, [st.empty_gpu(3)]) in (he.HE_ELEVEL,
                                                                                              he.HE_ENOKEY)
    st7 = Setup(12, 8, 3, 3, seed=64)
    x7 = st7.to_gpu(st7.encrypt(z, 8))
    assert _code(he.he_poly_eval_ps15, st7.ctx, [x7], coeffs, 2.0 ** 62, [st7.empty_gpu(8)]) == he.HE_ENOKEY
    raw7 = torch.zeros(2 * 8 * st7.P.N + 2, dtype=torch.int64, device="cuda")
    assert _code(he.he_poly_eval_ps15, st7.ctx, [x7], coeffs, 2.0 ** 62,
                 [he.Ciphertext(raw7[2:], 8, 1.0)]) == he.HE_EINVAL  # output 16 bytes off


def test_hoisted_rotation_errors():
    he = lib()
    st = Setup(12, 3, 1, 3, seed=65)
    st.upload_rot(1)
    z = S.complex_slots(st.seed, st.P.n_slots, -1, 1)
    x3 = st.to_gpu(st.encrypt(z, 3))
    x2 = st.to_gpu(st.encrypt(z, 2), room=3)
    y = [st.empty_gpu(3), st.empty_gpu(3)]
    assert _code(he.he_rotate_hoisted, st.ctx, [x3], [1, 4], y) == he.HE_ENOKEY
    assert _code(he.he_rotate_hoisted, st.ctx, [x3, x2], [1], y) == he.HE_ELEVEL
    assert _code(he.he_rotate_hoisted, st.ctx, [x3], [1, 1], [y[0], x3]) == he.HE_EINVAL  # aliases the input
    raw = torch.zeros(2 * 3 * st.P.N + 1, dtype=torch.int64, device="cuda")
    assert _code(he.he_rotate_hoisted, st.ctx, [x3], [1], [he.Ciphertext(raw[1:], 3, 1.0)]) == he.HE_EINVAL
    # the context still rotates correctly afterwards
    he.he_rotate_hoisted(st.ctx, [x3], [1], y[:1])
    he.he_sync(st.ctx)
    want = C.rotate_hoisted(st.encrypt(z, 3), [1], {1: st.oracle_rot_key(1)}, st.P)[0]
    assert np.array_equal(st.from_gpu(y[0]), want["c"])


def test_rotation_sum_errors():
    he = lib()
    st = Setup(12, 3, 1, 3, seed=66)
    st.upload_rot(1)
    z = S.complex_slots(st.seed, st.P.n_slots, -1, 1)
    x3 = st.to_gpu(st.encrypt(z, 3))
    x3b = st.to_gpu(st.encrypt(z, 3, scale=2.0 ** 30))
    y = [st.empty_gpu(3)]
    assert _code(he.he_rotate_sum, st.ctx, [x3, x3], [1, 4], None, y) == he.HE_ENOKEY
    assert _code(he.he_rotate_sum, st.ctx, [x3, x3b], [1, 1], None, y) == he.HE_ELEVEL  # scales differ
    assert _code(he.he_rotate_sum, st.ctx, [x3], [1], None, [x3]) == he.HE_EINVAL  # output aliases a term
    assert _code(he.he_rotate_sum, st.ctx, [x3] * 65, [1] * 65, None, y) == he.HE_EINVAL  # more than 64 terms
    assert _code(he.he_rotate_sum, st.ctx, [], [], None, y) == he.HE_EINVAL  # no terms and no base
    he.he_rotate_sum(st.ctx, [x3], [1], None, y)  # and still works
    he.he_sync(st.ctx)
    want = C.rotate_sum([st.encrypt(z, 3)], [1], {1: st.oracle_rot_key(1)}, st.P)
    assert np.array_equal(st.from_gpu(y[0]), want["c"])


def test_rotation_sum_hoisted_errors():
    he = lib()
    st = Setup(12, 3, 1, 3, seed=67)
    st.upload_rot(1)
    z = S.complex_slots(st.seed, st.P.n_slots, -1, 1)
    x3 = st.to_gpu(st.encrypt(z, 3))
    x2 = st.to_gpu(st.encrypt(z, 2), room=3)
    y = [st.empty_gpu(3), st.empty_gpu(3)]
    assert _code(he.he_rotate_sum_hoisted, st.ctx, [x3], [1, 4], y[:1]) == he.HE_ENOKEY
    assert _code(he.he_rotate_sum_hoisted, st.ctx, [x3, x2], [1], y) == he.HE_ELEVEL
    assert _code(he.he_rotate_sum_hoisted, st.ctx, [x3], [1], [x3]) == he.HE_EINVAL  # aliases the input
    assert _code(he.he_rotate_sum_hoisted, st.ctx, [x3], [], y[:1]) == he.HE_EINVAL  # no steps
    assert _code(he.he_rotate_sum_hoisted, st.ctx, [x3], [1] * 65, y[:1]) == he.HE_EINVAL  # above 64 steps
    he.he_rotate_sum_hoisted(st.ctx, [x3], [1, 1], y[:1])  # and still works
    he.he_sync(st.ctx)
    want = C.rotate_sum_hoisted(st.encrypt(z, 3), [1, 1], {1: st.oracle_rot_key(1)}, st.P)
    assert np.array_equal(st.from_gpu(y[0]), want["c"])
