"""Python binding of libhe.so (the C ABI in include/he.h).

Argument marshalling only: every function here forwards to the C entry point
of the same name.  Device buffers are torch tensors (int64 storage holding
uint64 residues); host buffers are numpy arrays.  There is no fallback: if
libhe.so is missing the import fails.
"""
import ctypes
import os

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "libhe.so")

if not os.path.exists(_LIB_PATH):
    raise ImportError("libhe.so not built: run `python -m homomorphic_encrypted_transformer_b200.build` "
                      "(or __graft_entry__.build())")

_lib = ctypes.CDLL(_LIB_PATH)

HE_OK = 0
HE_EINVAL = -1
HE_ELEVEL = -2
HE_ENOKEY = -3
HE_EDOMAIN = -4
HE_ENOMEM = -5
HE_ECUDA = -6
HE_ETIMEOUT = -7
HE_KEY_ROTATION = 0
HE_KEY_RELIN = 1
HE_KEYGEN_SEEDED_A = 1

PROF = {"ntt_fwd_cols": 0, "ntt_fwd_rows": 1, "ntt_inv_rows": 2, "ntt_inv_cols": 3, "modup": 4, "ks_inner": 5,
        "moddown_conv": 6, "moddown_combine": 7, "automorph": 8, "elementwise": 9, "rescale": 10, "pmult": 11}

_CODES = {HE_EINVAL: "HE_EINVAL", HE_ELEVEL: "HE_ELEVEL", HE_ENOKEY: "HE_ENOKEY", HE_EDOMAIN: "HE_EDOMAIN",
          HE_ENOMEM: "HE_ENOMEM", HE_ECUDA: "HE_ECUDA", HE_ETIMEOUT: "HE_ETIMEOUT"}


class HEError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__("%s (%d): %s" % (_CODES.get(code, "?"), code, msg))
        self.code = code


class he_params(ctypes.Structure):
    _fields_ = [("log_n", ctypes.c_int), ("n_q", ctypes.c_int), ("n_p", ctypes.c_int), ("dnum", ctypes.c_int),
                ("q0_bits", ctypes.c_int), ("q_bits", ctypes.c_int), ("p_bits", ctypes.c_int),
                ("q", ctypes.POINTER(ctypes.c_uint64)), ("p", ctypes.POINTER(ctypes.c_uint64))]


class he_ct(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("level", ctypes.c_int), ("scale", ctypes.c_double),
                ("is_ntt", ctypes.c_int)]


_vp = ctypes.c_void_p
_i = ctypes.c_int
_u64p = ctypes.POINTER(ctypes.c_uint64)


def _sig(name, res, *args):
    f = getattr(_lib, name)
    f.restype = res
    f.argtypes = list(args)
    return f


_sig("he_derive_primes", _i, ctypes.POINTER(he_params), _vp, _vp)
_sig("he_ctx_create", _i, ctypes.POINTER(he_params), _vp, ctypes.POINTER(_vp))
_sig("he_ctx_destroy", _i, _vp)
_sig("he_set_stream", _i, _vp, _vp)
_sig("he_sync", _i, _vp)
_sig("he_last_error", ctypes.c_char_p, _vp)
_sig("he_get_primes", _i, _vp, _u64p)
_sig("he_get_psi", _i, _vp, _u64p)
_sig("he_keygen_upload", _i, _vp, _i, ctypes.c_int32, _vp, _vp, _vp)
_sig("he_key_download", _i, _vp, _i, ctypes.c_int32, _vp)
_sig("he_keygen_seeded", _i, _vp, ctypes.c_uint64, _vp, _i, _i)
_sig("he_keygen_seeded_ex", _i, _vp, ctypes.c_uint64, _vp, _i, _i, _i)
_sig("he_sample_key_a_seeded", _i, ctypes.c_uint64, ctypes.c_uint64, _i, _vp, _i, _i, _vp)
_sig("he_sample_secret", _i, ctypes.c_uint64, _i, _vp)
_sig("he_sample_key_draws", _i, ctypes.c_uint64, ctypes.c_uint64, _i, _vp, _i, _i, _vp, _vp)
_sig("he_gaussian_cdt", _i, _vp)
_sig("he_key_digits", _i, _vp)
_sig("he_ntt_fwd", _i, _vp, _vp, _i, _i, _i)
_sig("he_ntt_inv", _i, _vp, _vp, _i, _i, _i)
_sig("he_rotate", _i, _vp, ctypes.POINTER(he_ct), ctypes.c_int32, ctypes.POINTER(he_ct))
_sig("he_rotate_batch", _i, _vp, ctypes.POINTER(he_ct), _vp, ctypes.POINTER(he_ct), _i)
_sig("he_rotate_hoisted", _i, _vp, ctypes.POINTER(he_ct), _i, _vp, _i, ctypes.POINTER(he_ct))
_sig("he_rotate_sum", _i, _vp, ctypes.POINTER(he_ct), _i, _i, _vp, ctypes.POINTER(he_ct), ctypes.POINTER(he_ct))
_sig("he_rotate_sum_hoisted", _i, _vp, ctypes.POINTER(he_ct), _i, _vp, _i, ctypes.POINTER(he_ct))
_sig("he_attention_scores", _i, _vp, ctypes.POINTER(he_ct), ctypes.POINTER(he_ct), _i, _i, _vp, _i,
     ctypes.POINTER(he_ct))
_sig("he_attention_output", _i, _vp, ctypes.POINTER(he_ct), ctypes.POINTER(he_ct), _i, _vp, _i, ctypes.POINTER(he_ct))
_sig("he_rotate_batch_host", _i, _vp, _vp, _i, _vp, _vp, _i)
_sig("he_rotate_batch_host_wire", _i, _vp, _vp, _i, _vp, _vp, _i)
_sig("he_ct_wire_bytes", ctypes.c_longlong, _vp, _i, _i)
_sig("he_ct_pack", _i, _vp, _i, _i, _vp, _i, _vp)
_sig("he_ct_unpack", _i, _vp, _i, _i, _vp, _i, _vp)
_sig("he_hmult_relin_rescale", _i, _vp, ctypes.POINTER(he_ct), ctypes.POINTER(he_ct), ctypes.POINTER(he_ct))
_sig("he_rescale", _i, _vp, ctypes.POINTER(he_ct))
_sig("he_rescale_noalloc", _i, _vp, ctypes.POINTER(he_ct), ctypes.POINTER(he_ct))
_sig("he_add", _i, _vp, ctypes.POINTER(he_ct), ctypes.POINTER(he_ct), ctypes.POINTER(he_ct))
_sig("he_mul_const", _i, _vp, ctypes.POINTER(he_ct), ctypes.c_int64, ctypes.POINTER(he_ct))
_sig("he_add_const", _i, _vp, ctypes.POINTER(he_ct), ctypes.c_int64)
_sig("he_drop_level", _i, _vp, ctypes.POINTER(he_ct), _i, ctypes.POINTER(he_ct))
_sig("he_pmult_accum_bsgs", _i, _vp, ctypes.POINTER(he_ct), _i, _vp, ctypes.c_double, _i, _i, _i, _i, _i,
     ctypes.POINTER(he_ct))
_sig("he_poly_eval_ps15", _i, _vp, ctypes.POINTER(he_ct), _i, _vp, ctypes.c_double, ctypes.POINTER(he_ct))
_sig("he_profile_enable", _i, _vp, _i)
_sig("he_profile_read", _i, _vp, _i, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_longlong),
     ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_double))
_sig("he_profile_read_fp", _i, _vp, _i, ctypes.POINTER(ctypes.c_double))
_sig("he_launch_count", ctypes.c_longlong, _vp, _i)
_sig("he_probe_copy", _i, _vp, _vp, _vp, ctypes.c_size_t)
_sig("he_probe_int", _i, _vp, _i, _vp)
_sig("he_probe_fp", _i, _vp, _i, _vp)
_sig("he_probe_int_threads", ctypes.c_longlong, _vp)
_sig("he_probe_int_mults_per_iter", _i)

LIB_PATH = _LIB_PATH


class Context:
    """Owns an he_ctx*.  N, L, K, primes are host-side copies."""

    def __init__(self, ptr, params):
        self.ptr = ptr
        self.log_n = params.log_n
        self.N = 1 << params.log_n
        self.L = params.n_q
        self.K = params.n_p
        self.dnum = params.dnum
        pr = (ctypes.c_uint64 * (self.L + self.K))()
        _check(self, _lib.he_get_primes(ptr, pr))
        self.primes = [int(v) for v in pr]
        ps = (ctypes.c_uint64 * (self.L + self.K))()
        _check(self, _lib.he_get_psi(ptr, ps))
        self.psi = [int(v) for v in ps]

    def __del__(self):
        # at interpreter exit the module's globals may already be gone
        if getattr(self, "ptr", None) and _lib is not None:
            _lib.he_ctx_destroy(self.ptr)
            self.ptr = None


def _check(ctx, rc):
    if rc != HE_OK:
        msg = _lib.he_last_error(ctx.ptr if ctx is not None else None)
        raise HEError(rc, msg.decode() if msg else "")


def _stream_handle(stream):
    if stream is None:
        return None
    return ctypes.c_void_p(int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream))


class Ciphertext:
    """Device ciphertext: `data` is a torch tensor with room for [2][level][N]
    uint64 (any int64 tensor of at least that many elements, contiguous)."""

    def __init__(self, data, level, scale, is_ntt=True):
        self.data = data
        self.level = int(level)
        self.scale = float(scale)
        self.is_ntt = bool(is_ntt)

    def _c(self):
        return he_ct(ctypes.c_void_p(self.data.data_ptr()), self.level, self.scale, 1 if self.is_ntt else 0)

    def _update(self, c):
        self.level = c.level
        self.scale = c.scale
        self.is_ntt = bool(c.is_ntt)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if hasattr(t, "data_ptr") else ctypes.c_void_p(t.ctypes.data)


# ----------------------------------------------------------------- wrappers

def he_ctx_create(log_n, n_q, n_p, dnum, stream=None, **kw):
    prm, keep = _params(log_n, n_q, n_p, dnum, **kw)
    out = ctypes.c_void_p()
    rc = _lib.he_ctx_create(ctypes.byref(prm), _stream_handle(stream), ctypes.byref(out))
    if rc != HE_OK:
        raise HEError(rc, "he_ctx_create failed")
    return Context(out, prm)


def _params(log_n, n_q, n_p, dnum, q=None, p=None, q0_bits=0, q_bits=0, p_bits=0):
    prm = he_params(log_n, n_q, n_p, dnum, q0_bits, q_bits, p_bits, None, None)
    keep = []
    if q is not None:
        qa = (ctypes.c_uint64 * n_q)(*[int(v) for v in q])
        pa = (ctypes.c_uint64 * n_p)(*[int(v) for v in p])
        prm.q = ctypes.cast(qa, _u64p)
        prm.p = ctypes.cast(pa, _u64p)
        keep = [qa, pa]
    return prm, keep


def he_derive_primes(log_n, n_q, n_p, dnum, **kw):
    """Host-only: (primes, psi) the library derives for this parameter set."""
    prm, keep = _params(log_n, n_q, n_p, dnum, **kw)
    pr = np.zeros(n_q + n_p, dtype=np.uint64)
    ps = np.zeros(n_q + n_p, dtype=np.uint64)
    rc = _lib.he_derive_primes(ctypes.byref(prm), _ptr(pr), _ptr(ps))
    if rc != HE_OK:
        raise HEError(rc, "he_derive_primes: invalid parameters")
    return [int(v) for v in pr], [int(v) for v in ps]


def he_ctx_destroy(ctx):
    if ctx.ptr:
        _check(ctx, _lib.he_ctx_destroy(ctx.ptr))
        ctx.ptr = None


def he_last_error(ctx):
    m = _lib.he_last_error(ctx.ptr)
    return m.decode() if m else ""


def he_get_primes(ctx):
    return list(ctx.primes)


def he_get_psi(ctx):
    return list(ctx.psi)


def he_set_stream(ctx, stream):
    _check(ctx, _lib.he_set_stream(ctx.ptr, _stream_handle(stream)))


def he_sync(ctx):
    _check(ctx, _lib.he_sync(ctx.ptr))


def he_key_digits(ctx):
    return _lib.he_key_digits(ctx.ptr)


def he_keygen_upload(ctx, kind, step, s, a, e):
    s = np.ascontiguousarray(s, dtype=np.int8)
    a = np.ascontiguousarray(a, dtype=np.uint64)
    e = np.ascontiguousarray(e, dtype=np.int32)
    nd = he_key_digits(ctx)
    if s.size < ctx.N or a.size < nd * len(ctx.primes) * ctx.N or e.size < nd * ctx.N:
        raise ValueError("he_keygen_upload: s needs N, a digits*(L+K)*N and e digits*N entries")
    _check(ctx, _lib.he_keygen_upload(ctx.ptr, kind, int(step), _ptr(s), _ptr(a), _ptr(e)))


def he_keygen_seeded(ctx, seed, rot_steps, with_relin):
    st = np.ascontiguousarray(list(rot_steps), dtype=np.int32)
    _check(ctx, _lib.he_keygen_seeded(ctx.ptr, int(seed), _ptr(st), len(st), 1 if with_relin else 0))


def he_keygen_seeded_ex(ctx, seed, rot_steps, with_relin, flags):
    st = np.ascontiguousarray(list(rot_steps), dtype=np.int32)
    _check(ctx, _lib.he_keygen_seeded_ex(ctx.ptr, int(seed), _ptr(st), len(st), 1 if with_relin else 0,
                                         int(flags)))


def he_sample_secret(seed, log_n):
    """Host-only: the ternary secret of a seed (int8[2^log_n])."""
    out = np.empty(1 << log_n, dtype=np.int8)
    rc = _lib.he_sample_secret(int(seed), int(log_n), _ptr(out))
    if rc != HE_OK:
        raise HEError(rc, "he_sample_secret: bad arguments")
    return out


def he_sample_key_draws(seed, key_id, log_n, primes, digits):
    """Host-only: (a [digits][len(primes)][N] uint64, e [digits][N] int32) of one key."""
    pr = np.ascontiguousarray(primes, dtype=np.uint64)
    n = 1 << log_n
    a = np.empty((digits, len(pr), n), dtype=np.uint64)
    e = np.empty((digits, n), dtype=np.int32)
    rc = _lib.he_sample_key_draws(int(seed), int(key_id), int(log_n), _ptr(pr), len(pr), int(digits), _ptr(a),
                                  _ptr(e))
    if rc != HE_OK:
        raise HEError(rc, "he_sample_key_draws: bad arguments")
    return a, e


def he_sample_key_a_seeded(seed, key_id, log_n, primes, digits):
    """Host-only: the seeded a-half of one key, [digits][len(primes)][N] uint64."""
    pr = np.ascontiguousarray(primes, dtype=np.uint64)
    a = np.empty((digits, len(pr), 1 << log_n), dtype=np.uint64)
    rc = _lib.he_sample_key_a_seeded(int(seed), int(key_id), int(log_n), _ptr(pr), len(pr), int(digits), _ptr(a))
    if rc != HE_OK:
        raise HEError(rc, "he_sample_key_a_seeded: bad arguments")
    return a


def he_gaussian_cdt():
    """Host-only: the error sampler's 38 thresholds."""
    out = np.empty(38, dtype=np.uint64)
    rc = _lib.he_gaussian_cdt(_ptr(out))
    if rc != HE_OK:
        raise HEError(rc, "he_gaussian_cdt")
    return [int(v) for v in out]


def he_key_download(ctx, kind, step):
    nd = he_key_digits(ctx)
    out = np.empty((nd, 2, ctx.L + ctx.K, ctx.N), dtype=np.uint64)
    _check(ctx, _lib.he_key_download(ctx.ptr, kind, int(step), _ptr(out)))
    return out


def he_ntt_fwd(ctx, d, n_polys, n_limbs, first_prime):
    _check(ctx, _lib.he_ntt_fwd(ctx.ptr, _ptr(d), n_polys, n_limbs, first_prime))


def he_ntt_inv(ctx, d, n_polys, n_limbs, first_prime):
    _check(ctx, _lib.he_ntt_inv(ctx.ptr, _ptr(d), n_polys, n_limbs, first_prime))


def he_rotate(ctx, ct_in, step, ct_out):
    ci, co = ct_in._c(), ct_out._c()
    _check(ctx, _lib.he_rotate(ctx.ptr, ctypes.byref(ci), int(step), ctypes.byref(co)))
    ct_out._update(co)


def he_rotate_batch(ctx, cts_in, steps, cts_out):
    n = len(cts_in)
    ai = (he_ct * n)(*[c._c() for c in cts_in])
    ao = (he_ct * n)(*[c._c() for c in cts_out])
    st = np.ascontiguousarray(steps, dtype=np.int32)
    _check(ctx, _lib.he_rotate_batch(ctx.ptr, ai, _ptr(st), ao, n))
    for c, o in zip(cts_out, ao):
        c._update(o)


def he_rotate_hoisted(ctx, cts_in, steps, cts_out):
    """cts_out[i * len(steps) + s] = hoisted rotation of cts_in[i] by steps[s]."""
    n_in, n_steps = len(cts_in), len(steps)
    if len(cts_out) != n_in * n_steps:
        raise ValueError("he_rotate_hoisted: need len(cts_in) * len(steps) outputs")
    ai = (he_ct * max(1, n_in))(*[c._c() for c in cts_in])
    ao = (he_ct * max(1, len(cts_out)))(*[c._c() for c in cts_out])
    st = np.ascontiguousarray(steps, dtype=np.int32)
    _check(ctx, _lib.he_rotate_hoisted(ctx.ptr, ai, n_in, _ptr(st), n_steps, ao))
    for c, o in zip(cts_out, ao):
        c._update(o)


def he_rotate_sum(ctx, z, steps, base, cts_out):
    """cts_out[o] = base[o] + sum_g rot_{steps[g]}(z[o * len(steps) + g]), one
    ModDown per output; base may be None."""
    n_out, n_terms = len(cts_out), len(steps)
    if len(z) != n_out * n_terms or (base is not None and len(base) != n_out):
        raise ValueError("he_rotate_sum: need len(cts_out) * len(steps) terms and one base per output")
    az = (he_ct * max(1, len(z)))(*[c._c() for c in z])
    ab = (he_ct * n_out)(*[c._c() for c in base]) if base is not None else None
    ao = (he_ct * max(1, n_out))(*[c._c() for c in cts_out])
    st = np.ascontiguousarray(steps, dtype=np.int32)
    _check(ctx, _lib.he_rotate_sum(ctx.ptr, az, n_out, n_terms, _ptr(st), ab, ao))
    for c, o in zip(cts_out, ao):
        c._update(o)


def he_rotate_sum_hoisted(ctx, cts_in, steps, cts_out):
    """cts_out[i] = sum_s rot_{steps[s]}(cts_in[i]), one ModUp and one ModDown each."""
    if len(cts_out) != len(cts_in):
        raise ValueError("he_rotate_sum_hoisted: one output per input")
    n_in = len(cts_in)
    ai = (he_ct * max(1, n_in))(*[c._c() for c in cts_in])
    ao = (he_ct * max(1, n_in))(*[c._c() for c in cts_out])
    st = np.ascontiguousarray(steps, dtype=np.int32)
    _check(ctx, _lib.he_rotate_sum_hoisted(ctx.ptr, ai, n_in, _ptr(st), len(st), ao))
    for c, o in zip(cts_out, ao):
        c._update(o)


def he_attention_scores(ctx, q, k, n_tok, d, offsets, s_out):
    """s_out[i] = the scores of token offset offsets[i] (see he.h)."""
    if len(s_out) != len(offsets):
        raise ValueError("he_attention_scores: one output per offset")
    cq, ck = q._c(), k._c()
    ao = (he_ct * max(1, len(s_out)))(*[c._c() for c in s_out])
    off = np.ascontiguousarray(offsets, dtype=np.int32)
    _check(ctx, _lib.he_attention_scores(ctx.ptr, ctypes.byref(cq), ctypes.byref(ck), n_tok, d, _ptr(off), len(off), ao))
    for c, o in zip(s_out, ao):
        c._update(o)


def he_attention_output(ctx, a, v, n_tok, offsets, out):
    """out = sum_i HMRR(a[i], drop(rot_{offsets[i]}(v))) (see he.h)."""
    if len(a) != len(offsets):
        raise ValueError("he_attention_output: one weight ciphertext per offset")
    aa = (he_ct * max(1, len(a)))(*[c._c() for c in a])
    cv, co = v._c(), out._c()
    off = np.ascontiguousarray(offsets, dtype=np.int32)
    _check(ctx, _lib.he_attention_output(ctx.ptr, aa, ctypes.byref(cv), n_tok, _ptr(off), len(off), ctypes.byref(co)))
    out._update(co)


def he_rotate_batch_host(ctx, h_in, level, steps, h_out):
    """h_in, h_out: host arrays (numpy or pinned torch CPU tensors) of [n][2][level][N] uint64."""
    st = np.ascontiguousarray(steps, dtype=np.int32)
    need = len(st) * 2 * int(level) * ctx.N * 8
    if 1 <= level <= ctx.L and (_nbytes(h_in) < need or _nbytes(h_out) < need):  # (a bad level: the library's error)
        raise ValueError("he_rotate_batch_host: buffers shorter than %d bytes" % need)
    _check(ctx, _lib.he_rotate_batch_host(ctx.ptr, _ptr(h_in), level, _ptr(st), _ptr(h_out), len(st)))


def _nbytes(a):
    return a.nbytes if isinstance(a, np.ndarray) else a.numel() * a.element_size()


def _wire_primes(primes, level):
    pr = np.ascontiguousarray(list(primes)[:max(int(level), 0)], dtype=np.uint64)
    if len(pr) != level:
        raise ValueError("wire format: level %d needs %d primes, got %d" % (level, level, len(pr)))
    return pr


def he_ct_wire_bytes(primes, level, log_n):
    """Bytes of one ciphertext at `level` in the packed wire format (host only)."""
    pr = _wire_primes(primes, level)
    v = _lib.he_ct_wire_bytes(_ptr(pr), int(level), int(log_n))
    if v < 0:
        raise HEError(int(v), "he_ct_wire_bytes: bad arguments")
    return int(v)


def he_ct_pack(primes, level, log_n, cts):
    """Host [n][2][level][N] uint64 -> n packed ciphertexts (uint8, back to back)."""
    pr = _wire_primes(primes, level)
    a = np.ascontiguousarray(cts, dtype=np.uint64)
    per = 2 * level << log_n
    n = a.size // per
    if a.size != n * per:
        raise ValueError("he_ct_pack: expected [n][2][level][N] residues")
    out = np.empty(n * he_ct_wire_bytes(primes, level, log_n), dtype=np.uint8)
    rc = _lib.he_ct_pack(_ptr(pr), int(level), int(log_n), _ptr(a), n, _ptr(out))
    if rc != HE_OK:
        raise HEError(rc, "he_ct_pack: bad arguments or a residue not below its prime")
    return out


def he_ct_unpack(primes, level, log_n, packed, n):
    """n packed ciphertexts -> host [n][2][level][N] uint64."""
    pr = _wire_primes(primes, level)
    p = np.ascontiguousarray(packed, dtype=np.uint8)
    if p.size < n * he_ct_wire_bytes(primes, level, log_n):
        raise ValueError("he_ct_unpack: buffer shorter than n packed ciphertexts")
    out = np.empty((n, 2, level, 1 << log_n), dtype=np.uint64)
    rc = _lib.he_ct_unpack(_ptr(pr), int(level), int(log_n), _ptr(p), int(n), _ptr(out))
    if rc != HE_OK:
        raise HEError(rc, "he_ct_unpack: bad arguments")
    return out


def he_rotate_batch_host_wire(ctx, h_in, level, steps, h_out):
    """h_in, h_out: host buffers (numpy or pinned torch CPU uint8 tensors) of
    len(steps) packed ciphertexts each (he_ct_wire_bytes apiece)."""
    st = np.ascontiguousarray(steps, dtype=np.int32)
    need = len(st) * he_ct_wire_bytes(ctx.primes, level, ctx.log_n)
    if _nbytes(h_in) < need or _nbytes(h_out) < need:
        raise ValueError("he_rotate_batch_host_wire: buffers shorter than %d bytes" % need)
    _check(ctx, _lib.he_rotate_batch_host_wire(ctx.ptr, _ptr(h_in), level, _ptr(st), _ptr(h_out), len(st)))


def he_hmult_relin_rescale(ctx, a, b, out):
    ca, cb, co = a._c(), b._c(), out._c()
    _check(ctx, _lib.he_hmult_relin_rescale(ctx.ptr, ctypes.byref(ca), ctypes.byref(cb), ctypes.byref(co)))
    out._update(co)


def he_rescale(ctx, ct):
    c = ct._c()
    _check(ctx, _lib.he_rescale(ctx.ptr, ctypes.byref(c)))
    ct._update(c)


def he_rescale_noalloc(ctx, ct_in, ct_out):
    """Out-of-place rescale that allocates no device memory (see include/he.h)."""
    ci, co = ct_in._c(), ct_out._c()
    _check(ctx, _lib.he_rescale_noalloc(ctx.ptr, ctypes.byref(ci), ctypes.byref(co)))
    ct_out._update(co)


def he_add(ctx, a, b, out):
    ca, cb, co = a._c(), b._c(), out._c()
    _check(ctx, _lib.he_add(ctx.ptr, ctypes.byref(ca), ctypes.byref(cb), ctypes.byref(co)))
    out._update(co)


def he_mul_const(ctx, a, K, out):
    ca, co = a._c(), out._c()
    _check(ctx, _lib.he_mul_const(ctx.ptr, ctypes.byref(ca), int(K), ctypes.byref(co)))
    out._update(co)


def he_add_const(ctx, a, K):
    ca = a._c()
    _check(ctx, _lib.he_add_const(ctx.ptr, ctypes.byref(ca), int(K)))
    a._update(ca)


def he_drop_level(ctx, a, level, out):
    ca, co = a._c(), out._c()
    _check(ctx, _lib.he_drop_level(ctx.ptr, ctypes.byref(ca), int(level), ctypes.byref(co)))
    out._update(co)


def he_pmult_accum_bsgs(ctx, xs, n_in, d_pt, pt_scale, n_out, bs, gs, slot_stride, n_groups, ys):
    ax = (he_ct * len(xs))(*[c._c() for c in xs])
    ay = (he_ct * len(ys))(*[c._c() for c in ys])
    _check(ctx, _lib.he_pmult_accum_bsgs(ctx.ptr, ax, n_in, _ptr(d_pt), float(pt_scale), n_out, bs, gs,
                                         slot_stride, n_groups, ay))
    for c, o in zip(ys, ay):
        c._update(o)


def he_poly_eval_ps15(ctx, xs, coeffs, top_scale, outs):
    n = len(xs)
    ax = (he_ct * n)(*[c._c() for c in xs])
    ao = (he_ct * n)(*[c._c() for c in outs])
    cf = np.ascontiguousarray(coeffs, dtype=np.float64)
    assert cf.shape == (16,)
    _check(ctx, _lib.he_poly_eval_ps15(ctx.ptr, ax, n, _ptr(cf), float(top_scale), ao))
    for c, o in zip(outs, ao):
        c._update(o)


def he_profile_enable(ctx, enable):
    _check(ctx, _lib.he_profile_enable(ctx.ptr, 1 if enable else 0))


def he_profile_read(ctx, cls):
    """(total ms, launches, algorithmic HBM bytes, modular multiplications) of one class."""
    ms = ctypes.c_double()
    n = ctypes.c_longlong()
    b = ctypes.c_double()
    m = ctypes.c_double()
    _check(ctx, _lib.he_profile_read(ctx.ptr, cls, ctypes.byref(ms), ctypes.byref(n), ctypes.byref(b),
                                     ctypes.byref(m)))
    return ms.value, n.value, b.value, m.value


def he_profile_read_fp(ctx, cls):
    """Modular multiplications of one class that ran on the FP64 pipe."""
    m = ctypes.c_double()
    _check(ctx, _lib.he_profile_read_fp(ctx.ptr, cls, ctypes.byref(m)))
    return m.value


def he_launch_count(ctx, reset=False):
    return int(_lib.he_launch_count(ctx.ptr, 1 if reset else 0))


def he_probe_copy(ctx, dst, src, n_words):
    _check(ctx, _lib.he_probe_copy(ctx.ptr, _ptr(dst), _ptr(src), n_words))


def he_probe_int(ctx, iters, sink):
    _check(ctx, _lib.he_probe_int(ctx.ptr, iters, _ptr(sink)))


def he_probe_fp(ctx, iters, sink):
    _check(ctx, _lib.he_probe_fp(ctx.ptr, iters, _ptr(sink)))


def he_probe_int_threads(ctx):
    return int(_lib.he_probe_int_threads(ctx.ptr))


def he_probe_int_mults_per_iter():
    return int(_lib.he_probe_int_mults_per_iter())
