"""Oracle: a plain, slow, obviously correct CPU implementation of RNS-CKKS.

TEST INFRASTRUCTURE ONLY.  Only tests/, the smoke check (__graft_entry__.smoke)
and bench.py's CPU-baseline / reference leg may import this package.  It
shares no code with the CUDA library: both sides receive the same random
draws from `seeded_inputs` and nothing else.

What the pages fix (AEGIS: Scaling Long-Sequence Homomorphic Encrypted
Transformer Inference, gist.science summary):
  * section 1 "Problem", item 2: ciphertexts are RNS polynomials split into
    modulus limbs along a modulus chain; rotation and key switching are the
    operations that tie the limbs together;
  * section 1 item 3: the scheme is CKKS;
  * section 1 item 1: tokens sit in fixed slots of a packed ciphertext;
  * section 2.2: the FFN is a local plaintext-weight x ciphertext polynomial
    product per output group;
  * section 2.3: Softmax is evaluated by a polynomial approximation;
  * the French page's summary: public-key encryption.
The pages give no formula, parameter or schedule below that.  Every step here
follows the textbook method it names:
  * RNS-CKKS: Cheon, Han, Kim, Kim, Song, "A Full RNS Variant of Approximate
    Homomorphic Encryption", SAC 2018 (CHKKS);
  * hybrid key switching with dnum digits: Han, Ki, "Better Bootstrapping for
    Approximate Homomorphic Encryption", CT-RSA 2020, section 3 (HK);
  * Paterson-Stockmeyer polynomial evaluation (1973);
  * hoisted rotations: Halevi, Shoup, "Faster Homomorphic Linear
    Transformations in HElib", CRYPTO 2018, section 5;
  * one ModDown for a sum of rotations: Bossuat, Mouchet, Troncoso-Pastoriza,
    Hubaux, "Efficient Bootstrapping for Approximate Homomorphic Encryption
    with Non-Sparse Keys", EUROCRYPT 2021, section 4.
Readings taken where the pages are silent are marked "Reading:" below.

Parity pins for every function live in tests/test_oracle_*.py.

Representation: an RNS polynomial is a numpy uint64 array [rows][N] of
canonical residues; `mods` lists the modulus of each row.  A ciphertext is a
dict {"c": uint64 [2][level][N], "level", "scale", "ntt"}.
"""
import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

from . import _core

_POOL = None


def _pool():
    global _POOL
    if _POOL is None:
        _POOL = ThreadPoolExecutor(max_workers=max(1, int(os.environ.get("ORACLE_THREADS", os.cpu_count() or 1))))
    return _POOL


def n_threads():
    return _pool()._max_workers


def _map(fn, items):
    items = list(items)
    if len(items) <= 1:
        return [fn(x) for x in items]
    return list(_pool().map(fn, items))


# --------------------------------------------------------------------------
# Number theory on Python integers
# --------------------------------------------------------------------------

_MR_BASES = (2, 3, 5, 7, 11, 13, 17, 19, 23, 29, 31, 37)


def is_prime(n):
    """Deterministic Miller-Rabin for n < 3.3e24 (bases 2..37, Sorenson-Webster 2015)."""
    if n < 2:
        return False
    for p in _MR_BASES:
        if n % p == 0:
            return n == p
    d, s = n - 1, 0
    while d % 2 == 0:
        d //= 2
        s += 1
    for a in _MR_BASES:
        x = pow(a, d, n)
        if x == 1 or x == n - 1:
            continue
        for _ in range(s - 1):
            x = x * x % n
            if x == n - 1:
                break
        else:
            return False
    return True


def prime_scan(bits, two_n):
    """Primes q = 1 (mod two_n) below 2^bits, largest first."""
    k = ((1 << bits) - 2) // two_n
    while k > 0:
        q = k * two_n + 1
        if q < (1 << bits) and is_prime(q):
            yield q
        k -= 1


def smallest_primitive_root(q, order):
    """The smallest primitive `order`-th root of unity mod q (order a power of 2
    dividing q-1).  Any primitive root x generates all of them as x^e, e odd;
    the smallest one is found by listing them all."""
    assert (q - 1) % order == 0
    half = order // 2
    g = 2
    while True:
        x = pow(g, (q - 1) // order, q)
        if pow(x, half, q) == q - 1:
            break
        g += 1
    x2 = x * x % q
    best, cur = x, x
    for _ in range(half - 1):
        cur = cur * x2 % q
        if cur < best:
            best = cur
    return best


def crt(residues, mods):
    """Integer in [0, prod(mods)) with the given residues (object array over columns)."""
    Q = math.prod(mods)
    acc = np.zeros(residues.shape[1], dtype=object)
    for r, q in zip(residues, mods):
        qh = Q // q
        coef = pow(qh, -1, q)
        acc = acc + ((r.astype(object) * coef) % q) * qh
    return acc % Q


def centered(x, Q):
    """Representative in (-Q/2, Q/2]."""
    x = np.asarray(x, dtype=object) % Q
    return np.where(x > Q // 2, x - Q, x)


# --------------------------------------------------------------------------
# Parameters
# --------------------------------------------------------------------------

class Params:
    """RNS-CKKS parameter set.

    Reading (the pages give no parameters): N = 2^log_n; the ciphertext
    modulus chain Q = q_0 ... q_{L-1} with q_0 of q0_bits and the others of
    q_bits; K special primes p_k of p_bits; every prime = 1 (mod 2N).  Primes
    are taken from a downward scan per bit size in this order: q_0, then
    p_0..p_{K-1}, then q_1..q_{L-1}.  With 60-bit q_0 and p this makes q_0 the
    largest 60-bit prime = 1 mod 2N and the p_k the next K below it; the
    40-bit q_i descend from the largest.

    Hybrid key switching (HK section 3): alpha = ceil(L / dnum); at level l
    (l limbs q_0..q_{l-1}) digit j holds q_{j alpha} .. q_{min((j+1) alpha, l)-1};
    the last digit may be partial.
    """

    def __init__(self, log_n, n_q, n_p, dnum, q0_bits=60, q_bits=40, p_bits=60, q=None, p=None):
        self.log_n = log_n
        self.N = 1 << log_n
        self.n_slots = self.N // 2
        self.L = n_q
        self.K = n_p
        self.dnum = dnum
        if q is None:
            scans = {}

            def take(bits):
                if bits not in scans:
                    scans[bits] = prime_scan(bits, 2 * self.N)
                return next(scans[bits])

            q0 = take(q0_bits)
            p = [take(p_bits) for _ in range(n_p)]
            q = [q0] + [take(q_bits) for _ in range(n_q - 1)]
        self.q = [int(v) for v in q]
        self.p = [int(v) for v in p]
        self.mods = self.q + self.p  # prime index space: 0..L-1 = q, L..L+K-1 = p
        self.alpha = -(-n_q // dnum)
        self.P = math.prod(self.p)
        self.psi = [smallest_primitive_root(m, 2 * self.N) for m in self.mods]

    def digits(self, level):
        a = self.alpha
        return [list(range(j * a, min((j + 1) * a, level))) for j in range(-(-level // a))]

    def n_digits(self, level=None):
        return len(self.digits(self.L if level is None else level))

    def psi_of(self, mod):
        return self.psi[self.mods.index(mod)]

    def galois_elt(self, step):
        """k = 5^(step mod n) mod 2N: the automorphism X -> X^k that rotates slots left by `step`."""
        return pow(5, step % self.n_slots, 2 * self.N)


# --------------------------------------------------------------------------
# Row-wise RNS arithmetic (each row of an array has its own modulus)
# --------------------------------------------------------------------------

def ntt_rows(a, mods, params):
    """Forward negacyclic NTT of every row (returns a new array)."""
    out = np.ascontiguousarray(a, dtype=np.uint64).copy()
    L = _core.lib()

    def one(i):
        row = out[i]
        L.ora_ntt_fwd(_core.ptr(row), params.log_n, mods[i], params.psi_of(mods[i]))

    _map(one, range(len(mods)))
    return out


def intt_rows(a, mods, params):
    out = np.ascontiguousarray(a, dtype=np.uint64).copy()
    L = _core.lib()

    def one(i):
        row = out[i]
        L.ora_ntt_inv(_core.ptr(row), params.log_n, mods[i], params.psi_of(mods[i]))

    _map(one, range(len(mods)))
    return out


def mul_rows(a, b, mods):
    a = np.ascontiguousarray(a, dtype=np.uint64)
    b = np.ascontiguousarray(b, dtype=np.uint64)
    out = np.empty_like(a)
    L = _core.lib()

    def one(i):
        L.ora_vec_mul(_core.ptr(a[i]), _core.ptr(b[i]), _core.ptr(out[i]), a.shape[1], mods[i])

    _map(one, range(len(mods)))
    return out


def scale_rows(a, consts, mods):
    """out[i] = a[i] * consts[i] mod mods[i] (consts are Python ints, reduced here)."""
    a = np.ascontiguousarray(a, dtype=np.uint64)
    out = np.empty_like(a)
    L = _core.lib()

    def one(i):
        L.ora_vec_scale(_core.ptr(a[i]), int(consts[i]) % mods[i], _core.ptr(out[i]), a.shape[1], mods[i])

    _map(one, range(len(mods)))
    return out


def add_rows(a, b, mods):
    q = np.array(mods, dtype=np.uint64)[:, None]
    return (a + b) % q


def sub_rows(a, b, mods):
    q = np.array(mods, dtype=np.uint64)[:, None]
    return (a + (q - b)) % q


def neg_rows(a, mods):
    q = np.array(mods, dtype=np.uint64)[:, None]
    return (q - a) % q


def to_residues(coeffs, mods):
    """Signed integer coefficients (int array or object array) -> [len(mods)][N] residues."""
    c = np.asarray(coeffs)
    out = np.empty((len(mods), c.shape[0]), dtype=np.uint64)
    if c.dtype == object:
        for i, q in enumerate(mods):
            out[i] = np.array([int(v) % q for v in c], dtype=np.uint64)
    else:
        c = c.astype(np.int64)
        for i, q in enumerate(mods):
            out[i] = np.mod(c, np.int64(q)).astype(np.uint64)
    return out


def automorph_coeff_rows(a, k, mods, params):
    """a(X) -> a(X^k) mod X^N + 1 on coefficient-domain rows."""
    a = np.ascontiguousarray(a, dtype=np.uint64)
    out = np.empty_like(a)
    L = _core.lib()

    def one(i):
        L.ora_automorph_coeff(_core.ptr(a[i]), _core.ptr(out[i]), params.log_n, k, mods[i])

    _map(one, range(len(mods)))
    return out


def automorph_ntt_rows(a, k, mods, params):
    """The automorphism applied to evaluation-domain rows, by its definition:
    back to coefficients, substitute X -> X^k, forward again."""
    return ntt_rows(automorph_coeff_rows(intt_rows(a, mods, params), k, mods, params), mods, params)


def base_conv(x, src, dst, centred=False):
    """Fast base conversion (CHKKS section 2.2) of coefficient-domain rows x
    (moduli `src`) onto the moduli `dst`, without overflow correction:
        Conv(x)_t = sum_i y_i (Q/q_i)  mod t,  y_i = [x_i (Q/q_i)^-1]_{q_i},
    Q = prod(src).  With centred=False, y_i is taken in [0, q_i) and the
    result is the residue of X + u Q, 0 <= u < len(src), X the CRT value of
    x in [0, Q).  With centred=True, y_i is taken in (-q_i/2, q_i/2) and the
    result is the residue of X_c + v Q with X_c the representative of x in
    (-Q/2, Q/2) and |v| <= len(src)/2."""
    Q = math.prod(src)
    qhat_inv = np.array([pow(Q // q, -1, q) for q in src], dtype=np.uint64)
    src_a = np.array(src, dtype=np.uint64)
    x = np.ascontiguousarray(x, dtype=np.uint64)
    out = np.empty((len(dst), x.shape[1]), dtype=np.uint64)
    L = _core.lib()

    def one(t):
        dst_a = np.array([dst[t]], dtype=np.uint64)
        qhat_mod = np.array([[(Q // q) % dst[t]] for q in src], dtype=np.uint64)
        o = np.empty((1, x.shape[1]), dtype=np.uint64)
        L.ora_base_conv(_core.ptr(x), len(src), _core.ptr(src_a), _core.ptr(qhat_inv), _core.ptr(o),
                        1, _core.ptr(dst_a), _core.ptr(qhat_mod), x.shape[1], 1 if centred else 0)
        out[t] = o[0]

    _map(one, range(len(dst)))
    return out


# --------------------------------------------------------------------------
# Encoding (CHKKS section 2 / Cheon-Kim-Kim-Song 2017 canonical embedding)
# --------------------------------------------------------------------------

def _slot_exponents(params):
    """e_j = 5^j mod 2N for j < n: slot j is the value at zeta^(e_j), zeta = exp(i pi / N)."""
    two_n = 2 * params.N
    e = np.empty(params.n_slots, dtype=np.int64)
    cur = 1
    for j in range(params.n_slots):
        e[j] = cur
        cur = cur * 5 % two_n
    return e


def round_half_away(x):
    return np.where(x >= 0, np.floor(x + 0.5), np.ceil(x - 0.5))


def encode_coeffs(z, scale, params):
    """Integer coefficients m_i = round((2 scale / N) Re sum_j z_j zeta^(-e_j i)).

    Computed by an FFT: with v the vector over odd exponents e (v at e_j = z_j,
    v at 2N - e_j = conj z_j), m_i = (scale / N) zeta^-i sum_m v_(2m+1) exp(-2 pi i m i / N)."""
    N = params.N
    z = np.asarray(z, dtype=np.complex128)
    assert z.shape == (params.n_slots,)
    e = _slot_exponents(params)
    v = np.zeros(N, dtype=np.complex128)  # v[m] = value at zeta^(2m+1)
    v[(e - 1) // 2] = z
    v[(2 * N - e - 1) // 2] = np.conj(z)
    i = np.arange(N)
    m = np.fft.fft(v) * np.exp(-1j * np.pi * i / N) * (scale / N)
    return round_half_away(m.real)


def encode_coeffs_direct(z, scale, params):
    """The O(N^2) definition of encode_coeffs (pin for small N)."""
    N = params.N
    e = _slot_exponents(params)
    i = np.arange(N)
    ang = -np.pi * np.outer(e, i) / N
    s = (np.asarray(z)[:, None] * np.exp(1j * ang)).sum(axis=0)
    return round_half_away(2.0 * scale / N * s.real)


def decode_coeffs(m, scale, params):
    """Slots z_j = m(zeta^(e_j)) / scale from (real-valued) coefficients m."""
    N = params.N
    m = np.asarray(m, dtype=np.float64)
    i = np.arange(N)
    vals = np.fft.ifft(m * np.exp(1j * np.pi * i / N)) * N  # vals[m] = m(zeta^(2m+1))
    e = _slot_exponents(params)
    return vals[(e - 1) // 2] / scale


def decode_coeffs_direct(m, scale, params):
    N = params.N
    e = _slot_exponents(params)
    i = np.arange(N)
    return (np.asarray(m, dtype=np.float64)[None, :] * np.exp(1j * np.pi * np.outer(e, i) / N)).sum(axis=1) / scale


def encode(z, scale, level, params):
    """Plaintext in the evaluation domain at `level` (rows q_0..q_{level-1})."""
    m = encode_coeffs(z, scale, params)
    if np.max(np.abs(m)) < 2.0 ** 62:
        coeffs = m.astype(np.int64)
    else:
        coeffs = np.array([int(v) for v in m], dtype=object)
    mods = params.q[:level]
    return ntt_rows(to_residues(coeffs, mods), mods, params)


def decode(pt_ntt, level, scale, params):
    mods = params.q[:level]
    coef = intt_rows(pt_ntt, mods, params)
    Q = math.prod(mods)
    vals = centered(crt(coef, mods), Q)
    return decode_coeffs(np.array([float(v) for v in vals]), scale, params)


# --------------------------------------------------------------------------
# Keys and encryption
# --------------------------------------------------------------------------

def secret_ntt(s, mods, params):
    """Evaluation-domain residues of the ternary secret (int8 coefficients)."""
    return ntt_rows(to_residues(s, mods), mods, params)


def public_key(s, a, e, params):
    """pk = (-a s + e, a) over q_0..q_{L-1} (a given in the evaluation domain).
    Reading: public-key encryption (French page, summary sentence)."""
    mods = params.q
    s_n = secret_ntt(s, mods, params)
    e_n = ntt_rows(to_residues(e, mods), mods, params)
    b = add_rows(neg_rows(mul_rows(a, s_n, mods), mods), e_n, mods)
    return b, a.copy()


def encrypt(pk, pt_ntt, v, e0, e1, level, params):
    """ct = (v pk0 + e0 + m, v pk1 + e1) at `level`."""
    mods = params.q[:level]
    v_n = ntt_rows(to_residues(v, mods), mods, params)
    e0_n = ntt_rows(to_residues(e0, mods), mods, params)
    e1_n = ntt_rows(to_residues(e1, mods), mods, params)
    c0 = add_rows(add_rows(mul_rows(v_n, pk[0][:level], mods), e0_n, mods), pt_ntt, mods)
    c1 = add_rows(mul_rows(v_n, pk[1][:level], mods), e1_n, mods)
    return np.stack([c0, c1])


def decrypt(ct, s, params):
    """Evaluation-domain plaintext m = c0 + c1 s at the ciphertext's level."""
    level = ct["level"]
    mods = params.q[:level]
    s_n = secret_ntt(s, mods, params)
    return add_rows(ct["c"][0], mul_rows(ct["c"][1], s_n, mods), mods)


def decrypt_decode(ct, s, params):
    return decode(decrypt(ct, s, params), ct["level"], ct["scale"], params)


def make_ct(c, level, scale):
    return {"c": c, "level": level, "scale": float(scale), "ntt": True}


def switching_key(s, s_prime_ntt, a, e, params):
    """Hybrid switching key from s' to s (HK section 3), over all L+K primes.

    For digit j (primes D_j at the top level):
        b_j = -a_j s + e_j + g_j s',   g_j = P on limbs q_i with i in D_j,
                                        g_j = 0 on the other q_i and on every p_k,
    i.e. g_j = P * (Q/Q_j) * [(Q/Q_j)^-1]_{Q_j}.  a_j is given (evaluation
    domain); e_j is a small integer polynomial.  Returns (b, a), each
    [n_digits][L+K][N]."""
    mods = params.mods
    s_n = secret_ntt(s, mods, params)
    digits = params.digits(params.L)
    b_all = np.empty((len(digits), len(mods), params.N), dtype=np.uint64)
    for j, D in enumerate(digits):
        e_n = ntt_rows(to_residues(e[j], mods), mods, params)
        b = add_rows(neg_rows(mul_rows(a[j], s_n, mods), mods), e_n, mods)
        g = [(params.P % m) if (r in D) else 0 for r, m in enumerate(mods)]
        b = add_rows(b, scale_rows(s_prime_ntt, g, mods), mods)
        b_all[j] = b
    return b_all, np.ascontiguousarray(a[: len(digits)]).copy()


def rotation_key(s, step, a, e, params):
    """Key for s' = sigma_k(s), k = 5^step mod 2N (slot rotation by `step`)."""
    k = params.galois_elt(step)
    mods = params.mods
    s_rot = automorph_coeff_rows(to_residues(s, mods), k, mods, params)
    return switching_key(s, ntt_rows(s_rot, mods, params), a, e, params)


def relin_key(s, a, e, params):
    """Key for s' = s^2."""
    mods = params.mods
    s_n = secret_ntt(s, mods, params)
    return switching_key(s, mul_rows(s_n, s_n, mods), a, e, params)


# --------------------------------------------------------------------------
# Key switching (HK section 3: ModUp, inner product, ModDown)
# --------------------------------------------------------------------------

def modup(d_coeff, d_ntt, D, level, params):
    """Digit D of d (coefficient rows d_coeff, evaluation rows d_ntt, both over
    q_0..q_{level-1}) raised to q_0..q_{level-1}, p_0..p_{K-1} (evaluation
    domain).  Rows in D keep d's own residues; every other row is the NTT of
    the fast base conversion from the primes of D."""
    src = [params.q[i] for i in D]
    tgt_rows = [i for i in range(level) if i not in D] + list(range(level, level + params.K))
    ext_mods = params.q[:level] + params.p
    tgt_mods = [ext_mods[r] for r in tgt_rows]
    conv = base_conv(d_coeff[D], src, tgt_mods)
    conv_n = ntt_rows(conv, tgt_mods, params)
    out = np.empty((level + params.K, params.N), dtype=np.uint64)
    for i in D:
        out[i] = d_ntt[i]
    for r, t in enumerate(tgt_rows):
        out[t] = conv_n[r]
    return out


def moddown(x_ntt, level, params):
    """(x - Conv_{P->q}([x]_P)) * P^-1 mod q_i for i < level, evaluation domain.
    x_ntt rows: q_0..q_{level-1}, p_0..p_{K-1}.

    Reading: the conversion from P takes its terms in the centred range
    (base_conv(centred=True)), so the result is round(x / P) - v with
    |v| <= K/2 and no systematic offset.  The floor form (terms in [0, p_k))
    biases every coefficient of u1 by about -(K+1)/2; multiplied by the secret
    that bias reaches ~4e-5 at slot 0 for N = 2^16, K = 8, scale 2^40,
    which is above the 1e-5 slot tolerance."""
    qm = params.q[:level]
    xp = intt_rows(x_ntt[level:], params.p, params)
    conv = ntt_rows(base_conv(xp, params.p, qm, centred=True), qm, params)
    diff = sub_rows(x_ntt[:level], conv, qm)
    return scale_rows(diff, [pow(params.P, -1, q) for q in qm], qm)


def key_switch(d_ntt, level, evk, params):
    """(u0, u1) with u0 + u1 s ~ d s' (mod Q_level), for evaluation-domain d at `level`."""
    b, a = evk
    qm = params.q[:level]
    ext_mods = qm + params.p
    key_rows = list(range(level)) + list(range(params.L, params.L + params.K))
    d_coeff = intt_rows(d_ntt, qm, params)
    u0 = np.zeros((level + params.K, params.N), dtype=np.uint64)
    u1 = np.zeros_like(u0)
    for j, D in enumerate(params.digits(level)):
        ext = modup(d_coeff, d_ntt, D, level, params)
        u0 = add_rows(u0, mul_rows(ext, b[j][key_rows], ext_mods), ext_mods)
        u1 = add_rows(u1, mul_rows(ext, a[j][key_rows], ext_mods), ext_mods)
    return moddown(u0, level, params), moddown(u1, level, params)


def rotate(ct, step, evk, params):
    """rot_step(ct) = (sigma_k(c0), 0) + KS_evk(sigma_k(c1)), k = 5^step mod 2N:
    slot j of the result holds slot j + step of the input (left rotation)."""
    level = ct["level"]
    qm = params.q[:level]
    k = params.galois_elt(step)
    c0 = automorph_ntt_rows(ct["c"][0], k, qm, params)
    c1 = automorph_ntt_rows(ct["c"][1], k, qm, params)
    u0, u1 = key_switch(c1, level, evk, params)
    return make_ct(np.stack([add_rows(c0, u0, qm), u1]), level, ct["scale"])


def rotate_hoisted(ct, steps, keys, params):
    """Hoisted rotations of one ciphertext (Halevi-Shoup, "Faster
    homomorphic linear transformations in HElib", section 5): the digits of
    c1 are raised to Q_level and P once, and each rotation applies sigma_k to
    the raised digits in the evaluation domain before its inner product:

        rot_step(ct) = (sigma_k(c0) + ModDown(sum_j sigma_k(ModUp_j(c1)) (.) evk_j.b),
                                      ModDown(sum_j sigma_k(ModUp_j(c1)) (.) evk_j.a)).

    sigma_k is a signed permutation of coefficients and the fast base
    conversion maps -x to -Conv(x) only up to a multiple of the digit's
    modulus, so the residues differ from rotate()'s: sigma_k(ModUp_j(c1)) and
    ModUp_j(sigma_k(c1)) agree on the digit's own rows and differ by
    m Q_{D_j} (|m| <= |D_j|) per coefficient on the others.  Both are
    lifts of sigma_k(c1)'s digit, so the result decrypts to the same rotated
    slots.  keys: step -> switching key.  Returns one ciphertext per step."""
    level = ct["level"]
    qm = params.q[:level]
    ext_mods = qm + params.p
    key_rows = list(range(level)) + list(range(params.L, params.L + params.K))
    c1 = ct["c"][1]
    c1_coeff = intt_rows(c1, qm, params)
    raised = [modup(c1_coeff, c1, D, level, params) for D in params.digits(level)]
    out = []
    for step in steps:
        k = params.galois_elt(step)
        b, a = keys[step]
        u0 = np.zeros((level + params.K, params.N), dtype=np.uint64)
        u1 = np.zeros_like(u0)
        for j, ext in enumerate(raised):
            ext_k = automorph_ntt_rows(ext, k, ext_mods, params)
            u0 = add_rows(u0, mul_rows(ext_k, b[j][key_rows], ext_mods), ext_mods)
            u1 = add_rows(u1, mul_rows(ext_k, a[j][key_rows], ext_mods), ext_mods)
        c0 = automorph_ntt_rows(ct["c"][0], k, qm, params)
        out.append(make_ct(np.stack([add_rows(c0, moddown(u0, level, params), qm), moddown(u1, level, params)]),
                           level, ct["scale"]))
    return out


def rotate_sum(zs, steps, keys, params):
    """sum_g rot_{steps[g]}(zs[g]) with a single ModDown per polynomial
    (the ModDown hoisting of Bossuat, Mouchet, Troncoso-Pastoriza, Hubaux,
    "Efficient Bootstrapping for Approximate Homomorphic Encryption with
    Non-Sparse Keys", EUROCRYPT 2021, section 4): each rotation's key inner
    product stays in Q_level and P, the products are summed there, and

        result = (sum_g sigma_g(z0_g) + ModDown(sum_g u0_g),  ModDown(sum_g u1_g)),
        u_g = sum_j ModUp_j(sigma_g(z1_g)) (.) evk_{g,j}.

    ModDown rounds once instead of once per rotation, so the residues differ
    from the sum of rotate() results by the rounding of the sum; with one
    rotation they are rotate()'s.  keys: step -> switching key."""
    level = zs[0]["level"]
    qm = params.q[:level]
    ext_mods = qm + params.p
    key_rows = list(range(level)) + list(range(params.L, params.L + params.K))
    u0 = np.zeros((level + params.K, params.N), dtype=np.uint64)
    u1 = np.zeros_like(u0)
    c0 = np.zeros((level, params.N), dtype=np.uint64)
    for z, step in zip(zs, steps):
        k = params.galois_elt(step)
        b, a = keys[step]
        c0 = add_rows(c0, automorph_ntt_rows(z["c"][0], k, qm, params), qm)
        d = automorph_ntt_rows(z["c"][1], k, qm, params)
        d_coeff = intt_rows(d, qm, params)
        for j, D in enumerate(params.digits(level)):
            ext = modup(d_coeff, d, D, level, params)
            u0 = add_rows(u0, mul_rows(ext, b[j][key_rows], ext_mods), ext_mods)
            u1 = add_rows(u1, mul_rows(ext, a[j][key_rows], ext_mods), ext_mods)
    return make_ct(np.stack([add_rows(c0, moddown(u0, level, params), qm), moddown(u1, level, params)]),
                   level, zs[0]["scale"])


def rotate_sum_hoisted(ct, steps, keys, params):
    """sum_s rot_{steps[s]}(ct) of one ciphertext with one ModUp and one
    ModDown: the raised digits of c1 are shared by every step (as in
    rotate_hoisted) and the inner products are added over Q_level and P
    before a single ModDown (as in rotate_sum):

        result = (sum_s sigma_s(c0) + ModDown(sum_s sum_j sigma_s(ModUp_j(c1)) (.) evk_{s,j}.b),
                                      ModDown(sum_s sum_j sigma_s(ModUp_j(c1)) (.) evk_{s,j}.a)).

    With one step it is rotate_hoisted's; against the sum of rotate_hoisted
    results it differs by the rounding of one ModDown instead of several.
    keys: step -> switching key."""
    level = ct["level"]
    qm = params.q[:level]
    ext_mods = qm + params.p
    key_rows = list(range(level)) + list(range(params.L, params.L + params.K))
    c1 = ct["c"][1]
    c1_coeff = intt_rows(c1, qm, params)
    raised = [modup(c1_coeff, c1, D, level, params) for D in params.digits(level)]
    u0 = np.zeros((level + params.K, params.N), dtype=np.uint64)
    u1 = np.zeros_like(u0)
    c0 = np.zeros((level, params.N), dtype=np.uint64)
    for step in steps:
        k = params.galois_elt(step)
        b, a = keys[step]
        c0 = add_rows(c0, automorph_ntt_rows(ct["c"][0], k, qm, params), qm)
        for j, ext in enumerate(raised):
            ext_k = automorph_ntt_rows(ext, k, ext_mods, params)
            u0 = add_rows(u0, mul_rows(ext_k, b[j][key_rows], ext_mods), ext_mods)
            u1 = add_rows(u1, mul_rows(ext_k, a[j][key_rows], ext_mods), ext_mods)
    return make_ct(np.stack([add_rows(c0, moddown(u0, level, params), qm), moddown(u1, level, params)]),
                   level, ct["scale"])


# --------------------------------------------------------------------------
# Multiplication, rescale, helpers
# --------------------------------------------------------------------------

def tensor(a, b, params):
    """(a0 b0, a0 b1 + a1 b0, a1 b1) at the common level."""
    assert a["level"] == b["level"]
    qm = params.q[: a["level"]]
    a0, a1 = a["c"]
    b0, b1 = b["c"]
    d0 = mul_rows(a0, b0, qm)
    d1 = add_rows(mul_rows(a0, b1, qm), mul_rows(a1, b0, qm), qm)
    d2 = mul_rows(a1, b1, qm)
    return d0, d1, d2


def rescale(ct, params):
    """Divide by the last prime q_{l-1} (CHKKS section 3.3):
        c'_i = (c_i - [c_{l-1}]_{q_{l-1}}) * q_{l-1}^-1 mod q_i,  i < l-1,
    with [c_{l-1}] the coefficient representative in (-q_{l-1}/2, q_{l-1}/2),
    so that the result is round(c / q_{l-1}).
    Reading: the rounding (centred) form; the floor form leaves a bias of 1/2
    per coefficient of c0 and c1, which the secret turns into a slot error of
    order 1e-8 per rescale at N = 2^12 and more at larger N."""
    level = ct["level"]
    ql = params.q[level - 1]
    qm = params.q[: level - 1]
    out = np.empty((2, level - 1, params.N), dtype=np.uint64)
    for k in range(2):
        last = intt_rows(ct["c"][k][level - 1: level], [ql], params)[0]
        neg = last > np.uint64(ql // 2)  # stands for last - ql
        lifted = []
        for q in qm:
            r = last % np.uint64(q)
            r = np.where(neg, (r + np.uint64(q) - np.uint64(ql % q)) % np.uint64(q), r)
            lifted.append(r.astype(np.uint64))
        lifted = ntt_rows(np.stack(lifted), qm, params)
        diff = sub_rows(ct["c"][k][: level - 1], lifted, qm)
        out[k] = scale_rows(diff, [pow(ql, -1, q) for q in qm], qm)
    return make_ct(out, level - 1, ct["scale"] / ql)


def relinearize(d, level, rlk, params):
    d0, d1, d2 = d
    qm = params.q[:level]
    u0, u1 = key_switch(d2, level, rlk, params)
    return np.stack([add_rows(d0, u0, qm), add_rows(d1, u1, qm)])


def hmult_relin_rescale(a, b, rlk, params):
    """Tensor, relinearise with the s^2 key, rescale.  Scale: (s_a * s_b) / q_{l-1}."""
    level = a["level"]
    c = relinearize(tensor(a, b, params), level, rlk, params)
    return rescale(make_ct(c, level, a["scale"] * b["scale"]), params)


def add(a, b, params):
    assert a["level"] == b["level"]
    qm = params.q[: a["level"]]
    return make_ct(np.stack([add_rows(a["c"][k], b["c"][k], qm) for k in range(2)]), a["level"], a["scale"])


def mul_const(ct, K, params):
    """Multiply by the integer K (reduced mod each q_i)."""
    qm = params.q[: ct["level"]]
    return make_ct(np.stack([scale_rows(ct["c"][k], [K] * len(qm), qm) for k in range(2)]), ct["level"], ct["scale"])


def add_const(ct, K, params):
    """Add the constant polynomial K (every slot gains K / scale)."""
    qm = params.q[: ct["level"]]
    q = np.array(qm, dtype=np.uint64)[:, None]
    kk = np.array([K % m for m in qm], dtype=np.uint64)[:, None]
    c0 = (ct["c"][0] + kk) % q
    return make_ct(np.stack([c0, ct["c"][1].copy()]), ct["level"], ct["scale"])


def drop_level(ct, level):
    """Keep limbs q_0..q_{level-1}."""
    assert level <= ct["level"]
    return make_ct(np.ascontiguousarray(ct["c"][:, :level]).copy(), level, ct["scale"])


# --------------------------------------------------------------------------
# Plaintext-weight x ciphertext product: diagonal method with BSGS
# (AEGIS summary section 2.2: the FFN is a local polynomial multiplication)
# --------------------------------------------------------------------------

def bsgs_plaintext_slots(W, n_feat, n_tok, bs, gs):
    """Slot vectors of the BSGS diagonals of one n_feat x n_feat block W.

    Feature-major packing: slot f * n_tok + t holds feature f of token t, so a
    slot rotation by n_tok * r shifts features by r.  Diagonal d:
    diag_d[f] = W[f, (f + d) mod n_feat].  With d = bs g + b, the plaintext for
    (g, b) is diag_d pre-rotated right by bs g features:
        pt_{g,b}[f * n_tok + t] = diag_{bs g + b}[(f - bs g) mod n_feat].
    Returns complex array [gs][bs][n_feat * n_tok]."""
    assert bs * gs == n_feat
    f = np.arange(n_feat)
    out = np.empty((gs, bs, n_feat * n_tok), dtype=np.complex128)
    for g in range(gs):
        for b in range(bs):
            d = bs * g + b
            diag = W[f, (f + d) % n_feat]
            pre = diag[(f - bs * g) % n_feat]
            out[g, b] = np.repeat(pre, n_tok)
    return out


def pmult_accum(xs, pts, level, params):
    """sum_k pts[k] (.) xs[k] (both polys), evaluation domain, exact mod q."""
    qm = params.q[:level]
    acc = np.zeros((2, level, params.N), dtype=np.uint64)
    for x, pt in zip(xs, pts):
        for c in range(2):
            acc[c] = add_rows(acc[c], mul_rows(x["c"][c], pt, qm), qm)
    return acc


def bsgs_matvec(X, pt, bs, gs, slot_stride, keys, params, outputs, pt_scale, hoisted=False, one_moddown=False):
    """Y_i = rescale( sum_g rot_{slot_stride bs g}( sum_{j,b} pt[i][j][g][b] (.) rot_{slot_stride b}(X_j) ) ).

    X: list of n_in ciphertexts at one level; pt: callable (i, j, g, b) ->
    evaluation-domain plaintext rows at that level, encoded at pt_scale;
    keys: step -> switching key.
    Baby-step rotations of each X_j are plain rotations, or with hoisted=True
    the hoisted rotations of rotate_hoisted (one ModUp per X_j).  The
    giant-step sum is over rotated partial sums Z_g: plain rotations added
    one by one, or with one_moddown=True Z_0 + rotate_sum(Z_1..Z_{gs-1}) (one
    ModDown per output).  One rescale follows.
    Reading: one rescale after the whole accumulation."""
    level = X[0]["level"]
    qm = params.q[:level]
    n_in = len(X)
    if hoisted:
        steps = [slot_stride * b for b in range(1, bs)]
        baby = [[X[j]] + rotate_hoisted(X[j], steps, keys, params) for j in range(n_in)]
    else:
        baby = [[X[j] if b == 0 else rotate(X[j], slot_stride * b, keys[slot_stride * b], params)
                 for b in range(bs)] for j in range(n_in)]
    Y = {}
    for i in outputs:
        zs = []
        for g in range(gs):
            xs, pts = [], []
            for j in range(n_in):
                for b in range(bs):
                    xs.append(baby[j][b])
                    pts.append(pt(i, j, g, b))
            zs.append(make_ct(pmult_accum(xs, pts, level, params), level, X[0]["scale"] * pt_scale))
        giant = [slot_stride * bs * g for g in range(1, gs)]
        if one_moddown and gs > 1:
            r = rotate_sum(zs[1:], giant, keys, params)
            parts = [zs[0], r]
        else:
            parts = [zs[0]] + [rotate(z, st, keys[st], params) for z, st in zip(zs[1:], giant)]
        acc = parts[0]
        for z in parts[1:]:
            acc = make_ct(np.stack([add_rows(acc["c"][c], z["c"][c], qm) for c in range(2)]), level, acc["scale"])
        Y[i] = acc
    return Y


# --------------------------------------------------------------------------
# One encrypted attention head (AEGIS summary section 2.3: Q x K^T, a
# polynomial Softmax, A x V).  The pages name the three stages only.
# Reading: token-duplicated feature-major packing, d features x n tokens with
# d 2n = N/2; scores by token offset (the diagonal method over the token
# axis); the feature sum by log2(d) rotations; Softmax's exponential by the
# degree-15 polynomial, without the division by the row sums.
# --------------------------------------------------------------------------

def attention_pack(X, dup):
    """Slot vector of a d x n matrix X, feature-major with stride 2n:
    slot f 2n + t holds X[f][t mod n] for every t < 2n (dup: the token axis
    twice, so that a slot rotation by delta < n shifts every feature's tokens
    cyclically), or X[f][t] for t < n and 0 for t >= n."""
    d, n = X.shape
    out = np.zeros((d, 2 * n), dtype=np.complex128)
    out[:, :n] = X
    if dup:
        out[:, n:] = X
    return out.reshape(-1)


def attention_sum_steps(n_tok, d):
    """Steps of the feature sum sum_{h<d} rot_{2n h}(P), taken as two hoisted
    rotate-and-sums: d = d1 d2 with d1 = 2^ceil(log2(d) / 2), first over
    2n b (b < d1), then over 2n d1 a (a < d2); step 0 is the term itself."""
    lg = d.bit_length() - 1
    d1 = 1 << ((lg + 1) // 2)
    d2 = d // d1
    return [2 * n_tok * b for b in range(d1)], [2 * n_tok * d1 * a for a in range(d2)]


def attention_scores(q, k, n_tok, d, offsets, keys, rlk, params):
    """S_delta for each token offset delta (0 <= delta < n):
        P = HMRR(q, rot_delta(k)),  rot_delta(k) hoisted (one ModUp of k; delta = 0: k),
        S = sum_{h<d} rot_{2n h}(P) as two hoisted rotate-and-sums,
            T = sum_{b<d1} rot_{2n b}(P),  S = sum_{a<d2} rot_{2n d1 a}(T)
        (attention_sum_steps; each: the term itself plus rotate_sum_hoisted
        over the non-zero steps).
    q packs Q with zeros on t >= n, k packs K token-duplicated; then every
    feature block of S_delta holds sum_f Q[f][t] K[f][(t + delta) mod n] at
    t < n and 0 at t >= n (the sum wraps around the d 2n = N/2 slots).
    Reading: the pages give no schedule for the feature sum; two hoisted
    sums take two ModUps and two ModDowns per offset where log2(d) doubling
    rotations take log2(d) of each, and give the same slots."""
    assert d * 2 * n_tok == params.n_slots and d & (d - 1) == 0
    nz = [o for o in offsets if o % params.n_slots]
    rot = dict(zip(nz, rotate_hoisted(k, nz, keys, params)))
    out = []
    for o in offsets:
        acc = hmult_relin_rescale(q, rot[o] if o in rot else k, rlk, params)
        for st in attention_sum_steps(n_tok, d):
            nzs = [x for x in st if x]
            if nzs:
                acc = add(acc, rotate_sum_hoisted(acc, nzs, keys, params), params)
        out.append(acc)
    return out


def attention_av(a, v, offsets, keys, rlk, params):
    """O = rescale(relinearise(sum_delta a_delta (x) drop(rot_delta(v)))) over
    the offsets: the tensors of the products summed, then one
    relinearisation and one rescale; rot_delta(v) hoisted (one ModUp of v;
    delta = 0: v) and dropped to a_delta's level.  With a_delta = p(S_delta)
    replicated over the feature blocks and v token-duplicated, slot f 2n + t
    of O holds sum_delta p(S_delta[t]) V[f][(t + delta) mod n] for t < n.
    Reading: the pages give no order for relinearising and rescaling the
    products; both maps are linear up to their noise and rounding, so the sum
    is relinearised and rescaled once (every a_delta at one level and scale)."""
    nz = [o for o in offsets if o % params.n_slots]
    rot = dict(zip(nz, rotate_hoisted(v, nz, keys, params)))
    level = a[0]["level"]
    qm = params.q[:level]
    d = None
    for ad, o in zip(a, offsets):
        assert ad["level"] == level and ad["scale"] == a[0]["scale"]
        vv = drop_level(rot[o] if o in rot else v, level)
        t = tensor(ad, vv, params)
        d = t if d is None else tuple(add_rows(d[k], t[k], qm) for k in range(3))
    c = relinearize(d, level, rlk, params)
    return rescale(make_ct(c, level, a[0]["scale"] * v["scale"]), params)


# --------------------------------------------------------------------------
# Paterson-Stockmeyer evaluation of a degree-15 polynomial
# (AEGIS summary section 2.3: Softmax by polynomial approximation)
# --------------------------------------------------------------------------

PS_TOP_SCALE = 2.0 ** 62


def ps_const(c, T, q_lam, S):
    """Integer multiplier that takes a term c x^j (x^j at scale S) to scale T
    after one rescale by q_lam: round_half_away(c * T * q_lam / S), evaluated
    left to right in fp64."""
    v = c * T * float(q_lam) / S
    return int(round_half_away(np.float64(v)))


def ps_eval_deg15(x, coeffs, rlk, params, top_scale=PS_TOP_SCALE):
    """p(x) = sum_{k<=15} c_k x^k by Paterson-Stockmeyer with 4 baby powers.

    Reading (the pages give no schedule).  x at level l0 (24 at the top):
      x2 = HMRR(x, x)                    level l0-1
      x3 = HMRR(x2, drop(x, l0-1))       level l0-2
      x4 = HMRR(x2, x2)                  level l0-2
      q_i(x) = sum_{j<4} c_{4i+j} x^j, built at (lambda, T): each x^j, j >= 1,
        is dropped to lambda+1 limbs and multiplied by
        K = round_half_away(c T q_lambda / S_j); the three products (all at
        nominal scale T q_lambda) are summed and the sum rescaled once by
        q_lambda; the constant adds round_half_away(c_{4i} T).  Its declared
        scale is T.  (One rounding per block instead of one per term: the
        pages fix no order, and rescaling is linear up to that rounding.)
      Horner: acc = q_3 at (l0-3, top_scale);
        acc = HMRR(acc, drop(x4)) + q_i for i = 2, 1, 0, with q_i's products
        added before the product's rescale: at the product's level l (its
        scale T q_lambda, lambda = l-1, T = acc.scale x4.scale / q_lambda),
        acc = rescale(relin(acc (x) drop(x4)) + sum_{j>=1} K_j drop(x^j, l))
              + round_half_away(c_{4i} T),
        K_j as above at (lambda, T); one rescale per Horner step.  (Both
        rescales divide by the same q_lambda and the terms share the nominal
        scale T q_lambda, so one rounding replaces two.)  Result level l0-6.
    Reading: top_scale = 2^62.  The innermost block q_3 is later multiplied
    by x4^3 = x^12, up to 4^12 ~ 1.7e7 on [-4, 0].  Its absolute error is the
    rescale rounding noise (~7e4 in message units at N = 2^16) divided by its
    scale, and the rounding of K (relative 1/K, K ~ c_15 T for c_15 ~ 1/15!).
    At T = 2^40 either term alone exceeds 1e-5 after amplification; at
    T = 2^62 both stay below 1e-6, and every K stays below 2^63."""
    l0 = x["level"]
    hm = lambda a, b: hmult_relin_rescale(a, b, rlk, params)
    x2 = hm(x, x)
    x3 = hm(x2, drop_level(x, l0 - 1))
    x4 = hm(x2, x2)
    pw = {1: x, 2: x2, 3: x3}

    def build_q(i, lam, T):
        acc = None
        for j in (1, 2, 3):
            c = float(coeffs[4 * i + j])
            xj = drop_level(pw[j], lam + 1)
            K = ps_const(c, T, params.q[lam], xj["scale"])
            t = mul_const(xj, K, params)
            acc = t if acc is None else make_ct(
                np.stack([add_rows(acc["c"][k], t["c"][k], params.q[:lam + 1]) for k in range(2)]), lam + 1,
                T * float(params.q[lam]))
        acc = rescale(make_ct(acc["c"], lam + 1, T * float(params.q[lam])), params)
        acc = add_const(acc, int(round_half_away(np.float64(float(coeffs[4 * i]) * T))), params)
        return make_ct(acc["c"], lam, T)

    acc = build_q(3, l0 - 3, top_scale)
    for i in (2, 1, 0):
        lev = acc["level"]
        lam = lev - 1
        prod_scale = acc["scale"] * x4["scale"]
        T = prod_scale / params.q[lam]
        qm = params.q[:lev]
        c = relinearize(tensor(acc, drop_level(x4, lev), params), lev, rlk, params)
        for j in (1, 2, 3):
            xj = drop_level(pw[j], lev)
            K = ps_const(float(coeffs[4 * i + j]), T, params.q[lam], xj["scale"])
            t = mul_const(xj, K, params)
            c = np.stack([add_rows(c[k], t["c"][k], qm) for k in range(2)])
        acc = rescale(make_ct(c, lev, prod_scale), params)
        acc = add_const(acc, int(round_half_away(np.float64(float(coeffs[4 * i]) * T))), params)
        acc = make_ct(acc["c"], lam, T)
    return acc


def ps_eval_plain(z, coeffs):
    """fp64 Horner of the same polynomial (expected slots)."""
    r = np.zeros_like(np.asarray(z, dtype=np.complex128))
    for c in coeffs[::-1]:
        r = r * z + c
    return r
