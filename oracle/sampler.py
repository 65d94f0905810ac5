"""Oracle of the seeded key sampler (test infrastructure: only tests/,
__graft_entry__.smoke() and bench.py's oracle legs use oracle/).

The same rule as the library's he_keygen_seeded, written here on its own
from the published definitions; no code is shared with the library.

  * SplitMix64 (Steele, Lea, Flood, "Fast splittable pseudorandom number
    generators", OOPSLA 2014): the state advances by gamma =
    0x9E3779B97F4A7C15 and each output is mix64(state).  Output k (k >= 1)
    of a stream that starts at state s0 is therefore mix64(s0 + k gamma):
    the streams are counter-based, and numpy evaluates many outputs at once.
  * Streams: s0 = mix64(seed + gamma (1 + obj)),
    obj = tag 2^56 + key_id 2^24 + digit 2^8 + prime_index
    (tag 1 secret, 2 uniform key half, 3 key error).
  * Uniform residue mod q: outputs >> (64 - bitlen(q)), keeping those < q.
  * Ternary: outputs other than 2^64 - 1, mapped to (x mod 3) - 1.
  * Discrete Gaussian, sigma = 3.2, on [-19, 19]: thresholds
    T_i = floor(2^64 C_i), C_i = P(e <= -19 + i) with
    P(k) proportional to exp(-k^2 / (2 sigma^2)) = exp(-25 k^2 / 512),
    computed in exact decimal arithmetic; a draw x gives -19 + #{i: T_i <= x}.
  * Seeded a-halves (keys that store only b and regenerate a where it is
    used): tag 4, one stream per digit and prime; coefficient i of the row
    takes outputs 1 + i + t N, t = 0, 1, ..., 63 (so any coefficient is
    computed alone), the first whose top bitlen(q) bits are < q; if none of
    the 64 is, the last one's top bits minus q.

Parity pinned: SplitMix64's published first outputs (tests/golden), the
threshold table's symmetry and its agreement with an independent float
computation to 2^-40, the samplers' value ranges and frequencies, and the
seeded a-halves against the generator stepped one state at a time with
rejections forced (tests/test_oracle_sampler.py).
"""
from decimal import Decimal, getcontext

import numpy as np

GAMMA = 0x9E3779B97F4A7C15
M64 = (1 << 64) - 1
ERR_BOUND = 19
TAG_SECRET, TAG_KEY_A, TAG_KEY_E, TAG_KEY_A_SEEDED = 1, 2, 3, 4
A_SEEDED_TRIES = 64


def mix64(z):
    """The SplitMix64 output function on a numpy uint64 array (wrapping)."""
    z = np.asarray(z, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
    return z ^ (z >> np.uint64(31))


def obj_id(tag, key_id=0, digit=0, prime_index=0):
    return (tag << 56) | (key_id << 24) | (digit << 8) | prime_index


def stream_start(seed, obj):
    return int(mix64(np.uint64((seed + GAMMA * (1 + obj)) & M64)))


def outputs(s0, start, count):
    """Outputs start+1 .. start+count of the stream with initial state s0."""
    k = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return mix64(np.uint64(s0) + k * np.uint64(GAMMA))


def _accepted(s0, n, keep, chunk):
    """The first n outputs x of a stream for which keep(x) holds, in order."""
    got, pos = [], 0
    have = 0
    while have < n:
        x = outputs(s0, pos, chunk)
        pos += chunk
        x = keep(x)
        got.append(x)
        have += len(x)
    return np.concatenate(got)[:n]


def uniform(seed, obj, q, n):
    sh = np.uint64(64 - int(q).bit_length())
    qq = np.uint64(q)

    def keep(x):
        v = x >> sh
        return v[v < qq]

    return _accepted(stream_start(seed, obj), n, keep, n + n // 4 + 64)


def ternary(seed, obj, n):
    x = _accepted(stream_start(seed, obj), n, lambda v: v[v != np.uint64(M64)], n + 64)
    return ((x % np.uint64(3)).astype(np.int64) - 1).astype(np.int8)


def gaussian_cdt():
    """T_i = floor(2^64 C_i), i < 38, in exact decimal arithmetic (60 digits)."""
    getcontext().prec = 60
    rho = [(Decimal(-25 * k * k) / Decimal(512)).exp() for k in range(-ERR_BOUND, ERR_BOUND + 1)]
    total = sum(rho, Decimal(0))
    two64 = Decimal(2) ** 64
    out, acc = [], Decimal(0)
    for i in range(2 * ERR_BOUND):
        acc += rho[i]
        out.append(int((two64 * acc / total).to_integral_value(rounding="ROUND_FLOOR")))
    return out


_CDT = None


def gaussian(seed, obj, n):
    global _CDT
    if _CDT is None:
        _CDT = np.array(gaussian_cdt(), dtype=np.uint64)
    x = outputs(stream_start(seed, obj), 0, n)
    return (np.searchsorted(_CDT, x, side="right").astype(np.int64) - ERR_BOUND).astype(np.int32)


def secret(seed, n):
    """The ternary secret of a seed, int8[n]."""
    return ternary(seed, obj_id(TAG_SECRET), n)


def key_draws(seed, key_id, moduli, n, digits):
    """Random parts of one switching key: a [digits][len(moduli)][n] uniform
    residues and e [digits][n] discrete Gaussian."""
    a = np.empty((digits, len(moduli), n), dtype=np.uint64)
    e = np.empty((digits, n), dtype=np.int32)
    for j in range(digits):
        for r, q in enumerate(moduli):
            a[j, r] = uniform(seed, obj_id(TAG_KEY_A, key_id, j, r), q, n)
        e[j] = gaussian(seed, obj_id(TAG_KEY_E, key_id, j, 0), n)
    return a, e


def a_seeded_row(seed, obj, q, n, tries=A_SEEDED_TRIES):
    """One row of a seeded a-half: uint64[n], coefficient i from outputs
    1 + i + t n of the stream of obj (t < tries), by the rule above."""
    sh = np.uint64(64 - int(q).bit_length())
    qq = np.uint64(q)
    s0 = stream_start(seed, obj)
    out = np.zeros(n, dtype=np.uint64)
    todo = np.arange(n)
    for t in range(tries):
        x = outputs(s0, t * n, n)[todo] >> sh
        ok = x < qq
        out[todo[ok]] = x[ok]
        if t == tries - 1:
            out[todo[~ok]] = x[~ok] - qq
        todo = todo[~ok]
        if len(todo) == 0:
            break
    return out


def key_a_seeded(seed, key_id, moduli, n, digits):
    """The a-half of one switching key with seeded a: uint64
    [digits][len(moduli)][n], row r of digit j uniform mod moduli[r]."""
    a = np.empty((digits, len(moduli), n), dtype=np.uint64)
    for j in range(digits):
        for r, q in enumerate(moduli):
            a[j, r] = a_seeded_row(seed, obj_id(TAG_KEY_A_SEEDED, key_id, j, r), q, n)
    return a


def key_errors(seed, key_id, n, digits):
    """The errors of one switching key, int32 [digits][n] (the same draws as
    key_draws')."""
    return np.stack([gaussian(seed, obj_id(TAG_KEY_E, key_id, j, 0), n) for j in range(digits)])
