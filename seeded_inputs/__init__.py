"""Seeded synthetic inputs shared by the oracle and the CUDA path.

This module holds random draws only -- no CKKS arithmetic.  Everything the
scheme samples (secret, errors, the uniform halves of keys, encryption
randomness) is drawn here and handed to both sides as plain arrays, so the
oracle and the library never need a common sampler.  The workload inputs
(slot values, FFN weights, polynomial coefficients, rotation steps) come from
here too.

Generator: numpy PCG64 seeded through SeedSequence((master, stream, *sub)).
Stream ids are fixed in STREAMS; `sub` distinguishes objects of one kind
(e.g. the Galois element of a rotation key, or a ciphertext index).

Distributions (the pages name CKKS but give no parameters; these follow the
usual RLWE choices):
  * secret: iid uniform over {-1, 0, 1};
  * error: Gaussian sigma = 3.2 rounded half away from zero, clipped to
    [-19, 19] (six sigma);
  * uniform residues: iid uniform in [0, q) for each modulus q;
  * slots / weights / coefficients: as each workload states.
"""
import math

import numpy as np

STREAMS = {
    "secret": 1,
    "pk_a": 2,
    "pk_e": 3,
    "evk_a": 4,
    "evk_e": 5,
    "enc_v": 6,
    "enc_e0": 7,
    "enc_e1": 8,
    "slots": 9,
    "weights": 10,
    "poly_coeffs": 11,
    "rot_steps": 12,
    "rot_assign": 13,
    "ct_residues": 14,
    "pt_residues": 15,
    "ntt_residues": 16,
    "groups": 17,
    "normal_slots": 18,
}

SIGMA = 3.2
ERR_BOUND = 19

# Master seed of each workload: 0xAE615000 + workload index (0 = tiny CKKS,
# 1 = rotation batch, 2 = FFN1 128 tokens, 3 = FFN1 2048 tokens,
# 4 = degree-15 polynomial, 5 = attention head).
MASTER_BASE = 0xAE615000


def master_seed(workload_index):
    return MASTER_BASE + int(workload_index)


def rng(master, stream, *sub):
    sid = STREAMS[stream] if isinstance(stream, str) else int(stream)
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(master), sid] + [int(s) for s in sub])))


def ternary(master, stream, n, *sub):
    """n iid draws from {-1, 0, 1} as int8."""
    return rng(master, stream, *sub).integers(-1, 2, size=n, dtype=np.int64).astype(np.int8)


def gaussian(master, stream, shape, *sub):
    """Rounded Gaussian (sigma 3.2), half away from zero, clipped to +-19, as int32."""
    x = rng(master, stream, *sub).normal(0.0, SIGMA, size=shape)
    r = np.where(x >= 0, np.floor(x + 0.5), np.ceil(x - 0.5))
    return np.clip(r, -ERR_BOUND, ERR_BOUND).astype(np.int32)


def uniform_residues(master, stream, moduli, n, *sub, lead=()):
    """Array [*lead, len(moduli), n] of uint64, entry [..., i, :] uniform in [0, moduli[i])."""
    g = rng(master, stream, *sub)
    lead = tuple(lead)
    out = np.empty(lead + (len(moduli), n), dtype=np.uint64)
    flat = out.reshape(-1, len(moduli), n)
    for b in range(flat.shape[0]):
        for i, q in enumerate(moduli):
            flat[b, i] = g.integers(0, int(q), size=n, dtype=np.uint64)
    return out


def complex_slots(master, n_slots, lo, hi, *sub):
    """n_slots complex values with real and imaginary parts iid U[lo, hi]."""
    g = rng(master, "slots", *sub)
    return g.uniform(lo, hi, size=n_slots) + 1j * g.uniform(lo, hi, size=n_slots)


def real_slots(master, n_slots, lo, hi, *sub):
    """n_slots real values iid U[lo, hi] (as complex with zero imaginary part)."""
    g = rng(master, "slots", *sub)
    return g.uniform(lo, hi, size=n_slots).astype(np.complex128)


def normal_slots(master, n_slots, mean, std, lo, hi, *sub):
    """n_slots real values iid N(mean, std^2) clipped to [lo, hi] (as complex)."""
    g = rng(master, "normal_slots", *sub)
    return np.clip(g.normal(mean, std, size=n_slots), lo, hi).astype(np.complex128)


def weights(master, shape, lo, hi, *sub):
    return rng(master, "weights", *sub).uniform(lo, hi, size=shape)


def poly_coeffs(master, degree):
    """c_k = U[-1, 1] / k!, k = 0..degree."""
    u = rng(master, "poly_coeffs").uniform(-1.0, 1.0, size=degree + 1)
    return np.array([u[k] / math.factorial(k) for k in range(degree + 1)])


def rotation_steps(master, count, lo, hi):
    """`count` distinct integers drawn without replacement from [lo, hi]."""
    g = rng(master, "rot_steps")
    return [int(v) + lo for v in g.choice(hi - lo + 1, size=count, replace=False)]


def step_assignment(master, n_items, n_choices):
    """For each of n_items, a uniform index into n_choices."""
    return [int(v) for v in rng(master, "rot_assign").integers(0, n_choices, size=n_items)]


def choose_groups(master, n_groups, k):
    """k distinct indices out of n_groups (which token groups the oracle checks)."""
    return sorted(int(v) for v in rng(master, "groups").choice(n_groups, size=k, replace=False))


def key_draws(master, key_id, moduli, n, dnum):
    """Random parts of one switching key: a [dnum][len(moduli)][n] uniform residues
    (used directly as evaluation-domain values) and e [dnum][n] rounded Gaussian."""
    a = uniform_residues(master, "evk_a", moduli, n, key_id, lead=(dnum,))
    e = gaussian(master, "evk_e", (dnum, n), key_id)
    return a, e


def secret(master, n):
    return ternary(master, "secret", n)


def encryption_draws(master, ct_id, n):
    """Randomness of one public-key encryption: v ternary, e0 and e1 Gaussian."""
    return (ternary(master, "enc_v", n, ct_id),
            gaussian(master, "enc_e0", (n,), ct_id),
            gaussian(master, "enc_e1", (n,), ct_id))


def public_key_draws(master, moduli, n):
    a = uniform_residues(master, "pk_a", moduli, n)
    e = gaussian(master, "pk_e", (n,))
    return a, e
