"""Shared set-up for the GPU parity tests: one oracle parameter set and the
matching library context, keys uploaded from the same seeded draws, and
ciphertexts encrypted by the oracle."""
import numpy as np

from oracle import ckks as C
import seeded_inputs as S

RELIN_KEY_ID = 2  # Galois elements are odd, so 2 never names a rotation key


def lib():
    from homomorphic_encrypted_transformer_b200 import he

    return he


def dev(a):
    from homomorphic_encrypted_transformer_b200.torch_io import to_device

    return to_device(a)


def host(t, shape=None):
    from homomorphic_encrypted_transformer_b200.torch_io import to_host

    return to_host(t, shape)


class Setup:
    """Oracle params P, library context ctx, secret, public key."""

    def __init__(self, log_n, L, K, dnum, seed):
        he = lib()
        self.P = C.Params(log_n, L, K, dnum)
        self.seed = seed
        self.ctx = he.he_ctx_create(log_n, L, K, dnum)
        assert self.ctx.primes == self.P.mods
        self.s = S.secret(seed, self.P.N)
        pa, pe = S.public_key_draws(seed, self.P.q, self.P.N)
        self.pk = C.public_key(self.s, pa, pe, self.P)
        self._ok = {}

    def key_draws(self, key_id):
        return S.key_draws(self.seed, key_id, self.P.mods, self.P.N, self.P.dnum)

    def upload_rot(self, step):
        he = lib()
        a, e = self.key_draws(self.P.galois_elt(step))
        he.he_keygen_upload(self.ctx, he.HE_KEY_ROTATION, step, self.s, a, e)

    def oracle_rot_key(self, step):
        k = self.P.galois_elt(step)
        if ("rot", k) not in self._ok:
            a, e = self.key_draws(k)
            self._ok[("rot", k)] = C.rotation_key(self.s, step, a, e, self.P)
        return self._ok[("rot", k)]

    def upload_relin(self):
        he = lib()
        a, e = self.key_draws(RELIN_KEY_ID)
        he.he_keygen_upload(self.ctx, he.HE_KEY_RELIN, 0, self.s, a, e)

    def oracle_relin_key(self):
        if "relin" not in self._ok:
            a, e = self.key_draws(RELIN_KEY_ID)
            self._ok["relin"] = C.relin_key(self.s, a, e, self.P)
        return self._ok["relin"]

    def encrypt(self, z, level, scale=2.0 ** 40, ct_id=0):
        v, e0, e1 = S.encryption_draws(self.seed, ct_id, self.P.N)
        pt = C.encode(z, scale, level, self.P)
        return C.make_ct(C.encrypt(self.pk, pt, v, e0, e1, level, self.P), level, scale)

    def to_gpu(self, ct, room=None):
        he = lib()
        import torch

        room = room or ct["level"]
        t = torch.zeros(2 * room * self.P.N, dtype=torch.int64, device="cuda")
        t[: 2 * ct["level"] * self.P.N] = dev(ct["c"]).reshape(-1)
        return he.Ciphertext(t, ct["level"], ct["scale"])

    def empty_gpu(self, room):
        he = lib()
        import torch

        return he.Ciphertext(torch.zeros(2 * room * self.P.N, dtype=torch.int64, device="cuda"), room, 1.0)

    def from_gpu(self, gct):
        lev = gct.level
        return host(gct.data).reshape(-1)[: 2 * lev * self.P.N].reshape(2, lev, self.P.N)


def random_rows(seed, mods, n_polys, N):
    """[n_polys][len(mods)][N] canonical residues."""
    return S.uniform_residues(seed, "ntt_residues", mods, N, lead=(n_polys,))


class SeededASetup(Setup):
    """Setup whose keys come from he_keygen_seeded_ex(HE_KEYGEN_SEEDED_A):
    the secret and key errors of the library's stated sampler, a-halves by
    its counter rule (the keys store only b).  The oracle builds the same
    keys from oracle/sampler.py."""

    def __init__(self, log_n, L, K, dnum, seed):
        from oracle import sampler as R

        super().__init__(log_n, L, K, dnum, seed)
        self.s = R.secret(seed, self.P.N)
        pa, pe = S.public_key_draws(seed, self.P.q, self.P.N)
        self.pk = C.public_key(self.s, pa, pe, self.P)

    def key_draws(self, key_id):
        from oracle import sampler as R

        P = self.P
        return (R.key_a_seeded(self.seed, key_id, P.mods, P.N, P.dnum),
                R.key_errors(self.seed, key_id, P.N, P.dnum))

    def upload_rot(self, step):
        he = lib()
        he.he_keygen_seeded_ex(self.ctx, self.seed, [step], False, he.HE_KEYGEN_SEEDED_A)

    def upload_relin(self):
        he = lib()
        he.he_keygen_seeded_ex(self.ctx, self.seed, [], True, he.HE_KEYGEN_SEEDED_A)

    def stored_twin(self):
        """A second context holding the same keys in stored form (both halves
        uploaded through he_keygen_upload): its key switches must give the
        same residues."""
        he = lib()
        twin = Setup.__new__(Setup)
        twin.__dict__.update(self.__dict__)
        twin.ctx = he.he_ctx_create(self.P.log_n, self.P.L, self.P.K, self.P.dnum)
        twin._ok = self._ok
        return twin

    def upload_rot_stored(self, twin, step):
        he = lib()
        a, e = self.key_draws(self.P.galois_elt(step))
        he.he_keygen_upload(twin.ctx, he.HE_KEY_ROTATION, step, self.s, a, e)
