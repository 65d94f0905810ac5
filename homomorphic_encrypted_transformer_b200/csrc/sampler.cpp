// Seeded sampling of key material on the host, for he_keygen_seeded.
//
// The pages give only the distributions' names (CKKS keys: a ternary
// secret, uniform key halves, Gaussian errors); this sampler fixes them by a
// stated, reproducible rule so that a seed determines every key:
//
//  * Generator: SplitMix64 (Steele, Lea, Flood, "Fast splittable
//    pseudorandom number generators", OOPSLA 2014): state += gamma,
//    gamma = 0x9E3779B97F4A7C15, output = mix64(state) with
//    mix64(z) = z ^= z >> 30, z *= 0xBF58476D1CE4E5B9, z ^= z >> 27,
//    z *= 0x94D049BB133111EB, z ^= z >> 31.
//  * One stream per object: initial state mix64(seed + gamma (1 + obj)),
//    obj = (tag << 56) | (key_id << 24) | (digit << 8) | prime_index with
//    tag 1 = secret (other fields 0), 2 = uniform half a of a switching key
//    (one stream per digit and prime), 3 = error e of a switching key (one
//    stream per digit, prime_index 0).  key_id = the Galois element of a
//    rotation key, 2 for the relinearisation key.
//  * Uniform residue mod q: draws x >> (64 - bitlen(q)) until one is < q.
//  * Ternary: draws x until x < 2^64 - 1 (a multiple of 3 of values), then
//    (x mod 3) - 1.
//  * Error: discrete Gaussian, sigma = 3.2, on [-19, 19] (six sigma), by
//    inversion of the cumulative table T_i = floor(2^64 C_i), i < 38, with
//    C_i the probability of values <= -19 + i; a draw x gives -19 + the
//    number of T_i <= x.  The table is computed in quad precision; the
//    oracle computes it with exact decimal arithmetic and a test compares
//    the two.
//  * Seeded a-halves (keys that store only b): tag 4, one stream per digit
//    and prime; coefficient i takes outputs 1 + i + t N, t = 0..63, the
//    first whose top bitlen(q) bits are < q (if none, the last one's top bits
//    minus q).  Any coefficient is computed alone, so the kernels regenerate
//    a where they use it (keyseed.cuh).
#include <quadmath.h>
#include <stdint.h>

#include <mutex>
#include <vector>

#include "../../include/he.h"

namespace he_sampler {

constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;
constexpr int kErrBound = 19;
constexpr int kCdt = 2 * kErrBound;  // 38 thresholds for 39 values

static inline uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

struct Stream {
    uint64_t state;
    uint64_t next() {
        state += kGamma;
        return mix64(state);
    }
};

static Stream stream(uint64_t seed, uint64_t obj) { return Stream{mix64(seed + kGamma * (1 + obj))}; }

static uint64_t obj_id(uint64_t tag, uint64_t key_id, uint64_t digit, uint64_t prime) {
    return (tag << 56) | (key_id << 24) | (digit << 8) | prime;
}

static int bitlen(uint64_t q) { return 64 - __builtin_clzll(q); }

constexpr uint64_t kTagSeededA = 4;
constexpr int kSeededTries = 64;

// Output k (k >= 1) of the stream that starts at state s0.
static uint64_t output_at(uint64_t s0, uint64_t k) { return mix64(s0 + kGamma * k); }

static void seeded_a_row(uint64_t s0, uint64_t q, uint64_t* out, int n) {
    const int sh = 64 - bitlen(q);
    for (int i = 0; i < n; i++) {
        uint64_t x = 0;
        bool ok = false;
        for (int t = 0; t < kSeededTries && !ok; t++) {
            x = output_at(s0, 1 + (uint64_t)i + (uint64_t)t * n) >> sh;
            ok = x < q;
        }
        out[i] = ok ? x : x - q;
    }
}

static void uniform(Stream& st, uint64_t q, uint64_t* out, int n) {
    const int sh = 64 - bitlen(q);
    for (int i = 0; i < n; i++) {
        uint64_t x;
        do x = st.next() >> sh;
        while (x >= q);
        out[i] = x;
    }
}

static void ternary(Stream& st, int8_t* out, int n) {
    for (int i = 0; i < n; i++) {
        uint64_t x;
        do x = st.next();
        while (x == ~0ull);
        out[i] = (int8_t)((int)(x % 3) - 1);
    }
}

static void cdt(uint64_t* t) {
    // rho(k) = exp(-k^2 / (2 sigma^2)) = exp(-25 k^2 / 512) for sigma = 3.2;
    // C_i = sum_{k <= -19+i} rho(k) / sum rho
    __float128 rho[2 * kErrBound + 1], total = 0;
    for (int k = -kErrBound; k <= kErrBound; k++) {
        rho[k + kErrBound] = expq(-((__float128)(25 * k * k)) / (__float128)512);
        total += rho[k + kErrBound];
    }
    __float128 acc = 0;
    const __float128 two64 = ldexpq((__float128)1, 64);
    for (int i = 0; i < kCdt; i++) {
        acc += rho[i];
        t[i] = (uint64_t)floorq(two64 * (acc / total));
    }
}

static const uint64_t* cdt_table() {
    static uint64_t t[kCdt];
    static std::once_flag once;
    std::call_once(once, [] { cdt(t); });
    return t;
}

static void gaussian(Stream& st, int32_t* out, int n) {
    const uint64_t* t = cdt_table();
    for (int i = 0; i < n; i++) {
        const uint64_t x = st.next();
        int c = 0;
        for (int j = 0; j < kCdt; j++) c += x >= t[j];
        out[i] = c - kErrBound;
    }
}

}  // namespace he_sampler

using namespace he_sampler;

namespace he {
uint64_t seeded_a_stream_start(uint64_t seed, uint64_t key_id, int digit, int prime_index) {
    return stream(seed, obj_id(kTagSeededA, key_id, digit, prime_index)).state;
}
}  // namespace he

extern "C" int he_gaussian_cdt(uint64_t* out) {
    if (!out) return HE_EINVAL;
    const uint64_t* t = cdt_table();
    for (int i = 0; i < kCdt; i++) out[i] = t[i];
    return HE_OK;
}

extern "C" int he_sample_secret(uint64_t seed, int log_n, int8_t* s_out) {
    if (!s_out || log_n < 1 || log_n > 20) return HE_EINVAL;
    Stream st = stream(seed, obj_id(1, 0, 0, 0));
    ternary(st, s_out, 1 << log_n);
    return HE_OK;
}

extern "C" int he_sample_key_draws(uint64_t seed, uint64_t key_id, int log_n, const uint64_t* primes, int n_primes,
                                   int digits, uint64_t* a_out, int32_t* e_out) {
    if (!primes || !a_out || !e_out || log_n < 1 || log_n > 20 || n_primes < 1 || n_primes > 255 || digits < 1 ||
        digits > 255 || key_id >= (1ull << 32))
        return HE_EINVAL;
    for (int r = 0; r < n_primes; r++)
        if (primes[r] < 2) return HE_EINVAL;
    const int N = 1 << log_n;
    for (int j = 0; j < digits; j++) {
        for (int r = 0; r < n_primes; r++) {
            Stream st = stream(seed, obj_id(2, key_id, j, r));
            uniform(st, primes[r], a_out + ((size_t)j * n_primes + r) * N, N);
        }
        Stream se = stream(seed, obj_id(3, key_id, j, 0));
        gaussian(se, e_out + (size_t)j * N, N);
    }
    return HE_OK;
}

extern "C" int he_sample_key_a_seeded(uint64_t seed, uint64_t key_id, int log_n, const uint64_t* primes, int n_primes,
                                      int digits, uint64_t* a_out) {
    if (!primes || !a_out || log_n < 1 || log_n > 20 || n_primes < 1 || n_primes > 255 || digits < 1 ||
        digits > 255 || key_id >= (1ull << 32))
        return HE_EINVAL;
    for (int r = 0; r < n_primes; r++)
        if (primes[r] < 2) return HE_EINVAL;
    const int N = 1 << log_n;
    for (int j = 0; j < digits; j++)
        for (int r = 0; r < n_primes; r++)
            seeded_a_row(stream(seed, obj_id(kTagSeededA, key_id, j, r)).state, primes[r],
                         a_out + ((size_t)j * n_primes + r) * N, N);
    return HE_OK;
}
