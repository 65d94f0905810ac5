// Seeded a-halves of switching keys, regenerated where they are used.
//
// A key with a seeded a-half stores only b_j = -a_j s + e_j + P g_j s'; the
// uniform a_j is a function of (seed, key, digit, prime, coefficient) that
// any kernel evaluates on its own (SplitMix64 of Steele, Lea and Flood,
// OOPSLA 2014, used as a counter-based generator):
//   s0 = mix64(seed + gamma (1 + obj)), obj = 4 2^56 + key_id 2^24 + j 2^8 + r
//   x_t = mix64(s0 + gamma (1 + i + t N)) >> (64 - bitlen(q_r)),  t = 0..63
//   a_j[r][i] = the first x_t < q_r, or x_63 - q_r if there is none.
// gamma = 0x9E3779B97F4A7C15.  The key keeps s0 per digit and prime (the
// host computes it); a kernel pays two 64-bit multiplies per coefficient,
// and more only on a rejection, which is rare: the primes of the chain sit
// just below a power of two.
#pragma once
#include <stdint.h>

namespace he {

constexpr uint64_t kSeedGamma = 0x9E3779B97F4A7C15ull;
constexpr int kSeedTries = 64;

__device__ __forceinline__ uint64_t seed_mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

// Tries 1..63 of coefficient i (x0: the rejected first try).
static __device__ __noinline__ uint64_t seeded_a_retry(uint64_t s0, uint32_t i, uint32_t n, uint64_t q, int sh, uint64_t x0) {
    uint64_t x = x0;
    for (int t = 1; t < kSeedTries; t++) {
        x = seed_mix64(s0 + kSeedGamma * (1 + (uint64_t)i + (uint64_t)t * n)) >> sh;
        if (x < q) return x;
    }
    return x - q;
}

// a[i] of the row with stream start s0 and prime q, n = N; sh = 64 - bitlen(q).
__device__ __forceinline__ uint64_t seeded_a(uint64_t s0, uint32_t i, uint32_t n, uint64_t q, int sh) {
    const uint64_t x = seed_mix64(s0 + kSeedGamma * (1 + (uint64_t)i)) >> sh;
    return x < q ? x : seeded_a_retry(s0, i, n, q, sh, x);
}

}  // namespace he
