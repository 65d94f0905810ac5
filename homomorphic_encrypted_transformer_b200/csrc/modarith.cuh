// Device modular arithmetic for primes q < 2^60 held in 64-bit words.
//
// Methods (all published, written here from their definitions):
//  - Shoup's precomputed-quotient product (Harvey, "Faster arithmetic for
//    number-theoretic transforms", J. Symb. Comp. 2014, section 2): for a
//    fixed w < q and w' = floor(w 2^64 / q), any a < 2^64 gives
//    a w - floor(a w' / 2^64) q in [0, 2q).
//  - Montgomery reduction (Montgomery 1985) with R = 2^64: for x < q 2^64,
//    REDC(x) = (x + m q) / 2^64, m = (x mod 2^64)(-q^-1) mod 2^64, lies in
//    [0, 2q) and equals x R^-1 mod q.
//  - Harvey's lazy butterflies keep NTT values in [0, 4q) (q < 2^62).
#pragma once
#include <stdint.h>

namespace he {

// Per-prime constants, laid out for one 64-byte load.
struct DevPrime {
    uint64_t q;
    uint64_t qinv_neg;   // -q^-1 mod 2^64 (Montgomery)
    uint64_t r2;         // 2^128 mod q  (to Montgomery form via REDC(a r2))
    uint64_t one_shoup;  // floor(2^64 / q)  (Shoup product by 1)
    uint64_t r1;         // 2^64 mod q
    uint64_t r1_shoup;   // floor(r1 2^64 / q)
    uint64_t n_inv;      // N^-1 mod q
    uint64_t n_inv_shoup;
};

__device__ __forceinline__ uint64_t csub(uint64_t a, uint64_t m) { return a >= m ? a - m : a; }

// Shoup product, result in [0, 2q).
__device__ __forceinline__ uint64_t mul_shoup_lazy(uint64_t a, uint64_t w, uint64_t w_shoup, uint64_t q) {
    uint64_t hi = __umul64hi(a, w_shoup);
    return a * w - hi * q;
}

__device__ __forceinline__ uint64_t mul_shoup(uint64_t a, uint64_t w, uint64_t w_shoup, uint64_t q) {
    return csub(mul_shoup_lazy(a, w, w_shoup, q), q);
}

// a mod q for any 64-bit a, result in [0, q).
__device__ __forceinline__ uint64_t reduce64(uint64_t a, const DevPrime& p) {
    uint64_t hi = __umul64hi(a, p.one_shoup);
    return csub(a - hi * p.q, p.q);
}

// Montgomery REDC of the 128-bit value hi:lo < q 2^64; result in [0, 2q).
__device__ __forceinline__ uint64_t redc_lazy(uint64_t hi, uint64_t lo, uint64_t q, uint64_t qinv_neg) {
    uint64_t m = lo * qinv_neg;
    uint64_t mh = __umul64hi(m, q);
    // lo + m q = 0 mod 2^64; the carry out of the low word is (lo != 0).
    return hi + mh + (lo != 0 ? 1ull : 0ull);
}

// a b R^-1 mod q in [0, q) for a, b < q.
__device__ __forceinline__ uint64_t mont_mul(uint64_t a, uint64_t b, const DevPrime& p) {
    uint64_t lo = a * b;
    uint64_t hi = __umul64hi(a, b);
    return csub(redc_lazy(hi, lo, p.q, p.qinv_neg), p.q);
}

// a b mod q for a, b < q (two Montgomery steps: a b R^-1, then times R^2 R^-1).
__device__ __forceinline__ uint64_t mul_mod(uint64_t a, uint64_t b, const DevPrime& p) {
    return mont_mul(mont_mul(a, b, p), p.r2, p);
}

// 128-bit accumulator helpers.
struct U128 {
    uint64_t lo, hi;
};

__device__ __forceinline__ void mac128(U128& acc, uint64_t a, uint64_t b) {
    uint64_t lo = a * b;
    uint64_t hi = __umul64hi(a, b);
    acc.lo += lo;
    acc.hi += hi + (acc.lo < lo ? 1ull : 0ull);
}

// acc += hi 2^64 + lo
__device__ __forceinline__ void add128(U128& acc, uint64_t lo, uint64_t hi) {
    acc.lo += lo;
    acc.hi += hi + (acc.lo < lo ? 1ull : 0ull);
}

// Any 128-bit value mod q: (hi mod q) 2^64 + lo = (hi mod q)(2^64 mod q) + lo.
__device__ __forceinline__ uint64_t reduce128(const U128& x, const DevPrime& p) {
    uint64_t h = reduce64(x.hi, p);
    uint64_t t = mul_shoup_lazy(h, p.r1, p.r1_shoup, p.q);  // [0, 2q)
    uint64_t l = mul_shoup_lazy(x.lo, 1ull, p.one_shoup, p.q);  // [0, 2q)
    uint64_t s = t + l;                                      // [0, 4q)
    s = csub(s, 2 * p.q);
    return csub(s, p.q);
}

__device__ __forceinline__ uint64_t add_mod(uint64_t a, uint64_t b, uint64_t q) { return csub(a + b, q); }
__device__ __forceinline__ uint64_t sub_mod(uint64_t a, uint64_t b, uint64_t q) { return a >= b ? a - b : a + q - b; }

}  // namespace he
