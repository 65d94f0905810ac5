// Hybrid key switching (Han-Ki, CT-RSA 2020, section 3) and rotation.
//
//   KS_evk(d) = ModDown( sum_j ModUp_j(d) (.) evk_j ),
//   ModUp_j: coefficients of digit j's primes -> fast base conversion onto
//            every prime of Q_level and P, back to the evaluation domain;
//   ModDown: (x - Conv_{P->q}([x]_P)) * P^-1 with the conversion terms taken
//            in the centred range, so the result is round(x/P) - v, |v| <= K/2.
//   rot_r(ct) = (sigma_k(c0), 0) + KS_{evk_r}(sigma_k(c1)),  k = 5^r mod 2N.
#include <algorithm>
#include <set>

#include "he_internal.h"
#include "keyseed.cuh"
#include "ntt.cuh"

namespace he {

constexpr int kMaxDigits = 15;

// x[k] = d[automorph_src(j0 + k)], k < 16, j0 even.  sigma_k maps the
// aligned pair {2m, 2m+1} onto an aligned pair (src(j ^ 1) = src(j) ^ 1), so
// each pair is one 16-byte load, swapped when src(j0 + 2k) is odd.  With
// k = 0 this is a plain load.
template <int LOGN, typename T>
__device__ __forceinline__ void gather_load16(T (&x)[16], const uint64_t* __restrict__ d, int j0, uint64_t galois) {
#pragma unroll
    for (int k = 0; k < 8; k++) {
        const int s = automorph_src(j0 + 2 * k, LOGN, galois);
        const ulonglong2 v = __ldg(reinterpret_cast<const ulonglong2*>(d + (s & ~1)));
        const bool sw = s & 1;
        x[2 * k] = to_elem(sw ? v.y : v.x, T());
        x[2 * k + 1] = to_elem(sw ? v.x : v.y, T());
    }
}

// First pass of the inverse NTT of sigma_{g_i}(d_i), the automorphism folded
// into its loads: coef[i][t] = inverse row pass of (d_i[t][automorph_src(.)]).
// Rows t of Q_level have prime index t.  Grid (ROW_TILES, n level).
template <int LOGN>
__global__ void __launch_bounds__(NttCfg<LOGN>::ROW_THREADS, NTT_MIN_BLOCKS)
    k_inv_rows_gather(PtrList din, GalList gal, uint64_t* __restrict__ coef, int level,
                      const DevPrime* __restrict__ pr, const ulonglong2* __restrict__ tw_all,
                      const double* __restrict__ twd_all, const FpMod* __restrict__ fpm) {
    using Cf = NttCfg<LOGN>;
    __shared__ uint64_t sm[Cf::TR * Cf::ROW_PITCH];
    const int y = blockIdx.y, i = y / level, t = y - i * level;
    const uint64_t q = pr[t].q;
    const int r = blockIdx.x * Cf::TR + threadIdx.x / (Cf::C / 16);
    const int j0 = r * Cf::C + 16 * row_lane<LOGN>();
    const uint64_t* d = din.p[i] + (size_t)t * Cf::N;
    uint64_t* out = coef + (size_t)y * Cf::N + (size_t)r * Cf::C;
    const uint64_t g = gal.g[i];
    if (q < kFpPrimeLimit) {
        double x[16];
        gather_load16<LOGN>(x, d, j0, g);
        inv_rows_core<LOGN>(x, reinterpret_cast<double*>(sm), out, r, twd_all + (size_t)t * Cf::N, fpm[t]);
    } else {
        uint64_t x[16];
        gather_load16<LOGN>(x, d, j0, g);
        inv_rows_core<LOGN>(x, sm, out, r, tw_all + (size_t)t * Cf::N, q);
    }
}

// ModUp of digit j at one level.  Rows of Q_level and P are numbered
// t = 0..n_rows-1 (q_0..q_{level-1}, then p_0..p_{K-1}); the digit owns rows
// src_row..src_row+n_src-1 and its targets are all the other rows, stored
// compactly: target row t sits at position t (t < src_row) or t - n_src.
// ext layout: [digit][ciphertext][n_rows - n_src][N].
// Entries per group of k_ks_inner_grp (one thread applies its key words to
// each in turn): 16 measured best, by a little, for the rotation batch,
// hoisted rotations and relinearisation batches (caps of 1 to 16 tried).
constexpr int kKsGroupMax = 16;
// Outputs per thread of k_ks_inner_sum_mo.
constexpr int kKsSumMo = 4;

struct ModupArgs {
    int n_digits;
    int n_src[kMaxDigits];
    int src_row[kMaxDigits];
    long long ext_off[kMaxDigits];  // first limb of digit j's block, per ciphertext count 1
    const ulonglong2* src[kMaxDigits];
    const ulonglong2* mat[kMaxDigits];
    uint8_t tprime[64];  // prime index of each of the level+K rows
};

// Target-side constants of one conversion, staged in shared memory.
struct ConvTarget {
    uint64_t q, qinv_neg, one_shoup, pad;
};

// The conversion matrices are stored in Montgomery form (m 2^64 mod t), so a
// sum of at most 16 products y m' with y < 2^60 stays below t 2^64 and one
// REDC returns sum(y m) mod t.
__device__ __forceinline__ uint64_t redc_t(const U128& x, const ConvTarget& p) {
    return csub(redc_lazy(x.hi, x.lo, p.q, p.qinv_neg), p.q);
}

constexpr int kConvMaxTargets = 64;

// Targets of one ModUp conversion split by arithmetic path; entries are
// positions tt (0..n_rows-|D_j|-1) in the digit's output block.
constexpr int kConvMaxInt = 32;
struct ConvLists {
    int n_fp, n_int;
    uint8_t fp_tt[kConvMaxTargets];
    uint8_t int_tt[kConvMaxInt];
};

// ModUp of digit j (NS source primes at rows s0..s0+NS-1), one launch per digit:
//   ext_j[i][tt][c] = sum_s [x_s qhat_inv_s]_{q_s} (qhat_s mod t)   (coefficient domain)
// for every target row t (all rows of Q_level and P outside the digit).
//  - targets below 2^41 (two per iteration): signed FP64 rounded-quotient
//    products, one reduction at the end;
//  - 60-bit targets, digit of 40-bit sources (NARROW): with y = y1 2^21 + y0
//    (y0 < 2^21, y1 < 2^20) and the Montgomery-form entry m' = m2 2^42 +
//    m1 2^21 + m0 (m0, m1 < 2^21, m2 < 2^18) the four sums
//      V0 = S y0 m0, V1 = S y0 m1 + y1 m0, V2 = S y0 m2 + y1 m1, V3 = S y1 m2
//    are exact doubles below 2^47 (NS <= 16); the 128-bit value
//    V0 + V1 2^21 + V2 2^42 + V3 2^63 = S y m' is assembled on the integer
//    pipe and one REDC gives S y m mod t;
//  - 60-bit targets of a digit whose first source alone is 60-bit (WIDE0,
//    the digit holding q_0): that residue splits in three 21-bit parts
//    (y = y2 2^42 + y1 2^21 + y0), adding V2 += y2 m0, V3 += y2 m1 and
//    V4 = y2 m2, all still exact (each sum below 2^48), and
//    V0 + V1 2^21 + V2 2^42 + V3 2^63 + V4 2^84 = S y m' (< 2^124);
//  - 60-bit targets of any other digit: 128-bit accumulation of the NS
//    products, one REDC.
// MODE: kConvNarrow, kConvWide0 or kConvGeneric.
constexpr int kConvGeneric = 0, kConvNarrow = 1, kConvWide0 = 2;

template <int NS, int MODE>
__global__ void __launch_bounds__(256, 4)  // measured: better than 3 blocks per SM despite small spills
    k_modup_conv(const uint64_t* __restrict__ coef, uint64_t* __restrict__ ext_j, const ulonglong2* __restrict__ src,
                 const ulonglong2* __restrict__ mat, ModupArgs a, const __grid_constant__ ConvLists cl,
                 const DevPrime* __restrict__ pr,
                 const FpMod* __restrict__ fpm, int level, int n_rows, int s0, int logn) {
    __shared__ double sm_fm[NS * kConvMaxTargets];  // [s][f]: FP64 targets in list order
    __shared__ FpMod sm_ff[kConvMaxTargets];
    __shared__ ConvTarget sm_ft[kConvMaxTargets];  // (wide sources: reduction into [0, 2t))
    constexpr bool SPLIT = MODE != kConvGeneric;  // 60-bit targets from exact FP64 partial sums
    __shared__ double2 sm_i01[SPLIT ? NS * kConvMaxInt : 1];
    __shared__ double sm_i2[SPLIT ? NS * kConvMaxInt : 1];
    __shared__ uint64_t sm_im[SPLIT ? 1 : NS * kConvMaxInt];
    __shared__ ConvTarget sm_it[kConvMaxInt];
    __shared__ int sm_ftt[kConvMaxTargets], sm_itt[kConvMaxInt];  // output rows, list order
    const int N = 1 << logn;
    const int n_tgt = n_rows - NS;
    const int n_fp = cl.n_fp, n_int = cl.n_int;
    for (int f = threadIdx.x; f < n_fp; f += blockDim.x) sm_ftt[f] = cl.fp_tt[f];
    for (int g = threadIdx.x; g < n_int; g += blockDim.x) sm_itt[g] = cl.int_tt[g];
    __syncthreads();
    for (int idx = threadIdx.x; idx < NS * n_fp; idx += blockDim.x) {
        int s = idx / n_fp, f = idx - s * n_fp;
        int tt = sm_ftt[f], t = tt < s0 ? tt : tt + NS;
        sm_fm[s * kConvMaxTargets + f] = (double)mat[(size_t)s * n_rows + t].y;  // exact: below 2^41
    }
    for (int idx = threadIdx.x; idx < NS * n_int; idx += blockDim.x) {
        int s = idx / n_int, g = idx - s * n_int;
        int tt = sm_itt[g], t = tt < s0 ? tt : tt + NS;
        uint64_t m = mat[(size_t)s * n_rows + t].x;
        if constexpr (SPLIT) {
            sm_i01[s * kConvMaxInt + g] =
                make_double2((double)(m & ((1ull << 21) - 1)), (double)((m >> 21) & ((1ull << 21) - 1)));
            sm_i2[s * kConvMaxInt + g] = (double)(m >> 42);
        } else {
            sm_im[s * kConvMaxInt + g] = m;
        }
    }
    for (int f = threadIdx.x; f < n_fp; f += blockDim.x) {
        int tt = sm_ftt[f], t = tt < s0 ? tt : tt + NS;
        DevPrime p = pr[a.tprime[t]];
        sm_ff[f] = fpm[a.tprime[t]];
        sm_ft[f] = ConvTarget{p.q, p.qinv_neg, p.one_shoup, 0};
    }
    for (int g = threadIdx.x; g < n_int; g += blockDim.x) {
        int tt = sm_itt[g], t = tt < s0 ? tt : tt + NS;
        DevPrime p = pr[a.tprime[t]];
        sm_it[g] = ConvTarget{p.q, p.qinv_neg, p.one_shoup, 0};
    }
    __syncthreads();
    int c = blockIdx.x * blockDim.x + threadIdx.x;
    int i = blockIdx.y;
    if (c >= N) return;
    uint64_t* o = ext_j + (size_t)i * n_tgt * N + c;
    if constexpr (SPLIT) {
        // Sources below 2^41 live as doubles only (the 60-bit source of a
        // WIDE0 digit as an integer); the targets below 2^41 go first, then
        // the 21-bit splits of the 60-bit targets are derived from the
        // doubles, so at most two forms of a source are live at a time.
        double yd[NS];
        uint64_t yw = 0;
#pragma unroll
        for (int s = 0; s < NS; s++) {
            const uint64_t q = pr[s0 + s].q;
            const ulonglong2 w = src[s];
            const uint64_t y = mul_shoup(coef[((size_t)i * level + s0 + s) * N + c], w.x, w.y, q);
            if (MODE == kConvWide0 && s == 0) {
                yw = y;
                yd[0] = 0.0;
            } else {
                yd[s] = u2d(y);
            }
        }
        // targets below 2^41, two at a time
        for (int f = 0; f < n_fp; f += 2) {
            const bool two = f + 1 < n_fp;
            const int f1 = two ? f + 1 : f;
            const FpMod F0 = sm_ff[f], F1 = sm_ff[f1];
            double acc0 = 0.0, acc1 = 0.0;
#pragma unroll
            for (int s = 0; s < NS; s++) {
                const double m0 = sm_fm[s * kConvMaxTargets + f], m1 = sm_fm[s * kConvMaxTargets + f1];
                double y0 = yd[s], y1 = yd[s];
                if (MODE == kConvWide0 && s == 0) {  // the 60-bit residue first drops to [0, 2t)
                    const ConvTarget t0 = sm_ft[f], t1 = sm_ft[f1];
                    y0 = u2d(yw - __umul64hi(yw, t0.one_shoup) * t0.q);
                    y1 = u2d(yw - __umul64hi(yw, t1.one_shoup) * t1.q);
                }
                acc0 = __dadd_rn(acc0, fp_mulmod_s(y0, m0, F0));
                acc1 = __dadd_rn(acc1, fp_mulmod_s(y1, m1, F1));
            }
            o[(size_t)sm_ftt[f] * N] = d2u(fp_canon(acc0, F0));
            if (two) o[(size_t)sm_ftt[f1] * N] = d2u(fp_canon(acc1, F1));
        }
        // 60-bit targets: y = y1 2^21 + y0 (y0 < 2^21, y1 < 2^20), and for the
        // WIDE0 source y = y2 2^42 + y1 2^21 + y0
        double y0[NS], y1[NS];
#pragma unroll
        for (int s = 0; s < NS; s++) {
            if (MODE == kConvWide0 && s == 0) {
                y0[0] = (double)(yw & ((1ull << 21) - 1));
                y1[0] = (double)((yw >> 21) & ((1ull << 21) - 1));
            } else {
                y1[s] = trunc(__dmul_rn(yd[s], 4.76837158203125e-07));  // exact: times 2^-21
                y0[s] = __fma_rn(-y1[s], 2097152.0, yd[s]);
            }
        }
        const double y2w = MODE == kConvWide0 ? (double)(yw >> 42) : 0.0;  // < 2^18
        for (int g = 0; g < n_int; g++) {
            double v0 = 0, v1 = 0, v2 = 0, v3 = 0, v4 = 0;
#pragma unroll
            for (int s = 0; s < NS; s++) {
                const double2 m01 = sm_i01[s * kConvMaxInt + g];
                const double m2 = sm_i2[s * kConvMaxInt + g];
                v0 = __fma_rn(y0[s], m01.x, v0);
                v1 = __fma_rn(y0[s], m01.y, __fma_rn(y1[s], m01.x, v1));
                v2 = __fma_rn(y0[s], m2, __fma_rn(y1[s], m01.y, v2));
                v3 = __fma_rn(y1[s], m2, v3);
                if (MODE == kConvWide0 && s == 0) {
                    v2 = __fma_rn(y2w, m01.x, v2);
                    v3 = __fma_rn(y2w, m01.y, v3);
                    v4 = __fma_rn(y2w, m2, v4);
                }
            }
            const uint64_t w0 = d2u(v0), w1 = d2u(v1), w2 = d2u(v2), w3 = d2u(v3);
            U128 acc = {w0, 0};
            add128(acc, w1 << 21, w1 >> 43);
            add128(acc, w2 << 42, w2 >> 22);
            add128(acc, w3 << 63, w3 >> 1);
            if constexpr (MODE == kConvWide0) add128(acc, 0, d2u(v4) << 20);
            o[(size_t)sm_itt[g] * N] = redc_t(acc, sm_it[g]);
        }
    } else {
        uint64_t y[NS];
        double yd[NS];  // y as a double (sources below 2^41)
#pragma unroll
        for (int s = 0; s < NS; s++) {
            const uint64_t q = pr[s0 + s].q;
            const ulonglong2 w = src[s];
            y[s] = mul_shoup(coef[((size_t)i * level + s0 + s) * N + c], w.x, w.y, q);
            yd[s] = u2d(q < kFpPrimeLimit ? y[s] : 0);
        }
        for (int g = 0; g < n_int; g++) {
            U128 acc = {0, 0};
#pragma unroll
            for (int s = 0; s < NS; s++) mac128(acc, y[s], sm_im[s * kConvMaxInt + g]);
            o[(size_t)sm_itt[g] * N] = redc_t(acc, sm_it[g]);
        }
        // targets below 2^41, two at a time
        for (int f = 0; f < n_fp; f += 2) {
            const bool two = f + 1 < n_fp;
            const int f1 = two ? f + 1 : f;
            const FpMod F0 = sm_ff[f], F1 = sm_ff[f1];
            double acc0 = 0.0, acc1 = 0.0;
#pragma unroll
            for (int s = 0; s < NS; s++) {
                const double m0 = sm_fm[s * kConvMaxTargets + f], m1 = sm_fm[s * kConvMaxTargets + f1];
                double y0 = yd[s], y1 = yd[s];
                if (pr[s0 + s].q >= kFpPrimeLimit) {  // a wide source residue first drops to [0, 2t)
                    const ConvTarget t0 = sm_ft[f], t1 = sm_ft[f1];
                    y0 = u2d(y[s] - __umul64hi(y[s], t0.one_shoup) * t0.q);
                    y1 = u2d(y[s] - __umul64hi(y[s], t1.one_shoup) * t1.q);
                }
                acc0 = __dadd_rn(acc0, fp_mulmod_s(y0, m0, F0));
                acc1 = __dadd_rn(acc1, fp_mulmod_s(y1, m1, F1));
            }
            o[(size_t)sm_ftt[f] * N] = d2u(fp_canon(acc0, F0));
            if (two) o[(size_t)sm_ftt[f1] * N] = d2u(fp_canon(acc1, F1));
        }
    }
}

// u[i][0/1][t][c] = sum_j x_j[t][c] * key_i,j[b/a][row(t)][c],
// x_j = sigma_{g_i}(d_i) on digit j's own rows (read through the
// automorphism: an aligned group of 32 indices maps onto one, so a warp's
// loads stay within the same 256 bytes), ext_j elsewhere.  Rows of primes
// below 2^41 (key stored as doubles) sum signed FP64 products, the others
// accumulate 128-bit products of the Montgomery-form key and reduce once.
// The ciphertext index is the fastest grid dimension: neighbouring blocks
// that share a key read the same key tile, which DRAM then serves once.
// ND = number of digits (compile time, so that every load of a thread is in
// flight at once).  HOIST: the raised digits belong to ciphertext xsrc[i] of
// ext (n_ext of them) and are read through sigma_{g_i} as well: the
// automorphism of a hoisted rotation, applied after ModUp.  SA: the keys
// store only their b-halves (key_digits of them); the a-halves are
// regenerated from their stream starts (keyseed.cuh) as canonical residues,
// and integer rows reduce their a-sums with reduce128 instead of REDC.
template <int ND, bool SA>
__device__ __forceinline__ void load_key_halves(const uint64_t* key, int j, int krow, int LK, int N, int c,
                                                ulonglong2& kb, ulonglong2& ka) {
    if constexpr (SA) {
        kb = __ldg(reinterpret_cast<const ulonglong2*>(key + ((size_t)j * LK + krow) * N + c));
    } else {
        kb = __ldg(reinterpret_cast<const ulonglong2*>(key + (((size_t)j * 2 + 0) * LK + krow) * N + c));
        ka = __ldg(reinterpret_cast<const ulonglong2*>(key + (((size_t)j * 2 + 1) * LK + krow) * N + c));
    }
}

// The a-halves of a seeded key at positions c, c + 1 of row krow, digits < ND.
template <int ND>
__device__ __forceinline__ void seeded_a_halves(const uint64_t* key, int key_digits, int krow, int LK, int N, int c,
                                                uint64_t q, ulonglong2 (&ka)[ND]) {
    const uint64_t* s0p = key + (size_t)key_digits * LK * N + krow;
    const int sh = __clzll(q);
#pragma unroll
    for (int j = 0; j < ND; j++) {
        const uint64_t s0 = __ldg(s0p + (size_t)j * LK);
        ka[j] = make_ulonglong2(seeded_a(s0, c, N, q, sh), seeded_a(s0, c + 1, N, q, sh));
    }
}

// An a-half word as the FP64 path multiplies it: stored keys hold the bits
// of a double, seeded ones the canonical residue.
template <bool SA>
__device__ __forceinline__ double key_a_fp(uint64_t w) {
    if constexpr (SA)
        return u2d(w);
    else
        return __longlong_as_double((long long)w);
}

// sum of the a-products mod q, [0, q): REDC of Montgomery-form stored keys,
// plain 128-bit reduction of canonical seeded ones
template <bool SA>
__device__ __forceinline__ uint64_t reduce_a_sum(const U128& x, const DevPrime& p) {
    if constexpr (SA)
        return reduce128(x, p);
    else
        return csub(redc_lazy(x.hi, x.lo, p.q, p.qinv_neg), p.q);
}

template <int ND, bool HOIST, bool SA>
__global__ void __launch_bounds__(256, 5)  // 5 blocks per SM: more loads in flight than at 4
    k_ks_inner(const uint64_t* __restrict__ ext, PtrList din, GalList gal, PtrList keys, IdxList xsrc,
               uint64_t* __restrict__ u, int n_rows, int level, int L, int LK, int n_ext, int key_digits,
               const DevPrime* __restrict__ pr, const FpMod* __restrict__ fpm, ModupArgs a, int logn) {
    const int N = 1 << logn;
    const int i = blockIdx.x, t = blockIdx.z;
    const int c = 2 * (blockIdx.y * blockDim.x + threadIdx.x);  // positions c, c+1
    if (c >= N) return;
    const uint64_t* key = keys.p[i];
    const int own = automorph_src(c, logn, gal.g[i]);  // the pair maps onto {own & ~1, own | 1}
    const bool own_sw = own & 1;
    const int krow = t < level ? t : L + (t - level);
    const int pidx = a.tprime[t];
    const DevPrime p = pr[pidx];
    const bool fp = p.q < kFpPrimeLimit;
    ulonglong2 xs[ND], kbs[ND], kas[ND];
#pragma unroll
    for (int j = 0; j < ND; j++) {
        const int s0 = a.src_row[j], ns = a.n_src[j];
        if (t >= s0 && t < s0 + ns) {
            const ulonglong2 v = __ldg(reinterpret_cast<const ulonglong2*>(din.p[i] + (size_t)t * N + (own & ~1)));
            xs[j] = own_sw ? make_ulonglong2(v.y, v.x) : v;
        } else {
            const int pos = t < s0 ? t : t - ns;
            const uint64_t* e =
                ext + ((size_t)a.ext_off[j] * n_ext + (size_t)(HOIST ? xsrc.i[i] : i) * (n_rows - ns) + pos) * N;
            if (HOIST) {
                const ulonglong2 v = __ldg(reinterpret_cast<const ulonglong2*>(e + (own & ~1)));
                xs[j] = own_sw ? make_ulonglong2(v.y, v.x) : v;
            } else {
                xs[j] = __ldg(reinterpret_cast<const ulonglong2*>(e + c));
            }
        }
        load_key_halves<ND, SA>(key, j, krow, LK, N, c, kbs[j], kas[j]);
    }
    if constexpr (SA) seeded_a_halves<ND>(key, key_digits, krow, LK, N, c, p.q, kas);
    ulonglong2 ob, oa;
    if (fp) {
        const FpMod m = fpm[pidx];
        double b0 = 0.0, b1 = 0.0, a0 = 0.0, a1 = 0.0;
#pragma unroll
        for (int j = 0; j < ND; j++) {
            const double x0 = u2d(xs[j].x), x1 = u2d(xs[j].y);
            b0 = __dadd_rn(b0, fp_mulmod_s(x0, __longlong_as_double((long long)kbs[j].x), m));
            b1 = __dadd_rn(b1, fp_mulmod_s(x1, __longlong_as_double((long long)kbs[j].y), m));
            a0 = __dadd_rn(a0, fp_mulmod_s(x0, key_a_fp<SA>(kas[j].x), m));
            a1 = __dadd_rn(a1, fp_mulmod_s(x1, key_a_fp<SA>(kas[j].y), m));
        }
        ob = make_ulonglong2(d2u(fp_canon(b0, m)), d2u(fp_canon(b1, m)));
        oa = make_ulonglong2(d2u(fp_canon(a0, m)), d2u(fp_canon(a1, m)));
    } else {
        U128 b0 = {0, 0}, b1 = {0, 0}, a0 = {0, 0}, a1 = {0, 0};
#pragma unroll
        for (int j = 0; j < ND; j++) {
            mac128(b0, xs[j].x, kbs[j].x);
            mac128(b1, xs[j].y, kbs[j].y);
            mac128(a0, xs[j].x, kas[j].x);
            mac128(a1, xs[j].y, kas[j].y);
        }
        ob = make_ulonglong2(csub(redc_lazy(b0.hi, b0.lo, p.q, p.qinv_neg), p.q),
                             csub(redc_lazy(b1.hi, b1.lo, p.q, p.qinv_neg), p.q));
        oa = make_ulonglong2(reduce_a_sum<SA>(a0, p), reduce_a_sum<SA>(a1, p));
    }
    uint64_t* o = u + ((size_t)i * 2 * n_rows) * N + c;
    *reinterpret_cast<ulonglong2*>(o + (size_t)t * N) = ob;
    *reinterpret_cast<ulonglong2*>(o + (size_t)(n_rows + t) * N) = oa;
}

// The inner product of k_ks_inner for a group of key switches that share one
// key (and so one Galois element): block x covers entries grp[x] ..
// grp[x + 1] - 1 (the last group ends at n).  Each thread reads (or, SA,
// regenerates) its key words once and applies them to every entry of the
// group in turn, instead of once per entry.
template <int ND, bool HOIST, bool SA>
__global__ void __launch_bounds__(256, 4)
    k_ks_inner_grp(const uint64_t* __restrict__ ext, PtrList din, GalList gal, PtrList keys, IdxList xsrc,
                   IdxList grp, int n_grp, int n, uint64_t* __restrict__ u, int n_rows, int level, int L, int LK,
                   int n_ext, int key_digits, const DevPrime* __restrict__ pr, const FpMod* __restrict__ fpm,
                   ModupArgs a, int logn) {
    const int N = 1 << logn;
    const int g = blockIdx.x, t = blockIdx.z;
    const int c = 2 * (blockIdx.y * blockDim.x + threadIdx.x);  // positions c, c+1
    if (c >= N) return;
    const int i0 = grp.i[g], i1 = g + 1 < n_grp ? grp.i[g + 1] : n;
    const uint64_t* key = keys.p[i0];
    const int own = automorph_src(c, logn, gal.g[i0]);  // the pair maps onto {own & ~1, own | 1}
    const bool own_sw = own & 1;
    const int krow = t < level ? t : L + (t - level);
    const int pidx = a.tprime[t];
    const DevPrime p = pr[pidx];
    const bool fp = p.q < kFpPrimeLimit;
    ulonglong2 kbs[ND], kas[ND];
#pragma unroll
    for (int j = 0; j < ND; j++) load_key_halves<ND, SA>(key, j, krow, LK, N, c, kbs[j], kas[j]);
    if constexpr (SA) seeded_a_halves<ND>(key, key_digits, krow, LK, N, c, p.q, kas);
    for (int i = i0; i < i1; i++) {
        ulonglong2 xs[ND];
#pragma unroll
        for (int j = 0; j < ND; j++) {
            const int s0 = a.src_row[j], ns = a.n_src[j];
            if (t >= s0 && t < s0 + ns) {
                const ulonglong2 v =
                    __ldg(reinterpret_cast<const ulonglong2*>(din.p[i] + (size_t)t * N + (own & ~1)));
                xs[j] = own_sw ? make_ulonglong2(v.y, v.x) : v;
            } else {
                const int pos = t < s0 ? t : t - ns;
                const uint64_t* e =
                    ext + ((size_t)a.ext_off[j] * n_ext + (size_t)(HOIST ? xsrc.i[i] : i) * (n_rows - ns) + pos) * N;
                if (HOIST) {
                    const ulonglong2 v = __ldg(reinterpret_cast<const ulonglong2*>(e + (own & ~1)));
                    xs[j] = own_sw ? make_ulonglong2(v.y, v.x) : v;
                } else {
                    xs[j] = __ldg(reinterpret_cast<const ulonglong2*>(e + c));
                }
            }
        }
        ulonglong2 ob, oa;
        if (fp) {
            const FpMod m = fpm[pidx];
            double b0 = 0.0, b1 = 0.0, a0 = 0.0, a1 = 0.0;
#pragma unroll
            for (int j = 0; j < ND; j++) {
                const double x0 = u2d(xs[j].x), x1 = u2d(xs[j].y);
                b0 = __dadd_rn(b0, fp_mulmod_s(x0, __longlong_as_double((long long)kbs[j].x), m));
                b1 = __dadd_rn(b1, fp_mulmod_s(x1, __longlong_as_double((long long)kbs[j].y), m));
                a0 = __dadd_rn(a0, fp_mulmod_s(x0, key_a_fp<SA>(kas[j].x), m));
                a1 = __dadd_rn(a1, fp_mulmod_s(x1, key_a_fp<SA>(kas[j].y), m));
            }
            ob = make_ulonglong2(d2u(fp_canon(b0, m)), d2u(fp_canon(b1, m)));
            oa = make_ulonglong2(d2u(fp_canon(a0, m)), d2u(fp_canon(a1, m)));
        } else {
            U128 b0 = {0, 0}, b1 = {0, 0}, a0 = {0, 0}, a1 = {0, 0};
#pragma unroll
            for (int j = 0; j < ND; j++) {
                mac128(b0, xs[j].x, kbs[j].x);
                mac128(b1, xs[j].y, kbs[j].y);
                mac128(a0, xs[j].x, kas[j].x);
                mac128(a1, xs[j].y, kas[j].y);
            }
            ob = make_ulonglong2(csub(redc_lazy(b0.hi, b0.lo, p.q, p.qinv_neg), p.q),
                                 csub(redc_lazy(b1.hi, b1.lo, p.q, p.qinv_neg), p.q));
            oa = make_ulonglong2(reduce_a_sum<SA>(a0, p), reduce_a_sum<SA>(a1, p));
        }
        uint64_t* o = u + ((size_t)i * 2 * n_rows) * N + c;
        *reinterpret_cast<ulonglong2*>(o + (size_t)t * N) = ob;
        *reinterpret_cast<ulonglong2*>(o + (size_t)(n_rows + t) * N) = oa;
    }
}

// Sum of G key inner products per output, for one ModDown of the sum:
// u[o][0/1][t][c] = sum_{g<G} sum_j x_{r,j}[t][c] * key_r,j[b/a][row(t)][c],
// r = o G + g, x_{r,j} as in k_ks_inner for key switch r (its own sigma on
// the digit's own rows, its raised digits elsewhere; HOIST: the raised
// digits of ciphertext xsrc[r], read through sigma_r).  FP64 rows add the
// signed products of all G switches (|sum| <= G ND 5q/8 < 2^51 for G <= 64,
// ND <= 15); integer rows reduce each switch's 128-bit sum once and add the
// results, kept in [0, 2q).
template <int ND, bool HOIST, bool SA>
__global__ void __launch_bounds__(256, 4)
    k_ks_inner_sum(const uint64_t* __restrict__ ext, PtrList din, GalList gal, PtrList keys, IdxList xsrc, int G,
                   uint64_t* __restrict__ u, int n_rows, int level, int L, int LK, int n_ext, int key_digits,
                   const DevPrime* __restrict__ pr, const FpMod* __restrict__ fpm, ModupArgs a, int logn) {
    const int N = 1 << logn;
    const int o = blockIdx.x, t = blockIdx.z;
    const int c = 2 * (blockIdx.y * blockDim.x + threadIdx.x);  // positions c, c+1
    if (c >= N) return;
    const int krow = t < level ? t : L + (t - level);
    const int pidx = a.tprime[t];
    const DevPrime p = pr[pidx];
    const bool fp = p.q < kFpPrimeLimit;
    const FpMod m = fpm[pidx];
    double fb0 = 0.0, fb1 = 0.0, fa0 = 0.0, fa1 = 0.0;
    uint64_t ib0 = 0, ib1 = 0, ia0 = 0, ia1 = 0;
    for (int g = 0; g < G; g++) {
        const int r = o * G + g;
        const uint64_t* key = keys.p[r];
        const int own = automorph_src(c, logn, gal.g[r]);
        const bool own_sw = own & 1;
        ulonglong2 xs[ND], kbs[ND], kas[ND];
#pragma unroll
        for (int j = 0; j < ND; j++) {
            const int s0 = a.src_row[j], ns = a.n_src[j];
            if (t >= s0 && t < s0 + ns) {
                const ulonglong2 v =
                    __ldg(reinterpret_cast<const ulonglong2*>(din.p[r] + (size_t)t * N + (own & ~1)));
                xs[j] = own_sw ? make_ulonglong2(v.y, v.x) : v;
            } else {
                const int pos = t < s0 ? t : t - ns;
                const uint64_t* e =
                    ext + ((size_t)a.ext_off[j] * n_ext + (size_t)(HOIST ? xsrc.i[r] : r) * (n_rows - ns) + pos) * N;
                if (HOIST) {
                    const ulonglong2 v = __ldg(reinterpret_cast<const ulonglong2*>(e + (own & ~1)));
                    xs[j] = own_sw ? make_ulonglong2(v.y, v.x) : v;
                } else {
                    xs[j] = __ldg(reinterpret_cast<const ulonglong2*>(e + c));
                }
            }
            load_key_halves<ND, SA>(key, j, krow, LK, N, c, kbs[j], kas[j]);
        }
        if constexpr (SA) seeded_a_halves<ND>(key, key_digits, krow, LK, N, c, p.q, kas);
        if (fp) {
#pragma unroll
            for (int j = 0; j < ND; j++) {
                const double x0 = u2d(xs[j].x), x1 = u2d(xs[j].y);
                fb0 = __dadd_rn(fb0, fp_mulmod_s(x0, __longlong_as_double((long long)kbs[j].x), m));
                fb1 = __dadd_rn(fb1, fp_mulmod_s(x1, __longlong_as_double((long long)kbs[j].y), m));
                fa0 = __dadd_rn(fa0, fp_mulmod_s(x0, key_a_fp<SA>(kas[j].x), m));
                fa1 = __dadd_rn(fa1, fp_mulmod_s(x1, key_a_fp<SA>(kas[j].y), m));
            }
        } else {
            U128 b0 = {0, 0}, b1 = {0, 0}, a0 = {0, 0}, a1 = {0, 0};
#pragma unroll
            for (int j = 0; j < ND; j++) {
                mac128(b0, xs[j].x, kbs[j].x);
                mac128(b1, xs[j].y, kbs[j].y);
                mac128(a0, xs[j].x, kas[j].x);
                mac128(a1, xs[j].y, kas[j].y);
            }
            const uint64_t q2 = 2 * p.q;
            ib0 = csub(ib0 + redc_lazy(b0.hi, b0.lo, p.q, p.qinv_neg), q2);
            ib1 = csub(ib1 + redc_lazy(b1.hi, b1.lo, p.q, p.qinv_neg), q2);
            ia0 = csub(ia0 + reduce_a_sum<SA>(a0, p), q2);
            ia1 = csub(ia1 + reduce_a_sum<SA>(a1, p), q2);
        }
    }
    ulonglong2 ob, oa;
    if (fp) {
        ob = make_ulonglong2(d2u(fp_canon(fb0, m)), d2u(fp_canon(fb1, m)));
        oa = make_ulonglong2(d2u(fp_canon(fa0, m)), d2u(fp_canon(fa1, m)));
    } else {
        ob = make_ulonglong2(csub(ib0, p.q), csub(ib1, p.q));
        oa = make_ulonglong2(csub(ia0, p.q), csub(ia1, p.q));
    }
    uint64_t* out = u + ((size_t)o * 2 * n_rows) * N + c;
    *reinterpret_cast<ulonglong2*>(out + (size_t)t * N) = ob;
    *reinterpret_cast<ulonglong2*>(out + (size_t)(n_rows + t) * N) = oa;
}

// The hoisted k_ks_inner_sum for MO outputs whose G terms use the same keys
// term by term (key of term g of output o = key of term g of output o0, as
// in the rotate-and-sum of several ciphertexts over one step list): one
// position per thread; each key word (or, SA, its regeneration) and each
// automorphism index serves all MO outputs of a term.  Block x covers
// outputs MO x .. MO x + MO - 1.  Measured against k_ks_inner_sum, this
// form wins for hoisted sums, whose terms gather from shared raised digits,
// and loses for plain sums (BSGS giant steps), whose per-term digits are
// the bulk of the reads and lose their 16-byte pair loads here.
template <int ND, bool SA, int MO>
__global__ void __launch_bounds__(256, 4)
    k_ks_inner_sum_mo(const uint64_t* __restrict__ ext, PtrList din, GalList gal, PtrList keys, IdxList xsrc, int G,
                      uint64_t* __restrict__ u, int n_rows, int level, int L, int LK, int n_ext, int key_digits,
                      const DevPrime* __restrict__ pr, const FpMod* __restrict__ fpm, ModupArgs a, int logn) {
    const int N = 1 << logn;
    const int o0 = blockIdx.x * MO, t = blockIdx.z;
    const int c = blockIdx.y * blockDim.x + threadIdx.x;
    if (c >= N) return;
    const int krow = t < level ? t : L + (t - level);
    const int pidx = a.tprime[t];
    const DevPrime p = pr[pidx];
    constexpr int KW = SA ? 1 : 2;  // stored halves per digit
    // x_{r,j} at this thread's position (digit j's own rows through sigma_r)
    auto load_x = [&](int r, int own, int j) -> uint64_t {
        const int s0 = a.src_row[j], ns = a.n_src[j];
        if (t >= s0 && t < s0 + ns) return __ldg(din.p[r] + (size_t)t * N + own);
        const int pos = t < s0 ? t : t - ns;
        return __ldg(ext + ((size_t)a.ext_off[j] * n_ext + (size_t)xsrc.i[r] * (n_rows - ns) + pos) * N + own);
    };
    uint64_t* out0 = u + ((size_t)o0 * 2 * n_rows) * N + c;
    const size_t ostride = (size_t)2 * n_rows * N;
    if (p.q < kFpPrimeLimit) {
        const FpMod m = fpm[pidx];
        double fb[MO], fa[MO];
#pragma unroll
        for (int o = 0; o < MO; o++) fb[o] = fa[o] = 0.0;
        for (int g = 0; g < G; g++) {
            const int r0 = o0 * G + g;
            const uint64_t* key = keys.p[r0];
            const int own = automorph_src(c, logn, gal.g[r0]);
            double kb[ND], ka[ND];
#pragma unroll
            for (int j = 0; j < ND; j++) {
                kb[j] = __longlong_as_double((long long)__ldg(key + ((size_t)j * KW * LK + krow) * N + c));
                if constexpr (!SA)
                    ka[j] = __longlong_as_double((long long)__ldg(key + ((size_t)(j * KW + 1) * LK + krow) * N + c));
            }
            if constexpr (SA) {
                const uint64_t* s0p = key + (size_t)key_digits * LK * N + krow;
                const int sh = __clzll(p.q);
#pragma unroll
                for (int j = 0; j < ND; j++) ka[j] = u2d(seeded_a(__ldg(s0p + (size_t)j * LK), c, N, p.q, sh));
            }
#pragma unroll
            for (int o = 0; o < MO; o++) {
                const int r = r0 + o * G;
#pragma unroll
                for (int j = 0; j < ND; j++) {
                    const double x = u2d(load_x(r, own, j));
                    fb[o] = __dadd_rn(fb[o], fp_mulmod_s(x, kb[j], m));
                    fa[o] = __dadd_rn(fa[o], fp_mulmod_s(x, ka[j], m));
                }
            }
        }
#pragma unroll
        for (int o = 0; o < MO; o++) {
            out0[o * ostride + (size_t)t * N] = d2u(fp_canon(fb[o], m));
            out0[o * ostride + (size_t)(n_rows + t) * N] = d2u(fp_canon(fa[o], m));
        }
    } else {
        const uint64_t q2 = 2 * p.q;
        uint64_t ib[MO], ia[MO];
#pragma unroll
        for (int o = 0; o < MO; o++) ib[o] = ia[o] = 0;
        for (int g = 0; g < G; g++) {
            const int r0 = o0 * G + g;
            const uint64_t* key = keys.p[r0];
            const int own = automorph_src(c, logn, gal.g[r0]);
            uint64_t kb[ND], ka[ND];
#pragma unroll
            for (int j = 0; j < ND; j++) {
                kb[j] = __ldg(key + ((size_t)j * KW * LK + krow) * N + c);
                if constexpr (!SA) ka[j] = __ldg(key + ((size_t)(j * KW + 1) * LK + krow) * N + c);
            }
            if constexpr (SA) {
                const uint64_t* s0p = key + (size_t)key_digits * LK * N + krow;
                const int sh = __clzll(p.q);
#pragma unroll
                for (int j = 0; j < ND; j++) ka[j] = seeded_a(__ldg(s0p + (size_t)j * LK), c, N, p.q, sh);
            }
#pragma unroll
            for (int o = 0; o < MO; o++) {
                const int r = r0 + o * G;
                U128 b = {0, 0}, aa = {0, 0};
#pragma unroll
                for (int j = 0; j < ND; j++) {
                    const uint64_t x = load_x(r, own, j);
                    mac128(b, x, kb[j]);
                    mac128(aa, x, ka[j]);
                }
                ib[o] = csub(ib[o] + redc_lazy(b.hi, b.lo, p.q, p.qinv_neg), q2);
                ia[o] = csub(ia[o] + reduce_a_sum<SA>(aa, p), q2);
            }
        }
#pragma unroll
        for (int o = 0; o < MO; o++) {
            out0[o * ostride + (size_t)t * N] = csub(ib[o], p.q);
            out0[o * ostride + (size_t)(n_rows + t) * N] = csub(ia[o], p.q);
        }
    }
}

// tmp[i][poly][r][c] = sum_k y'_k (P/p_k mod q_r), y_k = [x_k (P/p_k)^-1]_{p_k},
// y'_k = y_k or y_k - p_k (centred, |y'_k| < 2^59).  Two arithmetic paths:
//  - FP64 (targets below 2^41): with y'_k = a_k 2^40 + b_k 2^20 + c_k
//    (|a_k| < 2^19; b_k, c_k < 2^20) and m_kr = P/p_k mod q_r = h 2^21 + l
//    (h < 2^20, l < 2^21), every partial product is below 2^41 in magnitude,
//    so the six sums over k (KP <= 16 terms) are exact doubles below 2^45:
//      S = T_cl + 2^20 (T_bl + 2 T_ch) + 2^40 (T_al + 2 T_bh) + 2^61 T_ah,
//    and three rounded-quotient products by 2^20, 2^40, 2^61 mod q_r and one
//    reduction give S mod q_r.
//  - integer (the 60-bit q_0): since p_k (P/p_k) = P for every k, the centring
//    subtracts (number of negative terms) * P; the sum of the y_k products is
//    accumulated in 128 bits and reduced once.
template <int KP>
__global__ void __launch_bounds__(256)
    k_moddown_conv(const uint64_t* __restrict__ u, uint64_t* __restrict__ tmp, int level, int L,
                   const DevPrime* __restrict__ pr, const FpMod* __restrict__ fpm, const ulonglong2* __restrict__ pcoef,
                   const ulonglong2* __restrict__ mat, const uint64_t* __restrict__ negP, int logn) {
    __shared__ uint64_t sm_m[KP * kConvMaxTargets];
    __shared__ double2 sm_hl[KP * kConvMaxTargets];  // {h, l} of m_kr
    __shared__ ConvTarget sm_t[kConvMaxTargets];
    __shared__ FpMod sm_f[kConvMaxTargets];
    __shared__ double4 sm_pow[kConvMaxTargets];  // {2^20, 2^40, 2^61} mod q_r
    __shared__ uint64_t sm_neg[kConvMaxTargets];
    const int N = 1 << logn;
    for (int idx = threadIdx.x; idx < KP * level; idx += blockDim.x) {
        int k = idx / level, r = idx - k * level;
        ulonglong2 m = mat[(size_t)k * L + r];
        sm_m[k * kConvMaxTargets + r] = m.x;
        sm_hl[k * kConvMaxTargets + r] = make_double2((double)(m.y >> 21), (double)(m.y & ((1ull << 21) - 1)));
    }
    for (int r = threadIdx.x; r < level; r += blockDim.x) {
        DevPrime p = pr[r];
        sm_t[r] = ConvTarget{p.q, p.qinv_neg, p.one_shoup, 0};
        const FpMod f = fpm[r];
        sm_f[r] = f;
        sm_neg[r] = negP[r];
        if (p.q < kFpPrimeLimit) {
            const double p20 = fp_canon(1048576.0, f), p21 = fp_canon(2097152.0, f);
            const double p40 = fp_modmul(p20, p20, f);
            sm_pow[r] = make_double4(p20, p40, fp_modmul(p40, p21, f), 0.0);
        }
    }
    __syncthreads();
    int c = blockIdx.x * blockDim.x + threadIdx.x;
    int poly = blockIdx.y, i = blockIdx.z;  // poly in {0, 1}
    if (c >= N) return;
    const int n_rows = level + KP;
    const uint64_t* x = u + (((size_t)i * 2 + poly) * n_rows + level) * N + c;
    uint64_t y[KP];
    uint64_t n_neg = 0;
#pragma unroll
    for (int k = 0; k < KP; k++) {
        uint64_t p = pr[L + k].q;
        ulonglong2 w = pcoef[k];
        y[k] = mul_shoup(x[(size_t)k * N], w.x, w.y, p);
        n_neg += y[k] > (p >> 1) ? 1u : 0u;
    }
    uint64_t* o = tmp + (((size_t)i * 2 + poly) * level) * N + c;
    // integer targets first, so that y is dead before the split below
    for (int r = 0; r < level; r++) {
        const ConvTarget t = sm_t[r];
        if (t.q < kFpPrimeLimit) continue;
        U128 acc = {0, 0};
#pragma unroll
        for (int k = 0; k < KP; k++) mac128(acc, y[k], sm_m[k * kConvMaxTargets + r]);
        uint64_t w = n_neg * sm_neg[r];                      // < 16 q <= 2^64
        uint64_t wr = w - __umul64hi(w, t.one_shoup) * t.q;  // [0, 2q)
        uint64_t v = redc_t(acc, t) + wr;                    // [0, 3q)
        o[(size_t)r * N] = csub(csub(v, 2 * t.q), t.q);
    }
    double ya[KP], yb[KP], yc[KP];
#pragma unroll
    for (int k = 0; k < KP; k++) {
        const uint64_t p = pr[L + k].q;
        const long long v = y[k] > (p >> 1) ? (long long)(y[k] - p) : (long long)y[k];
        ya[k] = (double)(v >> 40);                        // exact: |.| < 2^19
        yb[k] = (double)((v >> 20) & ((1ll << 20) - 1));  // exact: < 2^20
        yc[k] = (double)(v & ((1ll << 20) - 1));          // exact: < 2^20
    }
    for (int r = 0; r < level; r++) {
        if (sm_t[r].q >= kFpPrimeLimit) continue;
        double t_ah = 0, t_al = 0, t_bh = 0, t_bl = 0, t_ch = 0, t_cl = 0;  // exact partial sums
#pragma unroll
        for (int k = 0; k < KP; k++) {
            const double2 m = sm_hl[k * kConvMaxTargets + r];
            t_ah = __fma_rn(ya[k], m.x, t_ah);
            t_al = __fma_rn(ya[k], m.y, t_al);
            t_bh = __fma_rn(yb[k], m.x, t_bh);
            t_bl = __fma_rn(yb[k], m.y, t_bl);
            t_ch = __fma_rn(yc[k], m.x, t_ch);
            t_cl = __fma_rn(yc[k], m.y, t_cl);
        }
        const FpMod f = sm_f[r];
        const double4 pw = sm_pow[r];
        double acc = fp_reduce_s(t_cl, f);
        acc = __dadd_rn(acc, fp_mulmod_s(__fma_rn(2.0, t_ch, t_bl), pw.x, f));
        acc = __dadd_rn(acc, fp_mulmod_s(__fma_rn(2.0, t_bh, t_al), pw.y, f));
        acc = __dadd_rn(acc, fp_mulmod_s(t_ah, pw.z, f));
        o[(size_t)r * N] = d2u(fp_canon(acc, f));
    }
}

// Outputs of ModDown: out_i = [2][level][N]; add0/add1 (or null) are added
// to the two polynomials, add0 read through sigma_{g_i} when sig_add0 is set.
struct MdOut {
    MutPtrList out;
    PtrList add0, add1;
    GalList gal;
    int sig_add0;
};

// Second pass of the forward NTT of tmp fused with the end of ModDown:
//   out_i[poly][t][c] = (u[poly][t][c] - NTT(tmp)[poly][t][c]) P^-1 + add_poly[t][c].
// tmp rows are [i][poly][t] (prime index t).  Grid (ROW_TILES, n 2 level).
template <int LOGN>
__global__ void __launch_bounds__(NttCfg<LOGN>::ROW_THREADS, NTT_MIN_BLOCKS)
    k_fwd_rows_moddown(const uint64_t* __restrict__ tmp, const uint64_t* __restrict__ u, MdOut mo, int level, int K,
                       const DevPrime* __restrict__ pr, const ulonglong2* __restrict__ pinv,
                       const ulonglong2* __restrict__ tw_all, const double* __restrict__ twd_all,
                       const FpMod* __restrict__ fpm) {
    using Cf = NttCfg<LOGN>;
    __shared__ uint64_t sm[Cf::TR * Cf::ROW_PITCH];
    const int y = blockIdx.y, i = y / (2 * level), rem = y - i * 2 * level;
    const int poly = rem / level, t = rem - poly * level;
    const uint64_t q = pr[t].q;
    const int r = blockIdx.x * Cf::TR + threadIdx.x / (Cf::C / 16);
    const int j0 = r * Cf::C + 16 * row_lane<LOGN>();
    const uint64_t* a = tmp + (size_t)y * Cf::N + (size_t)r * Cf::C;
    uint64_t v[16];
    if (q < kFpPrimeLimit) {
        const FpMod m = fpm[t];
        double x[16];
        row_load_strided<LOGN>(x, a);
        fwd_rows_core<LOGN>(x, reinterpret_cast<double*>(sm), r, twd_all + (size_t)t * Cf::N, m);
#pragma unroll
        for (int k = 0; k < 16; k++) v[k] = fwd_canon(x[k], m);
    } else {
        uint64_t x[16];
        row_load_strided<LOGN>(x, a);
        fwd_rows_core<LOGN>(x, sm, r, tw_all + (size_t)t * Cf::N, q);
#pragma unroll
        for (int k = 0; k < 16; k++) v[k] = fwd_canon(x[k], q);
    }
    const size_t off = (size_t)t * Cf::N + j0;  // within a [level][N] polynomial
    const uint64_t* up = u + (size_t)(i * 2 + poly) * (level + K) * Cf::N + off;
    uint64_t* op = mo.out.p[i] + (size_t)poly * level * Cf::N + off;
    const uint64_t* ad = poly == 0 ? mo.add0.p[i] : mo.add1.p[i];
    const uint64_t g = (poly == 0 && mo.sig_add0) ? mo.gal.g[i] : 0;
    const ulonglong2 w = pinv[t];
    const uint64_t* adt = ad ? ad + (size_t)t * Cf::N : nullptr;
#pragma unroll
    for (int k = 0; k < 4; k++) {
        uint64_t z[4];
        ldg256_ro(up + 4 * k, z[0], z[1], z[2], z[3]);
#pragma unroll
        for (int e = 0; e < 4; e++) z[e] = mul_shoup(z[e] + q - v[4 * k + e], w.x, w.y, q);
        if (adt) {
#pragma unroll
            for (int h = 0; h < 2; h++) {
                const int s = automorph_src(j0 + 4 * k + 2 * h, LOGN, g);
                const ulonglong2 av = __ldg(reinterpret_cast<const ulonglong2*>(adt + (s & ~1)));
                const bool sw = s & 1;
                z[2 * h] = add_mod(z[2 * h], sw ? av.y : av.x, q);
                z[2 * h + 1] = add_mod(z[2 * h + 1], sw ? av.x : av.y, q);
            }
        }
        stg256(op + 4 * k, z[0], z[1], z[2], z[3]);
    }
}

static ModupArgs modup_args(he_ctx* c, int level) {
    ModupArgs a;
    auto& tabs = c->modup[level];
    a.n_digits = (int)tabs.size();
    long long off = 0;
    for (int j = 0; j < a.n_digits; j++) {
        a.n_src[j] = tabs[j].n_src;
        a.src_row[j] = tabs[j].src_row;
        a.src[j] = tabs[j].d_src;
        a.mat[j] = tabs[j].d_mat;
        a.ext_off[j] = off;
        off += level + c->K - tabs[j].n_src;
    }
    std::vector<int> ep = ext_primes(c, level);
    for (size_t t = 0; t < ep.size(); t++) a.tprime[t] = (uint8_t)ep[t];
    return a;
}

static int lc(he_ctx* c, const char* what) {
    c->launches++;
    return check_cuda(c, cudaGetLastError(), what);
}

// coef [nm][level], ext [nm][sum_j (level+K-|D_j|)], u [n][2][level+K],
// tmp [n][2][level]: nm ciphertexts raised by ModUp, n key-switched.
size_t key_switch_scratch_words(const he_ctx* c, int nm, int n, int level) {
    size_t nd = (level + c->alpha - 1) / c->alpha, nr = level + c->K;
    size_t ext_rows = nd * nr - level;
    return (size_t)c->N * ((size_t)nm * (level + ext_rows) + (size_t)n * (2 * nr + 2 * level));
}

// Launches of the transform-fused kernels for the context's ring degree.
template <int LOGN>
static void launch_inv_rows_gather(he_ctx* c, const PtrList& din, const GalList& gal, uint64_t* coef, int n,
                                   int level) {
    using Cf = NttCfg<LOGN>;
    k_inv_rows_gather<LOGN><<<dim3(Cf::ROW_TILES, n * level), Cf::ROW_THREADS, 0, c->stream>>>(
        din, gal, coef, level, c->d_prime, c->d_tw_inv, c->d_twd_inv, c->d_fpmod);
}

template <int LOGN>
static void launch_fwd_rows_moddown(he_ctx* c, const uint64_t* tmp, const uint64_t* u, const MdOut& mo, int n,
                                    int level) {
    using Cf = NttCfg<LOGN>;
    k_fwd_rows_moddown<LOGN><<<dim3(Cf::ROW_TILES, n * 2 * level), Cf::ROW_THREADS, 0, c->stream>>>(
        tmp, u, mo, level, c->K, c->d_prime, c->d_md_pinv, c->d_tw_fwd, c->d_twd_fwd, c->d_fpmod);
}

#define HE_LOGN_SWITCH(c, CALL)                  \
    switch ((c)->log_n) {                        \
        case 10: CALL(10); break;                \
        case 11: CALL(11); break;                \
        case 12: CALL(12); break;                \
        case 13: CALL(13); break;                \
        case 14: CALL(14); break;                \
        case 15: CALL(15); break;                \
        case 16: CALL(16); break;                \
        default: break;                          \
    }

int key_switch_chunk(he_ctx* c, int n, int level, const KsIoList& io) {
    const int N = c->N, K = c->K, L = c->L, LK = L + K;
    const int n_rows = level + K;
    ModupArgs ma = modup_args(c, level);
    const int nd = ma.n_digits;
    // hoisted: ModUp raises the nm inputs hoist_d once (no automorphism) and
    // the inner product reads them through each output's sigma
    const bool hoist = !io.hoist_d.empty();
    const int nm = hoist ? (int)io.hoist_d.size() : n;
    if (nm > kMaxBatch || (hoist && (int)io.hoist_src.size() != n))
        return set_err(c, HE_EINVAL, "key switch: bad hoisting lists");
    // summed: n_md = n / G outputs, each the sum of G key switches
    const int G = io.sum_terms;
    const bool summed = G > 0;
    if (summed && n % G) return set_err(c, HE_EINVAL, "key switch: bad summed lists");
    const int n_md = summed ? n / G : n;
    uint64_t* base;
    int rc = scratch_slot(c, c->ks_slot, key_switch_scratch_words(c, nm, n_md, level), &base);
    if (rc) return rc;
    const int ext_rows = nd * n_rows - level;  // sum over digits of the target rows
    uint64_t* coef = base;
    uint64_t* ext = coef + (size_t)nm * level * N;
    uint64_t* u = ext + (size_t)nm * ext_rows * N;
    uint64_t* tmp = u + (size_t)n_md * 2 * n_rows * N;

    PtrList din, keys, mdin;
    GalList gal, mgal;
    IdxList xsrc;
    MdOut mo;
    mo.sig_add0 = io.sig_add0 ? 1 : 0;
    for (int i = 0; i < kMaxBatch; i++) {
        gal.g[i] = i < n ? io.galois[i] : 0;
        keys.p[i] = i < n ? io.key[i] : nullptr;
        din.p[i] = i < n ? io.d[i] : nullptr;
        mo.out.p[i] = i < n_md ? io.out[i] : nullptr;
        mo.add0.p[i] = i < n_md ? io.add0[i] : nullptr;
        mo.add1.p[i] = i < n_md ? io.add1[i] : nullptr;
        mdin.p[i] = hoist ? (i < nm ? io.hoist_d[i] : nullptr) : din.p[i];
        mgal.g[i] = hoist ? 0 : gal.g[i];
        xsrc.i[i] = hoist && i < n ? io.hoist_src[i] : i;
        if (hoist && i < n && (xsrc.i[i] < 0 || xsrc.i[i] >= nm || io.hoist_d[xsrc.i[i]] != io.d[i]))
            return set_err(c, HE_EINVAL, "key switch: output %d has no raised input", i);
    }
    mo.gal = gal;
    const int TB = 256;
    dim3 blk(TB);
    int gx = (N + TB - 1) / TB;

    const double limbB = 8.0 * N;
    const NttShape sh = ntt_shape(c->log_n);
    int sum_src = 0;
    for (int j = 0; j < nd; j++) sum_src += ma.n_src[j];
    std::vector<int> ep = ext_primes(c, level);
    int fp_q = 0;  // primes of Q_level on the FP64 path
    for (int t = 0; t < level; t++) fp_q += fp_prime(c, t);

    // sigma(d) (hoisted: d) back to coefficients: gathered row pass, then the
    // column pass
    prof_begin(c, HE_PROF_NTT_INV_ROWS);
#define HE_IRG(LN) launch_inv_rows_gather<LN>(c, mdin, mgal, coef, nm, level)
    HE_LOGN_SWITCH(c, HE_IRG)
#undef HE_IRG
    if ((rc = lc(c, "inv_rows_gather"))) return rc;
    prof_end(c, HE_PROF_NTT_INV_ROWS, 2.0 * nm * level * limbB, 0.5 * N * nm * level * sh.s2,
             0.5 * N * nm * fp_q * sh.s2);
    std::vector<int> qp = prime_range(0, level);
    if ((rc = ntt_inv_cols_set(c, rowset_contig(coef, level, N, qp), nm * level))) return rc;

    prof_begin(c, HE_PROF_MODUP);
    for (int j = 0; j < nd; j++) {
        uint64_t* ext_j = ext + (size_t)ma.ext_off[j] * nm * N;
        const int s0 = ma.src_row[j], ns = ma.n_src[j];
        bool narrow_j = true;  // every source prime of the digit below 2^41
        for (int s = 0; s < ns; s++) narrow_j = narrow_j && fp_prime(c, s0 + s);
        ConvLists cl;
        cl.n_fp = cl.n_int = 0;
        for (int tt = 0; tt < n_rows - ns; tt++) {
            const int t = tt < s0 ? tt : tt + ns;
            if (fp_prime(c, ep[t]))
                cl.fp_tt[cl.n_fp++] = (uint8_t)tt;
            else
                cl.int_tt[cl.n_int++] = (uint8_t)tt;
        }
        if (cl.n_int > kConvMaxInt) return set_err(c, HE_EINVAL, "key switch: %d wide targets unsupported", cl.n_int);
        // only the first source 60-bit (the digit holding q_0)?
        bool wide0 = !narrow_j && !fp_prime(c, s0);
        for (int s = 1; s < ns && wide0; s++) wide0 = fp_prime(c, s0 + s);
        const int mode = narrow_j ? kConvNarrow : (wide0 ? kConvWide0 : kConvGeneric);
        switch (ns * 3 + mode) {
#define HE_MU_LAUNCH(S, MD)                                                                                        \
    k_modup_conv<S, MD><<<dim3(gx, nm), blk, 0, c->stream>>>(coef, ext_j, ma.src[j], ma.mat[j], ma, cl, c->d_prime, \
                                                           c->d_fpmod, level, n_rows, s0, c->log_n)
#define HE_MU_CASE(S)                      \
    case 3 * S + kConvGeneric:             \
        HE_MU_LAUNCH(S, kConvGeneric);     \
        break;                             \
    case 3 * S + kConvNarrow:              \
        HE_MU_LAUNCH(S, kConvNarrow);      \
        break;                             \
    case 3 * S + kConvWide0:               \
        HE_MU_LAUNCH(S, kConvWide0);       \
        break;
            HE_MU_CASE(1) HE_MU_CASE(2) HE_MU_CASE(3) HE_MU_CASE(4) HE_MU_CASE(5) HE_MU_CASE(6) HE_MU_CASE(7)
            HE_MU_CASE(8) HE_MU_CASE(9) HE_MU_CASE(10) HE_MU_CASE(11) HE_MU_CASE(12) HE_MU_CASE(13)
            HE_MU_CASE(14) HE_MU_CASE(15) HE_MU_CASE(16)
#undef HE_MU_CASE
#undef HE_MU_LAUNCH
            default:
                return set_err(c, HE_EINVAL, "key switch: digit of %d primes unsupported", ns);
        }
        if ((rc = lc(c, "modup_conv"))) return rc;
    }
    {
        double prods = 0, prods_fp = 0;
        for (int j = 0; j < nd; j++) {
            prods += (double)ma.n_src[j] * (1 + n_rows - ma.n_src[j]);
            // FP64 pipe: 40-bit targets, and every target of a digit of 40-bit
            // sources (exact FP64 partial sums, six FMAs per product)
            int narrow_j = 1, wide0 = !fp_prime(c, ma.src_row[j]);  // digit all 40-bit / only its first source 60-bit
            for (int s = 0; s < ma.n_src[j]; s++) narrow_j &= fp_prime(c, ma.src_row[j] + s);
            for (int s = 1; s < ma.n_src[j]; s++) wide0 &= fp_prime(c, ma.src_row[j] + s);
            narrow_j |= wide0;
            for (int t = 0; t < n_rows; t++)
                if ((t < ma.src_row[j] || t >= ma.src_row[j] + ma.n_src[j]) && (narrow_j || fp_prime(c, ep[t])))
                    prods_fp += ma.n_src[j];
        }
        prof_end(c, HE_PROF_MODUP, (double)nm * (sum_src + ext_rows) * limbB, (double)nm * N * prods,
                 (double)nm * N * prods_fp);
    }
    for (int j = 0; j < nd; j++) {
        std::vector<int> tp;
        for (int t = 0; t < n_rows; t++)
            if (t < ma.src_row[j] || t >= ma.src_row[j] + ma.n_src[j]) tp.push_back(ep[t]);
        const int nt = (int)tp.size();
        RowSet rs = rowset_contig(ext + (size_t)ma.ext_off[j] * nm * N, nt, N, tp);
        if ((rc = ntt_fwd_set(c, rs, nm * nt))) return rc;
    }

    prof_begin(c, HE_PROF_KS_INNER);
    const int gx2 = (N / 2 + TB - 1) / TB;  // two positions per thread
    const int kd = he_key_digits(c);
    // groups of adjacent entries that share a key, at most kKsGroupMax each
    IdxList grp;
    int n_grp = 0;
    for (int i = 0; i < n; i++)
        if (i == 0 || io.key[i] != io.key[i - 1] || io.galois[i] != io.galois[i - 1] ||
            i - grp.i[n_grp - 1] >= kKsGroupMax)
            grp.i[n_grp++] = i;
    // single entries keep the lighter per-entry kernel (48 registers, five
    // blocks per SM against four)
    const bool grouped = !summed && n_grp < n;
    // hoisted sums whose outputs, kKsSumMo at a time, use the same key term
    // by term (rotate-and-sum of several ciphertexts over one step list)
    bool sum_mo = summed && hoist && n_md % kKsSumMo == 0;
    for (int o = 0; sum_mo && o < n_md; o++)
        for (int g = 0; g < G && sum_mo; g++) {
            const size_t r = (size_t)o * G + g, r0 = (size_t)(o - o % kKsSumMo) * G + g;
            sum_mo = io.key[r] == io.key[r0] && io.galois[r] == io.galois[r0];
        }
    switch (nd * 2 + (keys_seeded_a(c) ? 1 : 0)) {
#define HE_KS_LAUNCH(D, SA)                                                                                        \
    if (sum_mo)                                                                                                    \
        k_ks_inner_sum_mo<D, SA, kKsSumMo><<<dim3(n_md / kKsSumMo, gx, n_rows), blk, 0, c->stream>>>(             \
            ext, din, gal, keys, xsrc, G, u, n_rows, level, L, LK, nm, kd, c->d_prime, c->d_fpmod, ma, c->log_n);  \
    else if (summed && hoist)                                                                                      \
        k_ks_inner_sum<D, true, SA><<<dim3(n_md, gx2, n_rows), blk, 0, c->stream>>>(                               \
            ext, din, gal, keys, xsrc, G, u, n_rows, level, L, LK, nm, kd, c->d_prime, c->d_fpmod, ma, c->log_n);  \
    else if (summed)                                                                                               \
        k_ks_inner_sum<D, false, SA><<<dim3(n_md, gx2, n_rows), blk, 0, c->stream>>>(                              \
            ext, din, gal, keys, xsrc, G, u, n_rows, level, L, LK, nm, kd, c->d_prime, c->d_fpmod, ma, c->log_n);  \
    else if (grouped && hoist)                                                                                     \
        k_ks_inner_grp<D, true, SA><<<dim3(n_grp, gx2, n_rows), blk, 0, c->stream>>>(                              \
            ext, din, gal, keys, xsrc, grp, n_grp, n, u, n_rows, level, L, LK, nm, kd, c->d_prime, c->d_fpmod, ma, \
            c->log_n);                                                                                             \
    else if (grouped)                                                                                              \
        k_ks_inner_grp<D, false, SA><<<dim3(n_grp, gx2, n_rows), blk, 0, c->stream>>>(                             \
            ext, din, gal, keys, xsrc, grp, n_grp, n, u, n_rows, level, L, LK, nm, kd, c->d_prime, c->d_fpmod, ma, \
            c->log_n);                                                                                             \
    else if (hoist)                                                                                                \
        k_ks_inner<D, true, SA><<<dim3(n, gx2, n_rows), blk, 0, c->stream>>>(                                      \
            ext, din, gal, keys, xsrc, u, n_rows, level, L, LK, nm, kd, c->d_prime, c->d_fpmod, ma, c->log_n);     \
    else                                                                                                           \
        k_ks_inner<D, false, SA><<<dim3(n, gx2, n_rows), blk, 0, c->stream>>>(                                     \
            ext, din, gal, keys, xsrc, u, n_rows, level, L, LK, nm, kd, c->d_prime, c->d_fpmod, ma, c->log_n);
#define HE_KS_CASE(D)         \
    case 2 * D:               \
        HE_KS_LAUNCH(D, false) \
        break;                \
    case 2 * D + 1:           \
        HE_KS_LAUNCH(D, true)  \
        break;
        HE_KS_CASE(1) HE_KS_CASE(2) HE_KS_CASE(3) HE_KS_CASE(4) HE_KS_CASE(5) HE_KS_CASE(6) HE_KS_CASE(7)
        HE_KS_CASE(8) HE_KS_CASE(9) HE_KS_CASE(10) HE_KS_CASE(11) HE_KS_CASE(12) HE_KS_CASE(13) HE_KS_CASE(14)
        HE_KS_CASE(15)
#undef HE_KS_CASE
#undef HE_KS_LAUNCH
        default:
            return set_err(c, HE_EINVAL, "key switch: %d digits unsupported", nd);
    }
    if ((rc = lc(c, "ks_inner"))) return rc;
    {
        // raised digits of each raised input once, each distinct key once,
        // the products written once
        int fp_rows_ks = 0;
        for (int t = 0; t < n_rows; t++) fp_rows_ks += fp_prime(c, ep[t]);
        std::vector<const uint64_t*> kd(io.key.begin(), io.key.begin() + n);
        std::sort(kd.begin(), kd.end());
        const double n_keys = (double)(std::unique(kd.begin(), kd.end()) - kd.begin());
        const double key_halves = keys_seeded_a(c) ? 1.0 : 2.0;  // a-halves regenerated, not read
        prof_end(c, HE_PROF_KS_INNER,
                 ((double)nm * nd * n_rows + n_keys * key_halves * nd * n_rows + 2.0 * n_md * n_rows) * limbB,
                 (double)n * n_rows * N * 2.0 * nd, (double)n * fp_rows_ks * N * 2.0 * nd);
    }

    std::vector<int> pp = prime_range(L, K);
    RowSet prs = rowset(u + (size_t)level * N, (long long)n_rows * N, K, pp.data());
    if ((rc = ntt_inv_set(c, prs, n_md * 2 * K))) return rc;

    prof_begin(c, HE_PROF_MODDOWN_CONV);
    if (c->tc_moddown) {
        if ((rc = moddown_conv_tc(c, u, tmp, n_md, level))) return rc;
        c->launches--;  // counted once below
    } else {
        switch (K) {
#define HE_MD_CASE(KK)                                                                                          \
    case KK:                                                                                                    \
        k_moddown_conv<KK><<<dim3(gx, 2, n_md), blk, 0, c->stream>>>(u, tmp, level, L, c->d_prime, c->d_fpmod, \
                                                                  c->d_md_pcoef, c->d_md_mat, c->d_md_negP,    \
                                                                  c->log_n);                                   \
        break;
            HE_MD_CASE(1) HE_MD_CASE(2) HE_MD_CASE(3) HE_MD_CASE(4) HE_MD_CASE(5) HE_MD_CASE(6) HE_MD_CASE(7)
            HE_MD_CASE(8) HE_MD_CASE(9) HE_MD_CASE(10) HE_MD_CASE(11) HE_MD_CASE(12) HE_MD_CASE(13) HE_MD_CASE(14)
            HE_MD_CASE(15) HE_MD_CASE(16)
#undef HE_MD_CASE
            default:
                return set_err(c, HE_EINVAL, "key switch: K = %d unsupported", K);
        }
    }
    if ((rc = lc(c, "moddown_conv"))) return rc;
    {
        int fp_t = 0;
        for (int r = 0; r < level; r++) fp_t += fp_prime(c, r);
        prof_end(c, HE_PROF_MODDOWN_CONV, 2.0 * n_md * (K + level) * limbB,
                 2.0 * n_md * N * (K + (double)K * (level - fp_t) + 2.0 * K * fp_t),
                 2.0 * n_md * N * 2.0 * K * fp_t);
    }

    // back to the evaluation domain: column pass, then the row pass fused
    // with (u - tmp) P^-1 + add
    if ((rc = ntt_fwd_cols_set(c, rowset_contig(tmp, level, N, qp), n_md * 2 * level))) return rc;
    prof_begin(c, HE_PROF_MODDOWN_COMBINE);
#define HE_FRM(LN) launch_fwd_rows_moddown<LN>(c, tmp, u, mo, n_md, level)
    HE_LOGN_SWITCH(c, HE_FRM)
#undef HE_FRM
    if ((rc = lc(c, "fwd_rows_moddown"))) return rc;
    {
        int n_add = 0;
        for (int i = 0; i < n_md; i++)
            n_add += (io.add0[i] != nullptr) + (io.add1[i] != nullptr);
        prof_end(c, HE_PROF_MODDOWN_COMBINE, (6.0 * n_md + n_add) * level * limbB,
                 2.0 * n_md * level * N * (1.0 + 0.5 * sh.s2), 2.0 * n_md * fp_q * N * 0.5 * sh.s2);
    }
    return HE_OK;
}

int key_switch(he_ctx* c, int level, const KsIoList& io) {
    int n = (int)io.d.size();
    for (int i0 = 0; i0 < n; i0 += kMaxBatch) {
        int m = std::min(kMaxBatch, n - i0);
        KsIoList sub;
        sub.sig_add0 = io.sig_add0;
        sub.galois.assign(io.galois.begin() + i0, io.galois.begin() + i0 + m);
        sub.key.assign(io.key.begin() + i0, io.key.begin() + i0 + m);
        sub.d.assign(io.d.begin() + i0, io.d.begin() + i0 + m);
        sub.out.assign(io.out.begin() + i0, io.out.begin() + i0 + m);
        sub.add0.assign(io.add0.begin() + i0, io.add0.begin() + i0 + m);
        sub.add1.assign(io.add1.begin() + i0, io.add1.begin() + i0 + m);
        int rc = key_switch_chunk(c, m, level, sub);
        if (rc) return rc;
    }
    return HE_OK;
}

// Key switching of a batch split in two halves on two streams: the first
// half on the context's stream, the second on an auxiliary stream with its
// own scratch, forked from and joined back into the context's stream by
// events.  Each half is a chain of ALU-heavy and memory-heavy kernels; run
// side by side, one half's key inner product streams keys while the other
// converts or transforms.  The split falls on a key boundary (entries that
// share a key are adjacent), so each key is still read once per half at
// most (a batch with a single key, as in relinearisation, splits in the
// middle and each half reads the key once).  Results are the same as
// key_switch's.  With profiling on, or for small batches, one stream does
// everything in order.
int key_switch_split(he_ctx* c, int level, const KsIoList& io) {
    const int n = (int)io.d.size();
    if (c->prof_on || n < 16) return key_switch(c, level, io);
    int k = n / 2;
    while (k < n && io.key[k] == io.key[k - 1]) k++;  // next key boundary at or after n/2
    if (k == n) {                                      // else the last one before it
        k = n / 2;
        while (k > 0 && io.key[k] == io.key[k - 1]) k--;
    }
    if (k == 0) k = n / 2;  // one key for all
    int rc;
    if (!c->aux && (rc = check_cuda(c, cudaStreamCreateWithFlags(&c->aux, cudaStreamNonBlocking), "aux stream")))
        return rc;
    if (!c->ev_fork && (rc = check_cuda(c, cudaEventCreateWithFlags(&c->ev_fork, cudaEventDisableTiming), "event")))
        return rc;
    if (!c->ev_join && (rc = check_cuda(c, cudaEventCreateWithFlags(&c->ev_join, cudaEventDisableTiming), "event")))
        return rc;
    auto part = [&](int a, int b) {
        KsIoList h;
        h.sig_add0 = io.sig_add0;
        h.galois.assign(io.galois.begin() + a, io.galois.begin() + b);
        h.key.assign(io.key.begin() + a, io.key.begin() + b);
        h.d.assign(io.d.begin() + a, io.d.begin() + b);
        h.out.assign(io.out.begin() + a, io.out.begin() + b);
        h.add0.assign(io.add0.begin() + a, io.add0.begin() + b);
        h.add1.assign(io.add1.begin() + a, io.add1.begin() + b);
        return h;
    };
    if ((rc = check_cuda(c, cudaEventRecord(c->ev_fork, c->stream), "fork")) ||
        (rc = check_cuda(c, cudaStreamWaitEvent(c->aux, c->ev_fork, 0), "fork")))
        return rc;
    rc = key_switch(c, level, part(0, k));
    cudaStream_t main = c->stream;
    if (!rc) {
        c->stream = c->aux;
        c->ks_slot = 4;
        rc = key_switch(c, level, part(k, n));
        c->stream = main;
        c->ks_slot = 0;
    }
    // join whatever was enqueued on the auxiliary stream, also after an error
    int rj = check_cuda(c, cudaEventRecord(c->ev_join, c->aux), "join");
    if (!rj) rj = check_cuda(c, cudaStreamWaitEvent(c->stream, c->ev_join, 0), "join");
    return rc ? rc : rj;
}

static int ct_ok(he_ctx* c, const he_ct* x, const char* what) {
    if (!x || !x->data) return set_err(c, HE_EINVAL, "%s: null ciphertext", what);
    if ((uintptr_t)x->data & 31) return set_err(c, HE_EINVAL, "%s: ciphertext not 32-byte aligned", what);
    if (x->level < 1 || x->level > c->L) return set_err(c, HE_ELEVEL, "%s: level %d out of range", what, x->level);
    if (!x->is_ntt) return set_err(c, HE_EDOMAIN, "%s: ciphertext not in the evaluation domain", what);
    return HE_OK;
}

int rotate_many(he_ctx* c, const he_ct* in, const int32_t* steps, he_ct* out, int n) {
    if (n < 0) return set_err(c, HE_EINVAL, "rotate: negative count");
    if (n == 0) return HE_OK;
    if (!in || !out || !steps) return set_err(c, HE_EINVAL, "rotate: null argument");
    int level = in[0].level;
    for (int i = 0; i < n; i++) {
        int rc = ct_ok(c, &in[i], "rotate");
        if (rc) return rc;
        if (in[i].level != level) return set_err(c, HE_ELEVEL, "rotate: mixed levels in a batch");
        if (!out[i].data || ((uintptr_t)out[i].data & 31)) return set_err(c, HE_EINVAL, "rotate: null or unaligned output");
        if (out[i].data == in[i].data) return set_err(c, HE_EINVAL, "rotate: output aliases input");
    }
    // group by Galois element so that each key is streamed once per group
    std::map<uint64_t, std::vector<int>> groups;
    for (int i = 0; i < n; i++) {
        uint64_t g = galois_elt(c, steps[i]);
        if (g != 1 && !c->rot_keys.count(g))
            return set_err(c, HE_ENOKEY, "rotate: no key for step %d (galois %llu)", steps[i], (unsigned long long)g);
        groups[g].push_back(i);
    }
    // one key-switching pass over every ciphertext, ordered by key
    const size_t ct_words = (size_t)2 * level * c->N;
    KsIoList io;
    io.sig_add0 = true;
    for (auto& kv : groups) {
        if (kv.first == 1) {  // rotation by a multiple of N/2: identity
            for (int i : kv.second) {
                int rc = check_cuda(c, cudaMemcpyAsync(out[i].data, in[i].data, ct_words * 8,
                                                       cudaMemcpyDeviceToDevice, c->stream),
                                    "rotate copy");
                if (rc) return rc;
            }
            continue;
        }
        const uint64_t* key = c->rot_keys[kv.first].d;
        for (int i : kv.second) {
            io.galois.push_back(kv.first);
            io.key.push_back(key);
            io.d.push_back(in[i].data + (size_t)level * c->N);
            io.out.push_back(out[i].data);
            io.add0.push_back(in[i].data);
            io.add1.push_back(nullptr);
        }
    }
    if (!io.d.empty()) {
        int rc = key_switch_split(c, level, io);
        if (rc) return rc;
    }
    for (int i = 0; i < n; i++) {
        out[i].level = level;
        out[i].scale = in[i].scale;
        out[i].is_ntt = 1;
    }
    return HE_OK;
}

// Hoisted rotations (Halevi-Shoup, CRYPTO 2018, section 5):
// out[i n_steps + s] = (sigma_k(c0) + ModDown(sum_j sigma_k(ModUp_j(c1)) (.) evk_j.b),
//                        ModDown(sum_j sigma_k(ModUp_j(c1)) (.) evk_j.a)),  k = 5^steps[s],
// for the inputs in[i] = (c0, c1).  ModUp runs once per input and chunk of
// steps; each output reads the raised digits through its automorphism inside
// the inner product.  Outputs are ordered step-major within a chunk, so
// neighbouring inner-product blocks share a key tile.  Steps whose Galois
// element is 1 are copies.
int rotate_hoisted_many(he_ctx* c, const he_ct* in, int n_in, const int32_t* steps, int n_steps, he_ct* out) {
    if (n_in < 0 || n_steps < 0) return set_err(c, HE_EINVAL, "rotate_hoisted: negative count");
    if (n_in == 0 || n_steps == 0) return HE_OK;
    if (!in || !out || !steps) return set_err(c, HE_EINVAL, "rotate_hoisted: null argument");
    const int level = in[0].level;
    std::set<const uint64_t*> ins;
    for (int i = 0; i < n_in; i++) {
        int rc = ct_ok(c, &in[i], "rotate_hoisted");
        if (rc) return rc;
        if (in[i].level != level) return set_err(c, HE_ELEVEL, "rotate_hoisted: mixed levels");
        ins.insert(in[i].data);
    }
    for (long long o = 0; o < (long long)n_in * n_steps; o++) {
        if (!out[o].data || ((uintptr_t)out[o].data & 31))
            return set_err(c, HE_EINVAL, "rotate_hoisted: null or unaligned output %lld", o);
        if (ins.count(out[o].data)) return set_err(c, HE_EINVAL, "rotate_hoisted: output %lld aliases an input", o);
    }
    std::vector<int> eff;  // steps that key-switch
    std::vector<uint64_t> gal(n_steps);
    for (int s = 0; s < n_steps; s++) {
        gal[s] = galois_elt(c, steps[s]);
        if (gal[s] == 1) continue;
        if (!c->rot_keys.count(gal[s]))
            return set_err(c, HE_ENOKEY, "rotate_hoisted: no key for step %d (galois %llu)", steps[s],
                           (unsigned long long)gal[s]);
        eff.push_back(s);
    }
    const size_t N = c->N, ct_words = (size_t)2 * level * N;
    for (int s = 0; s < n_steps; s++)
        if (gal[s] == 1)
            for (int i = 0; i < n_in; i++) {
                int rc = check_cuda(c, cudaMemcpyAsync(out[(size_t)i * n_steps + s].data, in[i].data, ct_words * 8,
                                                       cudaMemcpyDeviceToDevice, c->stream), "rotate_hoisted copy");
                if (rc) return rc;
            }
    // chunks of ms steps x mi inputs, at most kMaxBatch outputs each
    const int ne = (int)eff.size();
    const int ms = std::min(ne, kMaxBatch), mi = ne ? std::max(1, kMaxBatch / ms) : 1;
    for (int e0 = 0; e0 < ne; e0 += ms)
        for (int i0 = 0; i0 < n_in; i0 += mi) {
            const int se = std::min(ne, e0 + ms), ie = std::min(n_in, i0 + mi);
            KsIoList io;
            io.sig_add0 = true;
            for (int i = i0; i < ie; i++) io.hoist_d.push_back(in[i].data + (size_t)level * N);
            for (int e = e0; e < se; e++) {
                const int s = eff[e];
                const uint64_t* key = c->rot_keys[gal[s]].d;
                for (int i = i0; i < ie; i++) {
                    io.galois.push_back(gal[s]);
                    io.key.push_back(key);
                    io.d.push_back(in[i].data + (size_t)level * N);
                    io.out.push_back(out[(size_t)i * n_steps + s].data);
                    io.add0.push_back(in[i].data);
                    io.add1.push_back(nullptr);
                    io.hoist_src.push_back(i - i0);
                }
            }
            int rc = key_switch_chunk(c, (int)io.d.size(), level, io);
            if (rc) return rc;
        }
    for (int i = 0; i < n_in; i++)
        for (int s = 0; s < n_steps; s++) {
            he_ct& o = out[(size_t)i * n_steps + s];
            o.level = level;
            o.scale = in[i].scale;
            o.is_ntt = 1;
        }
    return HE_OK;
}

// First part of a sum of rotations: s_o = base_o + sum_g (sigma_g(z0_{o,g}), 0)
// over the key-switched terms (gal != 0) + z_{o,g} over the identity terms
// (gal == 0, both polynomials); the key switches' ModDown adds the rest.
// Term r = o G + g.  Positions c, c + 1 per thread: sigma maps the aligned
// pair onto an aligned pair, so every term is one 16-byte load.
// Grid (ceil(N/512), 2 level, outputs).
__global__ void k_rot_presum(PtrList z, GalList gal, PtrList base, MutPtrList s, int G, int level,
                             const DevPrime* __restrict__ pr, int logn) {
    const int N = 1 << logn;
    const int c = 2 * (blockIdx.x * blockDim.x + threadIdx.x), row = blockIdx.y, o = blockIdx.z;
    if (c >= N) return;
    const int poly = row / level, t = row - poly * level;
    const uint64_t q = pr[t].q;
    const size_t k = (size_t)row * N;  // this limb within a ciphertext
    ulonglong2 acc = base.p[o] ? *reinterpret_cast<const ulonglong2*>(base.p[o] + k + c) : make_ulonglong2(0, 0);
    for (int g = 0; g < G; g++) {
        const int r = o * G + g;
        const uint64_t gl = gal.g[r];
        if (gl == 0) {
            // may be the output itself (sums of identity terms only): a coherent load
            const ulonglong2 v = *reinterpret_cast<const ulonglong2*>(z.p[r] + k + c);
            acc = make_ulonglong2(add_mod(acc.x, v.x, q), add_mod(acc.y, v.y, q));
        } else if (poly == 0) {
            const int src = automorph_src(c, logn, gl);
            const ulonglong2 v = __ldg(reinterpret_cast<const ulonglong2*>(z.p[r] + k + (src & ~1)));
            const bool sw = src & 1;
            acc = make_ulonglong2(add_mod(acc.x, sw ? v.y : v.x, q), add_mod(acc.y, sw ? v.x : v.y, q));
        }
    }
    *reinterpret_cast<ulonglong2*>(s.p[o] + k + c) = acc;
}

// Sums of rotations with one ModDown per output (the ModDown hoisting of
// Bossuat, Mouchet, Troncoso-Pastoriza, Hubaux, EUROCRYPT 2021, section 4):
//   out[o] = base[o] + sum_g rot_{steps[g]}(z[o n_terms + g])
//          = (base0 + sum_g sigma_g(z0_g) + ModDown(sum_g u0_g),  base1 + ModDown(sum_g u1_g)),
//   u_g = sum_j ModUp_j(sigma_g(z1_g)) (.) evk_{g,j}.
// base may be null.  Terms whose Galois element is 1 are added as they are.
// Outputs go in chunks of floor(64 / n_terms): one pre-sum launch, then one
// key-switching pass of the chunk's terms in summed mode.
int rotate_sum_many(he_ctx* c, const he_ct* z, int n_out, int n_terms, const int32_t* steps, const he_ct* base,
                    he_ct* out) {
    if (n_out < 0 || n_terms < 0) return set_err(c, HE_EINVAL, "rotate_sum: negative count");
    if (n_out == 0) return HE_OK;
    if (n_terms > kMaxBatch) return set_err(c, HE_EINVAL, "rotate_sum: at most %d terms", kMaxBatch);
    if (!out || (n_terms && (!z || !steps)) || (!n_terms && !base))
        return set_err(c, HE_EINVAL, "rotate_sum: null argument");
    const int level = n_terms ? z[0].level : base[0].level;
    const double scale = n_terms ? z[0].scale : base[0].scale;
    std::set<const uint64_t*> ins;
    for (long long i = 0; i < (long long)n_out * n_terms; i++) {
        int rc = ct_ok(c, &z[i], "rotate_sum");
        if (rc) return rc;
        if (z[i].level != level || z[i].scale != scale) return set_err(c, HE_ELEVEL, "rotate_sum: mixed levels or scales");
        ins.insert(z[i].data);
    }
    for (int o = 0; base && o < n_out; o++) {
        int rc = ct_ok(c, &base[o], "rotate_sum");
        if (rc) return rc;
        if (base[o].level != level || base[o].scale != scale)
            return set_err(c, HE_ELEVEL, "rotate_sum: base level or scale differs");
        ins.insert(base[o].data);
    }
    for (int o = 0; o < n_out; o++) {
        if (!out[o].data || ((uintptr_t)out[o].data & 31))
            return set_err(c, HE_EINVAL, "rotate_sum: null or unaligned output %d", o);
        if (ins.count(out[o].data)) return set_err(c, HE_EINVAL, "rotate_sum: output %d aliases an input", o);
    }
    std::vector<uint64_t> gal(n_terms);
    int g_eff = 0;
    for (int g = 0; g < n_terms; g++) {
        gal[g] = galois_elt(c, steps[g]);
        if (gal[g] == 1) continue;
        if (!c->rot_keys.count(gal[g]))
            return set_err(c, HE_ENOKEY, "rotate_sum: no key for step %d (galois %llu)", steps[g],
                           (unsigned long long)gal[g]);
        g_eff++;
    }
    const size_t N = c->N, ctw = (size_t)2 * level * N;
    const int G = n_terms, mc = std::max(1, kMaxBatch / std::max(1, G));
    uint64_t* S = nullptr;
    if (g_eff) {
        int rc = scratch_slot(c, 2, ctw * std::min(mc, n_out), &S);
        if (rc) return rc;
    }
    for (int o0 = 0; o0 < n_out; o0 += mc) {
        const int m = std::min(mc, n_out - o0);
        PtrList zp, bp;
        GalList gl;
        MutPtrList sp;
        for (int i = 0; i < kMaxBatch; i++) {
            zp.p[i] = nullptr;
            gl.g[i] = 0;
            bp.p[i] = nullptr;
            sp.p[i] = nullptr;
        }
        for (int o = 0; o < m; o++) {
            for (int g = 0; g < G; g++) {
                zp.p[o * G + g] = z[(size_t)(o0 + o) * G + g].data;
                gl.g[o * G + g] = gal[g] == 1 ? 0 : gal[g];
            }
            bp.p[o] = base ? base[o0 + o].data : nullptr;
            sp.p[o] = g_eff ? S + (size_t)o * ctw : out[o0 + o].data;
        }
        prof_begin(c, HE_PROF_ELEMENTWISE);
        k_rot_presum<<<dim3((unsigned)((N / 2 + 255) / 256), 2 * level, m), 256, 0, c->stream>>>(
            zp, gl, bp, sp, G, level, c->d_prime, c->log_n);
        int rc = lc(c, "rot_presum");
        if (rc) return rc;
        prof_end(c, HE_PROF_ELEMENTWISE,
                 8.0 * m * ((double)(base ? 2 : 1) * ctw + (double)(G - g_eff) * ctw + (double)g_eff * ctw / 2));
        if (!g_eff) continue;
        KsIoList io;
        io.sig_add0 = false;
        io.sum_terms = g_eff;
        for (int o = 0; o < m; o++) {
            for (int g = 0; g < G; g++) {
                if (gal[g] == 1) continue;
                io.galois.push_back(gal[g]);
                io.key.push_back(c->rot_keys[gal[g]].d);
                io.d.push_back(z[(size_t)(o0 + o) * G + g].data + (size_t)level * N);
            }
            io.out.push_back(out[o0 + o].data);
            io.add0.push_back(S + (size_t)o * ctw);
            io.add1.push_back(S + (size_t)o * ctw + (size_t)level * N);
        }
        if ((rc = key_switch_chunk(c, m * g_eff, level, io))) return rc;
    }
    for (int o = 0; o < n_out; o++) {
        out[o].level = level;
        out[o].scale = scale;
        out[o].is_ntt = 1;
    }
    return HE_OK;
}

// Rotate-and-sum of single ciphertexts with one ModUp and one ModDown each
// (the hoisting of Halevi-Shoup combined with the ModDown hoisting of
// Bossuat et al.):
//   out[i] = sum_s rot_{steps[s]}(in[i])
//          = (sum_s sigma_s(c0) + ModDown(sum_s sum_j sigma_s(ModUp_j(c1)) (.) evk_{s,j}.b),
//                                 ModDown(sum_s sum_j sigma_s(ModUp_j(c1)) (.) evk_{s,j}.a)).
// Steps whose Galois element is 1 add in[i] unchanged.  Inputs go in chunks
// of floor(64 / n_steps): one pre-sum launch, then one key-switching pass in
// hoisted and summed mode.
int rotate_sum_hoisted_many(he_ctx* c, const he_ct* in, int n_in, const int32_t* steps, int n_steps, he_ct* out) {
    if (n_in < 0 || n_steps < 0) return set_err(c, HE_EINVAL, "rotate_sum_hoisted: negative count");
    if (n_in == 0) return HE_OK;
    if (n_steps < 1 || n_steps > kMaxBatch)
        return set_err(c, HE_EINVAL, "rotate_sum_hoisted: 1 to %d steps", kMaxBatch);
    if (!in || !out || !steps) return set_err(c, HE_EINVAL, "rotate_sum_hoisted: null argument");
    const int level = in[0].level;
    std::set<const uint64_t*> ins;
    for (int i = 0; i < n_in; i++) {
        int rc = ct_ok(c, &in[i], "rotate_sum_hoisted");
        if (rc) return rc;
        if (in[i].level != level) return set_err(c, HE_ELEVEL, "rotate_sum_hoisted: mixed levels");
        ins.insert(in[i].data);
    }
    for (int i = 0; i < n_in; i++) {
        if (!out[i].data || ((uintptr_t)out[i].data & 31))
            return set_err(c, HE_EINVAL, "rotate_sum_hoisted: null or unaligned output %d", i);
        if (ins.count(out[i].data)) return set_err(c, HE_EINVAL, "rotate_sum_hoisted: output %d aliases an input", i);
    }
    std::vector<uint64_t> gal(n_steps);
    int g_eff = 0;
    for (int s = 0; s < n_steps; s++) {
        gal[s] = galois_elt(c, steps[s]);
        if (gal[s] == 1) continue;
        if (!c->rot_keys.count(gal[s]))
            return set_err(c, HE_ENOKEY, "rotate_sum_hoisted: no key for step %d (galois %llu)", steps[s],
                           (unsigned long long)gal[s]);
        g_eff++;
    }
    const size_t N = c->N, ctw = (size_t)2 * level * N;
    const int G = n_steps, mc = std::max(1, kMaxBatch / G);
    uint64_t* S = nullptr;
    if (g_eff) {
        int rc = scratch_slot(c, 2, ctw * std::min(mc, n_in), &S);
        if (rc) return rc;
    }
    for (int i0 = 0; i0 < n_in; i0 += mc) {
        const int m = std::min(mc, n_in - i0);
        PtrList zp, bp;
        GalList gl;
        MutPtrList sp;
        for (int k = 0; k < kMaxBatch; k++) {
            zp.p[k] = nullptr;
            gl.g[k] = 0;
            bp.p[k] = nullptr;
            sp.p[k] = nullptr;
        }
        for (int o = 0; o < m; o++) {
            for (int g = 0; g < G; g++) {
                zp.p[o * G + g] = in[i0 + o].data;
                gl.g[o * G + g] = gal[g] == 1 ? 0 : gal[g];
            }
            sp.p[o] = g_eff ? S + (size_t)o * ctw : out[i0 + o].data;
        }
        prof_begin(c, HE_PROF_ELEMENTWISE);
        k_rot_presum<<<dim3((unsigned)((N / 2 + 255) / 256), 2 * level, m), 256, 0, c->stream>>>(
            zp, gl, bp, sp, G, level, c->d_prime, c->log_n);
        int rc = lc(c, "rot_presum");
        if (rc) return rc;
        prof_end(c, HE_PROF_ELEMENTWISE, 8.0 * m * ((double)(G - g_eff) * ctw + (double)g_eff * ctw / 2 + ctw));
        if (!g_eff) continue;
        KsIoList io;
        io.sig_add0 = false;
        io.sum_terms = g_eff;
        for (int o = 0; o < m; o++) {
            io.hoist_d.push_back(in[i0 + o].data + (size_t)level * N);
            for (int g = 0; g < G; g++) {
                if (gal[g] == 1) continue;
                io.galois.push_back(gal[g]);
                io.key.push_back(c->rot_keys[gal[g]].d);
                io.d.push_back(in[i0 + o].data + (size_t)level * N);
                io.hoist_src.push_back(o);
            }
            io.out.push_back(out[i0 + o].data);
            io.add0.push_back(S + (size_t)o * ctw);
            io.add1.push_back(S + (size_t)o * ctw + (size_t)level * N);
        }
        if ((rc = key_switch_chunk(c, m * g_eff, level, io))) return rc;
    }
    for (int i = 0; i < n_in; i++) {
        out[i].level = level;
        out[i].scale = in[i].scale;
        out[i].is_ntt = 1;
    }
    return HE_OK;
}

}  // namespace he

using namespace he;

extern "C" int he_rotate_sum_hoisted(he_ctx* c, const he_ct* in, int n_in, const int32_t* steps, int n_steps,
                                     he_ct* out) {
    if (!c) return HE_EINVAL;
    return rotate_sum_hoisted_many(c, in, n_in, steps, n_steps, out);
}

extern "C" int he_rotate_sum(he_ctx* c, const he_ct* z, int n_out, int n_terms, const int32_t* steps,
                             const he_ct* base, he_ct* out) {
    if (!c) return HE_EINVAL;
    return rotate_sum_many(c, z, n_out, n_terms, steps, base, out);
}

extern "C" int he_rotate_hoisted(he_ctx* c, const he_ct* in, int n_in, const int32_t* steps, int n_steps,
                                 he_ct* out) {
    if (!c) return HE_EINVAL;
    return rotate_hoisted_many(c, in, n_in, steps, n_steps, out);
}

extern "C" int he_rotate(he_ctx* c, const he_ct* in, int32_t step, he_ct* out) {
    if (!c) return HE_EINVAL;
    return rotate_many(c, in, &step, out, 1);
}

extern "C" int he_rotate_batch(he_ctx* c, const he_ct* in, const int32_t* steps, he_ct* out, int n) {
    if (!c) return HE_EINVAL;
    return rotate_many(c, in, steps, out, n);
}

// Host-buffer rotation, pipelined: the ciphertexts, ordered by Galois element
// (so that a chunk holds few distinct keys), go through the GPU in chunks of
// at most kIoChunk.  Two staging buffers per direction let chunk k+1's upload
// and chunk k-1's download (one copy engine each) overlap chunk k's rotation.
constexpr int kIoChunk = 8;

// Chunk sizes of a pipeline of n ciphertexts: 2 and 4 first and last (when n
// leaves at least one full chunk between them), so that the upload before the
// first rotation and the download after the last, when one copy engine works
// alone, are short; the rest in near-equal chunks of at most kIoChunk.
static std::vector<int> io_plan(int n) {
    std::vector<int> head;
    int rem = n;
    for (int r : {2, 4})
        if (rem >= 2 * r + kIoChunk) {
            head.push_back(r);
            rem -= 2 * r;
        }
    std::vector<int> plan = head;
    const int nm = (rem + kIoChunk - 1) / kIoChunk;
    for (int k = 0; k < nm; k++) plan.push_back(rem / nm + (k < rem % nm ? 1 : 0));
    plan.insert(plan.end(), head.rbegin(), head.rend());
    return plan;
}

static int io_setup(he_ctx* c, size_t words) {
    int rc;
    if (words > c->io_words) {
        cudaStreamSynchronize(c->stream);
        cudaFree(c->io_buf);
        c->io_buf = nullptr;
        c->io_words = 0;
        if ((rc = check_cuda(c, cudaMalloc(&c->io_buf, words * 8), "io buffer"))) return rc;
        c->io_words = words;
    }
    if (!c->io_h2d && (rc = check_cuda(c, cudaStreamCreateWithFlags(&c->io_h2d, cudaStreamNonBlocking), "io stream")))
        return rc;
    if (!c->io_d2h && (rc = check_cuda(c, cudaStreamCreateWithFlags(&c->io_d2h, cudaStreamNonBlocking), "io stream")))
        return rc;
    for (cudaEvent_t& e : c->io_ev)
        if (!e && (rc = check_cuda(c, cudaEventCreateWithFlags(&e, cudaEventDisableTiming), "io event"))) return rc;
    return HE_OK;
}

static int io_drain(he_ctx* c, int rc) {
    cudaStreamSynchronize(c->io_h2d);
    cudaStreamSynchronize(c->stream);
    cudaStreamSynchronize(c->io_d2h);
    return rc;
}

// The host-buffer pipeline; wire: the host buffers hold ciphertexts in the
// packed wire format (wire.cu), unpacked and packed on the device, so only
// the packed bytes cross the host link.
static int rotate_batch_host(he_ctx* c, const uint8_t* h_in, int level, const int32_t* steps, uint8_t* h_out, int n,
                             bool wire, const char* what) {
    if (!c) return HE_EINVAL;
    if (!h_in || !h_out || !steps || n < 0 || level < 1 || level > c->L)
        return set_err(c, HE_EINVAL, "%s: bad arguments", what);
    if (n == 0) return HE_OK;
    std::vector<uint64_t> gal(n);
    for (int i = 0; i < n; i++) {
        gal[i] = galois_elt(c, steps[i]);
        if (gal[i] != 1 && !c->rot_keys.count(gal[i]))
            return set_err(c, HE_ENOKEY, "%s: no key for step %d", what, steps[i]);
    }
    std::vector<int> order(n);
    for (int i = 0; i < n; i++) order[i] = i;
    std::stable_sort(order.begin(), order.end(), [&](int x, int y) { return gal[x] < gal[y]; });

    const size_t ct_words = (size_t)2 * level * c->N;
    const size_t link_bytes = wire ? wire_bytes(c, level) : ct_words * 8;  // per ciphertext across the link
    const size_t link_words = (link_bytes + 7) / 8;
    const int chunk = std::min(kIoChunk, n);
    int rc = io_setup(c, 4 * (size_t)chunk * ct_words + (wire ? 4 * (size_t)chunk * link_words : 0));
    if (rc) return rc;
    cudaEvent_t* up = c->io_ev;        // [2] upload of buffer b done
    cudaEvent_t* done = c->io_ev + 2;  // [2] rotation of buffer b done
    cudaEvent_t* down = c->io_ev + 4;  // [2] download of buffer b done
    const std::vector<int> plan = io_plan(n);
    for (int k = 0, i0 = 0; k < (int)plan.size(); i0 += plan[k], k++) {
        const int b = k & 1, m = plan[k];
        uint64_t* din = c->io_buf + (size_t)b * chunk * ct_words;
        uint64_t* dout = c->io_buf + (size_t)(2 + b) * chunk * ct_words;
        uint64_t* wbase = c->io_buf + 4 * (size_t)chunk * ct_words;
        uint8_t* lin = reinterpret_cast<uint8_t*>(wire ? wbase + (size_t)b * chunk * link_words : din);
        uint8_t* lout = reinterpret_cast<uint8_t*>(wire ? wbase + (size_t)(2 + b) * chunk * link_words : dout);
        const size_t lstride = wire ? link_words * 8 : ct_words * 8;  // bytes between staged ciphertexts
        // upload, once chunk k-2 no longer reads this buffer
        if (k >= 2) cudaStreamWaitEvent(c->io_h2d, done[b], 0);
        for (int j = 0; j < m; j++) {
            rc = check_cuda(c, cudaMemcpyAsync(lin + j * lstride, h_in + (size_t)order[i0 + j] * link_bytes,
                                               link_bytes, cudaMemcpyHostToDevice, c->io_h2d), "H2D");
            if (rc) return io_drain(c, rc);
        }
        cudaEventRecord(up[b], c->io_h2d);
        // rotate, once uploaded and once chunk k-2's download left the output buffer
        cudaStreamWaitEvent(c->stream, up[b], 0);
        if (k >= 2) cudaStreamWaitEvent(c->stream, down[b], 0);
        std::vector<he_ct> in(m), out(m);
        std::vector<int32_t> st(m);
        std::vector<uint64_t*> dins(m);
        std::vector<const uint64_t*> douts(m);
        for (int j = 0; j < m; j++) {
            in[j] = he_ct{din + j * ct_words, level, 1.0, 1};
            out[j] = he_ct{dout + j * ct_words, level, 1.0, 1};
            st[j] = steps[order[i0 + j]];
            dins[j] = in[j].data;
            douts[j] = out[j].data;
        }
        if (wire && lstride != link_bytes) return io_drain(c, set_err(c, HE_EINVAL, "%s: wire size", what));
        if (wire && (rc = wire_unpack_many(c, lin, level, dins))) return io_drain(c, rc);
        rc = rotate_many(c, in.data(), st.data(), out.data(), m);
        if (rc) return io_drain(c, rc);
        if (wire && (rc = wire_pack_many(c, douts, level, lout))) return io_drain(c, rc);
        cudaEventRecord(done[b], c->stream);
        // download
        cudaStreamWaitEvent(c->io_d2h, done[b], 0);
        for (int j = 0; j < m; j++) {
            rc = check_cuda(c, cudaMemcpyAsync(h_out + (size_t)order[i0 + j] * link_bytes, lout + j * lstride,
                                               link_bytes, cudaMemcpyDeviceToHost, c->io_d2h), "D2H");
            if (rc) return io_drain(c, rc);
        }
        cudaEventRecord(down[b], c->io_d2h);
    }
    rc = check_cuda(c, cudaStreamSynchronize(c->io_d2h), "D2H sync");
    if (rc) return io_drain(c, rc);
    return he_sync(c);
}

extern "C" int he_rotate_batch_host(he_ctx* c, const uint64_t* h_in, int level, const int32_t* steps,
                                    uint64_t* h_out, int n) {
    return rotate_batch_host(c, reinterpret_cast<const uint8_t*>(h_in), level, steps,
                             reinterpret_cast<uint8_t*>(h_out), n, false, "he_rotate_batch_host");
}

extern "C" int he_rotate_batch_host_wire(he_ctx* c, const uint8_t* h_in, int level, const int32_t* steps,
                                         uint8_t* h_out, int n) {
    return rotate_batch_host(c, h_in, level, steps, h_out, n, true, "he_rotate_batch_host_wire");
}
