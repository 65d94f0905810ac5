// Negacyclic NTT building blocks: 16 elements per thread in registers.
//
// Transform (textbook negacyclic NTT, bit-reversed output): storage index j
// of the output holds a(psi^(2 brev(j) + 1)).  Computed by the Cooley-Tukey
// decimation-in-time network with twiddles psi^brev(m+i) (Longa-Naehrig,
// "Speeding up the Number Theoretic Transform for Faster Ideal Lattice-Based
// Cryptography", CANS 2016, algorithms 1 and 2) with Harvey's lazy
// butterflies; the inverse is the Gentleman-Sande network with psi^-brev(m+i)
// and N^-1 folded into its last stage.
//
// N = R C, R = 2^S1 rows, C = 2^S2 columns, element j = r C + c.  Forward
// stages 0..S1-1 pair rows ("column pass"), stages S1..LOGN-1 pair elements
// of one row ("row pass"); the inverse runs the row stages first.  Each pass
// is two register sub-passes of up to four stages separated by one exchange
// through shared memory:
//   column pass, sub-pass A: thread (g, col) holds rows g + (R/16) k, k < 16;
//                sub-pass B: rows 16 g + k;
//   row pass,    sub-pass A: thread (row, p) holds columns p + (C/16) k;
//                sub-pass B: columns 16 p + k.
// In every sub-pass the stage with pair distance D (in those index units)
// pairs registers k and k + D, and the twiddle index is 2^s plus the pair's
// block number, which the formulas below derive from k and the thread's
// (g, row, p) without division.
#pragma once
#include "modarith.cuh"

namespace he {

template <int LOGN>
struct NttCfg {
    static constexpr int S1 = (LOGN + 1) / 2;
    static constexpr int S2 = LOGN - S1;
    static constexpr int R = 1 << S1;
    static constexpr int C = 1 << S2;
    static constexpr int N = 1 << LOGN;
    // column pass: TC columns x R rows per block, 16 elements per thread
    static constexpr int TC = C < 16 ? C : 16;
    static constexpr int COL_THREADS = R * TC / 16;
    static constexpr int COL_TILES = C / TC;
    // row pass: TR rows x C columns per block
    static constexpr int TR = (4096 / C) < R ? (4096 / C) : R;
    static constexpr int ROW_THREADS = TR * C / 16;
    static constexpr int ROW_TILES = R / TR;
    static constexpr int ROW_PITCH = C + C / 16;  // one pad word per 16 (bank spread)
    static constexpr size_t COL_SMEM = (size_t)R * TC * 8;
    static constexpr size_t ROW_SMEM = (size_t)TR * ROW_PITCH * 8;
    static_assert(S1 >= 4 && S1 <= 8 && S2 >= 4 && S2 <= 8, "two sub-passes of at most 4 stages");
};

// Harvey CT butterfly: x, y in [0, 4q) -> [0, 4q).
__device__ __forceinline__ void bfly_ct(uint64_t& x, uint64_t& y, const ulonglong2 w, uint64_t q, uint64_t two_q) {
    uint64_t a = csub(x, two_q);
    uint64_t t = mul_shoup_lazy(y, w.x, w.y, q);
    x = a + t;
    y = a + two_q - t;
}

// Harvey GS butterfly: x, y in [0, 2q) -> [0, 2q).
__device__ __forceinline__ void bfly_gs(uint64_t& x, uint64_t& y, const ulonglong2 w, uint64_t q, uint64_t two_q) {
    uint64_t a = x, b = y;
    x = csub(a + b, two_q);
    y = mul_shoup_lazy(a + two_q - b, w.x, w.y, q);
}

__device__ __forceinline__ ulonglong2 ldtw(const ulonglong2* p) { return __ldg(p); }

// 256-bit global accesses (sm_100 vector width); the address must be 32-byte
// aligned.  ldg256_ro goes through the read-only path: only for data that no
// thread writes during the kernel (tables, inputs of out-of-place kernels).
__device__ __forceinline__ void ldg256_ro(const double* p, double& a, double& b, double& c, double& d) {
    asm("ld.global.nc.v4.f64 {%0, %1, %2, %3}, [%4];" : "=d"(a), "=d"(b), "=d"(c), "=d"(d) : "l"(p));
}
__device__ __forceinline__ void ldg256_ro(const uint64_t* p, uint64_t& a, uint64_t& b, uint64_t& c, uint64_t& d) {
    asm("ld.global.nc.v4.u64 {%0, %1, %2, %3}, [%4];" : "=l"(a), "=l"(b), "=l"(c), "=l"(d) : "l"(p));
}
__device__ __forceinline__ void ldg256(const uint64_t* p, uint64_t& a, uint64_t& b, uint64_t& c, uint64_t& d) {
    asm volatile("ld.global.v4.u64 {%0, %1, %2, %3}, [%4];" : "=l"(a), "=l"(b), "=l"(c), "=l"(d) : "l"(p) : "memory");
}
__device__ __forceinline__ void stg256(uint64_t* p, uint64_t a, uint64_t b, uint64_t c, uint64_t d) {
    asm volatile("st.global.v4.u64 [%0], {%1, %2, %3, %4};" ::"l"(p), "l"(a), "l"(b), "l"(c), "l"(d) : "memory");
}

// Forward stages on 16 registers.  H stages (H <= 4) with register pair
// distance 2^(H-1-u) at stage u; the twiddle of the pair starting at k is
// tw[base(u) + (key(k) >> (H - u))] where key(k) = kofs + k, with
//   base(u) = (2^(s0+u)) + row_term << u.
// s0: global index of the first stage; kofs/row_term select the block.
// kofs is a multiple of 16, so the 16 >> (H - u) twiddles one thread uses at
// stage u are contiguous and start at a multiple of their count: pairs of
// them load as one 256-bit access.
template <int H, int U>
__device__ __forceinline__ void load_stage_tw_int(ulonglong2 (&w)[8], const ulonglong2* __restrict__ p) {
    constexpr int LC = 4 - H + U;
    if constexpr (LC == 0) {
        w[0] = ldtw(p);
    } else {
#pragma unroll
        for (int v = 0; v < (1 << LC) / 2; v++) {
            uint64_t a, b, c, d;
            ldg256_ro(reinterpret_cast<const uint64_t*>(p + 2 * v), a, b, c, d);
            w[2 * v] = make_ulonglong2(a, b);
            w[2 * v + 1] = make_ulonglong2(c, d);
        }
    }
}

template <int H, int U>
__device__ __forceinline__ void fwd_stage_int(uint64_t (&x)[16], const ulonglong2* __restrict__ tw, int s0,
                                              int row_term, int kofs, uint64_t q) {
    constexpr int D = 1 << (H - 1 - U);
    ulonglong2 w[8];
    load_stage_tw_int<H, U>(w, tw + (1 << (s0 + U)) + (row_term << U) + (kofs >> (H - U)));
#pragma unroll
    for (int k = 0; k < 16; k++) {
        if (k & D) continue;
        bfly_ct(x[k], x[k + D], w[k >> (H - U)], q, 2 * q);
    }
}

template <int H, int U>
__device__ __forceinline__ void inv_stage_int(uint64_t (&x)[16], const ulonglong2* __restrict__ tw, int s0,
                                              int row_term, int kofs, uint64_t q) {
    constexpr int D = 1 << (H - 1 - U);
    ulonglong2 w[8];
    load_stage_tw_int<H, U>(w, tw + (1 << (s0 + U)) + (row_term << U) + (kofs >> (H - U)));
#pragma unroll
    for (int k = 0; k < 16; k++) {
        if (k & D) continue;
        bfly_gs(x[k], x[k + D], w[k >> (H - U)], q, 2 * q);
    }
}

template <int H>
__device__ __forceinline__ void fwd_stages(uint64_t (&x)[16], const ulonglong2* __restrict__ tw, int s0, int row_term,
                                           int kofs, uint64_t q) {
    if constexpr (H > 0) fwd_stage_int<H, 0>(x, tw, s0, row_term, kofs, q);
    if constexpr (H > 1) fwd_stage_int<H, 1>(x, tw, s0, row_term, kofs, q);
    if constexpr (H > 2) fwd_stage_int<H, 2>(x, tw, s0, row_term, kofs, q);
    if constexpr (H > 3) fwd_stage_int<H, 3>(x, tw, s0, row_term, kofs, q);
}

// Inverse stages on 16 registers: the forward stages of fwd_stages<H> in
// reverse order with GS butterflies (same twiddle index formula, inverse
// table).  Stages u = H-1 down to ULO.
template <int H, int ULO = 0>
__device__ __forceinline__ void inv_stages(uint64_t (&x)[16], const ulonglong2* __restrict__ tw, int s0, int row_term,
                                           int kofs, uint64_t q) {
    if constexpr (H > 3 && ULO <= 3) inv_stage_int<H, 3>(x, tw, s0, row_term, kofs, q);
    if constexpr (H > 2 && ULO <= 2) inv_stage_int<H, 2>(x, tw, s0, row_term, kofs, q);
    if constexpr (H > 1 && ULO <= 1) inv_stage_int<H, 1>(x, tw, s0, row_term, kofs, q);
    if constexpr (H > 0 && ULO <= 0) inv_stage_int<H, 0>(x, tw, s0, row_term, kofs, q);
}

// ---------------------------------------------------------------------------
// FP64 arithmetic for primes below 2^41 (the 40-bit primes of the modulus
// chain).  Residues are integers held in doubles (exact below 2^53), signed
// and unreduced inside a transform; the modular product runs on the FP64
// pipe with a rounded quotient:
//   p_hi = fl(y w), p_lo = fma(y, w, -p_hi)          (y w = p_hi + p_lo exactly)
//   qh = nearest integer to p_hi (1/q)  (1.5 2^52 magic constant)
//   r = fma(-qh, q, p_hi) + p_lo                     (both steps exact)
// r = y w - qh q exactly, and for |y| <= Y, 0 <= w < q:
//   |r| <= q (1/2 + 2^-52 Y)  <=  5q/8  for Y <= 2^49
// (quotient off by at most 1/2 + 2^-53 Y/1, p_lo at most 2^-53 Y q).
// No branch and no range correction: sums and differences of such values
// stay exact integers, and the transforms below keep |y| <= 2^49 by
// construction (bounds at each use).
struct FpMod {
    double q, two_q, qinv, ninv;
};

constexpr uint64_t kFpPrimeLimit = 1ull << 41;

constexpr double kFpMagic = 6755399441055744.0;  // 1.5 * 2^52

// r = y w (mod q) with |r| < 5q/8, for |y| <= 2^49 and 0 <= w < q
__device__ __forceinline__ double fp_mulmod_s(double y, double w, const FpMod& m) {
    double ph = __dmul_rn(y, w);
    double pl = __fma_rn(y, w, -ph);
    double qh = __dsub_rn(__fma_rn(ph, m.qinv, kFpMagic), kFpMagic);
    return __dadd_rn(__fma_rn(-qh, m.q, ph), pl);
}

// r = x (mod q) with |r| <= q/2 (1 + 2^-51 |x|/q), for |x| <= 2^51
__device__ __forceinline__ double fp_reduce_s(double x, const FpMod& m) {
    double qh = __dsub_rn(__fma_rn(x, m.qinv, kFpMagic), kFpMagic);
    return __fma_rn(-qh, m.q, x);
}

// canonical [0, q) from |r| < q
__device__ __forceinline__ double fp_from_signed(double r, const FpMod& m) { return r < 0.0 ? __dadd_rn(r, m.q) : r; }

// canonical [0, q) from |x| <= 2^51
__device__ __forceinline__ double fp_canon(double x, const FpMod& m) { return fp_from_signed(fp_reduce_s(x, m), m); }

// canonical product y w mod q, |y| <= 2^49
__device__ __forceinline__ double fp_modmul(double y, double w, const FpMod& m) {
    return fp_from_signed(fp_mulmod_s(y, w, m), m);
}

__device__ __forceinline__ double fp_csub(double x, double c) { return x >= c ? __dsub_rn(x, c) : x; }

// exact conversions for integers in [0, 2^52)
__device__ __forceinline__ double u2d(uint64_t x) {
    return __dsub_rn(__longlong_as_double((long long)(x | 0x4330000000000000ull)), 4503599627370496.0);
}
__device__ __forceinline__ uint64_t d2u(double d) {
    return (uint64_t)__double_as_longlong(__dadd_rn(d, 4503599627370496.0)) & 0x000FFFFFFFFFFFFFull;
}

// CT butterfly on signed values: |x'|, |y'| <= max(|x|) + 5q/8
__device__ __forceinline__ void bfly_ct(double& x, double& y, double w, const FpMod& m) {
    double t = fp_mulmod_s(y, w, m);
    double a = x;
    x = __dadd_rn(a, t);
    y = __dsub_rn(a, t);
}

// GS butterfly on signed values: |x'| <= |x| + |y|, |y'| < 5q/8
__device__ __forceinline__ void bfly_gs(double& x, double& y, double w, const FpMod& m) {
    double a = x, b = y;
    x = __dadd_rn(a, b);
    y = fp_mulmod_s(__dsub_rn(a, b), w, m);
}

// The twiddles of stage u used by one thread are contiguous:
// tw[base(u) + (kofs >> (H - u)) + i], i < 16 >> (H - u) (kofs is a multiple
// of 16), and the start is a multiple of their count, so they load as
// 16-byte pairs.  LC = log2 of the count.
template <int LC>
__device__ __forceinline__ void load_stage_tw(double (&w)[8], const double* __restrict__ p) {
    if constexpr (LC == 0) {
        w[0] = __ldg(p);
    } else if constexpr (LC == 1) {
        double2 d = __ldg(reinterpret_cast<const double2*>(p));
        w[0] = d.x;
        w[1] = d.y;
    } else {
#pragma unroll
        for (int v = 0; v < (1 << LC) / 4; v++) ldg256_ro(p + 4 * v, w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
    }
}

template <int H, int U>
__device__ __forceinline__ void fwd_stage_fp(double (&x)[16], const double* __restrict__ tw, int s0, int row_term,
                                             int kofs, const FpMod& m) {
    constexpr int D = 1 << (H - 1 - U);
    double w[8];
    load_stage_tw<4 - H + U>(w, tw + (1 << (s0 + U)) + (row_term << U) + (kofs >> (H - U)));
#pragma unroll
    for (int k = 0; k < 16; k++) {
        if (k & D) continue;
        bfly_ct(x[k], x[k + D], w[k >> (H - U)], m);
    }
}

template <int H, int U>
__device__ __forceinline__ void inv_stage_fp(double (&x)[16], const double* __restrict__ tw, int s0, int row_term,
                                             int kofs, const FpMod& m) {
    constexpr int D = 1 << (H - 1 - U);
    double w[8];
    load_stage_tw<4 - H + U>(w, tw + (1 << (s0 + U)) + (row_term << U) + (kofs >> (H - U)));
#pragma unroll
    for (int k = 0; k < 16; k++) {
        if (k & D) continue;
        bfly_gs(x[k], x[k + D], w[k >> (H - U)], m);
    }
}

template <int H>
__device__ __forceinline__ void fwd_stages(double (&x)[16], const double* __restrict__ tw, int s0, int row_term,
                                           int kofs, const FpMod& m) {
    if constexpr (H > 0) fwd_stage_fp<H, 0>(x, tw, s0, row_term, kofs, m);
    if constexpr (H > 1) fwd_stage_fp<H, 1>(x, tw, s0, row_term, kofs, m);
    if constexpr (H > 2) fwd_stage_fp<H, 2>(x, tw, s0, row_term, kofs, m);
    if constexpr (H > 3) fwd_stage_fp<H, 3>(x, tw, s0, row_term, kofs, m);
}

template <int H, int ULO = 0>
__device__ __forceinline__ void inv_stages(double (&x)[16], const double* __restrict__ tw, int s0, int row_term,
                                           int kofs, const FpMod& m) {
    if constexpr (H > 3 && ULO <= 3) inv_stage_fp<H, 3>(x, tw, s0, row_term, kofs, m);
    if constexpr (H > 2 && ULO <= 2) inv_stage_fp<H, 2>(x, tw, s0, row_term, kofs, m);
    if constexpr (H > 1 && ULO <= 1) inv_stage_fp<H, 1>(x, tw, s0, row_term, kofs, m);
    if constexpr (H > 0 && ULO <= 0) inv_stage_fp<H, 0>(x, tw, s0, row_term, kofs, m);
}

// Last inverse stage, FP64: outputs |r| < 5q/8 (callers canonicalise).
__device__ __forceinline__ void inv_stage0_scaled(double (&x)[16], double w1, const FpMod& m) {
#pragma unroll
    for (int k = 0; k < 8; k++) {
        double a = x[k], b = x[k + 8];
        x[k] = fp_mulmod_s(__dadd_rn(a, b), m.ninv, m);
        x[k + 8] = fp_mulmod_s(__dsub_rn(a, b), w1, m);
    }
}

// Element formats.  Transform inputs and outputs are canonical uint64
// residues; between the two passes of a transform a limb holds the pass's
// raw state: unreduced uint64 (integer path: [0, 4q) forward, [0, 2q)
// inverse) or the bit pattern of a signed double (FP64 path).
__device__ __forceinline__ uint64_t to_elem(uint64_t v, uint64_t) { return v; }
__device__ __forceinline__ double to_elem(uint64_t v, double) { return u2d(v); }
__device__ __forceinline__ uint64_t raw_in(uint64_t v, uint64_t) { return v; }
__device__ __forceinline__ double raw_in(uint64_t v, double) { return __longlong_as_double((long long)v); }
__device__ __forceinline__ uint64_t raw_out(uint64_t v) { return v; }
__device__ __forceinline__ uint64_t raw_out(double v) { return (uint64_t)__double_as_longlong(v); }

// Forward outputs: integer path [0, 4q), FP64 path |x| <= 2^49.
__device__ __forceinline__ uint64_t reduce4q(uint64_t x, uint64_t q) { return csub(csub(x, 2 * q), q); }
__device__ __forceinline__ uint64_t fwd_canon(uint64_t x, uint64_t q) { return reduce4q(x, q); }
__device__ __forceinline__ uint64_t fwd_canon(double x, const FpMod& m) { return d2u(fp_canon(x, m)); }
// Inverse outputs: integer path canonical already, FP64 path |x| < q.
__device__ __forceinline__ uint64_t inv_canon(uint64_t x, uint64_t) { return x; }
__device__ __forceinline__ uint64_t inv_canon(double x, const FpMod& m) { return d2u(fp_from_signed(x, m)); }
// Inverse column pass input: the FP64 row pass leaves |x| <= 2^8 q; bring it
// to |x| < q/2 + 1 so that seven more doubling stages stay below 2^49.
__device__ __forceinline__ void inv_cols_prereduce(uint64_t (&)[16], uint64_t) {}
__device__ __forceinline__ void inv_cols_prereduce(double (&x)[16], const FpMod& m) {
#pragma unroll
    for (int k = 0; k < 16; k++) x[k] = fp_reduce_s(x[k], m);
}

// Last inverse stage (global stage 0, pair distance N/2, block 0): the sum is
// multiplied by N^-1 and the difference by psi^-brev(1) N^-1 (table entry 1).
// Registers k and k + 8 hold rows g and g + R/2.  Outputs canonical.
__device__ __forceinline__ void inv_stage0_scaled(uint64_t (&x)[16], const ulonglong2 w1, const ulonglong2 ninv,
                                                  uint64_t q) {
    const uint64_t two_q = 2 * q;
#pragma unroll
    for (int k = 0; k < 8; k++) {
        uint64_t a = x[k], b = x[k + 8];
        x[k] = mul_shoup(a + b, ninv.x, ninv.y, q);
        x[k + 8] = mul_shoup(a + two_q - b, w1.x, w1.y, q);
    }
}

// ---------------------------------------------------------------------------
// Row pass pieces shared by the plain transforms and the fused key-switching
// kernels.  Thread (rr, p) of a row-pass block owns columns 16 p + k of row
// r = tile * TR + rr; after the pass the 16 registers hold those columns.

// Blocks per SM the passes are compiled for: column passes 4 (64 registers),
// row passes 3 (80 registers; at 64 their spills cost more than the added
// occupancy gains).
constexpr int NTT_COL_MIN_BLOCKS = 4;
constexpr int NTT_MIN_BLOCKS = 3;

// shared-memory index of element i of a padded row (one pad word per 16)
__device__ __forceinline__ int padded(int i) { return i + (i >> 4); }

template <int LOGN>
__device__ __forceinline__ int row_lane() { return threadIdx.x % (NttCfg<LOGN>::C / 16); }

// x[k] = a[k], k < 16 (a 128-byte aligned; a may be rewritten by this kernel)
template <typename T>
__device__ __forceinline__ void row_load16(T (&x)[16], const uint64_t* a) {
#pragma unroll
    for (int v = 0; v < 4; v++) {
        uint64_t e0, e1, e2, e3;
        ldg256(a + 4 * v, e0, e1, e2, e3);
        x[4 * v] = to_elem(e0, T());
        x[4 * v + 1] = to_elem(e1, T());
        x[4 * v + 2] = to_elem(e2, T());
        x[4 * v + 3] = to_elem(e3, T());
    }
}

// a[k] = canonical x[k] (forward transform output), a 128-byte aligned
template <typename T, typename M>
__device__ __forceinline__ void row_store16(uint64_t* a, T (&x)[16], const M& m) {
#pragma unroll
    for (int v = 0; v < 4; v++)
        stg256(a + 4 * v, fwd_canon(x[4 * v], m), fwd_canon(x[4 * v + 1], m), fwd_canon(x[4 * v + 2], m),
               fwd_canon(x[4 * v + 3], m));
}

// x[k] = row[p + CS k], k < 16: the forward row pass's input, the column
// pass's raw state
template <int LOGN, typename T>
__device__ __forceinline__ void row_load_strided(T (&x)[16], const uint64_t* row) {
    constexpr int CS = NttCfg<LOGN>::C / 16;
    const int p = threadIdx.x % CS;
#pragma unroll
    for (int k = 0; k < 16; k++) x[k] = raw_in(row[p + CS * k], T());
}

// Brings the twiddles of the last four stages of row r, which thread p uses
// after the exchange, towards L1 while the first four stages run: one
// prefetch per stage (its twiddles span at most 128 bytes, line-aligned).
template <int LOGN, typename TW>
__device__ __forceinline__ void prefetch_row_tw(const TW* tw, int r, int p) {
    constexpr int S = NttCfg<LOGN>::S1 + 4, H = NttCfg<LOGN>::S2 - 4;
#pragma unroll
    for (int u = 0; u < H; u++) {
        const TW* a = tw + (1 << (S + u)) + ((r << 4) << u) + ((16 * p) >> (H - u));
        asm volatile("prefetch.global.L1 [%0];" ::"l"(a));
    }
}

// Forward row pass (stages S1..LOGN-1) on registers loaded from columns
// p + CS k of row r; returns columns 16 p + k in [0, 4q).
template <int LOGN, typename T, typename TW, typename M>
__device__ __forceinline__ void fwd_rows_core(T (&x)[16], T* sm, int r, const TW* tw, const M& m) {
    using Cf = NttCfg<LOGN>;
    constexpr int CS = Cf::C / 16;
    const int p = threadIdx.x % CS, rr = threadIdx.x / CS;
    T* s = sm + rr * Cf::ROW_PITCH;
    prefetch_row_tw<LOGN>(tw, r, p);
    fwd_stages<4>(x, tw, Cf::S1, r, 0, m);
#pragma unroll
    for (int k = 0; k < 16; k++) s[padded(p + CS * k)] = x[k];
    __syncthreads();
#pragma unroll
    for (int k = 0; k < 16; k++) x[k] = s[padded(16 * p + k)];
    fwd_stages<Cf::S2 - 4>(x, tw, Cf::S1 + 4, r << 4, 16 * p, m);
}

// Inverse row pass (stages LOGN-1..S1) on registers loaded from columns
// 16 p + k of row r; stores columns p + CS k of the raw result to out_row.
template <int LOGN, typename T, typename TW, typename M>
__device__ __forceinline__ void inv_rows_core(T (&x)[16], T* sm, uint64_t* out_row, int r, const TW* tw,
                                              const M& m) {
    using Cf = NttCfg<LOGN>;
    constexpr int CS = Cf::C / 16;
    const int p = threadIdx.x % CS, rr = threadIdx.x / CS;
    T* s = sm + rr * Cf::ROW_PITCH;
    inv_stages<Cf::S2 - 4>(x, tw, Cf::S1 + 4, r << 4, 16 * p, m);
#pragma unroll
    for (int k = 0; k < 16; k++) s[padded(16 * p + k)] = x[k];
    __syncthreads();
#pragma unroll
    for (int k = 0; k < 16; k++) x[k] = s[padded(p + CS * k)];
    inv_stages<4>(x, tw, Cf::S1, r, 0, m);
#pragma unroll
    for (int k = 0; k < 16; k++) out_row[p + CS * k] = raw_out(x[k]);
}

}  // namespace he
