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

__device__ __forceinline__ uint64_t reduce4q(uint64_t x, uint64_t q) { return csub(csub(x, 2 * q), q); }

__device__ __forceinline__ ulonglong2 ldtw(const ulonglong2* p) { return __ldg(p); }

// Forward stages on 16 registers.  H stages (H <= 4) with register pair
// distance 2^(H-1-u) at stage u; the twiddle of the pair starting at k is
// tw[base(u) + (key(k) >> (H - u))] where key(k) = kofs + k, with
//   base(u) = (2^(s0+u)) + row_term << u.
// s0: global index of the first stage; kofs/row_term select the block.
template <int H>
__device__ __forceinline__ void fwd_stages(uint64_t (&x)[16], const ulonglong2* __restrict__ tw, int s0, int row_term,
                                           int kofs, uint64_t q) {
    const uint64_t two_q = 2 * q;
#pragma unroll
    for (int u = 0; u < H; u++) {
        const int D = 1 << (H - 1 - u);
        const int base = (1 << (s0 + u)) + (row_term << u);
#pragma unroll
        for (int k = 0; k < 16; k++) {
            if (k & D) continue;
            ulonglong2 w = ldtw(tw + base + ((kofs + k) >> (H - u)));
            bfly_ct(x[k], x[k + D], w, q, two_q);
        }
    }
}

// Inverse stages on 16 registers: the forward stages of fwd_stages<H> in
// reverse order with GS butterflies (same twiddle index formula, inverse
// table).  Stages u = H-1 down to ULO.
template <int H, int ULO = 0>
__device__ __forceinline__ void inv_stages(uint64_t (&x)[16], const ulonglong2* __restrict__ tw, int s0, int row_term,
                                           int kofs, uint64_t q) {
    const uint64_t two_q = 2 * q;
#pragma unroll
    for (int u = H - 1; u >= ULO; u--) {
        const int D = 1 << (H - 1 - u);
        const int base = (1 << (s0 + u)) + (row_term << u);
#pragma unroll
        for (int k = 0; k < 16; k++) {
            if (k & D) continue;
            ulonglong2 w = ldtw(tw + base + ((kofs + k) >> (H - u)));
            bfly_gs(x[k], x[k + D], w, q, two_q);
        }
    }
}

// ---------------------------------------------------------------------------
// FP64 arithmetic for primes below 2^44 (the 40-bit primes of the modulus
// chain).  Residues are held as doubles (exact integers below 2^53) and the
// modular product runs on the FP64 pipe:
//   p_hi = fl(y w), p_lo = fma(y, w, -p_hi)          (y w = p_hi + p_lo exactly)
//   qh = round-to-nearest(p_hi / q) via the 1.5 2^52 magic constant
//   r = fma(-qh, q, p_hi) + p_lo                     (exact: |r| < q/2 + 2^30)
//   r < 0 ? r + q : r                                (result in [0, q))
// The remainder is exact because its true value is an integer far below
// 2^53, which one rounding of the FMA reproduces.  Checked against integer
// arithmetic on random and boundary inputs (y < 4q, w < q).
struct FpMod {
    double q, two_q, qinv, ninv;
};

constexpr uint64_t kFpPrimeLimit = 1ull << 44;

__device__ __forceinline__ double fp_modmul(double y, double w, const FpMod& m) {
    const double MAGIC = 6755399441055744.0;  // 1.5 * 2^52
    double ph = __dmul_rn(y, w);
    double pl = __fma_rn(y, w, -ph);
    double qh = __dsub_rn(__fma_rn(ph, m.qinv, MAGIC), MAGIC);
    double r = __dadd_rn(__fma_rn(-qh, m.q, ph), pl);
    return r < 0.0 ? __dadd_rn(r, m.q) : r;
}

__device__ __forceinline__ double fp_csub(double x, double c) { return x >= c ? __dsub_rn(x, c) : x; }

// exact conversions for integers below 2^52
__device__ __forceinline__ double u2d(uint64_t x) {
    return __dsub_rn(__longlong_as_double((long long)(x | 0x4330000000000000ull)), 4503599627370496.0);
}
__device__ __forceinline__ uint64_t d2u(double d) {
    return (uint64_t)__double_as_longlong(__dadd_rn(d, 4503599627370496.0)) & 0x000FFFFFFFFFFFFFull;
}

// CT butterfly, values in [0, 4q) -> [0, 4q)
__device__ __forceinline__ void bfly_ct(double& x, double& y, double w, const FpMod& m) {
    double a = fp_csub(x, m.two_q);
    double t = fp_modmul(y, w, m);
    x = __dadd_rn(a, t);
    y = __dadd_rn(a, __dsub_rn(m.two_q, t));
}

// GS butterfly, values in [0, 2q) -> [0, 2q)
__device__ __forceinline__ void bfly_gs(double& x, double& y, double w, const FpMod& m) {
    double a = x, b = y;
    x = fp_csub(__dadd_rn(a, b), m.two_q);
    y = fp_modmul(__dsub_rn(__dadd_rn(a, m.two_q), b), w, m);
}

__device__ __forceinline__ double reduce4q(double x, const FpMod& m) { return fp_csub(fp_csub(x, m.two_q), m.q); }

template <int H>
__device__ __forceinline__ void fwd_stages(double (&x)[16], const double* __restrict__ tw, int s0, int row_term,
                                           int kofs, const FpMod& m) {
#pragma unroll
    for (int u = 0; u < H; u++) {
        const int D = 1 << (H - 1 - u);
        const int base = (1 << (s0 + u)) + (row_term << u);
#pragma unroll
        for (int k = 0; k < 16; k++) {
            if (k & D) continue;
            double w = __ldg(tw + base + ((kofs + k) >> (H - u)));
            bfly_ct(x[k], x[k + D], w, m);
        }
    }
}

template <int H, int ULO = 0>
__device__ __forceinline__ void inv_stages(double (&x)[16], const double* __restrict__ tw, int s0, int row_term,
                                           int kofs, const FpMod& m) {
#pragma unroll
    for (int u = H - 1; u >= ULO; u--) {
        const int D = 1 << (H - 1 - u);
        const int base = (1 << (s0 + u)) + (row_term << u);
#pragma unroll
        for (int k = 0; k < 16; k++) {
            if (k & D) continue;
            double w = __ldg(tw + base + ((kofs + k) >> (H - u)));
            bfly_gs(x[k], x[k + D], w, m);
        }
    }
}

__device__ __forceinline__ void inv_stage0_scaled(double (&x)[16], double w1, const FpMod& m) {
#pragma unroll
    for (int k = 0; k < 8; k++) {
        double a = x[k], b = x[k + 8];
        x[k] = fp_modmul(__dadd_rn(a, b), m.ninv, m);
        x[k + 8] = fp_modmul(__dsub_rn(__dadd_rn(a, m.two_q), b), w1, m);
    }
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

// Blocks per SM the transforms are compiled for (register budget 85).
constexpr int NTT_MIN_BLOCKS = 3;

// shared-memory index of element i of a padded row (one pad word per 16)
__device__ __forceinline__ int padded(int i) { return i + (i >> 4); }

__device__ __forceinline__ uint64_t to_elem(uint64_t v, uint64_t) { return v; }
__device__ __forceinline__ double to_elem(uint64_t v, double) { return u2d(v); }
__device__ __forceinline__ uint64_t from_elem(uint64_t v) { return v; }
__device__ __forceinline__ uint64_t from_elem(double v) { return d2u(v); }

template <int LOGN>
__device__ __forceinline__ int row_lane() { return threadIdx.x % (NttCfg<LOGN>::C / 16); }

// x[k] = a[k], k < 16 (a 16-byte aligned)
template <typename T>
__device__ __forceinline__ void row_load16(T (&x)[16], const uint64_t* a) {
    const ulonglong2* in = reinterpret_cast<const ulonglong2*>(a);
#pragma unroll
    for (int k = 0; k < 8; k++) {
        ulonglong2 v = in[k];
        x[2 * k] = to_elem(v.x, T());
        x[2 * k + 1] = to_elem(v.y, T());
    }
}

// a[k] = x[k] reduced from [0, 4q) to [0, q)
template <typename T, typename M>
__device__ __forceinline__ void row_store16(uint64_t* a, T (&x)[16], const M& m) {
    ulonglong2* o = reinterpret_cast<ulonglong2*>(a);
#pragma unroll
    for (int k = 0; k < 8; k++)
        o[k] = make_ulonglong2(from_elem(reduce4q(x[2 * k], m)), from_elem(reduce4q(x[2 * k + 1], m)));
}

// x[k] = row[p + CS k], k < 16 (the forward row pass's input layout)
template <int LOGN, typename T>
__device__ __forceinline__ void row_load_strided(T (&x)[16], const uint64_t* row) {
    constexpr int CS = NttCfg<LOGN>::C / 16;
    const int p = threadIdx.x % CS;
#pragma unroll
    for (int k = 0; k < 16; k++) x[k] = to_elem(row[p + CS * k], T());
}

// Forward row pass (stages S1..LOGN-1) on registers loaded from columns
// p + CS k of row r; returns columns 16 p + k in [0, 4q).
template <int LOGN, typename T, typename TW, typename M>
__device__ __forceinline__ void fwd_rows_core(T (&x)[16], T* sm, int r, const TW* tw, const M& m) {
    using Cf = NttCfg<LOGN>;
    constexpr int CS = Cf::C / 16;
    const int p = threadIdx.x % CS, rr = threadIdx.x / CS;
    T* s = sm + rr * Cf::ROW_PITCH;
    fwd_stages<4>(x, tw, Cf::S1, r, 0, m);
#pragma unroll
    for (int k = 0; k < 16; k++) s[padded(p + CS * k)] = x[k];
    __syncthreads();
#pragma unroll
    for (int k = 0; k < 16; k++) x[k] = s[padded(16 * p + k)];
    fwd_stages<Cf::S2 - 4>(x, tw, Cf::S1 + 4, r << 4, 16 * p, m);
}

// Inverse row pass (stages LOGN-1..S1) on registers loaded from columns
// 16 p + k of row r; stores columns p + CS k of the result to out_row.
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
    for (int k = 0; k < 16; k++) out_row[p + CS * k] = from_elem(x[k]);
}

}  // namespace he
