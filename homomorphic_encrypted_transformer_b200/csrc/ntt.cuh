// Negacyclic NTT building blocks on shared-memory tiles.
//
// Transform (textbook negacyclic NTT, bit-reversed output): storage index j
// of the output holds a(psi^(2 brev(j) + 1)).  Computed by the Cooley-Tukey
// decimation-in-time network with twiddles psi^brev(m+i) (Longa-Naehrig,
// "Speeding up the Number Theoretic Transform for Faster Ideal Lattice-Based
// Cryptography", CANS 2016, algorithms 1 and 2), with Harvey's lazy
// butterflies.  The inverse is the Gentleman-Sande network with psi^-brev(m+i)
// and N^-1 folded into its last stage.
//
// N = R * C with R = 2^s1 rows and C = 2^s2 columns (index j = r C + c).
// Forward: stages 0..s1-1 pair rows (one column at a time: "column pass"),
// stages s1..logN-1 pair elements inside a row ("row pass").  Inverse: the
// row stages run first, then the column stages.
#pragma once
#include "modarith.cuh"

namespace he {

// Harvey CT butterfly: x, y in [0, 4q) -> [0, 4q).
__device__ __forceinline__ void bfly_ct(uint64_t& x, uint64_t& y, const ulonglong2 w, uint64_t q) {
    uint64_t two_q = 2 * q;
    uint64_t a = csub(x, two_q);
    uint64_t t = mul_shoup_lazy(y, w.x, w.y, q);
    x = a + t;
    y = a - t + two_q;
}

// Harvey GS butterfly: x, y in [0, 2q) -> [0, 2q).
__device__ __forceinline__ void bfly_gs(uint64_t& x, uint64_t& y, const ulonglong2 w, uint64_t q) {
    uint64_t two_q = 2 * q;
    uint64_t a = x, b = y;
    x = csub(a + b, two_q);
    y = mul_shoup_lazy(a - b + two_q, w.x, w.y, q);
}

// [0, 4q) -> [0, q)
__device__ __forceinline__ uint64_t reduce4q(uint64_t x, uint64_t q) { return csub(csub(x, 2 * q), q); }

// Column pass of the forward transform on a tile sm[R][tc] (row-major, tc
// columns of the limb).  Values enter canonical or in [0, 4q) and leave in
// [0, 4q).  tw_s: the R-1 twiddles psi^brev(1..R-1) staged in shared memory.
__device__ __forceinline__ void tile_fwd_cols(uint64_t* sm, int s1, int tc, const ulonglong2* tw_s, uint64_t q) {
    const int R = 1 << s1;
    for (int s = 0; s < s1; s++) {
        const int t = R >> (s + 1);
        for (int b = threadIdx.x; b < (R >> 1) * tc; b += blockDim.x) {
            int cc = b % tc, p = b / tc;
            int i = p / t, jr = 2 * i * t + (p - i * t);
            bfly_ct(sm[jr * tc + cc], sm[(jr + t) * tc + cc], tw_s[(1 << s) + i], q);
        }
        __syncthreads();
    }
}

// Row pass of the forward transform on a tile sm[tr][C] holding rows
// r0..r0+tr-1.  Leaves values in [0, 4q).  tw: the prime's full twiddle table.
__device__ __forceinline__ void tile_fwd_rows(uint64_t* sm, int s1, int s2, int tr, int r0, const ulonglong2* tw,
                                              uint64_t q) {
    const int C = 1 << s2;
    for (int s = 0; s < s2; s++) {
        const int t = C >> (s + 1);
        const int gs = s1 + s;
        for (int b = threadIdx.x; b < tr * (C >> 1); b += blockDim.x) {
            int rr = b >> (s2 - 1), p = b & ((C >> 1) - 1);
            int i = p / t, jc = 2 * i * t + (p - i * t);
            ulonglong2 w = tw[(1 << gs) + ((r0 + rr) << s) + i];
            bfly_ct(sm[rr * C + jc], sm[rr * C + jc + t], w, q);
        }
        __syncthreads();
    }
}

// Row pass of the inverse transform (stages with t = 1 .. C/2) on sm[tr][C].
// Values enter in [0, 2q) and leave in [0, 2q).
__device__ __forceinline__ void tile_inv_rows(uint64_t* sm, int logn, int s2, int tr, int r0, const ulonglong2* tw,
                                              uint64_t q) {
    const int C = 1 << s2;
    for (int u = 0; u < s2; u++) {
        const int t = 1 << u;
        const int h = 1 << (logn - 1 - u);  // N / (2t)
        for (int b = threadIdx.x; b < tr * (C >> 1); b += blockDim.x) {
            int rr = b >> (s2 - 1), p = b & ((C >> 1) - 1);
            int i = p >> u, jc = 2 * i * t + (p & (t - 1));
            int gi = ((r0 + rr) << (s2 - 1 - u)) + i;
            bfly_gs(sm[rr * C + jc], sm[rr * C + jc + t], tw[h + gi], q);
        }
        __syncthreads();
    }
}

// Column pass of the inverse transform (stages t = C .. N/2) on sm[R][tc],
// including N^-1: the last stage multiplies the sum by N^-1 (ninv) and the
// difference by psi^-brev(1) N^-1 (stored in the table at index 1).
// Values enter in [0, 2q) and leave canonical.
__device__ __forceinline__ void tile_inv_cols(uint64_t* sm, int logn, int s1, int s2, int tc, const ulonglong2* tw,
                                              ulonglong2 ninv, uint64_t q) {
    const int R = 1 << s1;
    for (int u = 0; u < s1; u++) {
        const int tr = 1 << u;                  // distance in rows
        const int h = 1 << (logn - 1 - s2 - u);  // N / (2t), t = tr C
        const bool last = (u == s1 - 1);
        for (int b = threadIdx.x; b < (R >> 1) * tc; b += blockDim.x) {
            int cc = b % tc, p = b / tc;
            int i = p >> u, jr = 2 * i * tr + (p & (tr - 1));
            uint64_t& x = sm[jr * tc + cc];
            uint64_t& y = sm[(jr + tr) * tc + cc];
            if (!last) {
                bfly_gs(x, y, tw[h + i], q);
            } else {
                uint64_t two_q = 2 * q;
                uint64_t a = x, bb = y;
                ulonglong2 w = tw[1];
                x = mul_shoup(a + bb, ninv.x, ninv.y, q);
                y = mul_shoup(a - bb + two_q, w.x, w.y, q);
            }
        }
        __syncthreads();
    }
}

}  // namespace he
