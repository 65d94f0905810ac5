// Shared launch-side types of the engine's kernels.
#pragma once
#include <stdint.h>

#include "modarith.cuh"

namespace he {

// A batch of limbs: row r lives at base + (r / per_group) * group_stride
// + (r % per_group) * N.  Its prime index is that of position rr = r %
// per_group in a list made of at most three runs of consecutive primes:
// rr < len0 -> first0 + rr; rr < len0 + len1 -> first1 + rr - len0;
// otherwise first2 + rr - len0 - len1.  (Q_level then P, or Q_level minus a
// digit then P, are such lists.)  Plain scalars keep the struct out of local
// memory when kernels index it.
struct RowSet {
    uint64_t* base;
    long long group_stride;  // in uint64 words
    int per_group;
    int first0, len0, first1, len1, first2;

    __host__ __device__ __forceinline__ int prime(int r) const {
        int rr = r % per_group;
        if (rr < len0) return first0 + rr;
        rr -= len0;
        if (rr < len1) return first1 + rr;
        return first2 + rr - len1;
    }
    __device__ __forceinline__ uint64_t* ptr(int r, int N) const {
        int g = r / per_group, rr = r - g * per_group;
        return base + (long long)g * group_stride + (long long)rr * N;
    }
};

// Per-ciphertext parameters of batched launches (at most 64 ciphertexts).
constexpr int kMaxBatch = 64;
struct PtrList {
    const uint64_t* p[kMaxBatch];
};
struct MutPtrList {
    uint64_t* p[kMaxBatch];
};
struct GalList {
    uint64_t g[kMaxBatch];
};
struct IdxList {
    int i[kMaxBatch];
};

// Evaluation-domain index whose value sigma_k moves to index j (k = 0: j):
// storage j is the point psi^(2 brev(j)+1); sigma_k(a) there is a(psi^((2 brev(j)+1) k)).
// An aligned block of 2^m indices maps onto an aligned block of 2^m indices.
__device__ __forceinline__ int automorph_src(int j, int logn, uint64_t k) {
    if (!k) return j;
    unsigned m = __brev((unsigned)j) >> (32 - logn);
    uint64_t e = ((2ull * m + 1) * k) & ((2ull << logn) - 1);
    unsigned m2 = (unsigned)((e - 1) >> 1);
    return (int)(__brev(m2) >> (32 - logn));
}

struct NttShape {
    int s1, s2;          // log2 of rows (R) and columns (C), N = R C
    int tc, tr;          // columns per column-pass tile, rows per row-pass tile
    int col_tiles, row_tiles;
    size_t smem_cols, smem_rows;
};

NttShape ntt_shape(int logn);

}  // namespace he
