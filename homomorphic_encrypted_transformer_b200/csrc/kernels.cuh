// Shared launch-side types of the engine's kernels.
#pragma once
#include <stdint.h>

#include "modarith.cuh"

namespace he {

// A batch of limbs: row r lives at base + (r / per_group) * group_stride
// + (r % per_group) * N and uses prime index prime_idx[r % per_group].
struct RowSet {
    uint64_t* base;
    long long group_stride;  // in uint64 words
    int per_group;
    uint8_t prime_idx[64];

    __device__ __forceinline__ int prime(int r) const { return prime_idx[r % per_group]; }
    __device__ __forceinline__ uint64_t* ptr(int r, int N) const {
        int g = r / per_group, rr = r - g * per_group;
        return base + (long long)g * group_stride + (long long)rr * N;
    }
};

struct NttShape {
    int s1, s2;          // log2 of rows (R) and columns (C), N = R C
    int tc, tr;          // columns per column-pass tile, rows per row-pass tile
    int col_tiles, row_tiles;
    size_t smem_cols, smem_rows;
};

NttShape ntt_shape(int logn);

}  // namespace he
