// Batched negacyclic NTT / inverse NTT over RNS limbs: a column pass and a
// row pass per transform, 16 elements per thread (see ntt.cuh).  Limbs of
// primes below 2^41 run the butterflies on the FP64 pipe, the others on the
// integer pipe (the branch is uniform per block: one limb per block).
#include "he_internal.h"
#include "kernels.cuh"
#include "ntt.cuh"

namespace he {

template <int LOGN, typename T, typename TW, typename M>
__device__ __forceinline__ void fwd_cols_body(T* sm, uint64_t* a, const TW* tw, const M& m) {
    using Cf = NttCfg<LOGN>;
    const int cc = threadIdx.x % Cf::TC, g = threadIdx.x / Cf::TC;
    constexpr int RS = Cf::R / 16;
    T x[16];
#pragma unroll
    for (int k = 0; k < 16; k++) x[k] = to_elem(a[(size_t)(g + RS * k) * Cf::C + cc], T());
    fwd_stages<4>(x, tw, 0, 0, 0, m);
#pragma unroll
    for (int k = 0; k < 16; k++) sm[(g + RS * k) * Cf::TC + cc] = x[k];
    __syncthreads();
#pragma unroll
    for (int k = 0; k < 16; k++) x[k] = sm[(16 * g + k) * Cf::TC + cc];
    fwd_stages<Cf::S1 - 4>(x, tw, 4, 0, 16 * g, m);
#pragma unroll
    for (int k = 0; k < 16; k++) a[(size_t)(16 * g + k) * Cf::C + cc] = raw_out(x[k]);
}

template <int LOGN, typename T, typename TW, typename M>
__device__ __forceinline__ void fwd_rows_body(T* sm, uint64_t* a, int r, const TW* tw, const M& m) {
    T x[16];
    row_load_strided<LOGN>(x, a);
    fwd_rows_core<LOGN>(x, sm, r, tw, m);
    row_store16(a + 16 * row_lane<LOGN>(), x, m);
}

template <int LOGN, typename T, typename TW, typename M>
__device__ __forceinline__ void inv_rows_body(T* sm, uint64_t* a, int r, const TW* tw, const M& m) {
    T x[16];
    row_load16(x, a + 16 * row_lane<LOGN>());
    inv_rows_core<LOGN>(x, sm, a, r, tw, m);
}

template <int LOGN>
__global__ void __launch_bounds__(NttCfg<LOGN>::COL_THREADS, NTT_COL_MIN_BLOCKS)
    k_ntt_fwd_cols(RowSet rs, const DevPrime* __restrict__ pr, const ulonglong2* __restrict__ tw_all,
                   const double* __restrict__ twd_all, const FpMod* __restrict__ fpm) {
    using Cf = NttCfg<LOGN>;
    __shared__ uint64_t sm[Cf::R * Cf::TC];
    const int row = blockIdx.y;
    const int pidx = rs.prime(row);
    const uint64_t q = pr[pidx].q;
    uint64_t* a = rs.ptr(row, Cf::N) + blockIdx.x * Cf::TC;
    if (q < kFpPrimeLimit)
        fwd_cols_body<LOGN>(reinterpret_cast<double*>(sm), a, twd_all + (size_t)pidx * Cf::N, fpm[pidx]);
    else
        fwd_cols_body<LOGN>(sm, a, tw_all + (size_t)pidx * Cf::N, q);
}

template <int LOGN>
__global__ void __launch_bounds__(NttCfg<LOGN>::ROW_THREADS, NTT_MIN_BLOCKS)
    k_ntt_fwd_rows(RowSet rs, const DevPrime* __restrict__ pr, const ulonglong2* __restrict__ tw_all,
                   const double* __restrict__ twd_all, const FpMod* __restrict__ fpm) {
    using Cf = NttCfg<LOGN>;
    __shared__ uint64_t sm[Cf::TR * Cf::ROW_PITCH];
    const int row = blockIdx.y;
    const int pidx = rs.prime(row);
    const uint64_t q = pr[pidx].q;
    const int r = blockIdx.x * Cf::TR + threadIdx.x / (Cf::C / 16);
    uint64_t* a = rs.ptr(row, Cf::N) + (size_t)r * Cf::C;
    if (q < kFpPrimeLimit)
        fwd_rows_body<LOGN>(reinterpret_cast<double*>(sm), a, r, twd_all + (size_t)pidx * Cf::N, fpm[pidx]);
    else
        fwd_rows_body<LOGN>(sm, a, r, tw_all + (size_t)pidx * Cf::N, q);
}

template <int LOGN>
__global__ void __launch_bounds__(NttCfg<LOGN>::ROW_THREADS, NTT_MIN_BLOCKS)
    k_ntt_inv_rows(RowSet rs, const DevPrime* __restrict__ pr, const ulonglong2* __restrict__ tw_all,
                   const double* __restrict__ twd_all, const FpMod* __restrict__ fpm) {
    using Cf = NttCfg<LOGN>;
    __shared__ uint64_t sm[Cf::TR * Cf::ROW_PITCH];
    const int row = blockIdx.y;
    const int pidx = rs.prime(row);
    const uint64_t q = pr[pidx].q;
    const int r = blockIdx.x * Cf::TR + threadIdx.x / (Cf::C / 16);
    uint64_t* a = rs.ptr(row, Cf::N) + (size_t)r * Cf::C;
    if (q < kFpPrimeLimit)
        inv_rows_body<LOGN>(reinterpret_cast<double*>(sm), a, r, twd_all + (size_t)pidx * Cf::N, fpm[pidx]);
    else
        inv_rows_body<LOGN>(sm, a, r, tw_all + (size_t)pidx * Cf::N, q);
}

__device__ __forceinline__ void inv_stage0(uint64_t (&x)[16], ulonglong2 w1, ulonglong2 ninv, uint64_t q) {
    inv_stage0_scaled(x, w1, ninv, q);
}
__device__ __forceinline__ void inv_stage0(double (&x)[16], double w1, int, const FpMod& m) {
    inv_stage0_scaled(x, w1, m);
}

template <int LOGN, typename T, typename TW, typename M, typename W1, typename NI>
__device__ __forceinline__ void inv_cols_body(T* sm, uint64_t* a, const TW* tw, const M& m, W1 w1, NI ninv) {
    using Cf = NttCfg<LOGN>;
    const int cc = threadIdx.x % Cf::TC, g = threadIdx.x / Cf::TC;
    constexpr int RS = Cf::R / 16;
    T x[16];
#pragma unroll
    for (int k = 0; k < 16; k++) x[k] = raw_in(a[(size_t)(16 * g + k) * Cf::C + cc], T());
    inv_cols_prereduce(x, m);
    inv_stages<Cf::S1 - 4>(x, tw, 4, 0, 16 * g, m);
#pragma unroll
    for (int k = 0; k < 16; k++) sm[(16 * g + k) * Cf::TC + cc] = x[k];
    __syncthreads();
#pragma unroll
    for (int k = 0; k < 16; k++) x[k] = sm[(g + RS * k) * Cf::TC + cc];
    inv_stages<4, 1>(x, tw, 0, 0, 0, m);
    inv_stage0(x, w1, ninv, m);
#pragma unroll
    for (int k = 0; k < 16; k++) a[(size_t)(g + RS * k) * Cf::C + cc] = inv_canon(x[k], m);
}

template <int LOGN>
__global__ void __launch_bounds__(NttCfg<LOGN>::COL_THREADS, NTT_COL_MIN_BLOCKS)
    k_ntt_inv_cols(RowSet rs, const DevPrime* __restrict__ pr, const ulonglong2* __restrict__ tw_all,
                   const ulonglong2* __restrict__ ninv_all, const double* __restrict__ twd_all,
                   const FpMod* __restrict__ fpm) {
    using Cf = NttCfg<LOGN>;
    __shared__ uint64_t sm[Cf::R * Cf::TC];
    const int row = blockIdx.y;
    const int pidx = rs.prime(row);
    const uint64_t q = pr[pidx].q;
    uint64_t* a = rs.ptr(row, Cf::N) + blockIdx.x * Cf::TC;
    if (q < kFpPrimeLimit) {
        const double* twd = twd_all + (size_t)pidx * Cf::N;
        inv_cols_body<LOGN>(reinterpret_cast<double*>(sm), a, twd, fpm[pidx], __ldg(twd + 1), 0);
    } else {
        const ulonglong2* tw = tw_all + (size_t)pidx * Cf::N;
        inv_cols_body<LOGN>(sm, a, tw, q, ldtw(tw + 1), ninv_all[pidx]);
    }
}

NttShape ntt_shape(int logn) {
    NttShape s;
    s.s1 = (logn + 1) / 2;
    s.s2 = logn - s.s1;
    int R = 1 << s.s1, C = 1 << s.s2;
    s.tc = C < 16 ? C : 16;
    s.tr = (4096 / C) < R ? (4096 / C) : R;
    s.col_tiles = C / s.tc;
    s.row_tiles = R / s.tr;
    s.smem_cols = (size_t)R * s.tc * 8;
    s.smem_rows = (size_t)s.tr * (C + C / 16) * 8;
    return s;
}

static int launch_check(he_ctx* c, const char* what) { return check_cuda(c, cudaGetLastError(), what); }

template <int LOGN>
static void launch_fwd(he_ctx* c, const RowSet& rs, int n_rows, int which) {
    using Cf = NttCfg<LOGN>;
    if (which == 0)
        k_ntt_fwd_cols<LOGN><<<dim3(Cf::COL_TILES, n_rows), Cf::COL_THREADS, 0, c->stream>>>(
            rs, c->d_prime, c->d_tw_fwd, c->d_twd_fwd, c->d_fpmod);
    else
        k_ntt_fwd_rows<LOGN><<<dim3(Cf::ROW_TILES, n_rows), Cf::ROW_THREADS, 0, c->stream>>>(
            rs, c->d_prime, c->d_tw_fwd, c->d_twd_fwd, c->d_fpmod);
}

template <int LOGN>
static void launch_inv(he_ctx* c, const RowSet& rs, int n_rows, int which) {
    using Cf = NttCfg<LOGN>;
    if (which == 0)
        k_ntt_inv_rows<LOGN><<<dim3(Cf::ROW_TILES, n_rows), Cf::ROW_THREADS, 0, c->stream>>>(
            rs, c->d_prime, c->d_tw_inv, c->d_twd_inv, c->d_fpmod);
    else
        k_ntt_inv_cols<LOGN><<<dim3(Cf::COL_TILES, n_rows), Cf::COL_THREADS, 0, c->stream>>>(
            rs, c->d_prime, c->d_tw_inv, c->d_inv_last, c->d_twd_inv, c->d_fpmod);
}

static void dispatch(he_ctx* c, const RowSet& rs, int n_rows, bool fwd, int which) {
    switch (c->log_n) {
#define HE_NTT_CASE(LN)                                \
    case LN:                                           \
        if (fwd)                                       \
            launch_fwd<LN>(c, rs, n_rows, which);      \
        else                                           \
            launch_inv<LN>(c, rs, n_rows, which);      \
        break;
        HE_NTT_CASE(10)
        HE_NTT_CASE(11)
        HE_NTT_CASE(12)
        HE_NTT_CASE(13)
        HE_NTT_CASE(14)
        HE_NTT_CASE(15)
        HE_NTT_CASE(16)
#undef HE_NTT_CASE
        default:
            break;
    }
}

// One pass of a transform, bracketed for the profile: the column pass does
// stages 0..S1-1, the row pass stages S1..LOGN-1 (each reads and writes
// every limb once).
static int ntt_pass(he_ctx* c, const RowSet& rs, int n_rows, bool fwd, int which) {
    if (n_rows <= 0) return HE_OK;
    NttShape sh = ntt_shape(c->log_n);
    const double bytes = 16.0 * c->N * n_rows, half = 0.5 * c->N * n_rows;
    const int cls = fwd ? (which == 0 ? HE_PROF_NTT_FWD_COLS : HE_PROF_NTT_FWD_ROWS)
                        : (which == 0 ? HE_PROF_NTT_INV_ROWS : HE_PROF_NTT_INV_COLS);
    const bool col_pass = fwd == (which == 0);
    prof_begin(c, cls);
    dispatch(c, rs, n_rows, fwd, which);
    int rc = launch_check(c, fwd ? "ntt_fwd" : "ntt_inv");
    if (rc) return rc;
    c->launches += 1;
    const int stages = col_pass ? sh.s1 : sh.s2;
    return prof_end(c, cls, bytes, half * stages, 0.5 * c->N * fp_rows(c, rs, n_rows) * stages);
}

template <int LOGN>
static cudaError_t preload_kernels() {
    cudaFuncAttributes a;
    cudaError_t e = cudaFuncGetAttributes(&a, k_ntt_fwd_cols<LOGN>);
    if (e == cudaSuccess) e = cudaFuncGetAttributes(&a, k_ntt_fwd_rows<LOGN>);
    if (e == cudaSuccess) e = cudaFuncGetAttributes(&a, k_ntt_inv_rows<LOGN>);
    if (e == cudaSuccess) e = cudaFuncGetAttributes(&a, k_ntt_inv_cols<LOGN>);
    return e;
}

int ntt_preload(he_ctx* c) {
    cudaError_t e = cudaErrorInvalidValue;
    switch (c->log_n) {
        case 10: e = preload_kernels<10>(); break;
        case 11: e = preload_kernels<11>(); break;
        case 12: e = preload_kernels<12>(); break;
        case 13: e = preload_kernels<13>(); break;
        case 14: e = preload_kernels<14>(); break;
        case 15: e = preload_kernels<15>(); break;
        case 16: e = preload_kernels<16>(); break;
        default: break;
    }
    return check_cuda(c, e, "transform kernels");
}

int ntt_fwd_set(he_ctx* c, const RowSet& rs, int n_rows) {
    int rc = ntt_pass(c, rs, n_rows, true, 0);
    return rc ? rc : ntt_pass(c, rs, n_rows, true, 1);
}

int ntt_inv_set(he_ctx* c, const RowSet& rs, int n_rows) {
    int rc = ntt_pass(c, rs, n_rows, false, 0);
    return rc ? rc : ntt_pass(c, rs, n_rows, false, 1);
}

int ntt_fwd_cols_set(he_ctx* c, const RowSet& rs, int n_rows) { return ntt_pass(c, rs, n_rows, true, 0); }

int ntt_inv_cols_set(he_ctx* c, const RowSet& rs, int n_rows) { return ntt_pass(c, rs, n_rows, false, 1); }

}  // namespace he

using namespace he;

extern "C" int he_ntt_fwd(he_ctx* c, uint64_t* d, int n_polys, int n_limbs, int first_prime) {
    if (!c) return HE_EINVAL;
    if (!d || n_polys < 0 || n_limbs < 0 || first_prime < 0 || first_prime + n_limbs > c->L + c->K ||
        ((uintptr_t)d & 31))
        return set_err(c, HE_EINVAL, "he_ntt_fwd: bad arguments");
    RowSet rs = rowset_contig(d, n_limbs, c->N, prime_range(first_prime, n_limbs));
    return ntt_fwd_set(c, rs, n_polys * n_limbs);
}

extern "C" int he_ntt_inv(he_ctx* c, uint64_t* d, int n_polys, int n_limbs, int first_prime) {
    if (!c) return HE_EINVAL;
    if (!d || n_polys < 0 || n_limbs < 0 || first_prime < 0 || first_prime + n_limbs > c->L + c->K ||
        ((uintptr_t)d & 31))
        return set_err(c, HE_EINVAL, "he_ntt_inv: bad arguments");
    RowSet rs = rowset_contig(d, n_limbs, c->N, prime_range(first_prime, n_limbs));
    return ntt_inv_set(c, rs, n_polys * n_limbs);
}
