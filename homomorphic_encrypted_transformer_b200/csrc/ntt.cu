// Batched negacyclic NTT / inverse NTT over RNS limbs (two passes per
// transform: column pass and row pass, see ntt.cuh).
#include "he_internal.h"
#include "kernels.cuh"
#include "ntt.cuh"

namespace he {

__global__ void k_ntt_fwd_cols(RowSet rs, const DevPrime* __restrict__ pr, const ulonglong2* __restrict__ tw_all,
                               int logn, int s1, int tc) {
    extern __shared__ uint64_t smem[];
    const int N = 1 << logn, R = 1 << s1, C = N >> s1;
    uint64_t* sm = smem;
    ulonglong2* tws = reinterpret_cast<ulonglong2*>(smem + R * tc);
    const int row = blockIdx.y;
    const int pidx = rs.prime(row);
    const uint64_t q = pr[pidx].q;
    const ulonglong2* tw = tw_all + (size_t)pidx * N;
    uint64_t* a = rs.ptr(row, N);
    const int col0 = blockIdx.x * tc;
    for (int e = threadIdx.x; e < R; e += blockDim.x) tws[e] = tw[e];
    for (int e = threadIdx.x; e < R * tc; e += blockDim.x) {
        int r = e / tc, cc = e - r * tc;
        sm[e] = a[(size_t)r * C + col0 + cc];
    }
    __syncthreads();
    tile_fwd_cols(sm, s1, tc, tws, q);
    for (int e = threadIdx.x; e < R * tc; e += blockDim.x) {
        int r = e / tc, cc = e - r * tc;
        a[(size_t)r * C + col0 + cc] = sm[e];
    }
}

__global__ void k_ntt_fwd_rows(RowSet rs, const DevPrime* __restrict__ pr, const ulonglong2* __restrict__ tw_all,
                               int logn, int s1, int tr) {
    extern __shared__ uint64_t smem[];
    const int N = 1 << logn, s2 = logn - s1, C = 1 << s2;
    const int row = blockIdx.y;
    const int pidx = rs.prime(row);
    const uint64_t q = pr[pidx].q;
    const ulonglong2* tw = tw_all + (size_t)pidx * N;
    uint64_t* a = rs.ptr(row, N) + (size_t)blockIdx.x * tr * C;
    for (int e = threadIdx.x; e < tr * C; e += blockDim.x) smem[e] = a[e];
    __syncthreads();
    tile_fwd_rows(smem, s1, s2, tr, blockIdx.x * tr, tw, q);
    for (int e = threadIdx.x; e < tr * C; e += blockDim.x) a[e] = reduce4q(smem[e], q);
}

__global__ void k_ntt_inv_rows(RowSet rs, const DevPrime* __restrict__ pr, const ulonglong2* __restrict__ tw_all,
                               int logn, int s1, int tr) {
    extern __shared__ uint64_t smem[];
    const int N = 1 << logn, s2 = logn - s1, C = 1 << s2;
    const int row = blockIdx.y;
    const int pidx = rs.prime(row);
    const uint64_t q = pr[pidx].q;
    const ulonglong2* tw = tw_all + (size_t)pidx * N;
    uint64_t* a = rs.ptr(row, N) + (size_t)blockIdx.x * tr * C;
    for (int e = threadIdx.x; e < tr * C; e += blockDim.x) smem[e] = a[e];
    __syncthreads();
    tile_inv_rows(smem, logn, s2, tr, blockIdx.x * tr, tw, q);
    for (int e = threadIdx.x; e < tr * C; e += blockDim.x) a[e] = smem[e];
}

__global__ void k_ntt_inv_cols(RowSet rs, const DevPrime* __restrict__ pr, const ulonglong2* __restrict__ tw_all,
                               const ulonglong2* __restrict__ ninv_all, int logn, int s1, int tc) {
    extern __shared__ uint64_t smem[];
    const int N = 1 << logn, R = 1 << s1, s2 = logn - s1, C = N >> s1;
    uint64_t* sm = smem;
    ulonglong2* tws = reinterpret_cast<ulonglong2*>(smem + R * tc);
    const int row = blockIdx.y;
    const int pidx = rs.prime(row);
    const uint64_t q = pr[pidx].q;
    const ulonglong2* tw = tw_all + (size_t)pidx * N;
    uint64_t* a = rs.ptr(row, N);
    const int col0 = blockIdx.x * tc;
    for (int e = threadIdx.x; e < R; e += blockDim.x) tws[e] = tw[e];
    for (int e = threadIdx.x; e < R * tc; e += blockDim.x) {
        int r = e / tc, cc = e - r * tc;
        sm[e] = a[(size_t)r * C + col0 + cc];
    }
    __syncthreads();
    tile_inv_cols(sm, logn, s1, s2, tc, tws, ninv_all[pidx], q);
    for (int e = threadIdx.x; e < R * tc; e += blockDim.x) {
        int r = e / tc, cc = e - r * tc;
        a[(size_t)r * C + col0 + cc] = sm[e];
    }
}

NttShape ntt_shape(int logn) {
    NttShape s;
    s.s1 = (logn + 1) / 2;
    s.s2 = logn - s.s1;
    int R = 1 << s.s1, C = 1 << s.s2;
    s.tc = C < 16 ? C : 16;
    s.tr = R * s.tc / C;
    s.col_tiles = C / s.tc;
    s.row_tiles = R / s.tr;
    s.smem_cols = (size_t)R * s.tc * 8 + (size_t)R * 16;
    s.smem_rows = (size_t)s.tr * C * 8;
    return s;
}

static int launch_check(he_ctx* c, const char* what) { return check_cuda(c, cudaGetLastError(), what); }

int ntt_fwd_set(he_ctx* c, const RowSet& rs, int n_rows) {
    if (n_rows <= 0) return HE_OK;
    NttShape sh = ntt_shape(c->log_n);
    dim3 g1(sh.col_tiles, n_rows), g2(sh.row_tiles, n_rows);
    const double bytes = 16.0 * c->N * n_rows, half = 0.5 * c->N * n_rows;
    prof_begin(c, HE_PROF_NTT_FWD_COLS);
    k_ntt_fwd_cols<<<g1, 256, sh.smem_cols, c->stream>>>(rs, c->d_prime, c->d_tw_fwd, c->log_n, sh.s1, sh.tc);
    int rc = launch_check(c, "ntt_fwd_cols");
    if (rc) return rc;
    prof_end(c, HE_PROF_NTT_FWD_COLS, bytes, half * sh.s1);
    prof_begin(c, HE_PROF_NTT_FWD_ROWS);
    k_ntt_fwd_rows<<<g2, 256, sh.smem_rows, c->stream>>>(rs, c->d_prime, c->d_tw_fwd, c->log_n, sh.s1, sh.tr);
    rc = launch_check(c, "ntt_fwd_rows");
    if (rc) return rc;
    c->launches += 2;
    return prof_end(c, HE_PROF_NTT_FWD_ROWS, bytes, half * sh.s2);
}

int ntt_inv_set(he_ctx* c, const RowSet& rs, int n_rows) {
    if (n_rows <= 0) return HE_OK;
    NttShape sh = ntt_shape(c->log_n);
    dim3 g1(sh.col_tiles, n_rows), g2(sh.row_tiles, n_rows);
    const double bytes = 16.0 * c->N * n_rows, half = 0.5 * c->N * n_rows;
    prof_begin(c, HE_PROF_NTT_INV_ROWS);
    k_ntt_inv_rows<<<g2, 256, sh.smem_rows, c->stream>>>(rs, c->d_prime, c->d_tw_inv, c->log_n, sh.s1, sh.tr);
    int rc = launch_check(c, "ntt_inv_rows");
    if (rc) return rc;
    prof_end(c, HE_PROF_NTT_INV_ROWS, bytes, half * sh.s2);
    prof_begin(c, HE_PROF_NTT_INV_COLS);
    k_ntt_inv_cols<<<g1, 256, sh.smem_cols, c->stream>>>(rs, c->d_prime, c->d_tw_inv, c->d_inv_last, c->log_n, sh.s1,
                                                          sh.tc);
    rc = launch_check(c, "ntt_inv_cols");
    if (rc) return rc;
    c->launches += 2;
    return prof_end(c, HE_PROF_NTT_INV_COLS, bytes, half * sh.s1);
}

int ntt_setup(he_ctx* c) {
    NttShape sh = ntt_shape(c->log_n);
    size_t m = sh.smem_cols > sh.smem_rows ? sh.smem_cols : sh.smem_rows;
    if (m > 48 * 1024) {
        const void* fns[] = {(const void*)k_ntt_fwd_cols, (const void*)k_ntt_fwd_rows, (const void*)k_ntt_inv_rows,
                             (const void*)k_ntt_inv_cols};
        for (const void* f : fns) {
            int rc = check_cuda(c, cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)m),
                                "ntt smem attribute");
            if (rc) return rc;
        }
    }
    return HE_OK;
}

}  // namespace he

using namespace he;

extern "C" int he_ntt_fwd(he_ctx* c, uint64_t* d, int n_polys, int n_limbs, int first_prime) {
    if (!c) return HE_EINVAL;
    if (!d || n_polys < 0 || n_limbs < 0 || first_prime < 0 || first_prime + n_limbs > c->L + c->K)
        return set_err(c, HE_EINVAL, "he_ntt_fwd: bad arguments");
    RowSet rs = rowset_contig(d, n_limbs, c->N, prime_range(first_prime, n_limbs));
    return ntt_fwd_set(c, rs, n_polys * n_limbs);
}

extern "C" int he_ntt_inv(he_ctx* c, uint64_t* d, int n_polys, int n_limbs, int first_prime) {
    if (!c) return HE_EINVAL;
    if (!d || n_polys < 0 || n_limbs < 0 || first_prime < 0 || first_prime + n_limbs > c->L + c->K)
        return set_err(c, HE_EINVAL, "he_ntt_inv: bad arguments");
    RowSet rs = rowset_contig(d, n_limbs, c->N, prime_range(first_prime, n_limbs));
    return ntt_inv_set(c, rs, n_polys * n_limbs);
}
