// Key generation, tensor product, rescale, elementwise helpers,
// HMult+relinearise+rescale and the Paterson-Stockmeyer driver.
#include <math.h>

#include <algorithm>

#include "he_internal.h"
#include "keyseed.cuh"
#include "ntt.cuh"

namespace he {

constexpr int TB = 256;

static int lc(he_ctx* c, const char* what) {
    c->launches++;
    return check_cuda(c, cudaGetLastError(), what);
}

struct RowConst {
    ulonglong2 v[kMaxPrimes];  // {value, shoup} per row
};

#define HE_NTT_LOGN_SWITCH(c, CALL)       \
    switch ((c)->log_n) {                 \
        case 10: CALL(10); break;         \
        case 11: CALL(11); break;         \
        case 12: CALL(12); break;         \
        case 13: CALL(13); break;         \
        case 14: CALL(14); break;         \
        case 15: CALL(15); break;         \
        case 16: CALL(16); break;         \
        default: break;                   \
    }

// ------------------------------------------------------------------ kernels

// out[r][c] = src[c] mod prime(r)   (src: signed 32-bit coefficients)
__global__ void k_signed_to_res(const int32_t* __restrict__ src, uint64_t* __restrict__ out, RowSet rs,
                                const DevPrime* __restrict__ pr, int logn) {
    const int N = 1 << logn;
    int c = blockIdx.x * blockDim.x + threadIdx.x, r = blockIdx.y;
    if (c >= N) return;
    uint64_t q = pr[rs.prime(r)].q;
    int32_t v = src[c];
    uint64_t m = v >= 0 ? (uint64_t)v % q : q - ((uint64_t)(-(int64_t)v) % q);
    rs.ptr(r, N)[c] = m == q ? 0 : m;
}

// out[r][c] = in[r][automorph_src(c)]
__global__ void k_automorph_rows(const uint64_t* __restrict__ in, uint64_t* __restrict__ out, uint64_t galois,
                                 int logn) {
    const int N = 1 << logn;
    int c = blockIdx.x * blockDim.x + threadIdx.x, r = blockIdx.y;
    if (c >= N) return;
    out[(size_t)r * N + c] = in[(size_t)r * N + automorph_src(c, logn, galois)];
}

__global__ void k_mul_rows(const uint64_t* __restrict__ a, const uint64_t* __restrict__ b, uint64_t* __restrict__ o,
                           const DevPrime* __restrict__ pr, int logn) {
    const int N = 1 << logn;
    int c = blockIdx.x * blockDim.x + threadIdx.x, r = blockIdx.y;
    if (c >= N) return;
    DevPrime p = pr[r];
    size_t k = (size_t)r * N + c;
    o[k] = mul_mod(a[k], b[k], p);
}

// One digit of a switching key, rows = all L+K primes:
//   b = -a s + e + gmod(r) s'  (gmod = P mod q_r on the digit's rows, else 0)
// stored in the form the inner product consumes: rows of primes below 2^41
// as doubles (FP64 products), the others in Montgomery form (x 2^64 mod prime).
__device__ __forceinline__ uint64_t key_store_form(uint64_t v, const DevPrime& p) {
    return p.q < kFpPrimeLimit ? (uint64_t)__double_as_longlong((double)v) : mont_mul(v, p.r2, p);
}

__global__ void k_keygen_digit(const uint64_t* __restrict__ a, const uint64_t* __restrict__ s,
                               const uint64_t* __restrict__ e, const uint64_t* __restrict__ sp, RowConst g,
                               uint64_t* __restrict__ kb, uint64_t* __restrict__ ka, const DevPrime* __restrict__ pr,
                               int logn) {
    const int N = 1 << logn;
    int c = blockIdx.x * blockDim.x + threadIdx.x, r = blockIdx.y;
    if (c >= N) return;
    DevPrime p = pr[r];
    size_t k = (size_t)r * N + c;
    uint64_t av = a[k];
    uint64_t as = mul_mod(av, s[k], p);
    uint64_t b = sub_mod(e[k], as, p.q);
    if (g.v[r].x) b = add_mod(b, mul_shoup(sp[k], g.v[r].x, g.v[r].y, p.q), p.q);
    kb[k] = key_store_form(b, p);
    if (ka) ka[k] = key_store_form(av, p);
}

// canonical residues of a stored key
__global__ void k_key_canonical(const uint64_t* __restrict__ in, uint64_t* __restrict__ out, int rows_per_poly,
                                const DevPrime* __restrict__ pr, int logn) {
    const int N = 1 << logn;
    int c = blockIdx.x * blockDim.x + threadIdx.x, r = blockIdx.y;
    if (c >= N) return;
    DevPrime p = pr[r % rows_per_poly];
    size_t k = (size_t)r * N + c;
    out[k] = p.q < kFpPrimeLimit ? (uint64_t)__longlong_as_double((long long)in[k]) : mont_mul(in[k], 1, p);
}

// canonical residues of a key with seeded a-halves, out [digits][2][LK][N]:
// b from its stored rows, a regenerated from the stream starts after them
__global__ void k_key_canonical_seeded(const uint64_t* __restrict__ in, uint64_t* __restrict__ out, int LK, int nd,
                                       const DevPrime* __restrict__ pr, int logn) {
    const int N = 1 << logn;
    int c = blockIdx.x * blockDim.x + threadIdx.x, R = blockIdx.y;
    if (c >= N) return;
    const int r = R % LK, half = (R / LK) & 1, j = R / (2 * LK);
    const DevPrime p = pr[r];
    uint64_t v;
    if (half == 0) {
        const uint64_t w = in[((size_t)j * LK + r) * N + c];
        v = p.q < kFpPrimeLimit ? (uint64_t)__longlong_as_double((long long)w) : mont_mul(w, 1, p);
    } else {
        const uint64_t s0 = in[(size_t)nd * LK * N + (size_t)j * LK + r];
        v = seeded_a(s0, c, N, p.q, __clzll(p.q));
    }
    out[(size_t)R * N + c] = v;
}


// Rescale of x (the sum of up to kRsTerms ciphertexts x_j, each at its own
// level lin_j with its first lv limbs kept and optionally times an integer
// K_j) by q_l = q_{lv-1}, in the layout of the key switch's ModDown:
//   last   = INTT(x_{lv-1})                                  (coefficients)
//   lift_r = [last]_{q_r} - (last > q_l/2 ? q_l : 0)          (r < lv-1, centred)
//   out_r  = (x_r - NTT(lift_r)) q_l^-1 mod q_r  (+ addend_r) (+ K0 on c0)
// k_rescale_gather_last forms x_{lv-1}; the forward column pass of
// NTT(lift_r) computes the lift as it loads `last`, and the row pass forms
// x_r and ends with the combine, so neither the sum nor a lifted limb
// crosses HBM and the rescale takes two transform launches where the
// unfused form took a lift, two passes and a combine.  Residue for residue
// the same values.
constexpr int kRsTerms = 4;

struct RescaleIo {
    PtrList in[kRsTerms];  // term j: x_{j,i} at level lin[j]
    int lin[kRsTerms];
    int nterm;             // 1..kRsTerms
    int with_k;            // terms times their constants (else one term, as it is)
    MutPtrList out;        // [2][lv-1][N]
    PtrList add;           // addend_i at level lv-1, or unused
};
struct RescaleK {
    RowConst k[kRsTerms];
};

// limb r of polynomial poly of the sum of the terms of ciphertext i at position c
__device__ __forceinline__ uint64_t rs_term_sum(const RescaleIo& io, const RescaleK& kk, int i, int poly, int r,
                                                size_t c, int N, uint64_t q) {
    if (!io.with_k) return io.in[0].p[i][((size_t)poly * io.lin[0] + r) * N + c];
    uint64_t acc = 0;
    for (int j = 0; j < io.nterm; j++) {
        const uint64_t x = io.in[j].p[i][((size_t)poly * io.lin[j] + r) * N + c];
        acc = add_mod(acc, mul_shoup(x, kk.k[j].v[r].x, kk.k[j].v[r].y, q), q);
    }
    return acc;
}

// last[i][poly] = x_{lv-1} of ciphertext i (still in the evaluation domain)
__global__ void k_rescale_gather_last(const RescaleIo io, const RescaleK kk, uint64_t* __restrict__ last, int lv,
                                      const DevPrime* __restrict__ pr, int logn) {
    const int N = 1 << logn;
    int c = blockIdx.x * blockDim.x + threadIdx.x, poly = blockIdx.y, i = blockIdx.z;
    if (c >= N) return;
    const int r = lv - 1;
    last[((size_t)i * 2 + poly) * N + c] = rs_term_sum(io, kk, i, poly, r, c, N, pr[r].q);
}

// Column pass of NTT(lift_r), the lift taken as the limb loads: rows
// y = ip (lv-1) + r of tmp receive the pass's raw state.
template <int LOGN, typename T, typename TW, typename M>
__device__ __forceinline__ void rescale_cols_body(T* sm, const uint64_t* last, uint64_t* a, const TW* tw,
                                                  const M& m, uint64_t q, uint64_t one_shoup, uint64_t ql,
                                                  uint64_t qlmod) {
    using Cf = NttCfg<LOGN>;
    const int cc = threadIdx.x % Cf::TC, g = threadIdx.x / Cf::TC;
    constexpr int RS = Cf::R / 16;
    T x[16];
#pragma unroll
    for (int k = 0; k < 16; k++) {
        const uint64_t v = last[(size_t)(g + RS * k) * Cf::C + cc];
        uint64_t w = csub(v - __umul64hi(v, one_shoup) * q, q);  // v mod q_r
        if (v > (ql >> 1)) w = sub_mod(w, qlmod, q);             // v - q_l
        x[k] = to_elem(w, T());
    }
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

template <int LOGN>
__global__ void __launch_bounds__(NttCfg<LOGN>::COL_THREADS, NTT_COL_MIN_BLOCKS)
    k_rescale_cols_lift(const uint64_t* __restrict__ last, uint64_t* __restrict__ tmp, int lm1, uint64_t ql,
                        const uint64_t* __restrict__ qmod, const DevPrime* __restrict__ pr,
                        const ulonglong2* __restrict__ tw_all, const double* __restrict__ twd_all,
                        const FpMod* __restrict__ fpm) {
    using Cf = NttCfg<LOGN>;
    __shared__ uint64_t sm[Cf::R * Cf::TC];
    const int y = blockIdx.y, ip = y / lm1, r = y - ip * lm1;
    const uint64_t q = pr[r].q, os = pr[r].one_shoup, qm = qmod[r];
    const uint64_t* l = last + (size_t)ip * Cf::N + blockIdx.x * Cf::TC;
    uint64_t* a = tmp + (size_t)y * Cf::N + blockIdx.x * Cf::TC;
    if (q < kFpPrimeLimit)
        rescale_cols_body<LOGN>(reinterpret_cast<double*>(sm), l, a, twd_all + (size_t)r * Cf::N, fpm[r], q, os,
                                ql, qm);
    else
        rescale_cols_body<LOGN>(sm, l, a, tw_all + (size_t)r * Cf::N, q, q, os, ql, qm);
}

// Starts bringing the 128-byte line at p into L2 (a hint: nothing waits on it).
__device__ __forceinline__ void prefetch_l2(const void* p) { asm volatile("prefetch.global.L2 [%0];" ::"l"(p)); }

// Row pass of NTT(lift_r), then the combine.
template <int LOGN>
__global__ void __launch_bounds__(NttCfg<LOGN>::ROW_THREADS, NTT_MIN_BLOCKS)
    k_rescale_rows_combine(const uint64_t* __restrict__ tmp, const RescaleIo io, const RescaleK kk, int lm1,
                           const RowConst k0, int add_k0, int with_add, const ulonglong2* __restrict__ qinv,
                           const DevPrime* __restrict__ pr, const ulonglong2* __restrict__ tw_all,
                           const double* __restrict__ twd_all, const FpMod* __restrict__ fpm) {
    using Cf = NttCfg<LOGN>;
    __shared__ uint64_t sm[Cf::TR * Cf::ROW_PITCH];
    const int y = blockIdx.y, ip = y / lm1, t = y - ip * lm1, i = ip >> 1, poly = ip & 1;
    const uint64_t q = pr[t].q;
    const int r = blockIdx.x * Cf::TR + threadIdx.x / (Cf::C / 16);
    const int j0 = r * Cf::C + 16 * row_lane<LOGN>();
    const uint64_t* a = tmp + (size_t)y * Cf::N + (size_t)r * Cf::C;
    if (io.nterm == 1)  // read after the stages (several terms' lines would crowd L2)
        prefetch_l2(io.in[0].p[i] + ((size_t)poly * io.lin[0] + t) * Cf::N + j0);
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
    uint64_t* op = io.out.p[i] + ((size_t)poly * lm1 + t) * Cf::N + j0;
    const uint64_t* ap = with_add ? io.add.p[i] + ((size_t)poly * lm1 + t) * Cf::N + j0 : nullptr;
    const ulonglong2 w = qinv[t];
    const bool k0_here = add_k0 && poly == 0;
    const uint64_t kv = k0.v[t].x;
    if (io.with_k) {
        // v <- sum_j K_j x_j - v (mod q), term by term, each term's 16
        // words read in consecutive loads
#pragma unroll
        for (int e = 0; e < 16; e++) v[e] = v[e] ? q - v[e] : 0;
        for (int j = 0; j < io.nterm; j++) {
            const uint64_t* xj = io.in[j].p[i] + ((size_t)poly * io.lin[j] + t) * Cf::N + j0;
            const ulonglong2 kj = kk.k[j].v[t];
#pragma unroll
            for (int k = 0; k < 4; k++) {
                uint64_t e4[4];
                ldg256_ro(xj + 4 * k, e4[0], e4[1], e4[2], e4[3]);
#pragma unroll
                for (int e = 0; e < 4; e++) v[4 * k + e] = add_mod(v[4 * k + e], mul_shoup(e4[e], kj.x, kj.y, q), q);
            }
        }
    }
#pragma unroll
    for (int k = 0; k < 4; k++) {
        uint64_t z[4];
        if (io.with_k) {
#pragma unroll
            for (int e = 0; e < 4; e++) z[e] = mul_shoup(v[4 * k + e], w.x, w.y, q);
        } else {
            ldg256_ro(io.in[0].p[i] + ((size_t)poly * io.lin[0] + t) * Cf::N + j0 + 4 * k, z[0], z[1], z[2], z[3]);
#pragma unroll
            for (int e = 0; e < 4; e++) z[e] = mul_shoup(z[e] + q - v[4 * k + e], w.x, w.y, q);
        }
        if (ap) {  // the addend may be the output itself: a coherent load
            uint64_t s0, s1, s2, s3;
            ldg256(ap + 4 * k, s0, s1, s2, s3);
            z[0] = add_mod(s0, z[0], q);
            z[1] = add_mod(s1, z[1], q);
            z[2] = add_mod(s2, z[2], q);
            z[3] = add_mod(s3, z[3], q);
        }
        if (k0_here) {
#pragma unroll
            for (int e = 0; e < 4; e++) z[e] = add_mod(z[e], kv, q);
        }
        stg256(op + 4 * k, z[0], z[1], z[2], z[3]);
    }
}

// dst_i[k] = src_i[k], k < words (16-byte copies)
__global__ void k_copy_many(PtrList src, MutPtrList dst, size_t words2) {
    const int i = blockIdx.y;
    const ulonglong2* s = reinterpret_cast<const ulonglong2*>(src.p[i]);
    ulonglong2* d = reinterpret_cast<ulonglong2*>(dst.p[i]);
    for (size_t k = (size_t)blockIdx.x * blockDim.x + threadIdx.x; k < words2; k += (size_t)gridDim.x * blockDim.x)
        d[k] = s[k];
}




// Batched helpers over n <= kMaxBatch ciphertexts (grid z = ciphertext), two
// adjacent coefficients per thread (16-byte accesses; limbs start on
// 16-byte boundaries).
__device__ __forceinline__ ulonglong2 ld2(const uint64_t* p) { return *reinterpret_cast<const ulonglong2*>(p); }
__device__ __forceinline__ void st2(uint64_t* p, uint64_t a, uint64_t b) {
    *reinterpret_cast<ulonglong2*>(p) = make_ulonglong2(a, b);
}

// out_i[poly][r] = K_r in_i[poly][r] for r < lv, in_i at level lin >= lv
// (limbs lv..lin-1 dropped on the way).
__global__ void k_mul_const_many(PtrList in, MutPtrList out, RowConst kc, int lin, int lv,
                                 const DevPrime* __restrict__ pr, int logn) {
    const int N = 1 << logn;
    const int c = 2 * (blockIdx.x * blockDim.x + threadIdx.x), y = blockIdx.y, i = blockIdx.z;
    if (c >= N) return;
    const int poly = y / lv, r = y - poly * lv;
    const uint64_t q = pr[r].q;
    const ulonglong2 x = ld2(in.p[i] + ((size_t)poly * lin + r) * N + c);
    st2(out.p[i] + ((size_t)poly * lv + r) * N + c, mul_shoup(x.x, kc.v[r].x, kc.v[r].y, q),
        mul_shoup(x.y, kc.v[r].x, kc.v[r].y, q));
}

// out_i = in_i keeping limbs r < lv of both polynomials (out_i != in_i)
__global__ void k_drop_many(PtrList in, MutPtrList out, int lin, int lv, int logn) {
    const int N = 1 << logn;
    const int c = 2 * (blockIdx.x * blockDim.x + threadIdx.x), y = blockIdx.y, i = blockIdx.z;
    if (c >= N) return;
    const int poly = y / lv, r = y - poly * lv;
    const ulonglong2 x = ld2(in.p[i] + ((size_t)poly * lin + r) * N + c);
    st2(out.p[i] + ((size_t)poly * lv + r) * N + c, x.x, x.y);
}

// o_i = a_i + b_i (level lv)
__global__ void k_add_many(PtrList a, PtrList b, MutPtrList o, int lv, const DevPrime* __restrict__ pr, int logn) {
    const int N = 1 << logn;
    const int c = 2 * (blockIdx.x * blockDim.x + threadIdx.x), y = blockIdx.y, i = blockIdx.z;
    if (c >= N) return;
    const size_t k = (size_t)y * N + c;
    const uint64_t q = pr[y % lv].q;
    const ulonglong2 u = ld2(a.p[i] + k), v = ld2(b.p[i] + k);
    st2(o.p[i] + k, add_mod(u.x, v.x, q), add_mod(u.y, v.y, q));
}

// c0 of io_i gains the constant polynomial K (every evaluation equals K)
__global__ void k_add_const_many(MutPtrList io, RowConst kc, const DevPrime* __restrict__ pr, int logn) {
    const int N = 1 << logn;
    const int c = 2 * (blockIdx.x * blockDim.x + threadIdx.x), r = blockIdx.y, i = blockIdx.z;
    if (c >= N) return;
    uint64_t* a = io.p[i] + (size_t)r * N + c;
    const uint64_t q = pr[r].q, kv = kc.v[r].x;
    const ulonglong2 u = ld2(a);
    st2(a, add_mod(u.x, kv, q), add_mod(u.y, kv, q));
}

// d_i = (a0 b0, a0 b1 + a1 b0, a1 b1) of the pairs (a_i, b_i), [3][level][N]
// a_i and b_i hold level or more limbs per polynomial: their c1 starts at
// limb room_a / room_b (the first `level` limbs of each polynomial are read).
// Two adjacent coefficients per thread (16-byte accesses).  Limbs of primes
// below 2^41 take signed FP64 rounded-quotient products (four per
// coefficient, one canonicalisation per output); the others Montgomery
// products, corrected by R^2 R^-1 after the sum.
__global__ void k_tensor_many(PtrList pa, PtrList pb, MutPtrList pd, int level, int room_a, int room_b,
                              const DevPrime* __restrict__ pr, const FpMod* __restrict__ fpm, int logn) {
    const int N = 1 << logn;
    const int c = 2 * (blockIdx.x * blockDim.x + threadIdx.x), r = blockIdx.y, i = blockIdx.z;
    if (c >= N) return;
    const uint64_t* a = pa.p[i];
    const uint64_t* b = pb.p[i];
    uint64_t* d = pd.p[i];
    const DevPrime p = pr[r];
    const size_t k0 = (size_t)r * N + c;
    const ulonglong2 A0 = __ldg(reinterpret_cast<const ulonglong2*>(a + k0));
    const ulonglong2 A1 = __ldg(reinterpret_cast<const ulonglong2*>(a + (size_t)(room_a + r) * N + c));
    const ulonglong2 B0 = __ldg(reinterpret_cast<const ulonglong2*>(b + k0));
    const ulonglong2 B1 = __ldg(reinterpret_cast<const ulonglong2*>(b + (size_t)(room_b + r) * N + c));
    const uint64_t a0[2] = {A0.x, A0.y}, a1[2] = {A1.x, A1.y}, b0[2] = {B0.x, B0.y}, b1[2] = {B1.x, B1.y};
    uint64_t o0[2], o1[2], o2[2];
    if (p.q < kFpPrimeLimit) {
        const FpMod m = fpm[r];
#pragma unroll
        for (int e = 0; e < 2; e++) {
            const double x0 = u2d(a0[e]), x1 = u2d(a1[e]), y0 = u2d(b0[e]), y1 = u2d(b1[e]);
            o0[e] = d2u(fp_modmul(x0, y0, m));
            o1[e] = d2u(fp_canon(__dadd_rn(fp_mulmod_s(x0, y1, m), fp_mulmod_s(x1, y0, m)), m));
            o2[e] = d2u(fp_modmul(x1, y1, m));
        }
    } else {
#pragma unroll
        for (int e = 0; e < 2; e++) {
            const uint64_t m00 = mont_mul(a0[e], b0[e], p), m01 = mont_mul(a0[e], b1[e], p),
                           m10 = mont_mul(a1[e], b0[e], p), m11 = mont_mul(a1[e], b1[e], p);
            o0[e] = mont_mul(m00, p.r2, p);
            o1[e] = mont_mul(add_mod(m01, m10, p.q), p.r2, p);
            o2[e] = mont_mul(m11, p.r2, p);
        }
    }
    *reinterpret_cast<ulonglong2*>(d + k0) = make_ulonglong2(o0[0], o0[1]);
    *reinterpret_cast<ulonglong2*>(d + (size_t)(level + r) * N + c) = make_ulonglong2(o1[0], o1[1]);
    *reinterpret_cast<ulonglong2*>(d + (size_t)(2 * level + r) * N + c) = make_ulonglong2(o2[0], o2[1]);
}

// d (+)= sum_i (a_i0 b_i0, a_i0 b_i1 + a_i1 b_i0, a_i1 b_i1) over the m pairs
// (a_i, b_i), d = [3][level][N] (accumulate: d holds the sum of earlier
// pairs, canonical); a_i / b_i as in k_tensor_many.  Two coefficients per
// thread.  FP64 limbs sum signed rounded-quotient products (each |.| < 5q/8,
// at most 2 kMaxBatch of them per output: below 2^48) and reduce once; q_0
// sums Montgomery products and corrects once by R^2 R^-1.
__global__ void k_tensor_sum(PtrList pa, PtrList pb, int m, uint64_t* __restrict__ d, int accumulate, int level,
                             int room_a, int room_b, const DevPrime* __restrict__ pr, const FpMod* __restrict__ fpm,
                             int logn) {
    const int N = 1 << logn;
    const int c = 2 * (blockIdx.x * blockDim.x + threadIdx.x), r = blockIdx.y;
    if (c >= N) return;
    const DevPrime p = pr[r];
    const size_t k0 = (size_t)r * N + c, ka = (size_t)(room_a + r) * N + c, kb = (size_t)(room_b + r) * N + c;
    uint64_t* dp[3] = {d + k0, d + (size_t)(level + r) * N + c, d + (size_t)(2 * level + r) * N + c};
    uint64_t o[3][2];
    if (p.q < kFpPrimeLimit) {
        const FpMod fm = fpm[r];
        double s[3][2] = {{0.0, 0.0}, {0.0, 0.0}, {0.0, 0.0}};
        for (int i = 0; i < m; i++) {
            const ulonglong2 A0 = __ldg(reinterpret_cast<const ulonglong2*>(pa.p[i] + k0));
            const ulonglong2 A1 = __ldg(reinterpret_cast<const ulonglong2*>(pa.p[i] + ka));
            const ulonglong2 B0 = __ldg(reinterpret_cast<const ulonglong2*>(pb.p[i] + k0));
            const ulonglong2 B1 = __ldg(reinterpret_cast<const ulonglong2*>(pb.p[i] + kb));
            const double x0[2] = {u2d(A0.x), u2d(A0.y)}, x1[2] = {u2d(A1.x), u2d(A1.y)};
            const double y0[2] = {u2d(B0.x), u2d(B0.y)}, y1[2] = {u2d(B1.x), u2d(B1.y)};
#pragma unroll
            for (int e = 0; e < 2; e++) {
                s[0][e] = __dadd_rn(s[0][e], fp_mulmod_s(x0[e], y0[e], fm));
                s[1][e] = __dadd_rn(s[1][e], __dadd_rn(fp_mulmod_s(x0[e], y1[e], fm), fp_mulmod_s(x1[e], y0[e], fm)));
                s[2][e] = __dadd_rn(s[2][e], fp_mulmod_s(x1[e], y1[e], fm));
            }
        }
#pragma unroll
        for (int h = 0; h < 3; h++) {
            if (accumulate) {
                const ulonglong2 prev = *reinterpret_cast<const ulonglong2*>(dp[h]);
                s[h][0] = __dadd_rn(s[h][0], u2d(prev.x));
                s[h][1] = __dadd_rn(s[h][1], u2d(prev.y));
            }
            o[h][0] = d2u(fp_canon(s[h][0], fm));
            o[h][1] = d2u(fp_canon(s[h][1], fm));
        }
    } else {
        uint64_t s[3][2] = {{0, 0}, {0, 0}, {0, 0}};
        for (int i = 0; i < m; i++) {
            const ulonglong2 A0 = __ldg(reinterpret_cast<const ulonglong2*>(pa.p[i] + k0));
            const ulonglong2 A1 = __ldg(reinterpret_cast<const ulonglong2*>(pa.p[i] + ka));
            const ulonglong2 B0 = __ldg(reinterpret_cast<const ulonglong2*>(pb.p[i] + k0));
            const ulonglong2 B1 = __ldg(reinterpret_cast<const ulonglong2*>(pb.p[i] + kb));
            const uint64_t a0[2] = {A0.x, A0.y}, a1[2] = {A1.x, A1.y}, b0[2] = {B0.x, B0.y}, b1[2] = {B1.x, B1.y};
#pragma unroll
            for (int e = 0; e < 2; e++) {
                s[0][e] = add_mod(s[0][e], mont_mul(a0[e], b0[e], p), p.q);
                s[1][e] = add_mod(s[1][e], add_mod(mont_mul(a0[e], b1[e], p), mont_mul(a1[e], b0[e], p), p.q), p.q);
                s[2][e] = add_mod(s[2][e], mont_mul(a1[e], b1[e], p), p.q);
            }
        }
#pragma unroll
        for (int h = 0; h < 3; h++) {
            const ulonglong2 prev = accumulate ? *reinterpret_cast<const ulonglong2*>(dp[h]) : make_ulonglong2(0, 0);
            o[h][0] = add_mod(prev.x, mont_mul(s[h][0], p.r2, p), p.q);
            o[h][1] = add_mod(prev.y, mont_mul(s[h][1], p.r2, p), p.q);
        }
    }
#pragma unroll
    for (int h = 0; h < 3; h++) *reinterpret_cast<ulonglong2*>(dp[h]) = make_ulonglong2(o[h][0], o[h][1]);
}

// --------------------------------------------------------------- host side

static uint64_t h_shoup(uint64_t w, uint64_t q) { return (uint64_t)(((unsigned __int128)w << 64) / q); }

static uint64_t int_mod(int64_t K, uint64_t q) {
    if (K >= 0) return (uint64_t)K % q;
    uint64_t m = (uint64_t)(-(K + 1)) % q;  // -(K+1) >= 0 without overflow
    return (q - 1 - m) % q;                 // K = -(m'+1) => q - 1 - m' mod q
}

static int ct_ok(he_ctx* c, const he_ct* x, const char* what) {
    if (!x || !x->data) return set_err(c, HE_EINVAL, "%s: null ciphertext", what);
    if ((uintptr_t)x->data & 31) return set_err(c, HE_EINVAL, "%s: ciphertext not 32-byte aligned", what);
    if (x->level < 1 || x->level > c->L) return set_err(c, HE_ELEVEL, "%s: level %d out of range", what, x->level);
    if (!x->is_ntt) return set_err(c, HE_EDOMAIN, "%s: ciphertext not in the evaluation domain", what);
    return HE_OK;
}

// One term of a fused rescale: ciphertexts in[i] at level lin, their first
// lv limbs kept, times the row constants *kc (or as they are: kc null).
struct RsTerm {
    const std::vector<const uint64_t*>* in;
    int lin;
    const RowConst* kc;
};

// The rescale path above for n ciphertexts: out_i = rescale(sum_j (K_j)
// in_{j,i}) (+ addend_i) (+ K0 on c0), at most kRsTerms terms; several
// terms need their constants.  An out_i equal to one of its inputs (in
// place) goes through a staging buffer: c1's limbs move down, which would
// overwrite input another block has still to read.
static int rescale_fused(he_ctx* c, const RsTerm* terms, int nterm, int lv, const std::vector<uint64_t*>& out,
                         const std::vector<const uint64_t*>& addend, bool add_k0, int64_t K0) {
    const int N = c->N, n = (int)out.size(), lm1 = lv - 1;
    if (nterm < 1 || nterm > kRsTerms || (nterm > 1 && !terms[0].kc))
        return set_err(c, HE_EINVAL, "rescale: %d terms", nterm);
    for (int j = 0; j < nterm; j++) {
        if (lv < 2 || terms[j].lin < lv)
            return set_err(c, HE_ELEVEL, "rescale: level %d of %d has no prime to drop", lv, terms[j].lin);
        if ((int)terms[j].in->size() != n || (!terms[j].kc) != (!terms[0].kc))
            return set_err(c, HE_EINVAL, "rescale: term lists");
    }
    const bool with_add = !addend.empty();
    if (with_add && (int)addend.size() != n) return set_err(c, HE_EINVAL, "rescale: addend list length");
    RescaleK kk;
    RowConst k0;
    for (int j = 0; j < nterm; j++)
        if (terms[j].kc) kk.k[j] = *terms[j].kc;
    for (int r = 0; r < lm1; r++) k0.v[r] = make_ulonglong2(add_k0 ? int_mod(K0, c->primes[r]) : 0, 0);
    const bool with_k = terms[0].kc != nullptr;
    const int gx = (N + TB - 1) / TB;
    const uint64_t ql = c->primes[lv - 1];
    const double limbB = 8.0 * N;
    const NttShape sh = ntt_shape(c->log_n);
    for (int i0 = 0; i0 < n; i0 += kMaxBatch) {
        const int m = std::min(kMaxBatch, n - i0);
        // per ciphertext: last limbs [2][N], transform rows [2][lm1][N], staging of in-place outputs [2][lm1][N]
        const size_t per = (size_t)N * (2 + 4 * lm1);
        uint64_t* base;
        int rc = scratch_slot(c, 1, per * m, &base);
        if (rc) return rc;
        uint64_t* last = base;
        uint64_t* tmp = last + (size_t)2 * m * N;
        uint64_t* stage = tmp + (size_t)2 * m * lm1 * N;
        RescaleIo io;
        io.nterm = nterm;
        io.with_k = with_k ? 1 : 0;
        for (int j = 0; j < kRsTerms; j++) io.lin[j] = j < nterm ? terms[j].lin : 0;
        PtrList sback;
        MutPtrList dback;
        int n_back = 0, fp_rows_n = 0;
        for (int r = 0; r < lm1; r++) fp_rows_n += fp_prime(c, r);
        for (int i = 0; i < m; i++) {
            bool inplace = false;
            for (int j = 0; j < nterm; j++) {
                io.in[j].p[i] = (*terms[j].in)[i0 + i];
                inplace = inplace || out[i0 + i] == io.in[j].p[i];
            }
            io.add.p[i] = with_add ? addend[i0 + i] : nullptr;
            io.out.p[i] = inplace ? stage + (size_t)i * 2 * lm1 * N : out[i0 + i];
            if (inplace) {
                sback.p[n_back] = io.out.p[i];
                dback.p[n_back++] = out[i0 + i];
            }
        }
        prof_begin(c, HE_PROF_RESCALE);
        k_rescale_gather_last<<<dim3(gx, 2, m), TB, 0, c->stream>>>(io, kk, last, lv, c->d_prime, c->log_n);
        if ((rc = lc(c, "rescale_gather"))) return rc;
        prof_end(c, HE_PROF_RESCALE, (2.0 + 2.0 * nterm) * m * limbB, with_k ? 2.0 * nterm * m * N : 0);
        std::vector<int> pl(1, lv - 1);
        if ((rc = ntt_inv_set(c, rowset_contig(last, 1, N, pl), 2 * m))) return rc;
        const double rows = 2.0 * m * lm1, rows_fp = 2.0 * m * fp_rows_n;
        prof_begin(c, HE_PROF_NTT_FWD_COLS);
#define HE_RS_COLS(LN)                                                                                             \
    k_rescale_cols_lift<LN><<<dim3(NttCfg<LN>::COL_TILES, 2 * m * lm1), NttCfg<LN>::COL_THREADS, 0, c->stream>>>( \
        last, tmp, lm1, ql, c->d_rs_qmod + (size_t)lm1 * c->L, c->d_prime, c->d_tw_fwd, c->d_twd_fwd, c->d_fpmod)
        HE_NTT_LOGN_SWITCH(c, HE_RS_COLS)
#undef HE_RS_COLS
        if ((rc = lc(c, "rescale_cols"))) return rc;
        prof_end(c, HE_PROF_NTT_FWD_COLS, (rows + 2.0 * m) * limbB, 0.5 * N * rows * sh.s1, 0.5 * N * rows_fp * sh.s1);
        prof_begin(c, HE_PROF_RESCALE);
#define HE_RS_ROWS(LN)                                                                                              \
    k_rescale_rows_combine<LN><<<dim3(NttCfg<LN>::ROW_TILES, 2 * m * lm1), NttCfg<LN>::ROW_THREADS, 0, c->stream>>>( \
        tmp, io, kk, lm1, k0, add_k0 ? 1 : 0, with_add ? 1 : 0, c->d_rs_inv + (size_t)lm1 * c->L, c->d_prime,        \
        c->d_tw_fwd, c->d_twd_fwd, c->d_fpmod)
        HE_NTT_LOGN_SWITCH(c, HE_RS_ROWS)
#undef HE_RS_ROWS
        if ((rc = lc(c, "rescale_rows"))) return rc;
        prof_end(c, HE_PROF_RESCALE, ((with_add ? 3.0 : 2.0) + nterm) * rows * limbB,
                 0.5 * N * rows * sh.s2 + (with_k ? 1.0 + nterm : 1.0) * N * rows, 0.5 * N * rows_fp * sh.s2);
        if (n_back) {
            prof_begin(c, HE_PROF_RESCALE);
            k_copy_many<<<dim3(c->sm_count * 4, n_back), TB, 0, c->stream>>>(sback, dback, (size_t)lm1 * N);
            if ((rc = lc(c, "rescale_copy"))) return rc;
            prof_end(c, HE_PROF_RESCALE, 4.0 * n_back * lm1 * limbB);
        }
    }
    return HE_OK;
}

int rescale_many(he_ctx* c, const std::vector<const uint64_t*>& in, const std::vector<uint64_t*>& out, int level,
                 const std::vector<const uint64_t*>& addend) {
    const RsTerm t{&in, level, nullptr};
    return rescale_fused(c, &t, 1, level, out, addend, false, 0);
}

static RowConst row_const_shoup(const he_ctx* c, int level, int64_t K);

// HMult + relinearisation + rescale of n pairs at one level.
int hmrr_many(he_ctx* c, const std::vector<const uint64_t*>& a, const std::vector<const uint64_t*>& b,
              const std::vector<uint64_t*>& out, int level, int room_a, int room_b,
              const std::vector<const uint64_t*>& addend, const PreRescaleTerms* pre) {
    const int N = c->N, n = (int)a.size();
    const int n_pre = pre ? (int)pre->in.size() : 0;
    if (n_pre > kRsTerms - 1 || (pre && ((int)pre->lin.size() != n_pre || (int)pre->K.size() != n_pre)))
        return set_err(c, HE_EINVAL, "hmult: %d terms before the rescale", n_pre);
    for (int j = 0; j < n_pre; j++)
        if ((int)pre->in[j].size() != n || pre->lin[j] < level)
            return set_err(c, HE_EINVAL, "hmult: term %d before the rescale", j);
    if (pre && !addend.empty()) return set_err(c, HE_EINVAL, "hmult: an addend and terms before the rescale");
    if (!c->relin.d) return set_err(c, HE_ENOKEY, "hmult: no relinearisation key");
    if (level < 2) return set_err(c, HE_ELEVEL, "hmult: level %d cannot be rescaled", level);
    if (room_a == 0) room_a = level;
    if (room_b == 0) room_b = level;
    if (room_a < level || room_b < level) return set_err(c, HE_ELEVEL, "hmult: input room below level %d", level);
    const int gx2 = (N / 2 + TB - 1) / TB;
    int fp_l = 0;
    for (int r = 0; r < level; r++) fp_l += fp_prime(c, r);
    const size_t per = (size_t)5 * level * N;  // d0 d1 d2 | relinearised [2][level]
    const int chunk = 64;
    for (int i0 = 0; i0 < n; i0 += chunk) {
        int m = std::min(chunk, n - i0);
        uint64_t* base;
        int rc = scratch_slot(c, 2, per * m, &base);
        if (rc) return rc;
        KsIoList io;
        PtrList pa, pb;
        MutPtrList pd;
        for (int i = 0; i < m; i++) {
            pa.p[i] = a[i0 + i];
            pb.p[i] = b[i0 + i];
            pd.p[i] = base + per * i;
        }
        prof_begin(c, HE_PROF_ELEMENTWISE);
        k_tensor_many<<<dim3(gx2, level, m), TB, 0, c->stream>>>(pa, pb, pd, level, room_a, room_b, c->d_prime,
                                                                 c->d_fpmod, c->log_n);
        if ((rc = lc(c, "tensor"))) return rc;
        // 4 products per coefficient on FP64 limbs, 7 (with the corrections) on the others
        prof_end(c, HE_PROF_ELEMENTWISE, 7.0 * m * level * 8.0 * N, (7.0 * level - 3.0 * fp_l) * m * N,
                 4.0 * fp_l * m * N);
        for (int i = 0; i < m; i++) {
            uint64_t* d = base + per * i;
            io.galois.push_back(0);
            io.key.push_back(c->relin.d);
            io.d.push_back(d + (size_t)2 * level * N);
            io.out.push_back(d + (size_t)3 * level * N);
            io.add0.push_back(d);
            io.add1.push_back(d + (size_t)level * N);
        }
        if ((rc = key_switch_split(c, level, io))) return rc;
        std::vector<const uint64_t*> rin(io.out.begin(), io.out.end());
        std::vector<uint64_t*> rout(out.begin() + i0, out.begin() + i0 + m);
        if (pre) {
            // rescale(relinearised + sum_j K_j term_j) in one fused rescale,
            // the product taken with the constant 1
            std::vector<std::vector<const uint64_t*>> tin(n_pre);
            RowConst kc[kRsTerms];
            RsTerm t[kRsTerms];
            kc[0] = row_const_shoup(c, level, 1);
            t[0] = RsTerm{&rin, level, &kc[0]};
            for (int j = 0; j < n_pre; j++) {
                tin[j].assign(pre->in[j].begin() + i0, pre->in[j].begin() + i0 + m);
                kc[1 + j] = row_const_shoup(c, level, pre->K[j]);
                t[1 + j] = RsTerm{&tin[j], pre->lin[j], &kc[1 + j]};
            }
            if ((rc = rescale_fused(c, t, 1 + n_pre, level, rout, {}, pre->add_k0, pre->K0))) return rc;
            continue;
        }
        std::vector<const uint64_t*> radd;
        if (!addend.empty()) radd.assign(addend.begin() + i0, addend.begin() + i0 + m);
        if ((rc = rescale_many(c, rin, rout, level, radd))) return rc;
    }
    return HE_OK;
}

// out = rescale(relinearise(sum_i tensor(a_i, b_i))) of n pairs at one level
// (inputs as in hmrr_many; out apart from every input): the tensors summed
// in kMaxBatch-pair launches, then one key switch and one rescale.
int hmrr_sum(he_ctx* c, const std::vector<const uint64_t*>& a, const std::vector<const uint64_t*>& b, uint64_t* out,
             int level, int room_a, int room_b) {
    const int N = c->N, n = (int)a.size();
    if (n < 1 || (int)b.size() != n) return set_err(c, HE_EINVAL, "hmult sum: %d pairs", n);
    if (!c->relin.d) return set_err(c, HE_ENOKEY, "hmult: no relinearisation key");
    if (level < 2) return set_err(c, HE_ELEVEL, "hmult: level %d cannot be rescaled", level);
    if (room_a == 0) room_a = level;
    if (room_b == 0) room_b = level;
    if (room_a < level || room_b < level) return set_err(c, HE_ELEVEL, "hmult: input room below level %d", level);
    uint64_t* d;
    int rc = scratch_slot(c, 2, (size_t)5 * level * N, &d);  // d0 d1 d2 | relinearised [2][level]
    if (rc) return rc;
    int fp_l = 0;
    for (int r = 0; r < level; r++) fp_l += fp_prime(c, r);
    const int gx2 = (N / 2 + TB - 1) / TB;
    for (int i0 = 0; i0 < n; i0 += kMaxBatch) {
        const int m = std::min(kMaxBatch, n - i0);
        PtrList pa, pb;
        for (int i = 0; i < m; i++) {
            pa.p[i] = a[i0 + i];
            pb.p[i] = b[i0 + i];
        }
        prof_begin(c, HE_PROF_ELEMENTWISE);
        k_tensor_sum<<<dim3(gx2, level), TB, 0, c->stream>>>(pa, pb, m, d, i0 > 0 ? 1 : 0, level, room_a, room_b,
                                                             c->d_prime, c->d_fpmod, c->log_n);
        if ((rc = lc(c, "tensor_sum"))) return rc;
        prof_end(c, HE_PROF_ELEMENTWISE, (4.0 * m + (i0 > 0 ? 6.0 : 3.0)) * level * 8.0 * N,
                 4.0 * level * m * N + 3.0 * (level - fp_l) * N, 4.0 * fp_l * m * N);
    }
    KsIoList io;
    io.galois.push_back(0);
    io.key.push_back(c->relin.d);
    io.d.push_back(d + (size_t)2 * level * N);
    io.out.push_back(d + (size_t)3 * level * N);
    io.add0.push_back(d);
    io.add1.push_back(d + (size_t)level * N);
    if ((rc = key_switch_split(c, level, io))) return rc;
    return rescale_many(c, {d + (size_t)3 * level * N}, {out}, level);
}

// ---- batched helpers: n ciphertexts, kMaxBatch per launch

static RowConst row_const_shoup(const he_ctx* c, int level, int64_t K) {
    RowConst kc;
    for (int r = 0; r < level; r++) {
        uint64_t q = c->primes[r], v = int_mod(K, q);
        kc.v[r] = make_ulonglong2(v, h_shoup(v, q));
    }
    return kc;
}

// out_i = K in_i at level lv (in_i at level lin >= lv; out_i may equal in_i only when lin == lv)
int mul_const_many(he_ctx* c, const std::vector<const uint64_t*>& in, const std::vector<uint64_t*>& out, int lin,
                   int lv, int64_t K) {
    const RowConst kc = row_const_shoup(c, lv, K);
    const int n = (int)in.size(), gx2 = (c->N / 2 + TB - 1) / TB;
    for (int i0 = 0; i0 < n; i0 += kMaxBatch) {
        const int m = std::min(kMaxBatch, n - i0);
        PtrList pi;
        MutPtrList po;
        for (int i = 0; i < m; i++) {
            pi.p[i] = in[i0 + i];
            po.p[i] = out[i0 + i];
        }
        prof_begin(c, HE_PROF_ELEMENTWISE);
        k_mul_const_many<<<dim3(gx2, 2 * lv, m), TB, 0, c->stream>>>(pi, po, kc, lin, lv, c->d_prime, c->log_n);
        int rc = lc(c, "mul_const");
        if (rc) return rc;
        prof_end(c, HE_PROF_ELEMENTWISE, 4.0 * m * lv * 8.0 * c->N, 2.0 * m * lv * c->N);
    }
    return HE_OK;
}

// out_i = rescale(sum_j K_j in_{j,i}, each dropped to lv limbs) at level
// lv - 1, and, with add_k0, K0 added to c0 after that; in_{j,i} at level
// lin_j >= lv, out_i apart from every input; at most kRsTerms terms.  Equal,
// residue for residue, to mul_const_many of each term into a temporary,
// add_many of them, rescale_many of the sum and add_const_many (add_k0),
// without the intermediate ciphertexts in HBM.
int mul_const_sum_rescale_many(he_ctx* c, const std::vector<std::vector<const uint64_t*>>& in,
                               const std::vector<int>& lin, int lv, const std::vector<int64_t>& K,
                               const std::vector<uint64_t*>& out, bool add_k0, int64_t K0) {
    const int nterm = (int)in.size();
    if (nterm < 1 || nterm > kRsTerms || (int)lin.size() != nterm || (int)K.size() != nterm)
        return set_err(c, HE_EINVAL, "mul_const_sum_rescale: %d terms", nterm);
    RowConst kc[kRsTerms];
    RsTerm t[kRsTerms];
    for (int j = 0; j < nterm; j++) {
        kc[j] = row_const_shoup(c, lv, K[j]);
        t[j] = RsTerm{&in[j], lin[j], &kc[j]};
    }
    return rescale_fused(c, t, nterm, lv, out, {}, add_k0, K0);
}

// out_i = in_i keeping limbs < lv (out_i != in_i)
int drop_many(he_ctx* c, const std::vector<const uint64_t*>& in, const std::vector<uint64_t*>& out, int lin, int lv) {
    const int n = (int)in.size(), gx2 = (c->N / 2 + TB - 1) / TB;
    for (int i0 = 0; i0 < n; i0 += kMaxBatch) {
        const int m = std::min(kMaxBatch, n - i0);
        PtrList pi;
        MutPtrList po;
        for (int i = 0; i < m; i++) {
            pi.p[i] = in[i0 + i];
            po.p[i] = out[i0 + i];
        }
        prof_begin(c, HE_PROF_ELEMENTWISE);
        k_drop_many<<<dim3(gx2, 2 * lv, m), TB, 0, c->stream>>>(pi, po, lin, lv, c->log_n);
        int rc = lc(c, "drop");
        if (rc) return rc;
        prof_end(c, HE_PROF_ELEMENTWISE, 4.0 * m * lv * 8.0 * c->N);
    }
    return HE_OK;
}

// o_i = a_i + b_i at level lv (o_i may equal a_i or b_i)
int add_many(he_ctx* c, const std::vector<const uint64_t*>& a, const std::vector<const uint64_t*>& b,
             const std::vector<uint64_t*>& o, int lv) {
    const int n = (int)a.size(), gx2 = (c->N / 2 + TB - 1) / TB;
    for (int i0 = 0; i0 < n; i0 += kMaxBatch) {
        const int m = std::min(kMaxBatch, n - i0);
        PtrList pa, pb;
        MutPtrList po;
        for (int i = 0; i < m; i++) {
            pa.p[i] = a[i0 + i];
            pb.p[i] = b[i0 + i];
            po.p[i] = o[i0 + i];
        }
        prof_begin(c, HE_PROF_ELEMENTWISE);
        k_add_many<<<dim3(gx2, 2 * lv, m), TB, 0, c->stream>>>(pa, pb, po, lv, c->d_prime, c->log_n);
        int rc = lc(c, "add");
        if (rc) return rc;
        prof_end(c, HE_PROF_ELEMENTWISE, 6.0 * m * lv * 8.0 * c->N);
    }
    return HE_OK;
}

// io_i gains K/scale in every slot: K added to c0's constant polynomial
int add_const_many(he_ctx* c, const std::vector<uint64_t*>& io, int lv, int64_t K) {
    RowConst kc;
    for (int r = 0; r < lv; r++) kc.v[r] = make_ulonglong2(int_mod(K, c->primes[r]), 0);
    const int n = (int)io.size(), gx2 = (c->N / 2 + TB - 1) / TB;
    for (int i0 = 0; i0 < n; i0 += kMaxBatch) {
        const int m = std::min(kMaxBatch, n - i0);
        MutPtrList po;
        for (int i = 0; i < m; i++) po.p[i] = io[i0 + i];
        prof_begin(c, HE_PROF_ELEMENTWISE);
        k_add_const_many<<<dim3(gx2, lv, m), TB, 0, c->stream>>>(po, kc, c->d_prime, c->log_n);
        int rc = lc(c, "add_const");
        if (rc) return rc;
        prof_end(c, HE_PROF_ELEMENTWISE, 2.0 * m * lv * 8.0 * c->N);
    }
    return HE_OK;
}

int mul_const_raw(he_ctx* c, const uint64_t* in, uint64_t* out, int level, int64_t K) {
    return mul_const_many(c, {in}, {out}, level, level, K);
}

int add_const_raw(he_ctx* c, uint64_t* inout, int level, int64_t K) { return add_const_many(c, {inout}, level, K); }

int add_raw(he_ctx* c, const uint64_t* a, const uint64_t* b, uint64_t* out, int level) {
    return add_many(c, {a}, {b}, {out}, level);
}

// Keep limbs 0..new_level-1 of both polynomials: out = [2][new_level][N].
int drop_raw(he_ctx* c, const uint64_t* in, int level, uint64_t* out, int new_level) {
    const size_t N = c->N;
    if (out != in) return drop_many(c, {in}, {out}, level, new_level);
    if (new_level == level) return HE_OK;
    // in place: c1 rows move from offset level*N to new_level*N; ascending row
    // copies never overwrite a source row that is still to be read (the shift
    // is >= one row)
    for (int r = 0; r < new_level; r++) {
        int rc = check_cuda(c, cudaMemcpyAsync(out + (new_level + r) * N, in + (level + r) * N, N * 8,
                                               cudaMemcpyDeviceToDevice, c->stream), "drop");
        if (rc) return rc;
    }
    return HE_OK;
}

// fp64 bookkeeping of the polynomial evaluation.  The same expressions, in
// the same order, decide the integer constants.
static double round_half_away(double v) { return v >= 0 ? floor(v + 0.5) : ceil(v - 0.5); }

}  // namespace he

using namespace he;

// ------------------------------------------------------------------ keys

extern "C" int he_key_digits(const he_ctx* c) { return c ? (c->L + c->alpha - 1) / c->alpha : HE_EINVAL; }

namespace he {
bool keys_seeded_a(const he_ctx* c) {
    if (c->relin.d) return c->relin.seeded_a;
    return !c->rot_keys.empty() && c->rot_keys.begin()->second.seeded_a;
}
}  // namespace he

// Does the context hold keys of the other form than seeded_a?
static bool key_form_clash(const he_ctx* c, bool seeded_a) {
    if (c->relin.d && c->relin.seeded_a != seeded_a) return true;
    for (const auto& kv : c->rot_keys)
        if (kv.second.seeded_a != seeded_a) return true;
    return false;
}

// One switching key from host draws.  s0 (host [nd][LK], or null): the key
// keeps only its b-halves and these stream starts of its seeded a-halves.
static int keygen_one(he_ctx* c, int kind, int32_t step, const int8_t* s, const uint64_t* a, const int32_t* e,
                      const uint64_t* s0) {
    if (!c) return HE_EINVAL;
    if (!s || !a || !e || (kind != HE_KEY_ROTATION && kind != HE_KEY_RELIN))
        return set_err(c, HE_EINVAL, "he_keygen_upload: bad arguments");
    const int N = c->N, LK = c->L + c->K, nd = he_key_digits(c);
    const uint64_t galois = kind == HE_KEY_ROTATION ? galois_elt(c, step) : 0;
    if (kind == HE_KEY_ROTATION && galois == 1) return set_err(c, HE_EINVAL, "he_keygen_upload: identity rotation");
    if (key_form_clash(c, s0 != nullptr))
        return set_err(c, HE_EINVAL, "keygen: the context holds keys with %s a-halves", s0 ? "stored" : "seeded");
    for (int i = 0; i < N; i++)
        if (s[i] < -1 || s[i] > 1) return set_err(c, HE_EINVAL, "he_keygen_upload: secret not ternary");
    for (int j = 0; j < nd; j++)
        for (int r = 0; r < LK; r++)
            for (int i = 0; i < N; i += 4099)  // spot check: residues must be canonical
                if (a[((size_t)j * LK + r) * N + i] >= c->primes[r])
                    return set_err(c, HE_EINVAL, "he_keygen_upload: a not reduced");
    // work: s32 [N], e32 [nd][N], s_ntt [LK][N], sp [LK][N], e_ntt [LK][N], a [LK][N]
    size_t words = (size_t)N / 2 + (size_t)nd * N / 2 + 4 * (size_t)LK * N + 2;
    uint64_t* w;
    int rc = scratch_slot(c, 2, words, &w);
    if (rc) return rc;
    int32_t* s32 = (int32_t*)w;
    int32_t* e32 = s32 + N;
    uint64_t* s_ntt = w + (size_t)N / 2 + (size_t)nd * N / 2;  // 16-byte aligned (N >= 1024)
    uint64_t* sp = s_ntt + (size_t)LK * N;
    uint64_t* e_ntt = sp + (size_t)LK * N;
    uint64_t* a_d = e_ntt + (size_t)LK * N;
    std::vector<int32_t> s_h(s, s + N);
    rc = check_cuda(c, cudaMemcpyAsync(s32, s_h.data(), (size_t)N * 4, cudaMemcpyHostToDevice, c->stream), "keygen");
    if (!rc)
        rc = check_cuda(c, cudaMemcpyAsync(e32, e, (size_t)nd * N * 4, cudaMemcpyHostToDevice, c->stream), "keygen");
    if (rc) return rc;
    const int gx = (N + TB - 1) / TB;
    std::vector<int> all = prime_range(0, LK);
    RowSet rs_all = rowset_contig(s_ntt, LK, N, all);
    k_signed_to_res<<<dim3(gx, LK), TB, 0, c->stream>>>(s32, s_ntt, rs_all, c->d_prime, c->log_n);
    if ((rc = lc(c, "keygen s"))) return rc;
    if ((rc = ntt_fwd_set(c, rs_all, LK))) return rc;
    if (galois) {
        k_automorph_rows<<<dim3(gx, LK), TB, 0, c->stream>>>(s_ntt, sp, galois, c->log_n);
    } else {
        k_mul_rows<<<dim3(gx, LK), TB, 0, c->stream>>>(s_ntt, s_ntt, sp, c->d_prime, c->log_n);
    }
    if ((rc = lc(c, "keygen s'"))) return rc;
    Key key;
    key.seeded_a = s0 != nullptr;
    const int kw = key.seeded_a ? 1 : 2;  // stored halves per digit
    const size_t key_words = (size_t)nd * kw * LK * N + (key.seeded_a ? (size_t)nd * LK : 0);
    if ((rc = check_cuda(c, cudaMalloc(&key.d, key_words * 8), "key allocation"))) return rc;
    if (key.seeded_a &&
        (rc = check_cuda(c, cudaMemcpyAsync(key.d + (size_t)nd * LK * N, s0, (size_t)nd * LK * 8,
                                            cudaMemcpyHostToDevice, c->stream), "key stream starts"))) {
        cudaFree(key.d);
        return rc;
    }
    for (int j = 0; j < nd; j++) {
        RowSet rs_e = rowset_contig(e_ntt, LK, N, all);
        k_signed_to_res<<<dim3(gx, LK), TB, 0, c->stream>>>(e32 + (size_t)j * N, e_ntt, rs_e, c->d_prime, c->log_n);
        if ((rc = lc(c, "keygen e"))) break;
        if ((rc = ntt_fwd_set(c, rs_e, LK))) break;
        rc = check_cuda(c, cudaMemcpyAsync(a_d, a + (size_t)j * LK * N, (size_t)LK * N * 8, cudaMemcpyHostToDevice,
                                           c->stream), "keygen a");
        if (rc) break;
        RowConst g;
        for (int r = 0; r < LK; r++) {
            bool in_digit = r < c->L && r >= j * c->alpha && r < std::min((j + 1) * c->alpha, c->L);
            uint64_t v = in_digit ? c->h_Pmod[r] : 0;
            g.v[r] = make_ulonglong2(v, v ? h_shoup(v, c->primes[r]) : 0);
        }
        k_keygen_digit<<<dim3(gx, LK), TB, 0, c->stream>>>(
            a_d, s_ntt, e_ntt, sp, g, key.d + (size_t)(kw * j) * LK * N,
            key.seeded_a ? nullptr : key.d + (size_t)(kw * j + 1) * LK * N, c->d_prime, c->log_n);
        if ((rc = lc(c, "keygen digit"))) break;
        // the host arrays are read by the copies above: wait before reusing a_d
        if ((rc = check_cuda(c, cudaStreamSynchronize(c->stream), "keygen sync"))) break;
    }
    if (!rc) rc = check_cuda(c, cudaStreamSynchronize(c->stream), "keygen");
    if (rc) {
        cudaFree(key.d);
        return rc;
    }
    Key* slot = galois ? &c->rot_keys[galois] : &c->relin;
    if (slot->d) cudaFree(slot->d);
    *slot = key;
    return HE_OK;
}

extern "C" int he_keygen_upload(he_ctx* c, int kind, int32_t step, const int8_t* s, const uint64_t* a,
                                const int32_t* e) {
    return keygen_one(c, kind, step, s, a, e, nullptr);
}

extern "C" int he_keygen_seeded(he_ctx* c, uint64_t seed, const int32_t* rot_steps, int n_steps, int with_relin) {
    return he_keygen_seeded_ex(c, seed, rot_steps, n_steps, with_relin, 0);
}

extern "C" int he_keygen_seeded_ex(he_ctx* c, uint64_t seed, const int32_t* rot_steps, int n_steps, int with_relin,
                                   int flags) {
    if (!c) return HE_EINVAL;
    if (flags & ~HE_KEYGEN_SEEDED_A) return set_err(c, HE_EINVAL, "he_keygen_seeded: unknown flags %d", flags);
    const bool seeded_a = flags & HE_KEYGEN_SEEDED_A;
    if (n_steps < 0 || (n_steps > 0 && !rot_steps)) return set_err(c, HE_EINVAL, "he_keygen_seeded: bad step list");
    if (key_form_clash(c, seeded_a))
        return set_err(c, HE_EINVAL, "he_keygen_seeded: the context holds keys with %s a-halves",
                       seeded_a ? "stored" : "seeded");
    for (int i = 0; i < n_steps; i++)
        if (galois_elt(c, rot_steps[i]) == 1)
            return set_err(c, HE_EINVAL, "he_keygen_seeded: step %d is the identity rotation", rot_steps[i]);
    const int N = c->N, LK = c->L + c->K, nd = he_key_digits(c);
    std::vector<int8_t> s(N);
    std::vector<uint64_t> a((size_t)nd * LK * N);
    std::vector<int32_t> e((size_t)nd * N);
    int rc = he_sample_secret(seed, c->log_n, s.data());
    if (rc) return set_err(c, rc, "he_keygen_seeded: secret");
    std::vector<uint64_t> s0(seeded_a ? (size_t)nd * LK : 0);
    auto one = [&](int kind, int32_t step, uint64_t key_id) {
        int r = he_sample_key_draws(seed, key_id, c->log_n, c->primes.data(), LK, nd, a.data(), e.data());
        if (!r && seeded_a) r = he_sample_key_a_seeded(seed, key_id, c->log_n, c->primes.data(), LK, nd, a.data());
        if (r) return set_err(c, r, "he_keygen_seeded: key draws");
        if (seeded_a)
            for (int j = 0; j < nd; j++)
                for (int p = 0; p < LK; p++) s0[(size_t)j * LK + p] = seeded_a_stream_start(seed, key_id, j, p);
        return keygen_one(c, kind, step, s.data(), a.data(), e.data(), seeded_a ? s0.data() : nullptr);
    };
    for (int i = 0; i < n_steps; i++)
        if ((rc = one(HE_KEY_ROTATION, rot_steps[i], galois_elt(c, rot_steps[i])))) return rc;
    if (with_relin && (rc = one(HE_KEY_RELIN, 0, 2))) return rc;
    return HE_OK;
}

extern "C" int he_key_download(he_ctx* c, int kind, int32_t step, uint64_t* host_out) {
    if (!c) return HE_EINVAL;
    if (!host_out) return set_err(c, HE_EINVAL, "he_key_download: null output");
    const Key* k = nullptr;
    if (kind == HE_KEY_RELIN) {
        k = c->relin.d ? &c->relin : nullptr;
    } else if (kind == HE_KEY_ROTATION) {
        auto it = c->rot_keys.find(galois_elt(c, step));
        if (it != c->rot_keys.end()) k = &it->second;
    } else {
        return set_err(c, HE_EINVAL, "he_key_download: bad kind");
    }
    if (!k) return set_err(c, HE_ENOKEY, "he_key_download: no such key");
    const int N = c->N, LK = c->L + c->K, nd = he_key_digits(c);
    size_t words = (size_t)nd * 2 * LK * N;
    uint64_t* tmp;
    int rc = scratch_slot(c, 2, words, &tmp);
    if (rc) return rc;
    if (k->seeded_a)
        k_key_canonical_seeded<<<dim3((N + TB - 1) / TB, nd * 2 * LK), TB, 0, c->stream>>>(k->d, tmp, LK, nd,
                                                                                       c->d_prime, c->log_n);
    else
        k_key_canonical<<<dim3((N + TB - 1) / TB, nd * 2 * LK), TB, 0, c->stream>>>(k->d, tmp, LK, c->d_prime,
                                                                                c->log_n);
    if ((rc = lc(c, "key download"))) return rc;
    rc = check_cuda(c, cudaMemcpyAsync(host_out, tmp, words * 8, cudaMemcpyDeviceToHost, c->stream), "key D2H");
    if (rc) return rc;
    return he_sync(c);
}

// ---------------------------------------------------------- public operations

extern "C" int he_rescale(he_ctx* c, he_ct* x) {
    if (!c) return HE_EINVAL;
    int rc = ct_ok(c, x, "he_rescale");
    if (rc) return rc;
    if (x->level < 2) return set_err(c, HE_ELEVEL, "he_rescale: level 1 has no prime to drop");
    std::vector<const uint64_t*> in(1, x->data);
    std::vector<uint64_t*> out(1, x->data);
    rc = rescale_many(c, in, out, x->level);
    if (rc) return rc;
    x->scale = x->scale / (double)c->primes[x->level - 1];
    x->level -= 1;
    return HE_OK;
}

extern "C" int he_hmult_relin_rescale(he_ctx* c, const he_ct* a, const he_ct* b, he_ct* out) {
    if (!c) return HE_EINVAL;
    int rc;
    if ((rc = ct_ok(c, a, "hmult")) || (rc = ct_ok(c, b, "hmult"))) return rc;
    if (!out || !out->data || ((uintptr_t)out->data & 31)) return set_err(c, HE_EINVAL, "hmult: null or unaligned output");
    if (a->level != b->level) return set_err(c, HE_ELEVEL, "hmult: levels %d and %d differ", a->level, b->level);
    if (out->data == a->data || out->data == b->data) return set_err(c, HE_EINVAL, "hmult: output aliases an input");
    const int level = a->level;
    rc = hmrr_many(c, {a->data}, {b->data}, {out->data}, level);
    if (rc) return rc;
    out->level = level - 1;
    out->scale = (a->scale * b->scale) / (double)c->primes[level - 1];
    out->is_ntt = 1;
    return HE_OK;
}

extern "C" int he_add(he_ctx* c, const he_ct* a, const he_ct* b, he_ct* out) {
    if (!c) return HE_EINVAL;
    int rc;
    if ((rc = ct_ok(c, a, "he_add")) || (rc = ct_ok(c, b, "he_add"))) return rc;
    if (!out || !out->data) return set_err(c, HE_EINVAL, "he_add: null output");
    if (a->level != b->level) return set_err(c, HE_ELEVEL, "he_add: levels differ");
    rc = add_raw(c, a->data, b->data, out->data, a->level);
    if (rc) return rc;
    out->level = a->level;
    out->scale = a->scale;
    out->is_ntt = 1;
    return HE_OK;
}

extern "C" int he_mul_const(he_ctx* c, const he_ct* in, int64_t K, he_ct* out) {
    if (!c) return HE_EINVAL;
    int rc = ct_ok(c, in, "he_mul_const");
    if (rc) return rc;
    if (!out || !out->data) return set_err(c, HE_EINVAL, "he_mul_const: null output");
    rc = mul_const_raw(c, in->data, out->data, in->level, K);
    if (rc) return rc;
    out->level = in->level;
    out->scale = in->scale;
    out->is_ntt = 1;
    return HE_OK;
}

extern "C" int he_add_const(he_ctx* c, he_ct* x, int64_t K) {
    if (!c) return HE_EINVAL;
    int rc = ct_ok(c, x, "he_add_const");
    if (rc) return rc;
    return add_const_raw(c, x->data, x->level, K);
}

extern "C" int he_drop_level(he_ctx* c, const he_ct* in, int level, he_ct* out) {
    if (!c) return HE_EINVAL;
    int rc = ct_ok(c, in, "he_drop_level");
    if (rc) return rc;
    if (!out || !out->data) return set_err(c, HE_EINVAL, "he_drop_level: null output");
    if (level < 1 || level > in->level) return set_err(c, HE_ELEVEL, "he_drop_level: bad target level %d", level);
    rc = drop_raw(c, in->data, in->level, out->data, level);
    if (rc) return rc;
    out->level = level;
    out->scale = in->scale;
    out->is_ntt = 1;
    return HE_OK;
}

// --------------------------------------------------- Paterson-Stockmeyer

extern "C" int he_poly_eval_ps15(he_ctx* c, const he_ct* x, int n, const double* coeffs, double top_scale,
                                 he_ct* out) {
    if (!c) return HE_EINVAL;
    if (n < 0 || !coeffs || (n > 0 && (!x || !out))) return set_err(c, HE_EINVAL, "ps15: bad arguments");
    if (n == 0) return HE_OK;
    const int l0 = x[0].level, N = c->N;
    for (int i = 0; i < n; i++) {
        int rc = ct_ok(c, &x[i], "ps15");
        if (rc) return rc;
        if (x[i].level != l0) return set_err(c, HE_ELEVEL, "ps15: mixed levels");
        if (x[i].scale != x[0].scale) return set_err(c, HE_ELEVEL, "ps15: mixed scales");
        if (!out[i].data || ((uintptr_t)out[i].data & 31)) return set_err(c, HE_EINVAL, "ps15: null or unaligned output");
    }
    if (l0 < 7) return set_err(c, HE_ELEVEL, "ps15: needs level >= 7, got %d", l0);
    if (!c->relin.d) return set_err(c, HE_ENOKEY, "ps15: no relinearisation key");
    const size_t ctw = (size_t)2 * l0 * N;  // room of one ciphertext at the top level
    // per ciphertext: x2 x3 x4 acc
    const int nbuf = 4;
    uint64_t* pool = nullptr;
    int rc = scratch_slot(c, 3, ctw * nbuf * n, &pool);
    if (rc) return rc;
    auto buf = [&](int k, int i) { return pool + ctw * ((size_t)k * n + i); };
    auto bufs = [&](int k) {
        std::vector<uint64_t*> v(n);
        for (int i = 0; i < n; i++) v[i] = buf(k, i);
        return v;
    };
    auto cbufs = [&](int k) {
        std::vector<const uint64_t*> v(n);
        for (int i = 0; i < n; i++) v[i] = buf(k, i);
        return v;
    };
    enum { X2, X3, X4, ACC };
    std::vector<const uint64_t*> xd(n);
    for (int i = 0; i < n; i++) xd[i] = x[i].data;
    double sx = x[0].scale;
    // x2 = HMRR(x, x)
    if ((rc = hmrr_many(c, xd, xd, bufs(X2), l0))) goto done;
    {
        double s2 = (sx * sx) / (double)c->primes[l0 - 1];
        // x3 = HMRR(x2, drop(x, l0-1)): x read at level l0-1 in place
        if ((rc = hmrr_many(c, cbufs(X2), xd, bufs(X3), l0 - 1, l0 - 1, l0))) goto done;
        double s3 = (s2 * sx) / (double)c->primes[l0 - 2];
        // x4 = HMRR(x2, x2)
        if ((rc = hmrr_many(c, cbufs(X2), cbufs(X2), bufs(X4), l0 - 1))) goto done;
        double s4 = (s2 * s2) / (double)c->primes[l0 - 2];
        int pw_level[4] = {0, l0, l0 - 1, l0 - 2};
        double pw_scale[4] = {0, sx, s2, s3};

        // the terms of q_blk(x) at (lam, T): each x^j read at lam+1 limbs and
        // multiplied by its integer constant; the constant term K0
        auto q_terms = [&](int blk, int lam, double T) {
            PreRescaleTerms p;
            for (int j = 1; j <= 3; j++) {
                double cj = coeffs[4 * blk + j];
                double v = cj * T * (double)c->primes[lam] / pw_scale[j];
                p.K.push_back((int64_t)round_half_away(v));
                p.in.push_back(j == 1 ? xd : cbufs(j == 2 ? X2 : X3));
                p.lin.push_back(pw_level[j]);
            }
            p.add_k0 = true;
            p.K0 = (int64_t)round_half_away(coeffs[4 * blk] * T);
            return p;
        };
        int lev = l0 - 3;
        double T = top_scale;
        {
            // acc = q_3: the three terms summed and rescaled once, the
            // constant added (all in the launches of one rescale)
            const PreRescaleTerms p = q_terms(3, lev, T);
            if ((rc = mul_const_sum_rescale_many(c, p.in, p.lin, lev + 1, p.K, bufs(ACC), true, p.K0))) goto done;
        }
        std::vector<uint64_t*> od(n);
        for (int i = 0; i < n; i++) od[i] = out[i].data;
        // acc <- rescale(relin(acc (x) drop(x4)) + terms of q_blk) + K0: x4
        // read at the accumulator's level in place, the block's terms added
        // in the product's rescale, the last one written to the outputs
        for (int blk = 2; blk >= 0; blk--) {
            const int lev_in = lev;
            T = (T * s4) / (double)c->primes[lev - 1];
            lev -= 1;
            const PreRescaleTerms p = q_terms(blk, lev, T);
            if ((rc = hmrr_many(c, cbufs(ACC), cbufs(X4), blk == 0 ? od : bufs(ACC), lev_in, lev_in, l0 - 2, {}, &p)))
                goto done;
        }
        for (int i = 0; i < n; i++) {
            out[i].level = lev;
            out[i].scale = T;
            out[i].is_ntt = 1;
        }
    }
done:
    return rc;
}
