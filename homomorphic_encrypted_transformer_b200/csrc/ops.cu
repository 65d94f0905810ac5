// Key generation, tensor product, rescale, elementwise helpers,
// HMult+relinearise+rescale and the Paterson-Stockmeyer driver.
#include <math.h>

#include <algorithm>

#include "he_internal.h"
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
    ka[k] = key_store_form(av, p);
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

// d[i] = (a0 b0, a0 b1 + a1 b0, a1 b1), each [level][N]
__global__ void k_tensor(const uint64_t* __restrict__ a, const uint64_t* __restrict__ b, uint64_t* __restrict__ d,
                         int level, const DevPrime* __restrict__ pr, int logn) {
    const int N = 1 << logn;
    int c = blockIdx.x * blockDim.x + threadIdx.x, r = blockIdx.y;
    if (c >= N) return;
    DevPrime p = pr[r];
    size_t k0 = (size_t)r * N + c, k1 = (size_t)(level + r) * N + c;
    uint64_t a0 = a[k0], a1 = a[k1], b0 = b[k0], b1 = b[k1];
    // Montgomery products a0 b0 R^-1 etc.; the sum is taken before the final
    // correction by R^2 R^-1.
    uint64_t m00 = mont_mul(a0, b0, p), m01 = mont_mul(a0, b1, p), m10 = mont_mul(a1, b0, p),
             m11 = mont_mul(a1, b1, p);
    d[k0] = mont_mul(m00, p.r2, p);
    d[(size_t)(level + r) * N + c] = mont_mul(add_mod(m01, m10, p.q), p.r2, p);
    d[(size_t)(2 * level + r) * N + c] = mont_mul(m11, p.r2, p);
}

// Rescale, step 1: lift the (inverse-transformed) last limb x (coefficients
// mod q_l, l = level-1) to every q_i, i < l, as its centred representative.
__global__ void k_rescale_lift(const uint64_t* __restrict__ last, uint64_t* __restrict__ out, int lm1, uint64_t ql,
                               const uint64_t* __restrict__ qmod, const DevPrime* __restrict__ pr, int logn) {
    const int N = 1 << logn;
    int c = blockIdx.x * blockDim.x + threadIdx.x, r = blockIdx.y, poly = blockIdx.z;  // r < lm1
    if (c >= N) return;
    uint64_t x = last[(size_t)poly * N + c];
    DevPrime p = pr[r];
    uint64_t v = reduce64(x, p);
    if (x > (ql >> 1)) v = sub_mod(v, qmod[r], p.q);  // x - q_l
    out[((size_t)poly * lm1 + r) * N + c] = v;
}

// Rescale, step 2: out[poly][r] = (in[poly][r] - lift[poly][r]) q_l^-1
__global__ void k_rescale_combine(const uint64_t* __restrict__ in, const uint64_t* __restrict__ lift,
                                  uint64_t* __restrict__ out, int level, const ulonglong2* __restrict__ qinv,
                                  const DevPrime* __restrict__ pr, int logn) {
    const int N = 1 << logn;
    int c = blockIdx.x * blockDim.x + threadIdx.x, r = blockIdx.y, poly = blockIdx.z;
    if (c >= N) return;
    const int lm1 = level - 1;
    uint64_t q = pr[r].q;
    uint64_t x = in[((size_t)poly * level + r) * N + c];
    uint64_t y = lift[((size_t)poly * lm1 + r) * N + c];
    ulonglong2 w = qinv[r];
    out[((size_t)poly * lm1 + r) * N + c] = mul_shoup(x + q - y, w.x, w.y, q);
}

__global__ void k_add_ct(const uint64_t* __restrict__ a, const uint64_t* __restrict__ b, uint64_t* __restrict__ o,
                         int level, const DevPrime* __restrict__ pr, int logn) {
    const int N = 1 << logn;
    int c = blockIdx.x * blockDim.x + threadIdx.x, r = blockIdx.y;  // r < 2 level
    if (c >= N) return;
    uint64_t q = pr[r % level].q;
    size_t k = (size_t)r * N + c;
    o[k] = add_mod(a[k], b[k], q);
}

__global__ void k_mul_const(const uint64_t* __restrict__ a, uint64_t* __restrict__ o, RowConst kc, int level,
                            const DevPrime* __restrict__ pr, int logn) {
    const int N = 1 << logn;
    int c = blockIdx.x * blockDim.x + threadIdx.x, r = blockIdx.y;
    if (c >= N) return;
    int rr = r % level;
    uint64_t q = pr[rr].q;
    size_t k = (size_t)r * N + c;
    o[k] = mul_shoup(a[k], kc.v[rr].x, kc.v[rr].y, q);
}

__global__ void k_add_const(uint64_t* __restrict__ a, RowConst kc, const DevPrime* __restrict__ pr, int logn) {
    const int N = 1 << logn;
    int c = blockIdx.x * blockDim.x + threadIdx.x, r = blockIdx.y;  // rows of c0
    if (c >= N) return;
    size_t k = (size_t)r * N + c;
    a[k] = add_mod(a[k], kc.v[r].x, pr[r].q);
}

// --------------------------------------------------------------- host side

static uint64_t h_mulmod(uint64_t a, uint64_t b, uint64_t m) { return (uint64_t)((unsigned __int128)a * b % m); }
static uint64_t h_shoup(uint64_t w, uint64_t q) { return (uint64_t)(((unsigned __int128)w << 64) / q); }

static uint64_t int_mod(int64_t K, uint64_t q) {
    if (K >= 0) return (uint64_t)K % q;
    uint64_t m = (uint64_t)(-(K + 1)) % q;  // -(K+1) >= 0 without overflow
    return (q - 1 - m) % q;                 // K = -(m'+1) => q - 1 - m' mod q
}

int elementwise_setup(he_ctx* c) {
    (void)c;
    return HE_OK;
}

static int ct_ok(he_ctx* c, const he_ct* x, const char* what) {
    if (!x || !x->data) return set_err(c, HE_EINVAL, "%s: null ciphertext", what);
    if ((uintptr_t)x->data & 15) return set_err(c, HE_EINVAL, "%s: ciphertext not 16-byte aligned", what);
    if (x->level < 1 || x->level > c->L) return set_err(c, HE_ELEVEL, "%s: level %d out of range", what, x->level);
    if (!x->is_ntt) return set_err(c, HE_EDOMAIN, "%s: ciphertext not in the evaluation domain", what);
    return HE_OK;
}

int rescale_many(he_ctx* c, const std::vector<const uint64_t*>& in, const std::vector<uint64_t*>& out, int level) {
    const int N = c->N, n = (int)in.size(), lm1 = level - 1;
    if (level < 2) return set_err(c, HE_ELEVEL, "rescale: level %d has no prime to drop", level);
    uint64_t* base;
    // per ciphertext: last limbs [2][N], lifts [2][lm1][N], output [2][lm1][N]
    size_t per = (size_t)N * (2 + 4 * lm1);
    int rc = scratch_slot(c, 1, per * n, &base);
    if (rc) return rc;
    const int gx = (N + TB - 1) / TB;
    const uint64_t ql = c->primes[level - 1];
    for (int i = 0; i < n; i++) {
        uint64_t* last = base + per * i;
        uint64_t* lift = last + 2 * N;
        uint64_t* res = lift + (size_t)2 * lm1 * N;
        for (int poly = 0; poly < 2; poly++) {
            rc = check_cuda(c, cudaMemcpyAsync(last + (size_t)poly * N, in[i] + ((size_t)poly * level + lm1) * N,
                                               (size_t)N * 8, cudaMemcpyDeviceToDevice, c->stream), "rescale copy");
            if (rc) return rc;
        }
        std::vector<int> pl(1, level - 1);
        if ((rc = ntt_inv_set(c, rowset_contig(last, 1, N, pl), 2))) return rc;
        prof_begin(c, HE_PROF_RESCALE);
        k_rescale_lift<<<dim3(gx, lm1, 2), TB, 0, c->stream>>>(last, lift, lm1, ql, c->d_rs_qmod + (size_t)lm1 * c->L,
                                                               c->d_prime, c->log_n);
        if ((rc = lc(c, "rescale_lift"))) return rc;
        prof_end(c, HE_PROF_RESCALE);
        if ((rc = ntt_fwd_set(c, rowset_contig(lift, lm1, N, prime_range(0, lm1)), 2 * lm1))) return rc;
        uint64_t* dst = (out[i] == in[i]) ? res : out[i];
        prof_begin(c, HE_PROF_RESCALE);
        k_rescale_combine<<<dim3(gx, lm1, 2), TB, 0, c->stream>>>(in[i], lift, dst, level,
                                                                  c->d_rs_inv + (size_t)lm1 * c->L, c->d_prime,
                                                                  c->log_n);
        if ((rc = lc(c, "rescale_combine"))) return rc;
        prof_end(c, HE_PROF_RESCALE);
        if (dst != out[i]) {
            rc = check_cuda(c, cudaMemcpyAsync(out[i], dst, (size_t)2 * lm1 * N * 8, cudaMemcpyDeviceToDevice,
                                               c->stream), "rescale copy back");
            if (rc) return rc;
        }
    }
    return HE_OK;
}

// HMult + relinearisation + rescale of n pairs at one level.
int hmrr_many(he_ctx* c, const std::vector<const uint64_t*>& a, const std::vector<const uint64_t*>& b,
              const std::vector<uint64_t*>& out, int level) {
    const int N = c->N, n = (int)a.size();
    if (!c->relin.d) return set_err(c, HE_ENOKEY, "hmult: no relinearisation key");
    if (level < 2) return set_err(c, HE_ELEVEL, "hmult: level %d cannot be rescaled", level);
    const int gx = (N + TB - 1) / TB;
    const size_t per = (size_t)5 * level * N;  // d0 d1 d2 | relinearised [2][level]
    const int chunk = 64;
    for (int i0 = 0; i0 < n; i0 += chunk) {
        int m = std::min(chunk, n - i0);
        uint64_t* base;
        int rc = scratch_slot(c, 2, per * m, &base);
        if (rc) return rc;
        KsIoList io;
        for (int i = 0; i < m; i++) {
            uint64_t* d = base + per * i;
            prof_begin(c, HE_PROF_ELEMENTWISE);
            k_tensor<<<dim3(gx, level), TB, 0, c->stream>>>(a[i0 + i], b[i0 + i], d, level, c->d_prime, c->log_n);
            if ((rc = lc(c, "tensor"))) return rc;
            prof_end(c, HE_PROF_ELEMENTWISE);
            io.galois.push_back(0);
            io.key.push_back(c->relin.d);
            io.d.push_back(d + (size_t)2 * level * N);
            io.out.push_back(d + (size_t)3 * level * N);
            io.add0.push_back(d);
            io.add1.push_back(d + (size_t)level * N);
        }
        if ((rc = key_switch(c, level, io))) return rc;
        std::vector<const uint64_t*> rin(io.out.begin(), io.out.end());
        std::vector<uint64_t*> rout(out.begin() + i0, out.begin() + i0 + m);
        if ((rc = rescale_many(c, rin, rout, level))) return rc;
    }
    return HE_OK;
}

int mul_const_raw(he_ctx* c, const uint64_t* in, uint64_t* out, int level, int64_t K) {
    RowConst kc;
    for (int r = 0; r < level; r++) {
        uint64_t q = c->primes[r], v = int_mod(K, q);
        kc.v[r] = make_ulonglong2(v, h_shoup(v, q));
    }
    prof_begin(c, HE_PROF_ELEMENTWISE);
    k_mul_const<<<dim3((c->N + TB - 1) / TB, 2 * level), TB, 0, c->stream>>>(in, out, kc, level, c->d_prime,
                                                                             c->log_n);
    int rc = lc(c, "mul_const");
    prof_end(c, HE_PROF_ELEMENTWISE);
    return rc;
}

int add_const_raw(he_ctx* c, uint64_t* inout, int level, int64_t K) {
    RowConst kc;
    for (int r = 0; r < level; r++) kc.v[r] = make_ulonglong2(int_mod(K, c->primes[r]), 0);
    prof_begin(c, HE_PROF_ELEMENTWISE);
    k_add_const<<<dim3((c->N + TB - 1) / TB, level), TB, 0, c->stream>>>(inout, kc, c->d_prime, c->log_n);
    int rc = lc(c, "add_const");
    prof_end(c, HE_PROF_ELEMENTWISE);
    return rc;
}

int add_raw(he_ctx* c, const uint64_t* a, const uint64_t* b, uint64_t* out, int level) {
    prof_begin(c, HE_PROF_ELEMENTWISE);
    k_add_ct<<<dim3((c->N + TB - 1) / TB, 2 * level), TB, 0, c->stream>>>(a, b, out, level, c->d_prime, c->log_n);
    int rc = lc(c, "add");
    prof_end(c, HE_PROF_ELEMENTWISE);
    return rc;
}

// Keep limbs 0..new_level-1 of both polynomials: out = [2][new_level][N].
int drop_raw(he_ctx* c, const uint64_t* in, int level, uint64_t* out, int new_level) {
    const size_t N = c->N;
    int rc;
    if (out != in) {
        rc = check_cuda(c, cudaMemcpyAsync(out, in, new_level * N * 8, cudaMemcpyDeviceToDevice, c->stream), "drop");
        if (rc) return rc;
    }
    if (out != in || new_level != level) {
        // c1 rows move from offset level*N to new_level*N; ascending row copies never
        // overwrite a source row that is still to be read (the shift is >= one row).
        for (int r = 0; r < new_level; r++) {
            rc = check_cuda(c, cudaMemcpyAsync(out + (new_level + r) * N, in + (level + r) * N, N * 8,
                                               cudaMemcpyDeviceToDevice, c->stream), "drop");
            if (rc) return rc;
        }
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

extern "C" int he_keygen_upload(he_ctx* c, int kind, int32_t step, const int8_t* s, const uint64_t* a,
                                const int32_t* e) {
    if (!c) return HE_EINVAL;
    if (!s || !a || !e || (kind != HE_KEY_ROTATION && kind != HE_KEY_RELIN))
        return set_err(c, HE_EINVAL, "he_keygen_upload: bad arguments");
    const int N = c->N, LK = c->L + c->K, nd = he_key_digits(c);
    const uint64_t galois = kind == HE_KEY_ROTATION ? galois_elt(c, step) : 0;
    if (kind == HE_KEY_ROTATION && galois == 1) return set_err(c, HE_EINVAL, "he_keygen_upload: identity rotation");
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
    if ((rc = check_cuda(c, cudaMalloc(&key.d, (size_t)nd * 2 * LK * N * 8), "key allocation"))) return rc;
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
        k_keygen_digit<<<dim3(gx, LK), TB, 0, c->stream>>>(a_d, s_ntt, e_ntt, sp, g, key.d + (size_t)(2 * j) * LK * N,
                                                           key.d + (size_t)(2 * j + 1) * LK * N, c->d_prime,
                                                           c->log_n);
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
    if (!out || !out->data || ((uintptr_t)out->data & 15)) return set_err(c, HE_EINVAL, "hmult: null or unaligned output");
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
        if (!out[i].data) return set_err(c, HE_EINVAL, "ps15: null output");
    }
    if (l0 < 7) return set_err(c, HE_ELEVEL, "ps15: needs level >= 7, got %d", l0);
    if (!c->relin.d) return set_err(c, HE_ENOKEY, "ps15: no relinearisation key");
    const size_t ctw = (size_t)2 * l0 * N;  // room of one ciphertext at the top level
    // per ciphertext: x2 x3 x4 acc prod term qsum tmp
    const int nbuf = 8;
    uint64_t* pool = nullptr;
    int rc = scratch_slot(c, 3, ctw * nbuf * n, &pool);
    if (rc) return rc;
    auto buf = [&](int k, int i) { return pool + ctw * ((size_t)k * n + i); };
    enum { X2, X3, X4, ACC, PROD, TERM, QSUM, TMP };
    std::vector<const uint64_t*> vx(n), va(n), vb(n);
    std::vector<uint64_t*> vo(n);
    auto run_hmrr = [&](int level) { return hmrr_many(c, va, vb, vo, level); };
    double sx = x[0].scale;
    // x2 = HMRR(x, x)
    for (int i = 0; i < n; i++) {
        va[i] = x[i].data;
        vb[i] = x[i].data;
        vo[i] = buf(X2, i);
    }
    if ((rc = run_hmrr(l0))) goto done;
    {
        double s2 = (sx * sx) / (double)c->primes[l0 - 1];
        // x3 = HMRR(x2, drop(x, l0-1))
        for (int i = 0; i < n; i++) {
            if ((rc = drop_raw(c, x[i].data, l0, buf(TMP, i), l0 - 1))) goto done;
            va[i] = buf(X2, i);
            vb[i] = buf(TMP, i);
            vo[i] = buf(X3, i);
        }
        if ((rc = run_hmrr(l0 - 1))) goto done;
        double s3 = (s2 * sx) / (double)c->primes[l0 - 2];
        for (int i = 0; i < n; i++) {
            va[i] = buf(X2, i);
            vb[i] = buf(X2, i);
            vo[i] = buf(X4, i);
        }
        if ((rc = run_hmrr(l0 - 1))) goto done;
        double s4 = (s2 * s2) / (double)c->primes[l0 - 2];
        const uint64_t* pw_data[4] = {nullptr, nullptr, nullptr, nullptr};
        int pw_level[4] = {0, l0, l0 - 1, l0 - 2};
        double pw_scale[4] = {0, sx, s2, s3};

        // q_blk(x) at (lam, T) into dst buffers (level lam)
        auto build_q = [&](int blk, int lam, double T, int dst) -> int {
            int r;
            for (int j = 1; j <= 3; j++) {
                double cj = coeffs[4 * blk + j];
                double v = cj * T * (double)c->primes[lam] / pw_scale[j];
                int64_t K = (int64_t)round_half_away(v);
                for (int i = 0; i < n; i++) {
                    const uint64_t* src = j == 1 ? x[i].data : (j == 2 ? buf(X2, i) : buf(X3, i));
                    if ((r = drop_raw(c, src, pw_level[j], buf(TMP, i), lam + 1))) return r;
                    if ((r = mul_const_raw(c, buf(TMP, i), buf(TMP, i), lam + 1, K))) return r;
                }
                std::vector<const uint64_t*> rin(n);
                std::vector<uint64_t*> rout(n);
                for (int i = 0; i < n; i++) {
                    rin[i] = buf(TMP, i);
                    rout[i] = j == 1 ? buf(dst, i) : buf(TERM, i);
                }
                if ((r = rescale_many(c, rin, rout, lam + 1))) return r;
                if (j > 1)
                    for (int i = 0; i < n; i++)
                        if ((r = add_raw(c, buf(dst, i), buf(TERM, i), buf(dst, i), lam))) return r;
            }
            int64_t K0 = (int64_t)round_half_away(coeffs[4 * blk] * T);
            for (int i = 0; i < n; i++)
                if ((r = add_const_raw(c, buf(dst, i), lam, K0))) return r;
            return HE_OK;
        };
        (void)pw_data;
        int lev = l0 - 3;
        double T = top_scale;
        if ((rc = build_q(3, lev, T, ACC))) goto done;
        for (int blk = 2; blk >= 0; blk--) {
            for (int i = 0; i < n; i++) {
                if ((rc = drop_raw(c, buf(X4, i), l0 - 2, buf(TMP, i), lev))) goto done;
                va[i] = buf(ACC, i);
                vb[i] = buf(TMP, i);
                vo[i] = buf(PROD, i);
            }
            if ((rc = run_hmrr(lev))) goto done;
            T = (T * s4) / (double)c->primes[lev - 1];
            lev -= 1;
            if ((rc = build_q(blk, lev, T, QSUM))) goto done;
            for (int i = 0; i < n; i++)
                if ((rc = add_raw(c, buf(PROD, i), buf(QSUM, i), buf(ACC, i), lev))) goto done;
        }
        for (int i = 0; i < n; i++) {
            rc = check_cuda(c, cudaMemcpyAsync(out[i].data, buf(ACC, i), (size_t)2 * lev * N * 8,
                                               cudaMemcpyDeviceToDevice, c->stream), "ps15 out");
            if (rc) goto done;
            out[i].level = lev;
            out[i].scale = T;
            out[i].is_ntt = 1;
        }
    }
done:
    return rc;
}
