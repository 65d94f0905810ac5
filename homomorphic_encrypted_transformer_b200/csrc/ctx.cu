// Context creation: host-side number theory, RNS tables, device upload,
// error reporting, scratch and profiling.
#include <stdarg.h>
#include <stdio.h>

#include <algorithm>
#include <cstring>

#include "he_internal.h"
#include "ntt.cuh"

namespace he {

typedef unsigned __int128 u128;

// ---------------------------------------------------------------- host math

static uint64_t h_mulmod(uint64_t a, uint64_t b, uint64_t m) { return (uint64_t)((u128)a * b % m); }

static uint64_t h_powmod(uint64_t b, uint64_t e, uint64_t m) {
    uint64_t r = 1 % m;
    b %= m;
    while (e) {
        if (e & 1) r = h_mulmod(r, b, m);
        b = h_mulmod(b, b, m);
        e >>= 1;
    }
    return r;
}

static uint64_t h_inv(uint64_t a, uint64_t p) { return h_powmod(a, p - 2, p); }  // p prime

// Deterministic Miller-Rabin for 64-bit n (bases 2..37 suffice below 3.3e24).
static bool h_is_prime(uint64_t n) {
    static const uint64_t bases[] = {2, 3, 5, 7, 11, 13, 17, 19, 23, 29, 31, 37};
    if (n < 2) return false;
    for (uint64_t p : bases)
        if (n % p == 0) return n == p;
    uint64_t d = n - 1;
    int s = 0;
    while ((d & 1) == 0) {
        d >>= 1;
        s++;
    }
    for (uint64_t a : bases) {
        uint64_t x = h_powmod(a, d, n);
        if (x == 1 || x == n - 1) continue;
        bool comp = true;
        for (int r = 1; r < s; r++) {
            x = h_mulmod(x, x, n);
            if (x == n - 1) {
                comp = false;
                break;
            }
        }
        if (comp) return false;
    }
    return true;
}

// Downward scan of primes = 1 mod two_n below 2^bits.
struct PrimeScan {
    uint64_t two_n, k;
    PrimeScan(int bits, uint64_t tn) : two_n(tn), k((((u128)1 << bits) - 2) / tn) {}
    uint64_t next() {
        while (k > 0) {
            uint64_t q = k * two_n + 1;
            k--;
            if (h_is_prime(q)) return q;
        }
        return 0;
    }
};

// Smallest primitive `order`-th root of unity mod q (order a power of two).
static uint64_t h_min_primitive_root(uint64_t q, uint64_t order) {
    uint64_t half = order / 2, x = 0;
    for (uint64_t g = 2;; g++) {
        x = h_powmod(g, (q - 1) / order, q);
        if (h_powmod(x, half, q) == q - 1) break;
    }
    uint64_t x2 = h_mulmod(x, x, q), best = x, cur = x;
    for (uint64_t i = 1; i < half; i++) {
        cur = h_mulmod(cur, x2, q);
        if (cur < best) best = cur;
    }
    return best;
}

static uint64_t h_shoup(uint64_t w, uint64_t q) { return (uint64_t)(((u128)w << 64) / q); }

static unsigned h_brev(unsigned x, int bits) {
    unsigned r = 0;
    for (int b = 0; b < bits; b++) r |= ((x >> b) & 1u) << (bits - 1 - b);
    return r;
}

static DevPrime h_prime_consts(uint64_t q, int N) {
    DevPrime d;
    d.q = q;
    uint64_t inv = 1;  // Newton iteration for q^-1 mod 2^64 (q odd)
    for (int i = 0; i < 7; i++) inv *= 2 - q * inv;
    d.qinv_neg = (uint64_t)0 - inv;
    uint64_t r1 = (uint64_t)(((u128)1 << 64) % q);
    d.r1 = r1;
    d.r1_shoup = h_shoup(r1, q);
    d.r2 = h_mulmod(r1, r1, q);
    d.one_shoup = (uint64_t)(((u128)1 << 64) / q);
    d.n_inv = h_inv((uint64_t)N % q, q);
    d.n_inv_shoup = h_shoup(d.n_inv, q);
    return d;
}

// ------------------------------------------------------------ infrastructure

int set_err(he_ctx* c, int code, const char* fmt, ...) {
    if (c) {
        char buf[512];
        va_list ap;
        va_start(ap, fmt);
        vsnprintf(buf, sizeof buf, fmt, ap);
        va_end(ap);
        c->err = buf;
    }
    return code;
}

int check_cuda(he_ctx* c, cudaError_t e, const char* what) {
    if (e == cudaSuccess) return HE_OK;
    if (e == cudaErrorMemoryAllocation) {
        cudaGetLastError();
        return set_err(c, HE_ENOMEM, "%s: %s", what, cudaGetErrorString(e));
    }
    return set_err(c, HE_ECUDA, "%s: %s", what, cudaGetErrorString(e));
}

static bool alloc_forced_to_fail() {
    const char* v = getenv("HE_FAIL_ALLOC");
    return v && v[0] == '1';
}

template <typename T>
static int dev_alloc(he_ctx* c, T** p, size_t count, const char* what) {
    if (alloc_forced_to_fail()) return set_err(c, HE_ENOMEM, "%s: allocation refused (HE_FAIL_ALLOC=1)", what);
    return check_cuda(c, cudaMalloc((void**)p, count * sizeof(T)), what);
}

template <typename T>
static int upload(he_ctx* c, T** p, const std::vector<T>& h, const char* what) {
    int rc = dev_alloc(c, p, h.size(), what);
    if (rc) return rc;
    return check_cuda(c, cudaMemcpy(*p, h.data(), h.size() * sizeof(T), cudaMemcpyHostToDevice), what);
}

int scratch_slot(he_ctx* c, int slot, size_t words, uint64_t** out) {
    if (words > c->scratch_words[slot]) {
        // growing synchronises and allocates, which a stream capture cannot hold
        cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
        if (cudaStreamIsCapturing(c->stream, &cs) == cudaSuccess && cs != cudaStreamCaptureStatusNone)
            return set_err(c, HE_EINVAL,
                           "scratch slot %d must grow to %zu words during a stream capture: run the call once "
                           "before capturing it",
                           slot, words);
        if (c->scratch[slot]) {
            cudaStreamSynchronize(c->stream);
            cudaFree(c->scratch[slot]);
            c->scratch[slot] = nullptr;
            c->scratch_words[slot] = 0;
        }
        int rc = dev_alloc(c, &c->scratch[slot], words, "scratch");
        if (rc) return rc;
        c->scratch_words[slot] = words;
    }
    *out = c->scratch[slot];
    return HE_OK;
}

static cudaEvent_t ev_get(he_ctx* c) {
    if (!c->ev_pool.empty()) {
        cudaEvent_t e = c->ev_pool.back();
        c->ev_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
}

// Brackets one launch (or a short sequence of launches of one class) with
// events on the context's stream.  Nothing waits here; he_profile_read()
// collects the elapsed times.
void prof_begin(he_ctx* c, int cls) {
    if (!c->prof_on) return;
    ProfPending p;
    p.cls = cls;
    p.a = ev_get(c);
    p.b = nullptr;
    p.bytes = p.mults = p.mults_fp = 0;
    cudaEventRecord(p.a, c->stream);
    c->prof_pending.push_back(p);
}

int prof_end(he_ctx* c, int cls, double bytes, double mults, double mults_fp) {
    if (!c->prof_on || c->prof_pending.empty()) return HE_OK;
    ProfPending& p = c->prof_pending.back();
    if (p.cls != cls || p.b) return HE_OK;
    p.bytes = bytes;
    p.mults = mults;
    p.mults_fp = mults_fp;
    p.b = ev_get(c);
    cudaEventRecord(p.b, c->stream);
    return HE_OK;
}

static int prof_collect(he_ctx* c) {
    int rc = check_cuda(c, cudaStreamSynchronize(c->stream), "profile sync");
    if (rc) return rc;
    for (auto& p : c->prof_pending) {
        if (p.b) {
            float ms = 0;
            cudaEventElapsedTime(&ms, p.a, p.b);
            c->prof[p.cls].ms += ms;
            c->prof[p.cls].launches += 1;
            c->prof[p.cls].bytes += p.bytes;
            c->prof[p.cls].mults += p.mults;
            c->prof[p.cls].mults_fp += p.mults_fp;
            c->ev_pool.push_back(p.b);
        }
        c->ev_pool.push_back(p.a);
    }
    c->prof_pending.clear();
    return HE_OK;
}

bool fp_prime(const he_ctx* c, int prime_idx) { return c->primes[prime_idx] < kFpPrimeLimit; }

long long fp_rows(const he_ctx* c, const RowSet& rs, int n_rows) {
    long long per = 0, tail = 0;
    const int rem = n_rows % rs.per_group;
    for (int r = 0; r < rs.per_group; r++) {
        int f = fp_prime(c, rs.prime(r));
        per += f;
        if (r < rem) tail += f;
    }
    return (long long)(n_rows / rs.per_group) * per + tail;
}

uint64_t galois_elt(const he_ctx* c, int32_t step) {
    uint64_t n = (uint64_t)c->N / 2;
    int64_t r = ((int64_t)step % (int64_t)n + (int64_t)n) % (int64_t)n;
    return h_powmod(5, (uint64_t)r, 2 * (uint64_t)c->N);
}

RowSet rowset(uint64_t* base, long long group_stride, int per_group, const int* prime_idx) {
    RowSet r;
    r.base = base;
    r.group_stride = group_stride;
    r.per_group = per_group;
    // split the list into runs of consecutive primes (at most three are used)
    int first[3] = {0, 0, 0}, len[3] = {0, 0, 0}, runs = 0;
    for (int i = 0; i < per_group; i++) {
        if (runs > 0 && prime_idx[i] == first[runs - 1] + len[runs - 1]) {
            len[runs - 1]++;
        } else {
            if (runs == 3) abort();  // every caller passes at most three runs
            first[runs] = prime_idx[i];
            len[runs] = 1;
            runs++;
        }
    }
    r.first0 = first[0];
    r.len0 = len[0];
    r.first1 = first[1];
    r.len1 = len[1];
    r.first2 = first[2];
    return r;
}

std::vector<int> prime_range(int first, int count) {
    std::vector<int> v(count);
    for (int i = 0; i < count; i++) v[i] = first + i;
    return v;
}

std::vector<int> ext_primes(const he_ctx* c, int level) {
    std::vector<int> v;
    for (int i = 0; i < level; i++) v.push_back(i);
    for (int k = 0; k < c->K; k++) v.push_back(c->L + k);
    return v;
}

// Contiguous groups of per_group limbs of N words.
RowSet rowset_contig(uint64_t* base, int per_group, int N, const std::vector<int>& prime_idx) {
    return rowset(base, (long long)per_group * N, per_group, prime_idx.data());
}

// ------------------------------------------------------------------- tables

static int build_tables(he_ctx* c) {
    const int N = c->N, LK = c->L + c->K, L = c->L, K = c->K;
    c->hprime.resize(LK);
    std::vector<ulonglong2> tf((size_t)LK * N), ti((size_t)LK * N), il(LK);
    std::vector<double> tfd((size_t)LK * N), tid((size_t)LK * N);
    std::vector<FpMod> fpm(LK);
    std::vector<uint64_t> pw(N), pwi(N);
    for (int r = 0; r < LK; r++) {
        uint64_t q = c->primes[r], psi = c->psi[r], psi_i = h_inv(psi, q);
        c->hprime[r] = h_prime_consts(q, N);
        pw[0] = 1;
        pwi[0] = 1;
        for (int i = 1; i < N; i++) {
            pw[i] = h_mulmod(pw[i - 1], psi, q);
            pwi[i] = h_mulmod(pwi[i - 1], psi_i, q);
        }
        for (int k = 0; k < N; k++) {
            uint64_t w = pw[h_brev(k, c->log_n)], wi = pwi[h_brev(k, c->log_n)];
            if (k == 1) wi = h_mulmod(wi, c->hprime[r].n_inv, q);
            tf[(size_t)r * N + k] = make_ulonglong2(w, h_shoup(w, q));
            ti[(size_t)r * N + k] = make_ulonglong2(wi, h_shoup(wi, q));
            tfd[(size_t)r * N + k] = (double)w;  // exact for the primes the FP64 path serves
            tid[(size_t)r * N + k] = (double)wi;
        }
        il[r] = make_ulonglong2(c->hprime[r].n_inv, c->hprime[r].n_inv_shoup);
        fpm[r] = FpMod{(double)q, 2.0 * (double)q, 1.0 / (double)q, (double)c->hprime[r].n_inv};
    }
    int rc;
    if ((rc = upload(c, &c->d_prime, c->hprime, "prime table"))) return rc;
    if ((rc = upload(c, &c->d_tw_fwd, tf, "forward twiddles"))) return rc;
    if ((rc = upload(c, &c->d_tw_inv, ti, "inverse twiddles"))) return rc;
    if ((rc = upload(c, &c->d_inv_last, il, "N^-1 table"))) return rc;
    if ((rc = upload(c, &c->d_twd_fwd, tfd, "forward twiddles (fp64)"))) return rc;
    if ((rc = upload(c, &c->d_twd_inv, tid, "inverse twiddles (fp64)"))) return rc;
    if ((rc = upload(c, &c->d_fpmod, fpm, "fp64 prime constants"))) return rc;

    // ModUp conversion tables for every level and digit.
    c->modup.assign(L + 1, {});
    std::vector<ulonglong2> blob;
    std::vector<std::pair<size_t, size_t>> offs;  // per (level, digit): src offset, mat offset
    for (int lev = 1; lev <= L; lev++) {
        int nd = (lev + c->alpha - 1) / c->alpha;
        std::vector<int> rows = ext_primes(c, lev);
        for (int j = 0; j < nd; j++) {
            int s0 = j * c->alpha, s1 = std::min((j + 1) * c->alpha, lev);
            ConvTable t;
            t.n_src = s1 - s0;
            t.src_row = s0;
            size_t so = blob.size();
            for (int i = s0; i < s1; i++) {
                uint64_t qi = c->primes[i], prod = 1;
                for (int i2 = s0; i2 < s1; i2++)
                    if (i2 != i) prod = h_mulmod(prod, c->primes[i2] % qi, qi);
                uint64_t inv = h_inv(prod, qi);
                blob.push_back(make_ulonglong2(inv, h_shoup(inv, qi)));
            }
            size_t mo = blob.size();
            for (int i = s0; i < s1; i++) {
                for (int r : rows) {
                    uint64_t t_ = c->primes[r], prod = 1;
                    for (int i2 = s0; i2 < s1; i2++)
                        if (i2 != i) prod = h_mulmod(prod, c->primes[i2] % t_, t_);
                    // Montgomery form (x 2^64 mod t): the conversion reduces its
                    // 128-bit sum with one REDC, which divides by 2^64 again
                    uint64_t mont = h_mulmod(prod, (uint64_t)(((u128)1 << 64) % t_), t_);
                    blob.push_back(make_ulonglong2(mont, prod));
                }
            }
            offs.push_back({so, mo});
            c->modup[lev].push_back(t);
        }
    }
    ulonglong2* d_blob = nullptr;
    if ((rc = upload(c, &d_blob, blob, "modup tables"))) return rc;
    size_t k = 0;
    for (int lev = 1; lev <= L; lev++)
        for (auto& t : c->modup[lev]) {
            t.d_src = d_blob + offs[k].first;
            t.d_mat = d_blob + offs[k].second;
            k++;
        }

    // ModDown: centred conversion from P onto every q_i.
    std::vector<ulonglong2> pcoef(K), mat((size_t)K * L), pinv(L);
    std::vector<uint64_t> negP(L);
    c->h_Pmod.assign(L + K, 0);
    for (int kk = 0; kk < K; kk++) {
        uint64_t pk = c->primes[L + kk], prod = 1;
        for (int k2 = 0; k2 < K; k2++)
            if (k2 != kk) prod = h_mulmod(prod, c->primes[L + k2] % pk, pk);
        uint64_t inv = h_inv(prod, pk);
        pcoef[kk] = make_ulonglong2(inv, h_shoup(inv, pk));
        for (int i = 0; i < L; i++) {
            uint64_t qi = c->primes[i], pr = 1;
            for (int k2 = 0; k2 < K; k2++)
                if (k2 != kk) pr = h_mulmod(pr, c->primes[L + k2] % qi, qi);
            uint64_t mont = h_mulmod(pr, (uint64_t)(((u128)1 << 64) % qi), qi);  // Montgomery form
            mat[(size_t)kk * L + i] = make_ulonglong2(mont, pr);
        }
    }
    for (int i = 0; i < L; i++) {
        uint64_t qi = c->primes[i], P = 1;
        for (int kk = 0; kk < K; kk++) P = h_mulmod(P, c->primes[L + kk] % qi, qi);
        c->h_Pmod[i] = P;
        negP[i] = P ? qi - P : 0;
        uint64_t inv = h_inv(P, qi);
        pinv[i] = make_ulonglong2(inv, h_shoup(inv, qi));
    }
    if ((rc = upload(c, &c->d_md_pcoef, pcoef, "moddown coef"))) return rc;
    if ((rc = upload(c, &c->d_md_mat, mat, "moddown matrix"))) return rc;
    if ((rc = upload(c, &c->d_md_negP, negP, "moddown negP"))) return rc;
    if ((rc = upload(c, &c->d_md_pinv, pinv, "moddown pinv"))) return rc;

    // Rescale: dropping prime l onto q_i, i < l.
    std::vector<ulonglong2> rsi((size_t)L * L, make_ulonglong2(0, 0));
    std::vector<uint64_t> rsq((size_t)L * L, 0);
    for (int l = 1; l < L; l++)
        for (int i = 0; i < l; i++) {
            uint64_t qi = c->primes[i], ql = c->primes[l] % qi;
            uint64_t inv = h_inv(ql, qi);
            rsi[(size_t)l * L + i] = make_ulonglong2(inv, h_shoup(inv, qi));
            rsq[(size_t)l * L + i] = ql;
        }
    if ((rc = upload(c, &c->d_rs_inv, rsi, "rescale inv"))) return rc;
    if ((rc = upload(c, &c->d_rs_qmod, rsq, "rescale qmod"))) return rc;
    return HE_OK;
}

// Validates the parameter set and derives (or checks) the primes and their
// psi.  Host only.  Returns HE_OK or HE_EINVAL.
static int derive_params(const he_params* prm, std::vector<uint64_t>& primes, std::vector<uint64_t>& psi) {
    if (!prm) return HE_EINVAL;
    const int ln = prm->log_n, L = prm->n_q, K = prm->n_p, dnum = prm->dnum;
    if (ln < 10 || ln > 16 || L < 1 || K < 1 || L + K > kMaxPrimes || dnum < 1 || dnum > L) return HE_EINVAL;
    const int alpha = (L + dnum - 1) / dnum;
    if (K < alpha || alpha > 16 || K > 16 || (L + alpha - 1) / alpha > 15) return HE_EINVAL;
    const int b0 = prm->q0_bits ? prm->q0_bits : 60, bq = prm->q_bits ? prm->q_bits : 40,
              bp = prm->p_bits ? prm->p_bits : 60;
    if (b0 < 20 || b0 > 60 || bq < 20 || bq > 60 || bp < 20 || bp > 60) return HE_EINVAL;
    const uint64_t two_n = 2ull << ln;
    primes.clear();
    psi.clear();
    if (prm->q || prm->p) {
        if (!prm->q || !prm->p) return HE_EINVAL;
        for (int i = 0; i < L; i++) primes.push_back(prm->q[i]);
        for (int i = 0; i < K; i++) primes.push_back(prm->p[i]);
        for (size_t i = 0; i < primes.size(); i++) {
            uint64_t q = primes[i];
            if (q % two_n != 1 || q >= (1ull << 60) || !h_is_prime(q)) return HE_EINVAL;
            for (size_t k = 0; k < i; k++)
                if (primes[k] == q) return HE_EINVAL;
        }
    } else {
        std::map<int, PrimeScan> scans;
        auto take = [&](int bits) {
            auto it = scans.find(bits);
            if (it == scans.end()) it = scans.emplace(bits, PrimeScan(bits, two_n)).first;
            return it->second.next();
        };
        uint64_t q0 = take(b0);
        std::vector<uint64_t> ps, qs;
        for (int i = 0; i < K; i++) ps.push_back(take(bp));
        for (int i = 1; i < L; i++) qs.push_back(take(bq));
        primes.push_back(q0);
        for (uint64_t q : qs) primes.push_back(q);
        for (uint64_t p : ps) primes.push_back(p);
        for (uint64_t q : primes)
            if (q == 0) return HE_EINVAL;
    }
    for (uint64_t q : primes) psi.push_back(h_min_primitive_root(q, two_n));
    return HE_OK;
}

}  // namespace he

using namespace he;

extern "C" int he_derive_primes(const he_params* prm, uint64_t* primes_out, uint64_t* psi_out) {
    std::vector<uint64_t> pr, ps;
    int rc = derive_params(prm, pr, ps);
    if (rc) return rc;
    for (size_t i = 0; i < pr.size(); i++) {
        if (primes_out) primes_out[i] = pr[i];
        if (psi_out) psi_out[i] = ps[i];
    }
    return HE_OK;
}

extern "C" int he_ctx_create(const he_params* prm, void* stream, he_ctx** out) {
    if (!prm || !out) return HE_EINVAL;
    *out = nullptr;
    std::vector<uint64_t> primes, psi;
    int drc = derive_params(prm, primes, psi);
    if (drc) return drc;
    he_ctx* c = new he_ctx();
    c->log_n = prm->log_n;
    c->N = 1 << prm->log_n;
    c->L = prm->n_q;
    c->K = prm->n_p;
    c->dnum = prm->dnum;
    c->alpha = (c->L + c->dnum - 1) / c->dnum;
    c->stream = (cudaStream_t)stream;
    c->primes = primes;
    c->psi = psi;

    int rc = check_cuda(c, cudaGetDevice(&c->device), "cudaGetDevice");
    if (!rc) rc = check_cuda(c, cudaDeviceGetAttribute(&c->sm_count, cudaDevAttrMultiProcessorCount, c->device),
                             "multiprocessor count");
    if (!rc) rc = build_tables(c);
    if (!rc) rc = noalloc_setup(c);
    if (!rc) rc = check_cuda(c, cudaMalloc(&c->d_err, sizeof(int)), "error word");
    if (!rc) rc = check_cuda(c, cudaMemset(c->d_err, 0, sizeof(int)), "error word");
    if (!rc) rc = moddown_tc_setup(c);
    if (!rc) {
        // the FP64 conversion kernel unless "tc" selects the tensor-core one
        const char* v = getenv("HE_MODDOWN_CONV");
        c->tc_moddown = moddown_tc_available(c) && v && strcmp(v, "tc") == 0;
    }
    if (rc) {
        fprintf(stderr, "he_ctx_create: %s\n", c->err.c_str());
        he_ctx_destroy(c);
        return rc;
    }
    *out = c;
    return HE_OK;
}

extern "C" int he_ctx_destroy(he_ctx* c) {
    if (!c) return HE_EINVAL;
    cudaStreamSynchronize(c->stream);
    if (c->aux) cudaStreamSynchronize(c->aux), cudaStreamDestroy(c->aux);
    if (c->ev_fork) cudaEventDestroy(c->ev_fork);
    if (c->ev_join) cudaEventDestroy(c->ev_join);
    cudaFree(c->d_prime);
    cudaFree(c->d_tw_fwd);
    cudaFree(c->d_tw_inv);
    cudaFree(c->d_inv_last);
    cudaFree(c->d_twd_fwd);
    cudaFree(c->d_twd_inv);
    cudaFree(c->d_fpmod);
    if (c->L >= 1 && (int)c->modup.size() > 1 && !c->modup[1].empty()) cudaFree(c->modup[1][0].d_src);
    cudaFree(c->d_md_pcoef);
    cudaFree(c->d_md_mat);
    cudaFree(c->d_md_negP);
    cudaFree(c->d_md_pinv);
    cudaFree(c->d_rs_inv);
    cudaFree(c->d_rs_qmod);
    cudaFree(c->d_err);
    cudaFree(c->d_tc_btab);
    cudaFree(c->d_tc_tgt);
    for (auto& kv : c->rot_keys) cudaFree(kv.second.d);
    cudaFree(c->relin.d);
    for (int i = 0; i < kScratchSlots; i++) cudaFree(c->scratch[i]);
    cudaFree(c->io_buf);
    if (c->io_h2d) cudaStreamSynchronize(c->io_h2d), cudaStreamDestroy(c->io_h2d);
    if (c->io_d2h) cudaStreamSynchronize(c->io_d2h), cudaStreamDestroy(c->io_d2h);
    for (cudaEvent_t e : c->io_ev)
        if (e) cudaEventDestroy(e);
    for (auto& p : c->prof_pending) {
        if (p.a) cudaEventDestroy(p.a);
        if (p.b) cudaEventDestroy(p.b);
    }
    for (cudaEvent_t e : c->ev_pool) cudaEventDestroy(e);
    delete c;
    return HE_OK;
}

extern "C" int he_set_stream(he_ctx* c, void* s) {
    if (!c) return HE_EINVAL;
    c->stream = (cudaStream_t)s;
    return HE_OK;
}

extern "C" int he_sync(he_ctx* c) {
    if (!c) return HE_EINVAL;
    int rc = check_cuda(c, cudaStreamSynchronize(c->stream), "he_sync");
    if (rc || !c->d_err) return rc;
    int e = 0;
    if ((rc = check_cuda(c, cudaMemcpy(&e, c->d_err, sizeof(int), cudaMemcpyDeviceToHost), "he_sync"))) return rc;
    if (e) {
        cudaMemset(c->d_err, 0, sizeof(int));
        return set_err(c, HE_ETIMEOUT, "he_sync: a bounded device wait gave up (its results are not valid)");
    }
    return HE_OK;
}

extern "C" const char* he_last_error(const he_ctx* c) { return c ? c->err.c_str() : "null context"; }

extern "C" int he_get_primes(const he_ctx* c, uint64_t* out) {
    if (!c || !out) return HE_EINVAL;
    for (size_t i = 0; i < c->primes.size(); i++) out[i] = c->primes[i];
    return HE_OK;
}

extern "C" int he_get_psi(const he_ctx* c, uint64_t* out) {
    if (!c || !out) return HE_EINVAL;
    for (size_t i = 0; i < c->psi.size(); i++) out[i] = c->psi[i];
    return HE_OK;
}

extern "C" int he_profile_enable(he_ctx* c, int enable) {
    if (!c) return HE_EINVAL;
    int rc = prof_collect(c);
    if (rc) return rc;
    c->prof_on = enable != 0;
    for (auto& p : c->prof) p = ProfSlot();
    return HE_OK;
}

extern "C" int he_profile_read(he_ctx* c, int cls, double* ms, long long* launches, double* bytes,
                               double* mults) {
    if (!c || cls < 0 || cls >= HE_PROF_N) return HE_EINVAL;
    int rc = prof_collect(c);
    if (rc) return rc;
    if (ms) *ms = c->prof[cls].ms;
    if (launches) *launches = c->prof[cls].launches;
    if (bytes) *bytes = c->prof[cls].bytes;
    if (mults) *mults = c->prof[cls].mults;
    return HE_OK;
}

extern "C" int he_profile_read_fp(he_ctx* c, int cls, double* fp_mults) {
    if (!c || cls < 0 || cls >= HE_PROF_N) return HE_EINVAL;
    int rc = prof_collect(c);
    if (rc) return rc;
    if (fp_mults) *fp_mults = c->prof[cls].mults_fp;
    return HE_OK;
}

extern "C" long long he_launch_count(he_ctx* c, int reset) {
    if (!c) return -1;
    long long v = c->launches;
    if (reset) c->launches = 0;
    return v;
}
