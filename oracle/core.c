/*
 * Oracle core: plain, slow, obviously correct RNS polynomial arithmetic.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link or call this
 * file: only tests, the smoke check and the benchmark's CPU-baseline leg do.
 * It shares no code, header, table or constant generator with the CUDA path.
 *
 * Every modular product is the definition itself: ((unsigned __int128)a*b) % q.
 * No Montgomery, Barrett or Shoup form appears here, so a mistake in the GPU
 * reductions cannot be mirrored by the oracle.
 *
 * What the pages fix: the scheme is CKKS over an RNS modulus chain, ciphertext
 * polynomials are split into limbs, and rotation/relinearisation use key
 * switching (AEGIS, gist.science, section 1 "Problem" items 2-3).  The pages
 * give no formula below that level; this file follows the textbook negacyclic
 * number-theoretic transform and the RNS fast base conversion of
 * Cheon-Han-Kim-Kim-Song, "A Full RNS Variant of Approximate Homomorphic
 * Encryption" (SAC 2018), section 2.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef unsigned __int128 u128;

static uint64_t mulmod(uint64_t a, uint64_t b, uint64_t q) {
    return (uint64_t)(((u128)a * b) % q);
}

static uint64_t addmod(uint64_t a, uint64_t b, uint64_t q) {
    uint64_t s = a + b;            /* a, b < q < 2^63: no wrap */
    return s >= q ? s - q : s;
}

static uint64_t submod(uint64_t a, uint64_t b, uint64_t q) {
    return a >= b ? a - b : a + q - b;
}

uint64_t ora_powmod(uint64_t b, uint64_t e, uint64_t q) {
    uint64_t r = 1 % q;
    b %= q;
    while (e) {
        if (e & 1) r = mulmod(r, b, q);
        b = mulmod(b, b, q);
        e >>= 1;
    }
    return r;
}

/*
 * Evaluate the polynomial a(x) = sum_i a[i*stride] x^i of n terms at the n
 * points x_m = w^(2m+1), m = 0..n-1, where w has multiplicative order 2n.
 * out[m] = a(w^(2m+1)).
 *
 * Textbook even/odd split: a(x) = E(x^2) + x O(x^2).  Since x_m^2 = (w^2)^(2m+1)
 * and w^2 has order n, E and O are evaluated by the same routine on n/2 points,
 * and x_{m+n/2} = -x_m because w^n = -1.
 */
static void eval_odd(const uint64_t* a, size_t stride, size_t n, uint64_t w,
                     uint64_t q, uint64_t* out) {
    if (n == 1) {
        out[0] = a[0] % q;
        return;
    }
    size_t h = n / 2;
    uint64_t* e = (uint64_t*)malloc(sizeof(uint64_t) * h);
    uint64_t* o = (uint64_t*)malloc(sizeof(uint64_t) * h);
    uint64_t w2 = mulmod(w, w, q);
    eval_odd(a, 2 * stride, h, w2, q, e);
    eval_odd(a + stride, 2 * stride, h, w2, q, o);
    uint64_t x = w; /* x = w^(2m+1) */
    for (size_t m = 0; m < h; m++) {
        uint64_t t = mulmod(x, o[m], q);
        out[m] = addmod(e[m], t, q);
        out[m + h] = submod(e[m], t, q);
        x = mulmod(x, w2, q);
    }
    free(e);
    free(o);
}

/*
 * Cyclic transform F[k] = sum_m x[m*stride] w^(m k), k = 0..n-1, w of order n.
 * Textbook radix-2 decimation in time: F[k] = E[k] + w^k O[k], with
 * w^(k+n/2) = -w^k.
 */
static void dft_cyclic(const uint64_t* x, size_t stride, size_t n, uint64_t w,
                       uint64_t q, uint64_t* out) {
    if (n == 1) {
        out[0] = x[0] % q;
        return;
    }
    size_t h = n / 2;
    uint64_t* e = (uint64_t*)malloc(sizeof(uint64_t) * h);
    uint64_t* o = (uint64_t*)malloc(sizeof(uint64_t) * h);
    uint64_t w2 = mulmod(w, w, q);
    dft_cyclic(x, 2 * stride, h, w2, q, e);
    dft_cyclic(x + stride, 2 * stride, h, w2, q, o);
    uint64_t wk = 1;
    for (size_t k = 0; k < h; k++) {
        uint64_t t = mulmod(wk, o[k], q);
        out[k] = addmod(e[k], t, q);
        out[k + h] = submod(e[k], t, q);
        wk = mulmod(wk, w, q);
    }
    free(e);
    free(o);
}

static size_t bitrev(size_t j, int bits) {
    size_t r = 0;
    for (int b = 0; b < bits; b++) r |= ((j >> b) & 1) << (bits - 1 - b);
    return r;
}

/*
 * Forward negacyclic NTT, in place, on one limb of n = 2^logn coefficients.
 * Storage index j receives a(psi^(2*brev(j)+1)) where psi is a primitive
 * 2n-th root of unity mod q.
 */
void ora_ntt_fwd(uint64_t* a, int logn, uint64_t q, uint64_t psi) {
    size_t n = (size_t)1 << logn;
    uint64_t* v = (uint64_t*)malloc(sizeof(uint64_t) * n);
    eval_odd(a, 1, n, psi, q, v);
    for (size_t j = 0; j < n; j++) a[j] = v[bitrev(j, logn)];
    free(v);
}

/*
 * Inverse of ora_ntt_fwd: given the values at psi^(2m+1) (in the storage
 * order above), a_i = n^-1 psi^-i sum_m val[m] (psi^-2)^(m i).
 */
void ora_ntt_inv(uint64_t* a, int logn, uint64_t q, uint64_t psi) {
    size_t n = (size_t)1 << logn;
    uint64_t* val = (uint64_t*)malloc(sizeof(uint64_t) * n);
    uint64_t* f = (uint64_t*)malloc(sizeof(uint64_t) * n);
    for (size_t m = 0; m < n; m++) val[m] = a[bitrev(m, logn)];
    uint64_t psi_inv = ora_powmod(psi, q - 2, q);
    uint64_t w = mulmod(psi_inv, psi_inv, q);
    dft_cyclic(val, 1, n, w, q, f);
    uint64_t n_inv = ora_powmod((uint64_t)(n % q), q - 2, q);
    uint64_t pw = n_inv; /* n^-1 psi^-i */
    for (size_t i = 0; i < n; i++) {
        a[i] = mulmod(f[i], pw, q);
        pw = mulmod(pw, psi_inv, q);
    }
    free(val);
    free(f);
}

/* out[i] = a[i] * b[i] mod q */
void ora_vec_mul(const uint64_t* a, const uint64_t* b, uint64_t* out, size_t n, uint64_t q) {
    for (size_t i = 0; i < n; i++) out[i] = mulmod(a[i], b[i], q);
}

/* out[i] = a[i] * c mod q */
void ora_vec_scale(const uint64_t* a, uint64_t c, uint64_t* out, size_t n, uint64_t q) {
    for (size_t i = 0; i < n; i++) out[i] = mulmod(a[i], c, q);
}

/*
 * Fast base conversion (CHKKS SAC 2018, section 2.2, "Conv"):
 *   out_t[c] = sum_i y_i * qhat_mod[i][t]   mod dst[t],
 *   y_i = [ x_i[c] * qhat_inv[i] ]_{q_i}
 * with qhat_inv[i] = (Q/q_i)^-1 mod q_i and qhat_mod[i][t] = (Q/q_i) mod dst[t].
 * y_i is taken in [0, q_i) when centered == 0, and in (-q_i/2, q_i/2) when
 * centered != 0 (y_i > q_i/2 stands for y_i - q_i).
 * in: [n_src][n] residues, out: [n_dst][n].  No overflow correction.
 */
void ora_base_conv(const uint64_t* in, int n_src, const uint64_t* src_q,
                   const uint64_t* qhat_inv, uint64_t* out, int n_dst,
                   const uint64_t* dst_q, const uint64_t* qhat_mod, size_t n,
                   int centered) {
    uint64_t* y = (uint64_t*)malloc(sizeof(uint64_t) * n_src);
    for (size_t c = 0; c < n; c++) {
        for (int i = 0; i < n_src; i++)
            y[i] = mulmod(in[(size_t)i * n + c], qhat_inv[i], src_q[i]);
        for (int t = 0; t < n_dst; t++) {
            uint64_t acc = 0;
            for (int i = 0; i < n_src; i++) {
                uint64_t yt = y[i] % dst_q[t];
                if (centered && y[i] > src_q[i] / 2)
                    yt = submod(yt, src_q[i] % dst_q[t], dst_q[t]);
                acc = addmod(acc, mulmod(yt, qhat_mod[(size_t)i * n_dst + t], dst_q[t]), dst_q[t]);
            }
            out[(size_t)t * n + c] = acc;
        }
    }
    free(y);
}

/*
 * Ring automorphism in the coefficient domain: out(X) = a(X^k) mod (X^n + 1),
 * k odd.  Coefficient i moves to i*k mod 2n, negated when that lands in [n, 2n).
 */
void ora_automorph_coeff(const uint64_t* a, uint64_t* out, int logn, uint64_t k, uint64_t q) {
    size_t n = (size_t)1 << logn;
    size_t two_n = 2 * n;
    for (size_t i = 0; i < n; i++) {
        size_t e = (size_t)(((u128)i * k) % two_n);
        if (e < n) out[e] = a[i] % q;
        else out[e - n] = (q - a[i] % q) % q;
    }
}
