// One encrypted attention head (AEGIS summary section 2.3: Q x K^T, a
// polynomial Softmax, A x V), composed of the engine's batched operations.
//
// Packing: d features x n tokens with d 2n = N/2, feature-major with stride
// 2n.  Q sits at slot f 2n + t for t < n (zeros at t >= n); K and V are
// token-duplicated (slot f 2n + t holds X[f][t mod n] for every t < 2n), so
// that a slot rotation by delta < n shifts every feature's tokens cyclically.
//   scores:  P = HMRR(Q, rot_delta(K)), then S_delta = sum_{h<d} rot_{2n h}(P)
//            as two hoisted rotate-and-sums (d = d1 d2): every feature block holds
//            sum_f Q[f][t] K[f][(t + delta) mod n] at t < n (0 at t >= n);
//   Softmax: the caller shifts S_delta by a known bound and evaluates its
//            exponential with he_poly_eval_ps15 (no division by row sums);
//   output:  O = rescale(relinearise(sum_delta A_delta (x) drop(rot_delta(V)))):
//            the products' tensors summed, one relinearisation, one rescale.
// The rotations of K and of V by the offsets are hoisted (one ModUp each).
#include <algorithm>

#include "he_internal.h"

namespace he {

static int ct_check(he_ctx* c, const he_ct* x, const char* what) {
    if (!x || !x->data) return set_err(c, HE_EINVAL, "%s: null ciphertext", what);
    if ((uintptr_t)x->data & 31) return set_err(c, HE_EINVAL, "%s: ciphertext not 32-byte aligned", what);
    if (x->level < 1 || x->level > c->L) return set_err(c, HE_ELEVEL, "%s: level %d out of range", what, x->level);
    if (!x->is_ntt) return set_err(c, HE_EDOMAIN, "%s: ciphertext not in the evaluation domain", what);
    return HE_OK;
}

static int need_key(he_ctx* c, int32_t step, const char* what) {
    const uint64_t g = galois_elt(c, step);
    if (g != 1 && !c->rot_keys.count(g)) return set_err(c, HE_ENOKEY, "%s: no key for step %d", what, step);
    return HE_OK;
}

// Offsets in [0, n_tok); the non-zero ones (in order) and each offset's
// position among them (-1 for offset 0).
static int split_offsets(he_ctx* c, const int32_t* offsets, int n_off, int n_tok, std::vector<int32_t>& nz,
                         std::vector<int>& pos, const char* what) {
    for (int i = 0; i < n_off; i++) {
        if (offsets[i] < 0 || offsets[i] >= n_tok) return set_err(c, HE_EINVAL, "%s: offset %d outside [0, %d)", what,
                                                                  offsets[i], n_tok);
        pos.push_back(offsets[i] ? (int)nz.size() : -1);
        if (offsets[i]) nz.push_back(offsets[i]);
    }
    for (int32_t o : nz)
        if (int rc = need_key(c, o, what)) return rc;
    return HE_OK;
}

// Ranges [p, p + words) of two device buffers intersect.
static bool overlap(const uint64_t* a, size_t a_words, const uint64_t* b, size_t b_words) {
    return a < b + b_words && b < a + a_words;
}

// Rejects outputs (each `out_words` long) that overlap one another or one of
// the inputs (ins[i] with in_words[i] words).
static int check_outputs(he_ctx* c, const he_ct* out, int n_out, size_t out_words,
                         const std::vector<std::pair<const uint64_t*, size_t>>& ins, const char* what) {
    std::vector<const uint64_t*> o(n_out);
    for (int i = 0; i < n_out; i++) {
        o[i] = out[i].data;
        for (const auto& in : ins)
            if (overlap(o[i], out_words, in.first, in.second))
                return set_err(c, HE_EINVAL, "%s: output %d overlaps an input", what, i);
    }
    std::sort(o.begin(), o.end());
    for (int i = 1; i < n_out; i++)
        if (overlap(o[i - 1], out_words, o[i], out_words))
            return set_err(c, HE_EINVAL, "%s: outputs overlap one another", what);
    return HE_OK;
}

}  // namespace he

using namespace he;

extern "C" int he_attention_scores(he_ctx* c, const he_ct* q, const he_ct* k, int n_tok, int d,
                                   const int32_t* offsets, int n_off, he_ct* s) {
    if (!c) return HE_EINVAL;
    const char* what = "attention_scores";
    if (!s || !offsets || n_off < 1 || n_tok < 1 || d < 1 || (d & (d - 1)) ||
        (long long)d * 2 * n_tok != (long long)c->N / 2)
        return set_err(c, HE_EINVAL, "%s: bad arguments (need d a power of two, d 2 n_tok = N/2, n_off >= 1)", what);
    int rc;
    if ((rc = ct_check(c, q, what)) || (rc = ct_check(c, k, what))) return rc;
    const int l = q->level;
    if (k->level != l) return set_err(c, HE_ELEVEL, "%s: q and k at different levels", what);
    if (l < 2) return set_err(c, HE_ELEVEL, "%s: level %d cannot be rescaled", what, l);
    if (!c->relin.d) return set_err(c, HE_ENOKEY, "%s: no relinearisation key", what);
    std::vector<int32_t> nz;
    std::vector<int> pos;
    if ((rc = split_offsets(c, offsets, n_off, n_tok, nz, pos, what))) return rc;
    // feature-sum steps: 2n b (b < d1), then 2n d1 a (a < d2), d = d1 d2
    int lg = 0;
    while ((1 << lg) < d) lg++;
    const int d1 = 1 << ((lg + 1) / 2), d2 = d / d1;
    std::vector<int32_t> inner, outer;
    for (int b = 0; b < d1; b++) inner.push_back(2 * n_tok * b);
    for (int a2 = 0; a2 < d2; a2++) outer.push_back(2 * n_tok * d1 * a2);
    for (int32_t st : inner)
        if (st && (rc = need_key(c, st, what))) return rc;
    for (int32_t st : outer)
        if (st && (rc = need_key(c, st, what))) return rc;
    const size_t N = c->N, ctw = (size_t)2 * l * N, ctw1 = (size_t)2 * (l - 1) * N;
    for (int i = 0; i < n_off; i++)
        if (!s[i].data || ((uintptr_t)s[i].data & 31)) return set_err(c, HE_EINVAL, "%s: null or unaligned output", what);
    if ((rc = check_outputs(c, s, n_off, ctw1, {{q->data, ctw}, {k->data, ctw}}, what))) return rc;
    uint64_t* pool;
    if ((rc = scratch_slot(c, 3, ctw * nz.size() + ctw1 * n_off, &pool))) return rc;
    // rot_delta(k) for the non-zero offsets, hoisted
    std::vector<he_ct> rk(nz.size());
    for (size_t j = 0; j < nz.size(); j++) rk[j] = he_ct{pool + j * ctw, l, k->scale, 1};
    if (!nz.empty() && (rc = rotate_hoisted_many(c, k, 1, nz.data(), (int)nz.size(), rk.data()))) return rc;
    // P_delta = HMRR(q, rot_delta(k)) into the outputs
    std::vector<const uint64_t*> A, B;
    std::vector<uint64_t*> So, Tm;
    for (int i = 0; i < n_off; i++) {
        A.push_back(q->data);
        B.push_back(pos[i] < 0 ? k->data : rk[pos[i]].data);
        So.push_back(s[i].data);
        Tm.push_back(pool + ctw * nz.size() + ctw1 * i);
    }
    if ((rc = hmrr_many(c, A, B, So, l))) return rc;
    // the feature sum S = sum_{h<d} rot_{2n h}(P) as two hoisted
    // rotate-and-sums (one ModUp and one ModDown each; step 0 adds the term
    // itself): T = sum_b rot_{2n b}(P), S = sum_a rot_{2n d1 a}(T); the
    // rounds alternate between the outputs and the scratch
    const double scale = q->scale * k->scale / (double)c->primes[l - 1];
    std::vector<he_ct> sc(n_off), tc(n_off);
    for (int i = 0; i < n_off; i++) {
        sc[i] = he_ct{s[i].data, l - 1, scale, 1};
        tc[i] = he_ct{Tm[i], l - 1, scale, 1};
    }
    int rounds = 0;
    for (const std::vector<int32_t>* st : {&inner, &outer}) {
        if (st->size() < 2) continue;
        const std::vector<he_ct>& src = rounds % 2 ? tc : sc;
        std::vector<he_ct>& dst = rounds % 2 ? sc : tc;
        if ((rc = rotate_sum_hoisted_many(c, src.data(), n_off, st->data(), (int)st->size(), dst.data()))) return rc;
        rounds++;
    }
    if (rounds % 2)  // an odd number of rounds ends in the scratch
        for (int i = 0; i < n_off; i++)
            if ((rc = check_cuda(c, cudaMemcpyAsync(s[i].data, Tm[i], (size_t)2 * (l - 1) * c->N * 8,
                                                    cudaMemcpyDeviceToDevice, c->stream), "attention copy")))
                return rc;
    for (int i = 0; i < n_off; i++) {
        s[i].level = l - 1;
        s[i].scale = scale;
        s[i].is_ntt = 1;
    }
    return HE_OK;
}

extern "C" int he_attention_output(he_ctx* c, const he_ct* a, const he_ct* v, int n_tok, const int32_t* offsets,
                                   int n_off, he_ct* out) {
    if (!c) return HE_EINVAL;
    const char* what = "attention_output";
    if (!a || !out || !offsets || n_off < 1 || n_tok < 1) return set_err(c, HE_EINVAL, "%s: bad arguments", what);
    int rc;
    if ((rc = ct_check(c, v, what))) return rc;
    if (!out->data || ((uintptr_t)out->data & 31)) return set_err(c, HE_EINVAL, "%s: null or unaligned output", what);
    const int la = a[0].level, lv = v->level;
    for (int i = 0; i < n_off; i++) {
        if ((rc = ct_check(c, &a[i], what))) return rc;
        if (a[i].level != la || a[i].scale != a[0].scale)
            return set_err(c, HE_ELEVEL, "%s: mixed levels or scales among the weights", what);
    }
    if (la < 2 || lv < la) return set_err(c, HE_ELEVEL, "%s: weights at level %d, values at %d", what, la, lv);
    {
        const size_t n = c->N;
        std::vector<std::pair<const uint64_t*, size_t>> ins;
        for (int i = 0; i < n_off; i++) ins.push_back({a[i].data, (size_t)2 * la * n});
        ins.push_back({v->data, (size_t)2 * lv * n});
        if ((rc = check_outputs(c, out, 1, (size_t)2 * (la - 1) * n, ins, what))) return rc;
    }
    if (!c->relin.d) return set_err(c, HE_ENOKEY, "%s: no relinearisation key", what);
    std::vector<int32_t> nz;
    std::vector<int> pos;
    if ((rc = split_offsets(c, offsets, n_off, n_tok, nz, pos, what))) return rc;

    const size_t N = c->N, ctv = (size_t)2 * lv * N;
    uint64_t* pool = nullptr;
    if (!nz.empty() && (rc = scratch_slot(c, 3, ctv * nz.size(), &pool))) return rc;
    // rot_delta(v) for the non-zero offsets, hoisted; the products read them
    // at the weights' level in place
    std::vector<he_ct> rv(nz.size());
    for (size_t j = 0; j < nz.size(); j++) rv[j] = he_ct{pool + j * ctv, lv, v->scale, 1};
    if (!nz.empty() && (rc = rotate_hoisted_many(c, v, 1, nz.data(), (int)nz.size(), rv.data()))) return rc;
    // the products' tensors summed, then one relinearisation and one rescale
    std::vector<const uint64_t*> A, B;
    for (int i = 0; i < n_off; i++) {
        B.push_back(pos[i] < 0 ? v->data : rv[pos[i]].data);
        A.push_back(a[i].data);
    }
    if ((rc = hmrr_sum(c, A, B, out->data, la, la, lv))) return rc;
    out->level = la - 1;
    out->scale = a[0].scale * v->scale / (double)c->primes[la - 1];
    out->is_ntt = 1;
    return HE_OK;
}
