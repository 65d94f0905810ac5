// Plaintext-weight x ciphertext block product by the diagonal method with
// baby-step / giant-step (the FFN's local polynomial multiplication per
// output group, AEGIS summary section 2.2):
//   Y[t][i] = rescale( sum_g rot_{stride bs g}( sum_{j,b} pt[i][j][g][b] (.) rot_{stride b}(X[t][j]) ) )
#include <algorithm>

#include "he_internal.h"

namespace he {

int add_raw(he_ctx* c, const uint64_t* a, const uint64_t* b, uint64_t* out, int level);

// Z[t][g][poly][r][c] = sum_{j,b} pt[i][j][g][b][r][c] * B[t][j][b][poly][r][c]
// (128-bit accumulation, one reduction per output).  One thread per (r, c).
__global__ void k_pmult_accum(const uint64_t* __restrict__ pt_i, const uint64_t* __restrict__ B,
                              uint64_t* __restrict__ Z, int n_groups, int n_in, int gs, int bs, int level,
                              const DevPrime* __restrict__ pr, int logn) {
    const int N = 1 << logn;
    int c = blockIdx.x * blockDim.x + threadIdx.x, r = blockIdx.y;
    if (c >= N) return;
    const DevPrime p = pr[r];
    const size_t limb = (size_t)level * N, ctw = 2 * limb;
    const size_t off = (size_t)r * N + c;
    for (int g = 0; g < gs; g++) {
        for (int t = 0; t < n_groups; t++) {
            U128 a0 = {0, 0}, a1 = {0, 0};
            for (int j = 0; j < n_in; j++) {
                const uint64_t* ptj = pt_i + ((size_t)(j * gs + g) * bs) * limb + off;
                const uint64_t* bj = B + ((size_t)(t * n_in + j) * bs) * ctw + off;
                for (int b = 0; b < bs; b++) {
                    uint64_t w = ptj[(size_t)b * limb];
                    mac128(a0, w, bj[(size_t)b * ctw]);
                    mac128(a1, w, bj[(size_t)b * ctw + limb]);
                }
            }
            uint64_t* z = Z + (size_t)(t * gs + g) * ctw + off;
            z[0] = reduce128(a0, p);
            z[limb] = reduce128(a1, p);
        }
    }
}

}  // namespace he

using namespace he;

extern "C" int he_pmult_accum_bsgs(he_ctx* c, const he_ct* x, int n_in, const uint64_t* d_pt, double pt_scale,
                                   int n_out, int bs, int gs, int stride, int n_groups, he_ct* y) {
    if (!c) return HE_EINVAL;
    if (!x || !y || !d_pt || n_in < 1 || n_out < 1 || bs < 1 || gs < 1 || n_groups < 1 || stride < 1 ||
        (long long)n_in * bs > 255)
        return set_err(c, HE_EINVAL, "he_pmult_accum_bsgs: bad arguments");
    const int level = x[0].level, N = c->N;
    for (int i = 0; i < n_groups * n_in; i++) {
        if (!x[i].data || ((uintptr_t)x[i].data & 15) || !x[i].is_ntt) return set_err(c, HE_EINVAL, "he_pmult_accum_bsgs: bad input %d", i);
        if (x[i].level != level) return set_err(c, HE_ELEVEL, "he_pmult_accum_bsgs: mixed levels");
    }
    for (int i = 0; i < n_groups * n_out; i++)
        if (!y[i].data) return set_err(c, HE_EINVAL, "he_pmult_accum_bsgs: null output %d", i);
    if (level < 2) return set_err(c, HE_ELEVEL, "he_pmult_accum_bsgs: level %d cannot be rescaled", level);
    for (int b = 1; b < bs; b++)
        if (!c->rot_keys.count(galois_elt(c, stride * b)) && galois_elt(c, stride * b) != 1)
            return set_err(c, HE_ENOKEY, "he_pmult_accum_bsgs: no key for baby step %d", stride * b);
    for (int g = 1; g < gs; g++)
        if (!c->rot_keys.count(galois_elt(c, stride * bs * g)) && galois_elt(c, stride * bs * g) != 1)
            return set_err(c, HE_ENOKEY, "he_pmult_accum_bsgs: no key for giant step %d", stride * bs * g);

    const size_t ctw = (size_t)2 * level * N;
    const size_t nB = (size_t)n_groups * n_in * bs, nZ = (size_t)n_groups * gs;
    uint64_t* buf;
    int rc = scratch_slot(c, 3, ctw * (nB + 2 * nZ), &buf);
    if (rc) return rc;
    uint64_t* B = buf;
    uint64_t* Z = B + ctw * nB;
    uint64_t* Rg = Z + ctw * nZ;

    // baby steps: B[t][j][b] = rot_{stride b}(X[t][j])
    std::vector<he_ct> bin, bout;
    std::vector<int32_t> bsteps;
    for (int t = 0; t < n_groups; t++)
        for (int j = 0; j < n_in; j++) {
            const he_ct& xi = x[t * n_in + j];
            uint64_t* dst0 = B + ((size_t)(t * n_in + j) * bs) * ctw;
            rc = check_cuda(c, cudaMemcpyAsync(dst0, xi.data, ctw * 8, cudaMemcpyDeviceToDevice, c->stream),
                            "bsgs copy");
            if (rc) return rc;
            for (int b = 1; b < bs; b++) {
                bin.push_back(xi);
                bout.push_back(he_ct{dst0 + (size_t)b * ctw, level, xi.scale, 1});
                bsteps.push_back(stride * b);
            }
        }
    if (!bin.empty() && (rc = rotate_many(c, bin.data(), bsteps.data(), bout.data(), (int)bin.size()))) return rc;

    const int gx = (N + 255) / 256;
    const size_t pt_block = (size_t)n_in * gs * bs * level * N;
    for (int i = 0; i < n_out; i++) {
        prof_begin(c, HE_PROF_PMULT);
        k_pmult_accum<<<dim3(gx, level), 256, 0, c->stream>>>(d_pt + pt_block * i, B, Z, n_groups, n_in, gs, bs,
                                                              level, c->d_prime, c->log_n);
        c->launches++;
        if ((rc = check_cuda(c, cudaGetLastError(), "pmult_accum"))) return rc;
        prof_end(c, HE_PROF_PMULT);
        // giant steps
        std::vector<he_ct> gin, gout;
        std::vector<int32_t> gsteps;
        for (int t = 0; t < n_groups; t++)
            for (int g = 1; g < gs; g++) {
                gin.push_back(he_ct{Z + (size_t)(t * gs + g) * ctw, level, 1.0, 1});
                gout.push_back(he_ct{Rg + (size_t)(t * gs + g) * ctw, level, 1.0, 1});
                gsteps.push_back(stride * bs * g);
            }
        if (!gin.empty() && (rc = rotate_many(c, gin.data(), gsteps.data(), gout.data(), (int)gin.size())))
            return rc;
        std::vector<const uint64_t*> rin;
        std::vector<uint64_t*> rout;
        for (int t = 0; t < n_groups; t++) {
            uint64_t* dst = y[t * n_out + i].data;
            const uint64_t* z0 = Z + (size_t)(t * gs) * ctw;
            if (gs == 1) {
                rc = check_cuda(c, cudaMemcpyAsync(dst, z0, ctw * 8, cudaMemcpyDeviceToDevice, c->stream), "bsgs");
                if (rc) return rc;
            }
            for (int g = 1; g < gs; g++) {
                const uint64_t* src = g == 1 ? z0 : dst;
                if ((rc = add_raw(c, src, Rg + (size_t)(t * gs + g) * ctw, dst, level))) return rc;
            }
            rin.push_back(dst);
            rout.push_back(dst);
        }
        if ((rc = rescale_many(c, rin, rout, level))) return rc;
    }
    for (int i = 0; i < n_groups * n_out; i++) {
        y[i].level = level - 1;
        y[i].scale = (x[0].scale * pt_scale) / (double)c->primes[level - 1];
        y[i].is_ntt = 1;
    }
    return HE_OK;
}
