// Plaintext-weight x ciphertext block product by the diagonal method with
// baby-step / giant-step (the FFN's local polynomial multiplication per
// output group, AEGIS summary section 2.2):
//   Y[t][i] = rescale( sum_g rot_{stride bs g}( sum_{j,b} pt[i][j][g][b] (.) rot_{stride b}(X[t][j]) ) )
#include <algorithm>

#include "he_internal.h"
#include "ntt.cuh"

namespace he {


// Z[t][g][poly][r][c] = sum_{k < KB} pt[i][j][g][b][r][c] * B[t][k][poly][r][c],  k = j bs + b,
// a small modular matrix product per coefficient ([g x k] weights times
// [k x t] rotated inputs).  A block covers kPmCols columns of limb r and
// kPmG giant steps; the rotated inputs of up to TCH token groups for those
// columns are staged in shared memory once and read by all kPmG giant-step
// warps, while each thread streams its own weights.  Limbs of primes below
// 2^41 sum signed FP64 products (|.| < 5q/8 each, one reduction per output);
// the others accumulate 128-bit products and reduce once.
constexpr int kPmThreadsX = 32, kPmG = 8;

// Scratch words of sums and rotated sums a wave of output blocks may hold (8 GiB).
constexpr size_t kBsgsWaveWords = (size_t)1 << 30;

// 16-byte asynchronous copy global -> shared (both 16-byte aligned)
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(smem)),
                 "l"(gmem)
                 : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Element of the staged tile: the residue as a double (FP64 limbs) or as is.
__device__ __forceinline__ void stage_put(uint64_t* dst, uint64_t v, bool fp) {
    *dst = fp ? (uint64_t)__double_as_longlong(u2d(v)) : v;
}

// TCH token groups staged per pass, CPT adjacent columns and GPT giant steps
// per thread (kPmThreadsX * CPT columns and kPmG * GPT giant steps per block):
// each staged input feeds GPT products, each weight TCH * 2.
template <int TCH, int CPT, int GPT>
__global__ void __launch_bounds__(kPmThreadsX* kPmG)
    k_pmult_accum(const uint64_t* __restrict__ pt_i, const uint64_t* __restrict__ B, uint64_t* __restrict__ Z,
                  int n_groups, int n_in, int gs, int bs, int level, const DevPrime* __restrict__ pr,
                  const FpMod* __restrict__ fpm, int logn) {
    constexpr int COLS = kPmThreadsX * CPT;
    extern __shared__ __align__(16) uint64_t sB[];  // [TCH][KB][2][COLS]
    const int N = 1 << logn;
    const int KB = n_in * bs;
    const int tx = threadIdx.x % kPmThreadsX, tg = threadIdx.x / kPmThreadsX;
    // giant-step blocks of one column tile are neighbours: a second finds the tile in L2
    const int c0 = blockIdx.y * COLS, r = blockIdx.z, g0 = (blockIdx.x * kPmG + tg) * GPT;
    const DevPrime p = pr[r];
    const bool fp = p.q < kFpPrimeLimit;
    const FpMod m = fpm[r];
    const size_t limb = (size_t)level * N, ctw = 2 * limb;
    const size_t col = (size_t)r * N + c0;
    for (int t0 = 0; t0 < n_groups; t0 += TCH) {
        const int nt = min(TCH, n_groups - t0);
        __syncthreads();
        // stage the rotated inputs with asynchronous 16-byte copies (all of a
        // thread's copies in flight at once), then convert FP64 limbs in place
        for (int idx = threadIdx.x; idx < nt * KB * COLS; idx += blockDim.x) {
            const int cc2 = idx % (COLS / 2), rest = idx / (COLS / 2);  // rest = (t KB + k) 2 + poly
            const int poly = rest & 1, tk = rest >> 1, t = tk / KB, k = tk - t * KB;
            cp_async16(sB + (size_t)rest * COLS + 2 * cc2,
                       B + ((size_t)(t0 + t) * KB + k) * ctw + poly * limb + col + 2 * cc2);
        }
        cp_async_wait_all();
        __syncthreads();
        if (fp) {
            for (int idx = threadIdx.x; idx < nt * KB * 2 * COLS; idx += blockDim.x) stage_put(sB + idx, sB[idx], true);
            __syncthreads();
        }
        if (g0 >= gs) continue;
        const bool g1ok = GPT > 1 && g0 + 1 < gs;
        const uint64_t* w_base = pt_i + col + CPT * tx;
        if (fp) {
            double acc[GPT][TCH][2][CPT];
#pragma unroll
            for (int h = 0; h < GPT; h++)
#pragma unroll
                for (int t = 0; t < TCH; t++)
#pragma unroll
                    for (int e = 0; e < CPT; e++) acc[h][t][0][e] = acc[h][t][1][e] = 0.0;
#pragma unroll 4
            for (int k = 0; k < KB; k++) {
                const int j = k / bs, b = k - j * bs;
                double w[GPT][CPT];
#pragma unroll
                for (int h = 0; h < GPT; h++) {
                    const int g = (h == 0 || g1ok) ? g0 + h : g0;
                    const uint64_t* wp = w_base + ((size_t)(j * gs + g) * bs + b) * limb;
                    if constexpr (CPT == 2) {
                        const ulonglong2 v = __ldg(reinterpret_cast<const ulonglong2*>(wp));
                        w[h][0] = u2d(v.x);
                        w[h][1] = u2d(v.y);
                    } else {
                        w[h][0] = u2d(__ldg(wp));
                    }
                }
                const double* sk = reinterpret_cast<const double*>(sB) + (size_t)k * 2 * COLS + CPT * tx;
#pragma unroll
                for (int t = 0; t < TCH; t++) {
                    if (t < nt) {
                        const double* st = sk + (size_t)t * KB * 2 * COLS;
#pragma unroll
                        for (int e = 0; e < CPT; e++) {
                            const double b0 = st[e], b1 = st[COLS + e];
#pragma unroll
                            for (int h = 0; h < GPT; h++) {
                                acc[h][t][0][e] = __dadd_rn(acc[h][t][0][e], fp_mulmod_s(w[h][e], b0, m));
                                acc[h][t][1][e] = __dadd_rn(acc[h][t][1][e], fp_mulmod_s(w[h][e], b1, m));
                            }
                        }
                    }
                }
            }
#pragma unroll
            for (int h = 0; h < GPT; h++) {
                if (h > 0 && !g1ok) break;
#pragma unroll
                for (int t = 0; t < TCH; t++) {
                    if (t < nt) {
                        uint64_t* z = Z + ((size_t)(t0 + t) * gs + g0 + h) * ctw + col + CPT * tx;
#pragma unroll
                        for (int e = 0; e < CPT; e++) {
                            z[e] = d2u(fp_canon(acc[h][t][0][e], m));
                            z[limb + e] = d2u(fp_canon(acc[h][t][1][e], m));
                        }
                    }
                }
            }
        } else {
            for (int h = 0; h < GPT; h++) {
                if (h > 0 && !g1ok) break;
                const int g = g0 + h;
                U128 acc[TCH][2][CPT];
#pragma unroll
                for (int t = 0; t < TCH; t++)
#pragma unroll
                    for (int e = 0; e < CPT; e++) acc[t][0][e] = acc[t][1][e] = U128{0, 0};
#pragma unroll 4
                for (int k = 0; k < KB; k++) {
                    const int j = k / bs, b = k - j * bs;
                    const uint64_t* wp = w_base + ((size_t)(j * gs + g) * bs + b) * limb;
                    uint64_t w[CPT];
#pragma unroll
                    for (int e = 0; e < CPT; e++) w[e] = __ldg(wp + e);
                    const uint64_t* sk = sB + (size_t)k * 2 * COLS + CPT * tx;
#pragma unroll
                    for (int t = 0; t < TCH; t++) {
                        if (t < nt) {
                            const uint64_t* st = sk + (size_t)t * KB * 2 * COLS;
#pragma unroll
                            for (int e = 0; e < CPT; e++) {
                                mac128(acc[t][0][e], w[e], st[e]);
                                mac128(acc[t][1][e], w[e], st[COLS + e]);
                            }
                        }
                    }
                }
#pragma unroll
                for (int t = 0; t < TCH; t++) {
                    if (t < nt) {
                        uint64_t* z = Z + ((size_t)(t0 + t) * gs + g) * ctw + col + CPT * tx;
#pragma unroll
                        for (int e = 0; e < CPT; e++) {
                            z[e] = reduce128(acc[t][0][e], p);
                            z[limb + e] = reduce128(acc[t][1][e], p);
                        }
                    }
                }
            }
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
        if (!x[i].data || ((uintptr_t)x[i].data & 31) || !x[i].is_ntt) return set_err(c, HE_EINVAL, "he_pmult_accum_bsgs: bad input %d", i);
        if (x[i].level != level) return set_err(c, HE_ELEVEL, "he_pmult_accum_bsgs: mixed levels");
    }
    for (int i = 0; i < n_groups * n_out; i++)
        if (!y[i].data || ((uintptr_t)y[i].data & 31))
            return set_err(c, HE_EINVAL, "he_pmult_accum_bsgs: null or unaligned output %d", i);
    if ((uintptr_t)d_pt & 31) return set_err(c, HE_EINVAL, "he_pmult_accum_bsgs: plaintexts not 32-byte aligned");
    if (level < 2) return set_err(c, HE_ELEVEL, "he_pmult_accum_bsgs: level %d cannot be rescaled", level);
    for (int b = 1; b < bs; b++)
        if (!c->rot_keys.count(galois_elt(c, stride * b)) && galois_elt(c, stride * b) != 1)
            return set_err(c, HE_ENOKEY, "he_pmult_accum_bsgs: no key for baby step %d", stride * b);
    for (int g = 1; g < gs; g++)
        if (!c->rot_keys.count(galois_elt(c, stride * bs * g)) && galois_elt(c, stride * bs * g) != 1)
            return set_err(c, HE_ENOKEY, "he_pmult_accum_bsgs: no key for giant step %d", stride * bs * g);

    const size_t ctw = (size_t)2 * level * N;
    const size_t nB = (size_t)n_groups * n_in * bs;
    // output blocks run in waves: each block needs n_groups gs ciphertexts of
    // sums Z; a wave holds as many blocks as fit in kBsgsWaveWords (at least
    // one)
    const size_t per_block = (size_t)n_groups * gs * ctw;
    const int wave = std::max(1, std::min(n_out, (int)(kBsgsWaveWords / per_block)));
    uint64_t* buf;
    int rc = scratch_slot(c, 3, ctw * nB + per_block * wave, &buf);
    if (rc) return rc;
    uint64_t* B = buf;
    uint64_t* Z = B + ctw * nB;  // [wave][n_groups][gs]

    // baby steps: B[t][j][b] = rot_{stride b}(X[t][j]), the rotations b >= 1
    // hoisted (one ModUp per input X[t][j])
    std::vector<he_ct> bout;
    std::vector<int32_t> bsteps;
    for (int b = 1; b < bs; b++) bsteps.push_back(stride * b);
    for (int t = 0; t < n_groups; t++)
        for (int j = 0; j < n_in; j++) {
            const he_ct& xi = x[t * n_in + j];
            uint64_t* dst0 = B + ((size_t)(t * n_in + j) * bs) * ctw;
            rc = check_cuda(c, cudaMemcpyAsync(dst0, xi.data, ctw * 8, cudaMemcpyDeviceToDevice, c->stream),
                            "bsgs copy");
            if (rc) return rc;
            for (int b = 1; b < bs; b++) bout.push_back(he_ct{dst0 + (size_t)b * ctw, level, xi.scale, 1});
        }
    if (bs > 1 && (rc = rotate_hoisted_many(c, x, n_groups * n_in, bsteps.data(), bs - 1, bout.data()))) return rc;

    const size_t pt_block = (size_t)n_in * gs * bs * level * N;
    // one token group: 2 columns per thread.  Several: 2 groups staged per
    // pass, measured against 1, 3 and 4 for FFN1 at 2048 tokens (190 ms of
    // products against 225, 193 and 214): with 4 the 98 KB of staging leaves
    // 2 blocks per SM; with 1 the weights are re-read 16 times and bind.
    const int tch = n_groups == 1 ? 1 : 2, cpt = tch == 1 ? 2 : 1;
    const int smem = tch * n_in * bs * 2 * kPmThreadsX * cpt * 8;
    if (smem > 200 * 1024) return set_err(c, HE_EINVAL, "he_pmult_accum_bsgs: n_in*bs = %d too large", n_in * bs);
    const int gpt = 2;  // giant steps per thread
    const dim3 pgrid((gs + kPmG * gpt - 1) / (kPmG * gpt), N / (kPmThreadsX * cpt), level);
    int fp_l = 0;
    for (int r = 0; r < level; r++) fp_l += fp_prime(c, r);
    for (int i0 = 0; i0 < n_out; i0 += wave) {
        const int w = std::min(wave, n_out - i0);
        for (int ii = 0; ii < w; ii++) {
            uint64_t* Zi = Z + (size_t)ii * n_groups * gs * ctw;
            const uint64_t* pti = d_pt + pt_block * (i0 + ii);
            prof_begin(c, HE_PROF_PMULT);
            if (tch == 1) {
                cudaFuncSetAttribute(k_pmult_accum<1, 2, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
                k_pmult_accum<1, 2, 2><<<pgrid, kPmThreadsX * kPmG, smem, c->stream>>>(
                    pti, B, Zi, n_groups, n_in, gs, bs, level, c->d_prime, c->d_fpmod, c->log_n);
            } else {
                cudaFuncSetAttribute(k_pmult_accum<2, 1, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
                k_pmult_accum<2, 1, 2><<<pgrid, kPmThreadsX * kPmG, smem, c->stream>>>(
                    pti, B, Zi, n_groups, n_in, gs, bs, level, c->d_prime, c->d_fpmod, c->log_n);
            }
            c->launches++;
            if ((rc = check_cuda(c, cudaGetLastError(), "pmult_accum"))) return rc;
            // weights of the block once per staged pass of token groups, the
            // rotated inputs once, the sums written once
            const double passes = (n_groups + tch - 1) / tch;
            const double macs_per_limb = 2.0 * N * (double)gs * n_groups * n_in * bs;
            prof_end(c, HE_PROF_PMULT, 8.0 * ((double)pt_block * passes + (double)ctw * nB +
                                              (double)ctw * n_groups * gs),
                     macs_per_limb * level, macs_per_limb * fp_l);
        }
        // Y = Z_0 + sum_{g>=1} rot_{stride bs g}(Z_g) for every output of the
        // wave, one ModDown per output, then one rescale for the wave
        std::vector<he_ct> zg, z0, yo;
        std::vector<int32_t> gsteps;
        std::vector<const uint64_t*> rin;
        std::vector<uint64_t*> rout;
        for (int g = 1; g < gs; g++) gsteps.push_back(stride * bs * g);
        for (int u = 0; u < w * n_groups; u++) {
            const int ii = u / n_groups, t = u - ii * n_groups;
            z0.push_back(he_ct{Z + (size_t)u * gs * ctw, level, 1.0, 1});
            for (int g = 1; g < gs; g++) zg.push_back(he_ct{Z + ((size_t)u * gs + g) * ctw, level, 1.0, 1});
            yo.push_back(he_ct{y[t * n_out + i0 + ii].data, level, 1.0, 1});
            rin.push_back(yo.back().data);
            rout.push_back(yo.back().data);
        }
        if ((rc = rotate_sum_many(c, zg.data(), w * n_groups, gs - 1, gsteps.data(), z0.data(), yo.data())))
            return rc;
        if ((rc = rescale_many(c, rin, rout, level))) return rc;
    }
    for (int i = 0; i < n_groups * n_out; i++) {
        y[i].level = level - 1;
        y[i].scale = (x[0].scale * pt_scale) / (double)c->primes[level - 1];
        y[i].is_ntt = 1;
    }
    return HE_OK;
}
