// The ModDown base conversion as a split-integer GEMM on the tensor cores.
//
// For one polynomial, coefficient c and target prime q_r (r < level):
//   out_r[c] = sum_k y_k[c] m_kr  (mod q_r),   y_k = [x_k (P/p_k)^-1]_{p_k},
//   m_kr = (P/p_k) mod q_r,
// then corrected by n_neg (-P mod q_r) for the sources y_k > p_k/2 (the
// centred conversion: sum_k (y_k - p_k [y_k > p_k/2]) (P/p_k)).
// With y_k = sum_a y_ka 256^a and m_kr = sum_b m_krb 256^b (bytes),
//   sum_k y_k m_kr = sum_sigma 256^sigma C_r,sigma,
//   C_r,sigma = sum_{k,a} y_ka m_kr,(sigma-a),
// which is a GEMM of unsigned bytes with 32-bit accumulation:
//   A [128 coefficients x 64]: row c holds the K sources y_k as their eight
//     little-endian bytes (column 8k + a) -- the residues as they are;
//   B [64 x 16 per target]: column (r, sigma) holds byte sigma - a of m_kr
//     at row 8k + a (zero outside the byte range);
// every C_r,sigma < 64 * 255^2 < 2^22.  The epilogue recombines the
// sixteen columns of a target exactly: for primes below 2^41 on the FP64
// pipe, W_j = C_2j + 256 C_2j+1 (j < 7) times the 14-bit parts of
// 2^(16 j) mod q_r (exact partial sums below 2^48), or on the integer pipe as a
// 128-bit value (the 60-bit q_0 always, and a share of the 40-bit targets,
// so that both pipes work).
//
// tcgen05 (Blackwell fifth-generation tensor cores): one thread issues
// tcgen05.mma.cta_group::1.kind::i8 (M = 128, N = 16 targets-per-round x 16,
// K = 32 bytes per instruction, two per round) from shared-memory operands in
// the K-major interleaved layout (8-row x 16-byte core matrices), the
// accumulators live in tensor memory and each warp reads its 32 lanes with
// tcgen05.ld.  The operands are this CTA's own shared memory, written with
// ordinary stores; no TMA and no multicast.  The completion wait is bounded:
// on expiry the kernel records an error word that he_sync reports as
// HE_ETIMEOUT, and frees its tensor memory.
#include "he_internal.h"
#include "ntt.cuh"

namespace he {

constexpr int kTcM = 128;          // coefficients per tile (MMA M)
constexpr int kTcK = 64;           // bytes of A per coefficient row (8 sources x 8 bytes)
constexpr int kTcCols = 16;        // accumulator columns per target (shifts 0..15)
constexpr int kTcTgtRound = 8;     // targets per MMA round: N = 128
constexpr int kTcTmemCols = kTcTgtRound * kTcCols;
constexpr int kTcMaxTargets = 64;

// Epilogue constants of one target prime.
struct TcTarget {
    double e[7][3];  // 14-bit parts of 2^(16 j) mod q (FP64 recombination)
    FpMod fm;
    uint64_t q, negp;  // -P mod q (centring correction)
    uint64_t one_shoup, r1, r1_shoup;
    int use_int;  // recombine on the integer pipe
    int pad;
};

// ---- tcgen05 / mbarrier wrappers (PTX ISA 8.6+, sm_100a)

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

// Shared-memory matrix descriptor, K-major, no swizzle: core matrices of 8
// rows x 16 bytes (128 contiguous bytes); lbo = byte distance of the two
// 16-byte K chunks of one instruction, sbo = byte distance of consecutive
// 8-row groups; version 1 (bits 46-47) as Blackwell requires.
__device__ __forceinline__ uint64_t umma_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((addr >> 4) & 0x3FFF) | ((uint64_t)((lbo >> 4) & 0x3FFF) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFF) << 32) | (1ull << 46);
}

// Instruction descriptor of kind::i8: D s32, A and B unsigned 8-bit, both K-major.
__host__ __device__ constexpr uint32_t umma_idesc_u8(int m, int n) {
    return (2u << 4) | (0u << 7) | (0u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

__device__ __forceinline__ void mma_i8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, int accum) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accum));
}

__device__ __forceinline__ void mma_commit(uint64_t* mbar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(mbar))
                 : "memory");
}

__device__ __forceinline__ void mbar_init(uint64_t* mbar, int count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(mbar)), "r"(count) : "memory");
}

// Bounded wait on phase `parity`; returns false if it gave up.
__device__ __forceinline__ bool mbar_wait(uint64_t* mbar, uint32_t parity) {
    const uint32_t a = smem_u32(mbar);
    for (int it = 0; it < (1 << 22); it++) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}\n"
            : "=r"(done)
            : "r"(a), "r"(parity)
            : "memory");
        if (done) return true;
    }
    return false;
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
          "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// byte offset of (row, 16-byte chunk kc) in a K-major interleaved operand of 4 chunks per row
__device__ __forceinline__ int umma_off(int row, int kc) { return ((row >> 3) * 4 + kc) * 128 + (row & 7) * 16; }

// Recombination of one target's sixteen columns (FP64 pipe, q < 2^41).
__device__ __forceinline__ double tc_combine_fp(const uint32_t (&v)[16], const TcTarget& t, uint32_t n_neg) {
    double s0 = 0.0, s1 = 0.0, s2 = 0.0;
#pragma unroll
    for (int j = 0; j < 7; j++) {
        const double w = u2d((uint64_t)v[2 * j] + ((uint64_t)v[2 * j + 1] << 8));  // < 2^31, exact
        s0 = __fma_rn(w, t.e[j][0], s0);
        s1 = __fma_rn(w, t.e[j][1], s1);
        s2 = __fma_rn(w, t.e[j][2], s2);
    }
    double acc = fp_reduce_s(s0, t.fm);
    acc = __dadd_rn(acc, fp_mulmod_s(s1, 16384.0, t.fm));      // 2^14 < q
    acc = __dadd_rn(acc, fp_mulmod_s(s2, 268435456.0, t.fm));  // 2^28 < q
    acc = __fma_rn((double)n_neg, u2d(t.negp), acc);            // < 2^44
    return fp_canon(acc, t.fm);
}

// The same on the integer pipe: the 128-bit value sum_sigma C_sigma 2^(8 sigma)
// (below 2^123: it equals sum_k y_k m_kr), reduced once.
__device__ __forceinline__ uint64_t tc_combine_int(const uint32_t (&v)[16], const TcTarget& t, uint32_t n_neg) {
    U128 acc = {0, 0};
#pragma unroll
    for (int s = 0; s < 16; s++) {
        const uint64_t c = v[s];
        const int sh = 8 * s;
        if (sh < 64)
            add128(acc, c << sh, sh > 40 ? c >> (64 - sh) : 0);
        else
            add128(acc, 0, c << (sh - 64));
    }
    DevPrime p;
    p.q = t.q;
    p.one_shoup = t.one_shoup;
    p.r1 = t.r1;
    p.r1_shoup = t.r1_shoup;
    const uint64_t r = reduce128(acc, p);
    const uint64_t w = (uint64_t)n_neg * t.negp;  // < 16 q < 2^64
    return add_mod(r, reduce64(w, p), t.q);
}

// Persistent: each CTA loads the byte matrix B and the target constants
// once, then loops over work items (128-coefficient tile, polynomial,
// output).  256 threads: for the staging, thread t takes coefficient t % 128
// and sources 4 (t / 128) .. +3; in the epilogue warp w reads tensor-memory
// lanes 32 (w % 4) .. +31 (its coefficients) and recombines the targets of
// its half, t = w / 4 (mod 2), two targets' columns loaded per wait.
constexpr int kTcThreads = 256;

__global__ void __launch_bounds__(kTcThreads) k_moddown_conv_tc(const uint64_t* __restrict__ u,
                                                               uint64_t* __restrict__ tmp, int level, int L, int K,
                                                               int n_md, const DevPrime* __restrict__ pr,
                                                               const ulonglong2* __restrict__ pcoef,
                                                               const uint8_t* __restrict__ btab,
                                                               const TcTarget* __restrict__ tcon,
                                                               int* __restrict__ err, int logn) {
    __shared__ __align__(1024) uint8_t sA[kTcM * kTcK];
    extern __shared__ __align__(1024) uint8_t dyn[];
    uint8_t* sB = dyn;  // [level x 16 rows][64 bytes], K-major interleaved
    TcTarget* sT = reinterpret_cast<TcTarget*>(dyn + (size_t)level * kTcCols * kTcK);
    __shared__ uint64_t mbar;
    __shared__ uint32_t tmem_base;
    __shared__ uint32_t s_neg[2][kTcM];
    const int N = 1 << logn;
    const int tid = threadIdx.x, warp = tid >> 5;
    const int n_rows = level + K;
    const int tiles = N / kTcM, items = tiles * 2 * n_md;

    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base)),
                     "r"(kTcTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (tid == 0) {
        mbar_init(&mbar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    {
        const uint4* src = reinterpret_cast<const uint4*>(btab);
        uint4* dst = reinterpret_cast<uint4*>(sB);
        for (int idx = tid; idx < level * kTcCols * kTcK / 16; idx += kTcThreads) dst[idx] = src[idx];
        for (int r = tid; r < level; r += kTcThreads) sT[r] = tcon[r];
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = tmem_base;
    const uint32_t lane_addr = tbase + ((uint32_t)((warp & 3) * 32) << 16);
    const int half = warp >> 2, row = tid & (kTcM - 1), shalf = tid / kTcM;
    uint32_t phase = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < items && ok; it += gridDim.x) {
        const int tile = it % tiles, rest = it / tiles, poly = rest & 1, i = rest >> 1;
        // A: sources 4 shalf .. 4 shalf + 3 of coefficient `row`
        {
            const int c = tile * kTcM + row;
            const uint64_t* x = u + (((size_t)i * 2 + poly) * n_rows + level) * N + c;
            uint32_t neg = 0;
#pragma unroll
            for (int kk = 0; kk < 4; kk++) {
                const int k = 4 * shalf + kk;
                uint64_t y = 0;
                if (k < K) {
                    const uint64_t p = pr[L + k].q;
                    const ulonglong2 w = pcoef[k];
                    y = mul_shoup(x[(size_t)k * N], w.x, w.y, p);
                    neg += y > (p >> 1) ? 1u : 0u;
                }
                *reinterpret_cast<uint64_t*>(sA + umma_off(row, k >> 1) + (k & 1) * 8) = y;
            }
            s_neg[shalf][row] = neg;
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // stores visible to the tensor cores
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        const uint32_t n_neg = s_neg[0][(warp & 3) * 32 + (tid & 31)] + s_neg[1][(warp & 3) * 32 + (tid & 31)];
        uint64_t* out = tmp + (((size_t)i * 2 + poly) * level) * N + tile * kTcM + (warp & 3) * 32 + (tid & 31);
        const int rounds = (level + kTcTgtRound - 1) / kTcTgtRound;
        for (int rd = 0; rd < rounds; rd++) {
            const int r0 = rd * kTcTgtRound, nt = min(kTcTgtRound, level - r0);
            if (tid == 0) {
                const uint32_t idesc = umma_idesc_u8(kTcM, nt * kTcCols);
                for (int ks = 0; ks < 2; ks++) {
                    const uint64_t ad = umma_desc(smem_u32(sA) + ks * 2 * 128, 128, 512);
                    const uint64_t bd = umma_desc(smem_u32(sB) + (r0 * kTcCols / 8) * 512 + ks * 2 * 128, 128, 512);
                    mma_i8(tbase, ad, bd, idesc, ks);
                }
                mma_commit(&mbar);
            }
            ok = mbar_wait(&mbar, phase);
            phase ^= 1;
            tc_fence_after();
            if (ok) {
                // this half's targets of the round: t = half, half + 2, ...
                for (int t = half; t < nt; t += 4) {
                    uint32_t v[16], w2[16];
                    const bool two = t + 2 < nt;
                    tmem_ld16(lane_addr + t * kTcCols, v);
                    if (two) tmem_ld16(lane_addr + (t + 2) * kTcCols, w2);
                    tmem_ld_wait();
                    const TcTarget& T = sT[r0 + t];
                    out[(size_t)(r0 + t) * N] =
                        T.use_int ? tc_combine_int(v, T, n_neg) : d2u(tc_combine_fp(v, T, n_neg));
                    if (two) {
                        const TcTarget& T2 = sT[r0 + t + 2];
                        out[(size_t)(r0 + t + 2) * N] =
                            T2.use_int ? tc_combine_int(w2, T2, n_neg) : d2u(tc_combine_fp(w2, T2, n_neg));
                    }
                }
            }
            tc_fence_before();
            __syncthreads();  // tensor memory and A free again
            tc_fence_after();
            ok = __syncthreads_and(ok);
            if (!ok) break;
        }
    }
    if (!ok && tid == 0) atomicExch(err, 1);
    __syncthreads();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tbase), "r"(kTcTmemCols) : "memory");
}

// ---------------------------------------------------------------- host side

typedef unsigned __int128 u128;

static uint64_t t_mulmod(uint64_t a, uint64_t b, uint64_t m) { return (uint64_t)((u128)a * b % m); }

int moddown_tc_setup(he_ctx* c) {
    const int L = c->L, K = c->K;
    if (L > kTcMaxTargets || K > 8) return HE_OK;  // the GEMM form covers up to 8 special primes
    // B: row (r, sigma) of target r, byte 8k + a = byte (sigma - a) of (P/p_k) mod q_r
    std::vector<uint8_t> b((size_t)L * kTcCols * kTcK, 0);
    std::vector<TcTarget> tc(L);
    for (int r = 0; r < L; r++) {
        const uint64_t q = c->primes[r];
        for (int k = 0; k < K; k++) {
            uint64_t m = 1;
            for (int k2 = 0; k2 < K; k2++)
                if (k2 != k) m = t_mulmod(m, c->primes[L + k2] % q, q);
            for (int a = 0; a < 8; a++)
                for (int s = a; s < kTcCols; s++) {
                    const int bb = s - a;
                    const uint8_t byte = bb < 8 ? (uint8_t)(m >> (8 * bb)) : 0;
                    const int row = r * kTcCols + s, col = 8 * k + a;
                    b[((row >> 3) * 4 + (col >> 4)) * 128 + (row & 7) * 16 + (col & 15)] = byte;
                }
        }
        TcTarget& t = tc[r];
        const DevPrime& p = c->hprime[r];
        t.q = q;
        t.negp = (q - c->h_Pmod[r]) % q;
        t.one_shoup = p.one_shoup;
        t.r1 = p.r1;
        t.r1_shoup = p.r1_shoup;
        t.fm = FpMod{(double)q, 2.0 * (double)q, 1.0 / (double)q, 0.0};
        for (int j = 0; j < 7; j++) {
            uint64_t e = 1;
            for (int s = 0; s < 16 * j; s++) e = t_mulmod(e, 2, q);
            t.e[j][0] = (double)(e & 0x3FFF);
            t.e[j][1] = (double)((e >> 14) & 0x3FFF);
            t.e[j][2] = (double)(e >> 28);
        }
        // the integer pipe takes q_0 (60-bit) and every third 40-bit target
        t.use_int = q >= kFpPrimeLimit || (r % 3 == 1);
        t.pad = 0;
    }
    int rc = check_cuda(c, cudaMalloc(&c->d_tc_btab, b.size()), "tensor-core conversion table");
    if (!rc) rc = check_cuda(c, cudaMemcpy(c->d_tc_btab, b.data(), b.size(), cudaMemcpyHostToDevice), "tc table");
    if (!rc) rc = check_cuda(c, cudaMalloc(&c->d_tc_tgt, tc.size() * sizeof(TcTarget)), "tc targets");
    if (!rc)
        rc = check_cuda(c, cudaMemcpy(c->d_tc_tgt, tc.data(), tc.size() * sizeof(TcTarget), cudaMemcpyHostToDevice),
                        "tc targets");
    return rc;
}

bool moddown_tc_available(const he_ctx* c) { return c->d_tc_btab != nullptr; }

int moddown_conv_tc(he_ctx* c, const uint64_t* u, uint64_t* tmp, int n_md, int level) {
    const size_t smem = (size_t)level * kTcCols * kTcK + (size_t)level * sizeof(TcTarget);
    cudaFuncSetAttribute(k_moddown_conv_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)((size_t)kTcMaxTargets * (kTcCols * kTcK + sizeof(TcTarget))));
    // persistent CTAs: four per SM (tensor memory: 128 of 512 columns each)
    const int items = (c->N / kTcM) * 2 * n_md;
    const int grid = items < 4 * c->sm_count ? items : 4 * c->sm_count;
    k_moddown_conv_tc<<<grid, kTcThreads, smem, c->stream>>>(u, tmp, level, c->L, c->K, n_md, c->d_prime,
                                                            c->d_md_pcoef, (const uint8_t*)c->d_tc_btab,
                                                            (const TcTarget*)c->d_tc_tgt, c->d_err, c->log_n);
    c->launches++;
    return check_cuda(c, cudaGetLastError(), "moddown_conv_tc");
}

}  // namespace he
