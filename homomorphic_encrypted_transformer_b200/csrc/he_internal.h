// Internal state of the RNS-CKKS engine.  Not part of the ABI.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include <map>
#include <string>
#include <vector>

#include "../../include/he.h"
#include "kernels.cuh"
#include "modarith.cuh"

namespace he {

constexpr int kMaxPrimes = 64;
constexpr int kMaxDevices = 64;

// ModUp fast base conversion of one digit at one level, on device:
//   y_i = [x_i * qhat_inv_i]_{q_i} for the digit's source primes,
//   out_t = sum_i y_i * (qhat_i mod t) for every row t of Q_level and P
//   (rows of the digit itself reproduce x: the sum collapses to x_t there).
struct ConvTable {
    int n_src;
    int src_row;            // first row of the digit (its primes are rows src_row..src_row+n_src-1)
    ulonglong2* d_src;      // [n_src] {qhat_inv_i mod q_i, shoup}
    ulonglong2* d_mat;      // [n_src][level + K] {(qhat_i mod t) 2^64 mod t, qhat_i mod t}
};

struct FpMod;  // FP64 constants of a prime below 2^41 (ntt.cuh)

struct Key {
    // [digits][2][L+K][N] (b then a): rows of primes below 2^41 as doubles,
    // the others in Montgomery form (value * 2^64 mod p).  With seeded_a:
    // [digits][L+K][N] b-halves only, followed by the a-halves' stream starts
    // s0 [digits][L+K] (keyseed.cuh), from which the kernels regenerate a.
    uint64_t* d = nullptr;
    bool seeded_a = false;
};

// Do the context's keys store only b-halves?  (All keys of a context have
// one form.)
bool keys_seeded_a(const he_ctx* c);

// Stream start of row prime_index of digit `digit` of a seeded a-half (sampler.cpp).
uint64_t seeded_a_stream_start(uint64_t seed, uint64_t key_id, int digit, int prime_index);

struct ProfSlot {
    double ms = 0;
    long long launches = 0;
    double bytes = 0, mults = 0, mults_fp = 0;
};

struct ProfPending {
    int cls;
    cudaEvent_t a, b;
    double bytes, mults, mults_fp;
};

}  // namespace he

struct he_ctx {
    int log_n = 0, N = 0, L = 0, K = 0, dnum = 0, alpha = 0;
    std::vector<uint64_t> primes;  // L + K, prime index space
    std::vector<uint64_t> psi;
    cudaStream_t stream = nullptr;
    std::string err;
    int device = 0;
    int sm_count = 148;

    std::vector<he::DevPrime> hprime;
    he::DevPrime* d_prime = nullptr;   // [L+K]
    ulonglong2* d_tw_fwd = nullptr;    // [L+K][N] {psi^brev(i), shoup}
    ulonglong2* d_tw_inv = nullptr;    // [L+K][N] {psi^-brev(i), shoup}; entry 1 times N^-1
    ulonglong2* d_inv_last = nullptr;  // [L+K] {N^-1, shoup}
    double* d_twd_fwd = nullptr;       // [L+K][N] forward twiddles as doubles (exact below 2^53)
    double* d_twd_inv = nullptr;       // [L+K][N] inverse twiddles as doubles; entry 1 times N^-1
    he::FpMod* d_fpmod = nullptr;      // [L+K] {q, 2q, 1/q, N^-1} as doubles

    std::vector<std::vector<he::ConvTable>> modup;  // [level][digit], level 1..L
    ulonglong2* d_md_pcoef = nullptr;  // [K] {(P/p_k)^-1 mod p_k, shoup}
    ulonglong2* d_md_mat = nullptr;    // [K][L] {(P/p_k) 2^64 mod q_i, (P/p_k) mod q_i}
    uint64_t* d_md_negP = nullptr;     // [L] -P mod q_i (correction of a negative centred term)
    ulonglong2* d_md_pinv = nullptr;   // [L] {P^-1 mod q_i, shoup}
    std::vector<uint64_t> h_Pmod;      // [L+K] P mod prime (0 on the p's)
    ulonglong2* d_rs_inv = nullptr;    // [L][L] {q_l^-1 mod q_i, shoup}
    uint64_t* d_rs_qmod = nullptr;     // [L][L] q_l mod q_i

    std::map<uint64_t, he::Key> rot_keys;  // by Galois element
    he::Key relin;

    uint64_t* scratch[5] = {nullptr, nullptr, nullptr, nullptr, nullptr};
    size_t scratch_words[5] = {0, 0, 0, 0, 0};
    int ks_slot = 0;                    // scratch slot of key switching (4 on the auxiliary stream)
    cudaStream_t aux = nullptr;         // second stream of a split rotation batch
    cudaEvent_t ev_fork = nullptr, ev_join = nullptr;
    uint64_t* noalloc_scratch = nullptr;  // device address of he_rescale_noalloc's fixed array
    int* d_err = nullptr;                 // device error word: a bounded device wait gave up (he_sync reports it)
    void* d_tc_btab = nullptr;            // tensor-core ModDown conversion: byte matrix B (moddown_tc.cu)
    void* d_tc_tgt = nullptr;             // and its per-target recombination constants
    bool tc_moddown = false;              // ModDown conversion on the tensor cores
    uint64_t* io_buf = nullptr;  // device staging of the host-buffer entry point
    size_t io_words = 0;
    cudaStream_t io_h2d = nullptr, io_d2h = nullptr;  // its copy streams (one per direction)
    cudaEvent_t io_ev[6] = {};                         // per staging buffer: uploaded, rotated, downloaded

    bool prof_on = false;
    he::ProfSlot prof[HE_PROF_N];
    std::vector<he::ProfPending> prof_pending;
    std::vector<cudaEvent_t> ev_pool;
    long long launches = 0;
};

namespace he {

int set_err(he_ctx* c, int code, const char* fmt, ...);
int check_cuda(he_ctx* c, cudaError_t e, const char* what);

// Brackets launches of one class with events; prof_end records the
// algorithmic work of what it closes: HBM bytes, modular multiplications,
// and how many of those run on the FP64 pipe (primes below 2^41).
void prof_begin(he_ctx* c, int cls);
int prof_end(he_ctx* c, int cls, double bytes = 0, double mults = 0, double mults_fp = 0);

// Rows 0..n_rows-1 of a RowSet whose prime takes the FP64 path.
long long fp_rows(const he_ctx* c, const RowSet& rs, int n_rows);
bool fp_prime(const he_ctx* c, int prime_idx);

uint64_t galois_elt(const he_ctx* c, int32_t step);

RowSet rowset(uint64_t* base, long long group_stride, int per_group, const int* prime_idx);
RowSet rowset_contig(uint64_t* base, int per_group, int N, const std::vector<int>& prime_idx);
std::vector<int> prime_range(int first, int count);
// Rows of Q_level then all of P: 0..level-1, L..L+K-1
std::vector<int> ext_primes(const he_ctx* c, int level);

int ntt_fwd_set(he_ctx* c, const RowSet& rs, int n_rows);
int ntt_inv_set(he_ctx* c, const RowSet& rs, int n_rows);
// Single passes, for callers that fuse the other pass with their own work:
// the forward column pass (stages 0..S1-1) and the inverse column pass
// (stages S1-1..0, scaled by N^-1).
int ntt_fwd_cols_set(he_ctx* c, const RowSet& rs, int n_rows);
int ntt_inv_cols_set(he_ctx* c, const RowSet& rs, int n_rows);

// Key switching of polynomials d[i] (evaluation domain, [level][N] each) with
// one key.  Writes out[i] = [2][level][N]:
//   out0 = KS(d)_0 + add0[i],  out1 = KS(d)_1 + add1[i]   (null adds are skipped).
// With galois != 0 the switched polynomial is sigma_galois(d[i]), and add0 is
// also read through sigma_galois when sig_add0 is set (rotation).
// Entry i switches d[i] with key[i]; entries that share a key should be
// adjacent (the inner product then reads each key tile once from DRAM for
// all of them).
struct KsIoList {
    bool sig_add0 = false;
    std::vector<uint64_t> galois;  // 0: no automorphism
    std::vector<const uint64_t*> key;
    std::vector<const uint64_t*> d;
    std::vector<uint64_t*> out;
    std::vector<const uint64_t*> add0;
    std::vector<const uint64_t*> add1;
    // Hoisted mode (non-empty hoist_d): ModUp runs once on each hoist_d[m]
    // (evaluation rows, no automorphism) and output i takes the raised digits
    // of hoist_d[hoist_src[i]] through sigma_{galois[i]}; d[i] must then be
    // hoist_d[hoist_src[i]].
    std::vector<const uint64_t*> hoist_d;
    std::vector<int> hoist_src;
    // Summed mode (sum_terms > 0): the key switches o*sum_terms ..
    // o*sum_terms + sum_terms - 1 share output o: their inner products are
    // added in Q_level and P and brought down by one ModDown; out, add0 and
    // add1 then hold one entry per output.
    int sum_terms = 0;
};
int key_switch(he_ctx* c, int level, const KsIoList& io);
// key_switch of a plain (not hoisted, not summed) batch in two halves on two
// streams, forked from and joined back into the context's stream.
int key_switch_split(he_ctx* c, int level, const KsIoList& io);
int key_switch_chunk(he_ctx* c, int n, int level, const KsIoList& io);
size_t key_switch_scratch_words(const he_ctx* c, int n_raised, int n, int level);
// out_i = rot_{steps_i}(in_i)
int rotate_many(he_ctx* c, const he_ct* in, const int32_t* steps, he_ct* out, int n);
int rotate_hoisted_many(he_ctx* c, const he_ct* in, int n_in, const int32_t* steps, int n_steps, he_ct* out);
int rotate_sum_many(he_ctx* c, const he_ct* z, int n_out, int n_terms, const int32_t* steps, const he_ct* base,
                    he_ct* out);
int rotate_sum_hoisted_many(he_ctx* c, const he_ct* in, int n_in, const int32_t* steps, int n_steps, he_ct* out);

// Scratch slots: 0 = key switching internals, 1 = rescale temporaries,
// 2 = HMult temporaries, key generation and the pre-sums of the summed
// rotations, 3 = driver buffers (polynomial evaluation, BSGS), 4 = key
// switching on the auxiliary stream (the second half of a split rotation
// batch).  A call only uses slots below the ones its callers hold.
constexpr int kScratchSlots = 5;
int scratch_slot(he_ctx* c, int slot, size_t words, uint64_t** out);

// Packed wire format of ciphertexts (wire.cu): bytes of one ciphertext at
// `level`; device unpacking of n packed ciphertexts into ct_i and packing
// back (wire: device, 8-byte aligned, ciphertexts back to back).
size_t wire_bytes(const he_ctx* c, int level);
int wire_unpack_many(he_ctx* c, const uint8_t* wire, int level, const std::vector<uint64_t*>& ct);
int wire_pack_many(he_ctx* c, const std::vector<const uint64_t*>& ct, int level, uint8_t* wire);

// out[i] = rescale(in[i]) for n ciphertexts at `level` (out may equal in),
// plus addend[i] (a ciphertext at level - 1) when addend is not empty.
int rescale_many(he_ctx* c, const std::vector<const uint64_t*>& in, const std::vector<uint64_t*>& out, int level,
                 const std::vector<const uint64_t*>& addend = {});
// Batched helpers of the drivers (ops.cu): HMult + relinearisation + rescale
// of pairs at `level` (a_i, b_i with at least `level` limbs per polynomial:
// their c1 starts at limb room_a / room_b, 0 = level; out_i may be a_i or
// b_i of the same i; plus addend_i at level - 1 when addend is not empty); out_i = a_i +
// b_i at lv limbs (out may equal a); out_i = in_i keeping limbs < lv (out !=
// in).
// Terms added to the relinearised products before their rescale (at most
// three): term j of product i is in[j][i], at level lin[j] >= the product's
// level and read at that level, times the integer K[j]; with add_k0, K0 is
// added to c0 after the rescale.
struct PreRescaleTerms {
    std::vector<std::vector<const uint64_t*>> in;
    std::vector<int> lin;
    std::vector<int64_t> K;
    bool add_k0 = false;
    int64_t K0 = 0;
};
int hmrr_many(he_ctx* c, const std::vector<const uint64_t*>& a, const std::vector<const uint64_t*>& b,
              const std::vector<uint64_t*>& out, int level, int room_a = 0, int room_b = 0,
              const std::vector<const uint64_t*>& addend = {}, const PreRescaleTerms* pre = nullptr);
// out = rescale(relinearise(sum_i tensor(a_i, b_i))) of the pairs at `level`
// (a_i, b_i as in hmrr_many; out apart from every input).
int hmrr_sum(he_ctx* c, const std::vector<const uint64_t*>& a, const std::vector<const uint64_t*>& b, uint64_t* out,
             int level, int room_a = 0, int room_b = 0);
int add_many(he_ctx* c, const std::vector<const uint64_t*>& a, const std::vector<const uint64_t*>& b,
             const std::vector<uint64_t*>& o, int lv);
int drop_many(he_ctx* c, const std::vector<const uint64_t*>& in, const std::vector<uint64_t*>& out, int lin, int lv);

// Set-up of he_rescale_noalloc at context creation (noalloc.cu): looks up
// the device address of its fixed scratch array on the context's device and
// loads every kernel that entry point launches, so that its calls allocate
// nothing, the first one included.
int noalloc_setup(he_ctx* c);
// ModDown base conversion as a split-integer GEMM on the tensor cores
// (moddown_tc.cu): tables at context creation, then one launch per key switch
// writing the same canonical residues as k_moddown_conv.
int moddown_tc_setup(he_ctx* c);
bool moddown_tc_available(const he_ctx* c);
int moddown_conv_tc(he_ctx* c, const uint64_t* u, uint64_t* tmp, int n_md, int level);
// Loads the transform kernels of the context's ring degree (cudaFuncGetAttributes).
int ntt_preload(he_ctx* c);

}  // namespace he
