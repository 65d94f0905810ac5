/*
 * he.h -- C ABI of the B200 RNS-CKKS polynomial engine (libhe.so).
 *
 * The engine is the data-parallel hot path under encrypted Transformer
 * inference as AEGIS describes it (AEGIS: Scaling Long-Sequence Homomorphic
 * Encrypted Transformer Inference, gist.science summary): CKKS ciphertexts
 * are RNS polynomials split into modulus limbs along a modulus chain, and
 * the operations that dominate are key switching and rotation (section 1
 * "Problem", items 2-3), the local plaintext-weight x ciphertext product of
 * the FFN (section 2.2) and the polynomial approximation of Softmax (section
 * 2.3).  The pages define no API; the calls below follow that statement of
 * the problem.  Below the CKKS level the arithmetic is the textbook one:
 * Cheon-Han-Kim-Kim-Song, "A Full RNS Variant of Approximate Homomorphic
 * Encryption" (SAC 2018) and the hybrid key switching of Han-Ki (CT-RSA 2020).
 *
 * Conventions for every call
 *  - Return value: HE_OK (0) or a negative HE_E* code; he_last_error(ctx)
 *    then holds a one-line message.  Argument errors are reported before
 *    anything is enqueued.  CUDA errors of enqueued work are reported by the
 *    next call that checks the stream, or by he_sync().
 *  - Work is enqueued on the context's CUDA stream and is asynchronous
 *    unless stated otherwise.  Host buffers passed to a call may be reused
 *    as soon as it returns.
 *  - Residues are uint64 in canonical form [0, q).  N = 2^log_n.
 *  - Prime index space: 0..n_q-1 are q_0..q_{L-1} (the ciphertext modulus
 *    chain), n_q..n_q+n_p-1 are the special primes p_0..p_{K-1}.
 *  - A polynomial "limb" is N contiguous residues for one prime.  A
 *    ciphertext at level l (l limbs q_0..q_{l-1}) is [2][l][N] uint64,
 *    limb-major, c0 then c1, in the evaluation (NTT) domain: storage index j
 *    holds the value at psi^(2*brev(j)+1), psi the smallest primitive 2N-th
 *    root of unity mod the limb's prime.
 *  - Ciphertext and plaintext buffers are device memory owned by the caller,
 *    32-byte aligned.  The context owns its tables, keys and scratch, and
 *    frees them in he_ctx_destroy().
 *  - A context is not thread-safe: one host thread at a time.
 */
#ifndef HE_B200_H
#define HE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define HE_OK 0
#define HE_EINVAL (-1)   /* bad argument (null pointer, size, alignment, unsupported value) */
#define HE_ELEVEL (-2)   /* level or scale mismatch between operands */
#define HE_ENOKEY (-3)   /* no rotation / relinearisation key uploaded for the request */
#define HE_EDOMAIN (-4)  /* operand not in the evaluation (NTT) domain */
#define HE_ENOMEM (-5)   /* device allocation failed */
#define HE_ECUDA (-6)    /* CUDA runtime error (message in he_last_error) */
#define HE_ETIMEOUT (-7) /* a bounded device wait gave up (reported by he_sync) */

#define HE_KEY_ROTATION 0
#define HE_KEY_RELIN 1

typedef struct he_ctx he_ctx;

/*
 * Parameter set.  The pages fix none; the primes follow this rule unless
 * given explicitly: every prime = 1 (mod 2N); a downward scan per bit size
 * yields, in order, q_0 (q0_bits), p_0..p_{K-1} (p_bits), q_1..q_{L-1}
 * (q_bits).  alpha = ceil(n_q / dnum) primes per key-switching digit.
 * Requires 10 <= log_n <= 16, 1 <= n_q, 1 <= n_p, n_q + n_p <= 64,
 * 1 <= dnum <= n_q, and n_p >= alpha (the special modulus must cover a digit).
 * Zero bit sizes select 60 / 40 / 60.
 */
typedef struct {
    int log_n;
    int n_q;
    int n_p;
    int dnum;
    int q0_bits;
    int q_bits;
    int p_bits;
    const uint64_t* q; /* optional host array of n_q primes, or NULL */
    const uint64_t* p; /* optional host array of n_p primes, or NULL */
} he_params;

/* A ciphertext: data is a device pointer to [2][level][N] uint64, 32-byte
 * aligned (the transform passes move residues four at a time with 256-bit
 * accesses); calls reject other pointers with HE_EINVAL. */
typedef struct {
    uint64_t* data;
    int level;
    double scale;
    int is_ntt;
} he_ct;

/* Context ------------------------------------------------------------------ */

/* Host only (no device work): validates params and writes the n_q + n_p
 * primes (prime index order) and their psi.  Either output may be NULL. */
int he_derive_primes(const he_params* params, uint64_t* primes_out, uint64_t* psi_out);

/* Builds the RNS tables on the host (primes, roots, twiddles, conversion
 * constants) and uploads them.  cuda_stream: a cudaStream_t or NULL for the
 * legacy default stream.  Synchronous.  *out receives the context.
 * Environment: HE_MODDOWN_CONV=tc makes the context's key switches run the
 * ModDown base conversion as a split-integer GEMM on the tensor cores
 * (identical residues; slower than the default FP64 kernel on B200). */
int he_ctx_create(const he_params* params, void* cuda_stream, he_ctx** out);
int he_ctx_destroy(he_ctx* ctx);
/*
 * Later calls enqueue on cuda_stream.  CUDA graph capture: the operation
 * calls (transforms, rotations, HMult, rescale, the BSGS product, the
 * degree-15 evaluation, attention, the helpers) launch kernels and record
 * events only, so a sequence of them can be captured on the context's
 * stream and replayed, provided each call already ran once eagerly with
 * the same sizes (that run sizes the context's scratch).  A call that would
 * have to grow its scratch while the stream is being captured returns
 * HE_EINVAL before any CUDA work, leaving the capture intact.  Key
 * generation, key download, the host-buffer entry points, he_sync and
 * profiling synchronise and cannot be captured.
 */
int he_set_stream(he_ctx* ctx, void* cuda_stream);
/* Blocks until the context's stream is idle; returns HE_ECUDA on a pending
 * CUDA error, HE_ETIMEOUT if a bounded device wait gave up. */
int he_sync(he_ctx* ctx);
const char* he_last_error(const he_ctx* ctx);
/* Host copies of the n_q + n_p primes / of their psi (smallest primitive 2N-th roots). */
int he_get_primes(const he_ctx* ctx, uint64_t* out);
int he_get_psi(const he_ctx* ctx, uint64_t* out);

/* Keys --------------------------------------------------------------------- */

/*
 * Computes one switching key on the device from caller-supplied random
 * parts and keeps it in the context (hybrid key switching, Han-Ki section 3):
 *   for digit j < ceil(L/alpha), on every prime of Q and P,
 *     b_j = -a_j s + e_j + g_j s',  g_j = P on the primes of digit j, 0 elsewhere;
 *   s' = sigma_k(s), k = 5^(step mod N/2) mod 2N   (kind HE_KEY_ROTATION)
 *   s' = s^2                                        (kind HE_KEY_RELIN, step ignored)
 * s: host int8[N] ternary secret coefficients.
 * a: host uint64 [dnum][n_q+n_p][N], uniform residues, used as evaluation-domain values.
 * e: host int32 [dnum][N], small error coefficients.
 * Only the first ceil(L/alpha) digits of a and e are read.  Uploading a key
 * that exists replaces it.  Synchronous.
 */
int he_keygen_upload(he_ctx* ctx, int kind, int32_t step, const int8_t* s, const uint64_t* a,
                     const int32_t* e);
/*
 * Key generation from a seed (host sampling, then he_keygen_upload's device
 * computation): the secret and every key's random parts are drawn from
 * SplitMix64 streams of `seed` by the rule below, one rotation key per
 * entry of rot_steps (HE_EINVAL for a step whose Galois element is 1) and
 * the relinearisation key when with_relin != 0.  The context keeps the keys;
 * the caller keeps the seed, from which he_sample_secret gives the secret
 * for encryption and decryption.  Synchronous.
 *
 * Sampling rule (the pages name only the distributions; this fixes them so
 * that a seed determines every key):
 *  - SplitMix64 (Steele, Lea, Flood, "Fast splittable pseudorandom number
 *    generators", OOPSLA 2014): state += 0x9E3779B97F4A7C15, output
 *    mix64(state); one stream per object with initial state
 *    mix64(seed + 0x9E3779B97F4A7C15 (1 + obj)),
 *    obj = tag 2^56 + key_id 2^24 + digit 2^8 + prime_index, where
 *    tag 1 = the secret (other fields 0), 2 = the uniform half a of digit
 *    `digit` of a key on prime `prime_index`, 3 = the error of digit `digit`
 *    (prime_index 0); key_id = the Galois element 5^(step mod N/2) mod 2N of
 *    a rotation key, 2 for the relinearisation key.
 *  - uniform residue mod q: draws x >> (64 - bitlen(q)) until one is < q;
 *  - ternary secret coefficient: draws x until x != 2^64 - 1, then (x mod 3) - 1;
 *  - error coefficient: discrete Gaussian with sigma = 3.2 on [-19, 19]:
 *    -19 + the number of thresholds T_i <= x (he_gaussian_cdt).
 * The key itself is he_keygen_upload's: s' = sigma_k(s) or s^2,
 * b_j = -a_j s + e_j + P [prime in digit j] s'.
 */
int he_keygen_seeded(he_ctx* ctx, uint64_t seed, const int32_t* rot_steps, int n_steps, int with_relin);
/*
 * he_keygen_seeded with flags.  HE_KEYGEN_SEEDED_A: every key keeps only its
 * b-half (plus one 8-byte stream start per digit and prime) and the
 * key-switching kernels regenerate the uniform a-half where they read it
 * (the optional seeded a-halves of the hoisted-rotation design: half the key
 * bytes in HBM and per key switch).  a_j is then drawn by the counter rule
 * below instead of the sequential stream of tag 2; s and e are drawn as
 * above, and b_j = -a_j s + e_j + P [prime in digit j] s' as before.
 *  - stream start s0 = mix64(seed + 0x9E3779B97F4A7C15 (1 + obj)),
 *    obj = 4 2^56 + key_id 2^24 + digit 2^8 + prime_index;
 *  - coefficient i (evaluation-domain storage index) of that row is the
 *    first x_t = mix64(s0 + 0x9E3779B97F4A7C15 (1 + i + t N)) >> (64 -
 *    bitlen(q)), t = 0..63, with x_t < q, or x_63 - q if there is none.
 * All keys of a context have one form: HE_EINVAL if the context already
 * holds keys of the other form (he_keygen_upload makes stored-a keys).
 * he_key_download returns such a key whole (a regenerated on the device).
 */
#define HE_KEYGEN_SEEDED_A 1
int he_keygen_seeded_ex(he_ctx* ctx, uint64_t seed, const int32_t* rot_steps, int n_steps, int with_relin,
                        int flags);
/* Host only (no context, no device): the ternary secret of a seed, int8[N] (N = 2^log_n). */
int he_sample_secret(uint64_t seed, int log_n, int8_t* s_out);
/* Host only: the random parts of one switching key as he_keygen_seeded draws
 * them: a uint64 [digits][n_primes][N] (uniform mod primes[r] on row r) and
 * e int32 [digits][N].  key_id < 2^32. */
int he_sample_key_draws(uint64_t seed, uint64_t key_id, int log_n, const uint64_t* primes, int n_primes, int digits,
                        uint64_t* a_out, int32_t* e_out);
/* Host only: the a-half of one key as HE_KEYGEN_SEEDED_A defines it,
 * uint64 [digits][n_primes][N] (row r uniform mod primes[r], prime_index r).
 * key_id < 2^32. */
int he_sample_key_a_seeded(uint64_t seed, uint64_t key_id, int log_n, const uint64_t* primes, int n_primes,
                           int digits, uint64_t* a_out);
/* Host only: the 38 thresholds T_i = floor(2^64 C_i) of the error sampler,
 * C_i = P(e <= -19 + i) for the discrete Gaussian of sigma 3.2 on [-19, 19]. */
int he_gaussian_cdt(uint64_t* out);
/* Copies a key back in canonical residues: host uint64 [digits][2][n_q+n_p][N] (b then a). */
int he_key_download(he_ctx* ctx, int kind, int32_t step, uint64_t* host_out);
/* Number of key-switching digits at the top level, ceil(L / alpha). */
int he_key_digits(const he_ctx* ctx);

/* Transforms --------------------------------------------------------------- */

/*
 * In-place batched negacyclic NTT (coefficients -> evaluation values, storage
 * index j = value at psi^(2 brev(j)+1)) / its inverse (including N^-1).
 * d: device [n_polys][n_limbs][N], 32-byte aligned; limb i of every poly
 * uses prime index first_prime + i.  Inputs must be canonical; outputs are
 * canonical.
 */
int he_ntt_fwd(he_ctx* ctx, uint64_t* d, int n_polys, int n_limbs, int first_prime);
int he_ntt_inv(he_ctx* ctx, uint64_t* d, int n_polys, int n_limbs, int first_prime);

/* Operations --------------------------------------------------------------- */

/*
 * Slot rotation (AEGIS section 1 item 2: rotation needs key switching):
 *   rot_r(ct) = (sigma_k(c0), 0) + KS_{evk_r}(sigma_k(c1)),  k = 5^(r mod N/2) mod 2N,
 * slot j of the result = slot j + r of the input.  KS = ModUp (fast base
 * conversion of each digit onto the other primes), inner product with the
 * key, ModDown with centred conversion from P.  out gets in's level and
 * scale; out->data must not overlap in->data.
 */
int he_rotate(he_ctx* ctx, const he_ct* in, int32_t step, he_ct* out);
/* n independent rotations (in[i] by steps[i] into out[i]); all at one level.
 * Ciphertexts that share a step share one read of its key. */
int he_rotate_batch(he_ctx* ctx, const he_ct* in, const int32_t* steps, he_ct* out, int n);
/* Host-buffer form of he_rotate_batch: h_in / h_out are host [n][2][level][N];
 * the call copies in, rotates, copies out and waits.  The ciphertexts pass
 * through the GPU in chunks of 8, ordered by step, with uploads, rotations and
 * downloads of consecutive chunks overlapped (device staging: 4 chunks, held
 * by the context).  Pinned host memory gives full copy bandwidth.  h_out may
 * not overlap h_in.  Synchronous. */
int he_rotate_batch_host(he_ctx* ctx, const uint64_t* h_in, int level, const int32_t* steps,
                         uint64_t* h_out, int n);
/*
 * Packed wire format of ciphertexts, for host transfers: a residue mod q_r
 * takes b_r = ceil(bitlen(q_r) / 8) bytes, little-endian (5 for the 40-bit
 * primes of the chain, 8 for a 60-bit one); a ciphertext at `level` is, for
 * poly 0 then 1 and limb r = 0..level-1, its N residues of b_r bytes each:
 * he_ct_wire_bytes = 2 N sum_{r<level} b_r bytes (64% of 2 level N 8 at
 * N = 2^16, level 24).  Exact for canonical residues.  Host only (no
 * context, no device work): primes = q_0..q_{level-1} (he_get_primes or
 * he_derive_primes), N = 2^log_n.  he_ct_pack / he_ct_unpack convert n
 * ciphertexts between host [n][2][level][N] uint64 and n packed ciphertexts
 * back to back; he_ct_pack returns HE_EINVAL for a residue not below its
 * prime.  he_ct_wire_bytes returns HE_EINVAL (negative) for bad arguments.
 */
long long he_ct_wire_bytes(const uint64_t* primes, int level, int log_n);
int he_ct_pack(const uint64_t* primes, int level, int log_n, const uint64_t* in, int n, uint8_t* out);
int he_ct_unpack(const uint64_t* primes, int level, int log_n, const uint8_t* in, int n, uint64_t* out);
/* he_rotate_batch_host on packed host buffers: h_in / h_out hold n packed
 * ciphertexts each (he_ct_wire_bytes bytes apiece at the context's primes,
 * canonical
 * residues); they are unpacked and packed on the device, so only the packed
 * bytes cross the host link.  Same pipeline, staging and rules otherwise. */
int he_rotate_batch_host_wire(he_ctx* ctx, const uint8_t* h_in, int level, const int32_t* steps,
                              uint8_t* h_out, int n);
/*
 * Hoisted rotations (Halevi-Shoup, "Faster Homomorphic Linear Transformations
 * in HElib", CRYPTO 2018, section 5): every input rotated by every step, with
 * one ModUp per input shared by all its steps.  For in[i] = (c0, c1) and
 * k = 5^(steps[s] mod N/2) mod 2N,
 *   out[i*n_steps + s] = (sigma_k(c0) + ModDown(sum_j sigma_k(ModUp_j(c1)) (.) evk_j.b),
 *                                       ModDown(sum_j sigma_k(ModUp_j(c1)) (.) evk_j.a)),
 * sigma_k applied to the raised digits in the evaluation domain.  The
 * residues differ from he_rotate's (the fast base conversion commutes with
 * sigma_k only up to multiples of each digit's modulus), the decrypted slots
 * do not: slot j of out[i*n_steps + s] = slot j + steps[s] of in[i].
 * in: n_in device ciphertexts at one level, 32-byte aligned; out: n_in *
 * n_steps device ciphertexts, none overlapping an input, each given in[i]'s
 * level and scale.  A step whose Galois element is 1 copies.  Errors:
 * HE_EINVAL (null, unaligned, aliasing, negative counts), HE_ELEVEL (mixed or
 * out-of-range levels), HE_EDOMAIN (an input not in the evaluation domain),
 * HE_ENOKEY (a step without a rotation key); nothing is launched then.
 */
int he_rotate_hoisted(he_ctx* ctx, const he_ct* in, int n_in, const int32_t* steps, int n_steps, he_ct* out);
/*
 * Sums of rotations with one ModDown per sum (the ModDown hoisting of
 * Bossuat, Mouchet, Troncoso-Pastoriza, Hubaux, "Efficient Bootstrapping for
 * Approximate Homomorphic Encryption with Non-Sparse Keys", EUROCRYPT 2021,
 * section 4).  For o < n_out, with z_g = z[o*n_terms + g] = (z0_g, z1_g) and
 * k_g = 5^(steps[g] mod N/2) mod 2N:
 *   out[o] = base[o] + sum_g rot_{steps[g]}(z_g)
 *          = (b0 + sum_g sigma_g(z0_g) + ModDown(sum_g u0_g),  b1 + ModDown(sum_g u1_g)),
 *   u_g = sum_j ModUp_j(sigma_g(z1_g)) (.) evk_{g,j}   (kept over Q_level and P).
 * ModDown rounds once per sum, so the residues differ from adding he_rotate
 * results (by at most (n_terms+1)(K+1)/2 per coefficient) while the slots
 * agree.  Terms whose Galois element is 1 are added unchanged.
 * z: n_out*n_terms device ciphertexts (output-major), base: n_out ciphertexts
 * or NULL (then n_terms >= 1), all at one level and scale, 32-byte aligned;
 * n_terms <= 64.  out: n_out device ciphertexts with room for that level,
 * none overlapping an input; each gets the level and scale.  Errors:
 * HE_EINVAL (null, unaligned, aliasing, counts), HE_ELEVEL (mixed levels or
 * scales), HE_EDOMAIN, HE_ENOKEY (a step without a rotation key); nothing is
 * launched then.
 */
int he_rotate_sum(he_ctx* ctx, const he_ct* z, int n_out, int n_terms, const int32_t* steps, const he_ct* base,
                  he_ct* out);
/*
 * Rotate-and-sum of single ciphertexts with one ModUp and one ModDown each:
 * the hoisting of he_rotate_hoisted and the single ModDown of he_rotate_sum
 * together.  For in[i] = (c0, c1) and k_s = 5^(steps[s] mod N/2) mod 2N,
 *   out[i] = sum_s rot_{steps[s]}(in[i])
 *          = (sum_s sigma_s(c0) + ModDown(sum_s sum_j sigma_s(ModUp_j(c1)) (.) evk_{s,j}.b),
 *                                 ModDown(sum_s sum_j sigma_s(ModUp_j(c1)) (.) evk_{s,j}.a)).
 * Residues differ from adding he_rotate_hoisted results by the rounding of
 * one ModDown instead of n_steps (at most (n_steps+1)(K+1)/2 per
 * coefficient); the slots agree.  A step whose Galois element is 1 adds
 * in[i] unchanged.  in: n_in device ciphertexts at one level, 32-byte
 * aligned; 1 <= n_steps <= 64; out: n_in device ciphertexts with room for
 * that level, none overlapping an input, each given in[i]'s level and scale.
 * Errors: HE_EINVAL, HE_ELEVEL, HE_EDOMAIN, HE_ENOKEY as he_rotate_hoisted;
 * nothing is launched then.
 */
int he_rotate_sum_hoisted(he_ctx* ctx, const he_ct* in, int n_in, const int32_t* steps, int n_steps, he_ct* out);

/* Tensor, relinearise (key switch of d2 with the s^2 key), rescale.
 * a and b at the same level l >= 2; out at level l-1, scale (sa*sb)/q_{l-1}.
 * out->data must not overlap the inputs. */
int he_hmult_relin_rescale(he_ctx* ctx, const he_ct* a, const he_ct* b, he_ct* out);
/* Divide by q_{l-1} with rounding: c'_i = (c_i - [c_{l-1}]) q_{l-1}^-1 mod q_i with
 * [c_{l-1}] the centred coefficient representative.  In place: level-1, scale/q_{l-1}. */
int he_rescale(he_ctx* ctx, he_ct* inout);

/*
 * The same rescale as he_rescale, out of place, for callers that must not
 * allocate device memory while they run (runtimes that reserve and hand out
 * all device memory themselves, or that cannot afford the device-wide
 * synchronisation a cudaMalloc/cudaFree may cause).  The pages have no
 * counterpart: this is a deployment variant, not part of the method.
 * It calls no cudaMalloc/cudaFree and no allocating routine.  Its scratch is
 * a fixed device array of HE_NOALLOC_SCRATCH_WORDS uint64 (4.5 MiB) inside
 * libhe.so, held by every GPU that loads the library until the process exits.
 * he_ctx_create looks that array's address up on the context's device and
 * loads every kernel this call launches (CUDA otherwise loads them lazily,
 * on first use), so no call allocates, the first one included.  A context
 * does not survive cudaDeviceReset of its device.  All calls share the
 * array, so calls that overlap on the GPU race.  N must satisfy
 * 2N <= HE_NOALLOC_SCRATCH_WORDS (always true for log_n <= 16).  out must not
 * overlap in; it receives level-1 and scale/q_{level-1}.  Returns HE_EINVAL
 * while profiling is enabled.
 */
#define HE_NOALLOC_SCRATCH_WORDS 589824u
int he_rescale_noalloc(he_ctx* ctx, const he_ct* in, he_ct* out);

/* Helpers: ct + ct (same level; scale of a kept), ct * K (integer, any sign),
 * ct + K (K added to the constant coefficient: every slot gains K/scale),
 * keep limbs q_0..q_{level-1}.  out may equal the input. */
int he_add(he_ctx* ctx, const he_ct* a, const he_ct* b, he_ct* out);
int he_mul_const(he_ctx* ctx, const he_ct* in, int64_t K, he_ct* out);
int he_add_const(he_ctx* ctx, he_ct* inout, int64_t K);
int he_drop_level(he_ctx* ctx, const he_ct* in, int level, he_ct* out);

/*
 * Plaintext-weight x ciphertext block product by the diagonal method with
 * baby-step/giant-step (AEGIS section 2.2: the FFN is a local polynomial
 * multiplication per output group).  For each token group t < n_groups and
 * output block i < n_out:
 *   Y[t][i] = rescale( sum_g rot_{stride*bs*g}( sum_{j,b} pt[i][j][g][b] (.) rot_{stride*b}(X[t][j]) ) )
 * x: n_groups*n_in ciphertexts (group-major) at one level l >= 2.
 * d_pt: device [n_out][n_in][gs][bs][l][N] evaluation-domain plaintexts,
 *       encoded at pt_scale, 32-byte aligned.
 * y: n_groups*n_out ciphertexts (group-major) with room for level l; they
 *    come back at level l-1, scale x.scale*pt_scale/q_{l-1}.
 * The baby-step rotations rot_{stride*b}(X[t][j]) are the hoisted rotations of
 * he_rotate_hoisted (one ModUp per input); the giant-step sum of each output
 * is he_rotate_sum's (one ModDown per output).
 * Needs rotation keys for stride*b (0<b<bs) and stride*bs*g (0<g<gs).
 */
int he_pmult_accum_bsgs(he_ctx* ctx, const he_ct* x, int n_in, const uint64_t* d_pt, double pt_scale,
                        int n_out, int bs, int gs, int slot_stride, int n_groups, he_ct* y);

/*
 * One encrypted attention head (AEGIS section 2.3: Q x K^T, a polynomial
 * Softmax, A x V; the pages give no packing, this one is the engine's).
 * d features x n_tok tokens with d a power of two and d * 2 * n_tok = N/2,
 * feature-major with stride 2 n_tok: q holds Q[f][t] at slot f*2n + t for
 * t < n (zeros at t >= n); k and v are token-duplicated (slot f*2n + t holds
 * X[f][t mod n] for every t < 2n).
 * he_attention_scores: for each offset delta = offsets[i] in [0, n_tok),
 *   P = HMRR(q, rot_delta(k)), then s[i] = sum_{h<d} rot_{2n*h}(P) as two
 *   hoisted rotate-and-sums (he_rotate_sum_hoisted, step 0 adding the term
 *   itself): T = sum_{b<d1} rot_{2n*b}(P), s[i] = sum_{a<d2} rot_{2n*d1*a}(T),
 *   d1 = 2^ceil(log2(d)/2), d2 = d/d1; every feature block of s[i] then holds
 *   sum_f Q[f][t] K[f][(t + delta) mod n] at t < n (0 at t >= n).
 *   The rotations of k are hoisted (he_rotate_hoisted).  q and k at one
 *   level l >= 2; s[i] come back at level l-1, scale q.scale*k.scale/q_{l-1}.
 *   Needs rotation keys for the non-zero offsets, for 2n*b (0 < b < d1) and
 *   for 2n*d1*a (0 < a < d2), and the relinearisation key.
 * Softmax between the two calls is the caller's: shift each s[i] by a known
 * bound (he_add_const) and evaluate the exponential by he_poly_eval_ps15.
 * he_attention_output: out = rescale(relinearise(sum_i a[i] (x)
 *   drop(rot_{offsets[i]}(v)))): the products' tensors summed, then one
 *   relinearisation and one rescale; a[i] the n_off weights at one level
 *   la >= 2 and scale, v at level >= la; the rotations of v are hoisted
 *   (he_rotate_hoisted).  Slot f*2n + t of out holds
 *   sum_i A_i[t] V[f][(t + offsets[i]) mod n] for t < n.  out at la-1,
 *   scale a.scale*v.scale/q_{la-1}.
 * Outputs: s[i] each [2][l-1][N] words, out [2][la-1][N]; an output may not
 * overlap another output or any input.
 * Scratch (context-owned): the rotated copies, one ciphertext per offset
 * (scores), and the summed tensor (output).
 * Errors: HE_EINVAL (shape, offsets, null, unaligned, overlapping
 * buffers), HE_ELEVEL, HE_EDOMAIN, HE_ENOKEY; nothing is launched then.
 */
int he_attention_scores(he_ctx* ctx, const he_ct* q, const he_ct* k, int n_tok, int d, const int32_t* offsets,
                        int n_off, he_ct* s);
int he_attention_output(he_ctx* ctx, const he_ct* a, const he_ct* v, int n_tok, const int32_t* offsets, int n_off,
                        he_ct* out);

/*
 * Degree-15 polynomial sum_k c_k x^k by Paterson-Stockmeyer with 4 baby
 * powers (AEGIS section 2.3: Softmax by polynomial approximation):
 *   x2 = HMRR(x,x); x3 = HMRR(x2, drop(x)); x4 = HMRR(x2,x2);
 *   q_i = sum_{j<4} c_{4i+j} x^j built at (level, T): each x^j is dropped to
 *         level+1 and multiplied by K = round_half_away(c*T*q_level/S_j)
 *         (fp64, left to right); the three products are summed and the sum
 *         rescaled once; the constant adds round_half_away(c*T);
 *   acc = q_3 at (l0-3, top_scale); then for i = 2, 1, 0, at the product's
 *         level l (lambda = l-1, T = acc.scale*x4.scale/q_lambda):
 *         acc = rescale(relin(acc (x) drop(x4)) + sum_{j>=1} K_j drop(x^j))
 *               + round_half_away(c_{4i}*T), K_j as above at (lambda, T):
 *         q_i's products join the product before its rescale.
 * HMRR = he_hmult_relin_rescale.  x: n ciphertexts at level l0 >= 7;
 * out: n ciphertexts with room for level l0; they come back at level l0-6.
 */
int he_poly_eval_ps15(he_ctx* ctx, const he_ct* x, int n, const double* coeffs, double top_scale,
                      he_ct* out);

/* Measurement -------------------------------------------------------------- */

/* Kernel classes timed by the profiler. */
#define HE_PROF_NTT_FWD_COLS 0
#define HE_PROF_NTT_FWD_ROWS 1
#define HE_PROF_NTT_INV_ROWS 2
#define HE_PROF_NTT_INV_COLS 3
#define HE_PROF_MODUP 4
#define HE_PROF_KS_INNER 5
#define HE_PROF_MODDOWN_CONV 6
#define HE_PROF_MODDOWN_COMBINE 7
#define HE_PROF_AUTOMORPH 8
#define HE_PROF_ELEMENTWISE 9
#define HE_PROF_RESCALE 10
#define HE_PROF_PMULT 11
#define HE_PROF_N 12

/* enable != 0: every kernel launch is bracketed by CUDA events on the
 * context's stream and its time is added to its class.  Resets the totals. */
int he_profile_enable(he_ctx* ctx, int enable);
/* Waits for the stream, then returns total milliseconds and launches of one
 * class, and the algorithmic work of those launches: bytes that must cross
 * HBM (each input read once, each output written once) and 64-bit modular
 * multiplications (NTT butterflies, conversion and inner-product products).
 * Any output pointer may be NULL. */
int he_profile_read(he_ctx* ctx, int cls, double* total_ms, long long* launches, double* bytes,
                    double* modmuls);
/* Of the modular multiplications he_profile_read reports for a class, those
 * that ran on the FP64 pipe (residues of primes below 2^41); the rest ran on
 * the integer pipe. */
int he_profile_read_fp(he_ctx* ctx, int cls, double* fp_modmuls);
/* Kernels this context has launched since creation or the last reset. */
long long he_launch_count(he_ctx* ctx, int reset);

/* HBM copy probe: dst[i] = src[i] for n_words uint64 (device pointers),
 * grid-stride, 16-byte accesses.  Asynchronous. */
int he_probe_copy(he_ctx* ctx, uint64_t* dst, const uint64_t* src, size_t n_words);
/* Integer probe: every thread of a full-GPU grid runs `iters` rounds of
 * independent 64-bit Shoup modular multiplications in registers and writes
 * one word to sink[thread].  sink: device, >= he_probe_int_threads() words.
 * Asynchronous. */
int he_probe_int(he_ctx* ctx, int iters, uint64_t* sink);
long long he_probe_int_threads(he_ctx* ctx);
/* 64-bit modular multiplications one he_probe_int thread performs per iteration. */
int he_probe_int_mults_per_iter(void);
/* FP64 probe: as he_probe_int, with the FP64 rounded-quotient modular product
 * (the NTT's and the conversions' arithmetic for primes below 2^41) modulo
 * the context's largest such prime; same grid, same products per iteration.
 * HE_EINVAL when the context has no prime below 2^41.  Asynchronous. */
int he_probe_fp(he_ctx* ctx, int iters, uint64_t* sink);

#ifdef __cplusplus
}
#endif

#endif /* HE_B200_H */
