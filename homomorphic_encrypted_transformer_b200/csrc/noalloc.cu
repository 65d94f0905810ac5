// he_rescale_noalloc: the rescale of he_rescale with its scratch memory in a
// fixed device array of this library instead of memory the context allocates.
//
// Who needs it: callers that must not allocate device memory while they run.
// Examples are serving runtimes that reserve all of a GPU's memory up front
// and hand it out themselves, processes whose remaining device memory belongs
// to another allocator, and latency-sensitive callers that cannot afford the
// device-wide synchronisation a cudaMalloc/cudaFree may cause.  This entry
// point calls neither, nor any routine that allocates.
//
// The scratch array below (HE_NOALLOC_SCRATCH_WORDS uint64 = 4.5 MiB) is held
// by every GPU that loads the library until the process exits.  All calls
// share it and it keeps the last call's contents; two calls that overlap on
// the GPU (different streams or contexts without ordering) race on it.  Every
// word a call reads was written earlier in the same call, so nothing needs
// clearing between calls.
//
// Host code cannot use the array's name as a device address (in host code
// the symbol is a stand-in, not device memory).  he_ctx_create therefore
// looks the address up with cudaGetSymbolAddress on the context's device
// (current during creation) and keeps it in the context.  CUDA loads a
// module and its device arrays lazily, on first use; the lookup does that
// load for this file, and the set-up also loads every kernel the entry point
// launches, so the entry point's first call allocates nothing either.  A
// context does not survive a reset of its device (cudaDeviceReset frees all
// of its memory); contexts created after a reset look the address up again.
#include "he_internal.h"

namespace he {

// The centred last limb x (coefficients mod q_l) onto every q_r of a chunk:
// out[r] = [x]_{q_r} - (x > q_l/2 ? q_l : 0)  (pointers and tables offset to
// the chunk's first limb)
__global__ void k_rescale_lift(const uint64_t* __restrict__ last, uint64_t* __restrict__ out, int lm1, uint64_t ql,
                               const uint64_t* __restrict__ qmod, const DevPrime* __restrict__ pr, int logn) {
    const int N = 1 << logn;
    int c = blockIdx.x * blockDim.x + threadIdx.x, r = blockIdx.y, ip = blockIdx.z;
    if (c >= N) return;
    const uint64_t x = last[(size_t)ip * N + c];
    const DevPrime p = pr[r];
    uint64_t v = reduce64(x, p);
    if (x > (ql >> 1)) v = sub_mod(v, qmod[r], p.q);  // x - q_l
    out[((size_t)ip * lm1 + r) * N + c] = v;
}

// out[r] = (in[r] - lift[r]) q_l^-1 for the limbs of one chunk (pointers and
// tables offset to the chunk's first limb)
__global__ void k_noalloc_combine(const uint64_t* __restrict__ in, const uint64_t* __restrict__ lift,
                                  uint64_t* __restrict__ out, const ulonglong2* __restrict__ qinv,
                                  const DevPrime* __restrict__ pr, int logn) {
    const int N = 1 << logn;
    int c = blockIdx.x * blockDim.x + threadIdx.x, r = blockIdx.y;
    if (c >= N) return;
    const uint64_t q = pr[r].q;
    const ulonglong2 w = qinv[r];
    out[(size_t)r * N + c] = mul_shoup(in[(size_t)r * N + c] + q - lift[(size_t)r * N + c], w.x, w.y, q);
}

static __device__ __align__(256) uint64_t g_noalloc_scratch[HE_NOALLOC_SCRATCH_WORDS];

int noalloc_setup(he_ctx* c) {
    void* p = nullptr;
    int rc = check_cuda(c, cudaGetSymbolAddress(&p, g_noalloc_scratch), "he_rescale_noalloc set-up: cudaGetSymbolAddress");
    if (rc) return rc;
    cudaFuncAttributes a;
    rc = check_cuda(c, cudaFuncGetAttributes(&a, k_noalloc_combine), "he_rescale_noalloc set-up: combine kernel");
    if (!rc) rc = check_cuda(c, cudaFuncGetAttributes(&a, k_rescale_lift), "he_rescale_noalloc set-up: lift kernel");
    if (!rc) rc = ntt_preload(c);
    if (rc) return rc;
    c->noalloc_scratch = (uint64_t*)p;
    return HE_OK;
}

}  // namespace he

using namespace he;

extern "C" int he_rescale_noalloc(he_ctx* c, const he_ct* in, he_ct* out) {
    if (!c) return HE_EINVAL;
    if (!in || !in->data || !out || !out->data) return set_err(c, HE_EINVAL, "he_rescale_noalloc: null argument");
    if (((uintptr_t)in->data | (uintptr_t)out->data) & 31)
        return set_err(c, HE_EINVAL, "he_rescale_noalloc: ciphertext not 32-byte aligned");
    if (!in->is_ntt) return set_err(c, HE_EDOMAIN, "he_rescale_noalloc: input not in the evaluation domain");
    const int level = in->level, N = c->N, lm1 = level - 1;
    if (level < 2 || level > c->L)
        return set_err(c, HE_ELEVEL, "he_rescale_noalloc: level %d cannot be rescaled", level);
    const size_t in_words = (size_t)2 * level * N, out_words = (size_t)2 * lm1 * N;
    const uint64_t *ib = in->data, *ie = in->data + in_words;
    const uint64_t *ob = out->data, *oe = out->data + out_words;
    if (ib < oe && ob < ie) return set_err(c, HE_EINVAL, "he_rescale_noalloc: output overlaps the input");
    // scratch: the last limb [N] and a chunk of lifted limbs [chunk][N]
    if ((size_t)2 * N > HE_NOALLOC_SCRATCH_WORDS)
        return set_err(c, HE_EINVAL, "he_rescale_noalloc: N = %d needs %zu scratch words, the maximum is %u", N,
                       (size_t)2 * N, (unsigned)HE_NOALLOC_SCRATCH_WORDS);
    if (c->prof_on) return set_err(c, HE_EINVAL, "he_rescale_noalloc: not available while profiling is enabled");
    uint64_t* scratch = c->noalloc_scratch;
    if (!scratch) return set_err(c, HE_EINVAL, "he_rescale_noalloc: context has no scratch address");
    int rc;
    const int chunk = (int)(HE_NOALLOC_SCRATCH_WORDS / N) - 1;
    uint64_t* last = scratch;
    uint64_t* lift = scratch + N;
    const uint64_t ql = c->primes[lm1];
    const int gx = (N + 255) / 256;
    for (int poly = 0; poly < 2; poly++) {
        rc = check_cuda(c, cudaMemcpyAsync(last, in->data + ((size_t)poly * level + lm1) * N, (size_t)N * 8,
                                           cudaMemcpyDeviceToDevice, c->stream), "he_rescale_noalloc: copy");
        if (rc) return rc;
        std::vector<int> pl(1, lm1);
        if ((rc = ntt_inv_set(c, rowset_contig(last, 1, N, pl), 1))) return rc;
        for (int i0 = 0; i0 < lm1; i0 += chunk) {
            const int m = lm1 - i0 < chunk ? lm1 - i0 : chunk;
            k_rescale_lift<<<dim3(gx, m, 1), 256, 0, c->stream>>>(last, lift, lm1, ql,
                                                                 c->d_rs_qmod + (size_t)lm1 * c->L + i0,
                                                                 c->d_prime + i0, c->log_n);
            c->launches++;
            if ((rc = check_cuda(c, cudaGetLastError(), "he_rescale_noalloc: lift"))) return rc;
            if ((rc = ntt_fwd_set(c, rowset_contig(lift, m, N, prime_range(i0, m)), m))) return rc;
            k_noalloc_combine<<<dim3(gx, m, 1), 256, 0, c->stream>>>(
                in->data + ((size_t)poly * level + i0) * N, lift, out->data + ((size_t)poly * lm1 + i0) * N,
                c->d_rs_inv + (size_t)lm1 * c->L + i0, c->d_prime + i0, c->log_n);
            c->launches++;
            if ((rc = check_cuda(c, cudaGetLastError(), "he_rescale_noalloc: combine"))) return rc;
        }
    }
    out->level = lm1;
    out->scale = in->scale / (double)ql;
    out->is_ntt = 1;
    return HE_OK;
}
