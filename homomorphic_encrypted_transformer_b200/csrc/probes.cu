// Measurement probes run in the same process as the engine: an HBM copy
// (the denominator of the memory roofline) and register-only streams of
// modular products on the integer pipe (64-bit Shoup) and on the FP64 pipe
// (rounded-quotient products of primes below 2^41): the ceilings of the
// engine's two arithmetic paths.
#include "he_internal.h"
#include "ntt.cuh"

namespace he {

__global__ void k_probe_copy(const ulonglong2* __restrict__ src, ulonglong2* __restrict__ dst, size_t n2) {
    size_t stride = (size_t)gridDim.x * blockDim.x;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n2; i += stride) dst[i] = src[i];
}

constexpr int kProbeChains = 8;

__global__ void k_probe_int(int iters, uint64_t q, uint64_t w, uint64_t ws, uint64_t* __restrict__ sink) {
    uint64_t x[kProbeChains];
    size_t tid = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    for (int k = 0; k < kProbeChains; k++) x[k] = (tid * 0x9E3779B97F4A7C15ull + k) % q;
    for (int it = 0; it < iters; it++) {
#pragma unroll
        for (int k = 0; k < kProbeChains; k++) x[k] = mul_shoup_lazy(x[k], w, ws, q);
    }
    uint64_t acc = 0;
    for (int k = 0; k < kProbeChains; k++) acc ^= x[k];
    sink[tid] = acc;
}

__global__ void k_probe_fp(int iters, FpMod m, double w, uint64_t* __restrict__ sink) {
    double x[kProbeChains];
    size_t tid = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    for (int k = 0; k < kProbeChains; k++) x[k] = (double)((tid * 0x9E3779B97F4A7C15ull + k) % (uint64_t)m.q);
    for (int it = 0; it < iters; it++) {
#pragma unroll
        for (int k = 0; k < kProbeChains; k++) x[k] = fp_mulmod_s(x[k], w, m);
    }
    uint64_t acc = 0;
    for (int k = 0; k < kProbeChains; k++) acc ^= (uint64_t)__double_as_longlong(x[k]);
    sink[tid] = acc;
}

static int probe_grid(he_ctx* c) {
    int sms = 0;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, c->device);
    return sms > 0 ? sms * 8 : 148 * 8;
}

}  // namespace he

using namespace he;

extern "C" int he_probe_copy(he_ctx* c, uint64_t* dst, const uint64_t* src, size_t n_words) {
    if (!c) return HE_EINVAL;
    if (!dst || !src || (n_words & 1) || (((uintptr_t)dst | (uintptr_t)src) & 15))
        return set_err(c, HE_EINVAL, "he_probe_copy: need 16-byte aligned buffers and an even word count");
    k_probe_copy<<<probe_grid(c), 256, 0, c->stream>>>((const ulonglong2*)src, (ulonglong2*)dst, n_words / 2);
    c->launches++;
    return check_cuda(c, cudaGetLastError(), "probe_copy");
}

extern "C" long long he_probe_int_threads(he_ctx* c) { return c ? (long long)probe_grid(c) * 256 : -1; }

extern "C" int he_probe_int_mults_per_iter(void) { return kProbeChains; }

extern "C" int he_probe_int(he_ctx* c, int iters, uint64_t* sink) {
    if (!c) return HE_EINVAL;
    if (!sink || iters < 0) return set_err(c, HE_EINVAL, "he_probe_int: bad arguments");
    const DevPrime& p = c->hprime[0];
    uint64_t w = p.r1;  // any constant below q
    k_probe_int<<<probe_grid(c), 256, 0, c->stream>>>(iters, p.q, w, p.r1_shoup, sink);
    c->launches++;
    return check_cuda(c, cudaGetLastError(), "probe_int");
}

extern "C" int he_probe_fp(he_ctx* c, int iters, uint64_t* sink) {
    if (!c) return HE_EINVAL;
    if (!sink || iters < 0) return set_err(c, HE_EINVAL, "he_probe_fp: bad arguments");
    int best = -1;
    for (size_t i = 0; i < c->primes.size(); i++)
        if (c->primes[i] < kFpPrimeLimit && (best < 0 || c->primes[i] > c->primes[best])) best = (int)i;
    if (best < 0) return set_err(c, HE_EINVAL, "he_probe_fp: no prime below 2^41");
    const double q = (double)c->primes[best];
    FpMod m{q, 2.0 * q, 1.0 / q, 0.0};
    const double w = (double)(c->primes[best] / 3);  // any constant below q
    k_probe_fp<<<probe_grid(c), 256, 0, c->stream>>>(iters, m, w, sink);
    c->launches++;
    return check_cuda(c, cudaGetLastError(), "probe_fp");
}
