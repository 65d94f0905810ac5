// Measurement probes run in the same process as the engine: an HBM copy
// (the denominator of the memory roofline) and a register-only stream of
// 64-bit Shoup modular products (the integer-pipe ceiling of the NTT's
// butterfly arithmetic).
#include "he_internal.h"

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
