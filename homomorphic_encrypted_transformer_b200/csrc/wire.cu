// Packed wire format of ciphertexts for host transfers.
//
// A residue mod q_r takes b_r = ceil(bitlen(q_r) / 8) bytes, little-endian
// (5 for the 40-bit primes of the chain, 8 for the 60-bit q_0), instead of a
// full 64-bit word: a ciphertext at level l is, poly by poly and limb by
// limb, N residues of b_r bytes each, 2 N sum_{r<l} b_r bytes in all (64% of
// the unpacked size at N = 2^16, level 24).  Packing is exact for canonical
// residues.  The device kernels move groups of 8 residues (8 b_r bytes, so a
// group starts on an 8-byte boundary): thread g of limb (i, poly, r) turns
// b_r 64-bit words into 8 residues or back.
#include <algorithm>

#include "he_internal.h"

namespace he {

// Byte offsets of every limb of a packed ciphertext at `level`: limb (poly,
// r) starts at off[poly level + r]; off[2 level] is the ciphertext's size.
struct WireLayout {
    long long off[2 * kMaxPrimes + 1];
    uint8_t bytes[kMaxPrimes];  // b_r
};

static int residue_bytes(uint64_t q) { return (64 - __builtin_clzll(q) + 7) / 8; }

static WireLayout wire_layout(const uint64_t* primes, int level, int N) {
    WireLayout w;
    long long o = 0;
    for (int r = 0; r < level; r++) w.bytes[r] = (uint8_t)residue_bytes(primes[r]);
    for (int poly = 0; poly < 2; poly++)
        for (int r = 0; r < level; r++) {
            w.off[poly * level + r] = o;
            o += (long long)w.bytes[r] * N;
        }
    w.off[2 * level] = o;
    return w;
}

static WireLayout wire_layout(const he_ctx* c, int level) { return wire_layout(c->primes.data(), level, c->N); }

size_t wire_bytes(const he_ctx* c, int level) { return (size_t)wire_layout(c, level).off[2 * level]; }

// 8 residues <-> B words (residue k at bits [8 B k, 8 B k + 8 B) of the group)
template <int B>
__device__ __forceinline__ void unpack8(const uint64_t* src, uint64_t* dst) {
    uint64_t w[B];
#pragma unroll
    for (int j = 0; j < B; j++) w[j] = src[j];
    constexpr int BITS = 8 * B;
    constexpr uint64_t MASK = BITS == 64 ? ~0ull : (1ull << BITS) - 1;
#pragma unroll
    for (int k = 0; k < 8; k++) {
        const int bit = BITS * k, wi = bit >> 6, s = bit & 63;
        uint64_t v = w[wi] >> s;
        if (s + BITS > 64) v |= w[wi + 1] << (64 - s);
        dst[k] = v & MASK;
    }
}

template <int B>
__device__ __forceinline__ void pack8(const uint64_t* src, uint64_t* dst) {
    uint64_t w[B];
#pragma unroll
    for (int j = 0; j < B; j++) w[j] = 0;
    constexpr int BITS = 8 * B;
#pragma unroll
    for (int k = 0; k < 8; k++) {
        const int bit = BITS * k, wi = bit >> 6, s = bit & 63;
        const uint64_t v = src[k];
        w[wi] |= v << s;
        if (s + BITS > 64) w[wi + 1] |= v >> (64 - s);
    }
#pragma unroll
    for (int j = 0; j < B; j++) dst[j] = w[j];
}

// grid (groups of 8 residues, 2 level limbs, ciphertexts): packed bytes at
// wire + i wire_ct <-> ct_i [2][level][N] words
template <bool PACK>
__global__ void k_wire(const uint8_t* __restrict__ wire_in, uint8_t* __restrict__ wire_out, size_t wire_ct,
                       PtrList ct_in, MutPtrList ct_out, int level, const WireLayout lay, int logn) {
    const int N = 1 << logn;
    const int g = blockIdx.x * blockDim.x + threadIdx.x, y = blockIdx.y, i = blockIdx.z;
    if (g >= N / 8) return;
    const int r = y % level;
    const int B = lay.bytes[r];
    const size_t woff = (size_t)i * wire_ct + (size_t)lay.off[y] + (size_t)g * 8 * B;
    if constexpr (PACK) {
        const uint64_t* src = ct_in.p[i] + (size_t)y * N + 8 * g;
        uint64_t* dst = reinterpret_cast<uint64_t*>(wire_out + woff);
        switch (B) {
            case 1: pack8<1>(src, dst); break;
            case 2: pack8<2>(src, dst); break;
            case 3: pack8<3>(src, dst); break;
            case 4: pack8<4>(src, dst); break;
            case 5: pack8<5>(src, dst); break;
            case 6: pack8<6>(src, dst); break;
            case 7: pack8<7>(src, dst); break;
            default: pack8<8>(src, dst); break;
        }
    } else {
        const uint64_t* src = reinterpret_cast<const uint64_t*>(wire_in + woff);
        uint64_t* dst = ct_out.p[i] + (size_t)y * N + 8 * g;
        switch (B) {
            case 1: unpack8<1>(src, dst); break;
            case 2: unpack8<2>(src, dst); break;
            case 3: unpack8<3>(src, dst); break;
            case 4: unpack8<4>(src, dst); break;
            case 5: unpack8<5>(src, dst); break;
            case 6: unpack8<6>(src, dst); break;
            case 7: unpack8<7>(src, dst); break;
            default: unpack8<8>(src, dst); break;
        }
    }
}

// ct_i (i < n, device [2][level][N]) from n packed ciphertexts at wire
// (device, 8-byte aligned), or packed into it.
int wire_unpack_many(he_ctx* c, const uint8_t* wire, int level, const std::vector<uint64_t*>& ct) {
    const WireLayout lay = wire_layout(c, level);
    const int n = (int)ct.size(), gx = (c->N / 8 + 255) / 256;
    for (int i0 = 0; i0 < n; i0 += kMaxBatch) {
        const int m = std::min(kMaxBatch, n - i0);
        PtrList none{};
        MutPtrList out;
        for (int i = 0; i < m; i++) out.p[i] = ct[i0 + i];
        k_wire<false><<<dim3(gx, 2 * level, m), 256, 0, c->stream>>>(wire + (size_t)i0 * lay.off[2 * level], nullptr,
                                                                   (size_t)lay.off[2 * level], none, out, level, lay,
                                                                   c->log_n);
        c->launches++;
        int rc = check_cuda(c, cudaGetLastError(), "wire unpack");
        if (rc) return rc;
    }
    return HE_OK;
}

int wire_pack_many(he_ctx* c, const std::vector<const uint64_t*>& ct, int level, uint8_t* wire) {
    const WireLayout lay = wire_layout(c, level);
    const int n = (int)ct.size(), gx = (c->N / 8 + 255) / 256;
    for (int i0 = 0; i0 < n; i0 += kMaxBatch) {
        const int m = std::min(kMaxBatch, n - i0);
        PtrList in;
        MutPtrList none{};
        for (int i = 0; i < m; i++) in.p[i] = ct[i0 + i];
        k_wire<true><<<dim3(gx, 2 * level, m), 256, 0, c->stream>>>(nullptr, wire + (size_t)i0 * lay.off[2 * level],
                                                                  (size_t)lay.off[2 * level], in, none, level, lay,
                                                                  c->log_n);
        c->launches++;
        int rc = check_cuda(c, cudaGetLastError(), "wire pack");
        if (rc) return rc;
    }
    return HE_OK;
}

}  // namespace he

using namespace he;

static bool wire_args_ok(const uint64_t* primes, int level, int log_n) {
    if (!primes || level < 1 || level > kMaxPrimes || log_n < 3 || log_n > 20) return false;
    for (int r = 0; r < level; r++)
        if (primes[r] < 2) return false;
    return true;
}

extern "C" long long he_ct_wire_bytes(const uint64_t* primes, int level, int log_n) {
    if (!wire_args_ok(primes, level, log_n)) return HE_EINVAL;
    return wire_layout(primes, level, 1 << log_n).off[2 * level];
}

// Host-side packing (no device work): the same layout, byte by byte.
extern "C" int he_ct_pack(const uint64_t* primes, int level, int log_n, const uint64_t* in, int n, uint8_t* out) {
    if (!wire_args_ok(primes, level, log_n) || !in || !out || n < 0) return HE_EINVAL;
    const size_t N = (size_t)1 << log_n;
    const WireLayout lay = wire_layout(primes, level, (int)N);
    const size_t ctw = 2 * (size_t)level * N, ctb = (size_t)lay.off[2 * level];
    for (int i = 0; i < n; i++)
        for (int y = 0; y < 2 * level; y++) {
            const int r = y % level, B = lay.bytes[r];
            const uint64_t q = primes[r];
            const uint64_t* src = in + i * ctw + (size_t)y * N;
            uint8_t* dst = out + i * ctb + (size_t)lay.off[y];
            for (size_t k = 0; k < N; k++) {
                const uint64_t v = src[k];
                if (v >= q) return HE_EINVAL;  // not a canonical residue
                for (int b = 0; b < B; b++) dst[k * B + b] = (uint8_t)(v >> (8 * b));
            }
        }
    return HE_OK;
}

extern "C" int he_ct_unpack(const uint64_t* primes, int level, int log_n, const uint8_t* in, int n, uint64_t* out) {
    if (!wire_args_ok(primes, level, log_n) || !in || !out || n < 0) return HE_EINVAL;
    const size_t N = (size_t)1 << log_n;
    const WireLayout lay = wire_layout(primes, level, (int)N);
    const size_t ctw = 2 * (size_t)level * N, ctb = (size_t)lay.off[2 * level];
    for (int i = 0; i < n; i++)
        for (int y = 0; y < 2 * level; y++) {
            const int r = y % level, B = lay.bytes[r];
            const uint8_t* src = in + i * ctb + (size_t)lay.off[y];
            uint64_t* dst = out + i * ctw + (size_t)y * N;
            for (size_t k = 0; k < N; k++) {
                uint64_t v = 0;
                for (int b = 0; b < B; b++) v |= (uint64_t)src[k * B + b] << (8 * b);
                dst[k] = v;
            }
        }
    return HE_OK;
}
