// Error feedback around the codecs for the shapes the fused encoders do not take.
//
// Method: "Sparsified SGD with Memory" (abstract): the compressor keeps the part of
// each update it did not send in a memory and adds it to the next gradient.  Around
// QSGD: p = e + g is encoded, and e becomes p minus what a receiver decodes (p where
// no record was sent).  The fast encoders do all of this in their one pass.  Other
// shapes take three passes over the memory: ef_add (e <- e + g, so e holds p), the
// ordinary encoder reading p from e, and a residual pass that re-derives every
// sent level from the stream's scale and the same random words (Elias) or reads it
// from the codes (b-bit) and subtracts its decoded value.
#include <cuda_runtime.h>

#include <algorithm>

#include "../../include/qsgd.h"
#include "qsgd_device.cuh"
#include "qsgd_internal.h"

namespace qsgd {
namespace {

constexpr int kEfBlock = 256;

int ef_grid(uint64_t items) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const uint64_t want = (items + kEfBlock - 1) / kEfBlock;
    return static_cast<int>(std::max<uint64_t>(1, std::min<uint64_t>(want, static_cast<uint64_t>(sms) * 8)));
}

// e[i] <- e[i] + g[i]; float4 when both are 16-byte aligned (vec4).
template <bool kVec4>
__global__ void __launch_bounds__(kEfBlock) ef_add(const float* __restrict__ g, float* __restrict__ e, uint64_t n) {
    const uint64_t stride = static_cast<uint64_t>(gridDim.x) * kEfBlock;
    const uint64_t t0 = static_cast<uint64_t>(blockIdx.x) * kEfBlock + threadIdx.x;
    if (kVec4) {
        const uint64_t n4 = n / 4;
        for (uint64_t j = t0; j < n4; j += stride) {
            const float4 a = __ldcs(reinterpret_cast<const float4*>(g) + j);
            float4 b = __ldcs(reinterpret_cast<const float4*>(e) + j);
            b.x = __fadd_rn(b.x, a.x);
            b.y = __fadd_rn(b.y, a.y);
            b.z = __fadd_rn(b.z, a.z);
            b.w = __fadd_rn(b.w, a.w);
            __stcs(reinterpret_cast<float4*>(e) + j, b);
        }
        for (uint64_t i = 4 * n4 + t0; i < n; i += stride) e[i] = __fadd_rn(e[i], g[i]);
    } else {
        for (uint64_t i = t0; i < n; i += stride) e[i] = __fadd_rn(e[i], g[i]);
    }
}

// The 32-bit norm that heads bucket b of an Elias stream (bit offset offsets[b],
// MSB-first words), or 0 when the offset would read past the capacity.
__device__ __forceinline__ float stream_norm(const uint32_t* words, uint64_t cap_words, const uint64_t* offsets,
                                             uint64_t b) {
    const uint64_t off = offsets[b];
    if (cap_words * 32 < 32 || off > cap_words * 32 - 32) return 0.f;
    const uint64_t w = off >> 5;
    const uint32_t sh = static_cast<uint32_t>(off & 31u);
    const uint32_t bits = sh ? (words[w] << sh) | (words[w + 1] >> (32 - sh)) : words[w];
    return __uint_as_float(bits);
}

// Elias stream: one thread per 4 coordinates (one Philox block).  A bucket sent
// with norm N > 0 had scale s/N (the encoder's division); its level k is re-drawn
// from p and the same random word; e <- p - fl(fl(N/s) k) with the sign of p.
__global__ void __launch_bounds__(kEfBlock) ef_residual_elias(float* e, const uint32_t* __restrict__ words,
                                                              uint64_t cap_words, const uint64_t* __restrict__ offsets,
                                                              uint64_t n, uint32_t d, uint32_t s, PhiloxKey key) {
    const uint64_t nq = (n + 3) / 4;
    const uint64_t stride = static_cast<uint64_t>(gridDim.x) * kEfBlock;
    const float sf = __uint2float_rn(s);
    for (uint64_t j = static_cast<uint64_t>(blockIdx.x) * kEfBlock + threadIdx.x; j < nq; j += stride) {
        const uint4 r = philox4x32_10(j, key);
        const uint32_t rw[4] = {r.x, r.y, r.z, r.w};
        uint64_t cached = ~uint64_t(0);
        float sinv = 0.f, scale = 0.f;
        for (int c = 0; c < 4; ++c) {
            const uint64_t i = 4 * j + c;
            if (i >= n) break;
            const uint64_t b = i / d;
            if (b != cached) {
                cached = b;
                const float N = stream_norm(words, cap_words, offsets, b);
                const bool sent = N > 0.f && isfinite(N);
                sinv = sent ? __fdiv_rn(sf, N) : 0.f;
                scale = sent ? __fdiv_rn(N, sf) : 0.f;
            }
            if (sinv == 0.f || !isfinite(sinv)) continue;
            const float p = e[i];
            const uint32_t k = quantize_level(p, sinv, rw[c], s);
            if (k) e[i] = ef_residual(p, k, signbit(p), scale);
        }
    }
}

// b-bit codes: one thread per coordinate; code (sign << (b-1)) | k at bits
// [i b, i b + b), MSB-first; e <- p - fl(fl(norm/S) k) with the code's sign.
template <int B>
__global__ void __launch_bounds__(kEfBlock) ef_residual_bbit(float* e, const float* __restrict__ norms,
                                                             const uint32_t* __restrict__ codes, uint64_t n,
                                                             uint32_t d) {
    constexpr uint32_t S = (1u << (B - 1)) - 1u;
    const uint64_t stride = static_cast<uint64_t>(gridDim.x) * kEfBlock;
    for (uint64_t i = static_cast<uint64_t>(blockIdx.x) * kEfBlock + threadIdx.x; i < n; i += stride) {
        const uint64_t bit = i * B;  // a code never straddles a word (B divides 32)
        const uint32_t code = (codes[bit >> 5] >> (32 - B - (bit & 31u))) & ((1u << B) - 1u);
        const uint32_t k = code & S;
        if (!k) continue;
        const float scale = __fdiv_rn(norms[i / d], __uint2float_rn(S));
        e[i] = ef_residual(e[i], k, code >> (B - 1), scale);
    }
}

}  // namespace

cudaError_t launch_ef_add(const float* g, float* e, uint64_t n, cudaStream_t stream) {
    const bool vec4 = ((reinterpret_cast<uintptr_t>(g) | reinterpret_cast<uintptr_t>(e)) & 15u) == 0;
    if (vec4)
        ef_add<true><<<ef_grid(n / 4 + 1), kEfBlock, 0, stream>>>(g, e, n);
    else
        ef_add<false><<<ef_grid(n), kEfBlock, 0, stream>>>(g, e, n);
    return cudaGetLastError();
}

cudaError_t launch_ef_residual(float* e, const uint32_t* words, uint64_t cap_words, const uint64_t* offsets,
                               uint64_t n, uint32_t d, uint32_t s, uint64_t seed, cudaStream_t stream) {
    const PhiloxKey key{static_cast<uint32_t>(seed), static_cast<uint32_t>(seed >> 32)};
    ef_residual_elias<<<ef_grid((n + 3) / 4), kEfBlock, 0, stream>>>(e, words, cap_words, offsets, n, d, s, key);
    return cudaGetLastError();
}

cudaError_t launch_bbit_ef_residual(float* e, const float* norms, const uint32_t* codes, uint64_t n, uint32_t d,
                                    uint32_t b, cudaStream_t stream) {
    const int grid = ef_grid(n);
    switch (b) {
        case 2: ef_residual_bbit<2><<<grid, kEfBlock, 0, stream>>>(e, norms, codes, n, d); break;
        case 4: ef_residual_bbit<4><<<grid, kEfBlock, 0, stream>>>(e, norms, codes, n, d); break;
        default: ef_residual_bbit<8><<<grid, kEfBlock, 0, stream>>>(e, norms, codes, n, d); break;
    }
    return cudaGetLastError();
}

}  // namespace qsgd
