// Fixed-width b-bit QSGD (b = 2, 4, 8): encoder, decoder and decode-accumulate.
//
// Method: the "4-bit and 2-bit QSGD" of the claim "QSVRG, non-convex and multi-GPU
// bucketed training" of "QSGD (Quantized Stochastic Gradient Descent) with Elias
// Coding" (AIMech curated entry), with s = 2^(b-1) - 1 levels and the quantiser of
// the definition paragraph.  Layout (the page gives none): one fp32 norm per bucket
// in its own array; coordinate i's code (sign << (b-1)) | k at bits [i*b, i*b + b)
// of the code words, MSB-first, so every code sits at a fixed place and both
// directions are plain data-parallel passes with no prefix scan.
#include <cuda_runtime.h>

#include <algorithm>

#include "../../include/qsgd.h"
#include "qsgd_device.cuh"
#include "qsgd_internal.h"

namespace qsgd {
namespace {

constexpr uint32_t kAll = 0xFFFFFFFFu;
constexpr int kBbitBlock = 256;

// The b-bit code of one coordinate from its value and the random word drawn for it.
__device__ __forceinline__ uint32_t bbit_code(float v, float sinv, uint32_t r, uint32_t s, uint32_t b) {
    const uint32_t k = quantize_level(v, sinv, r, s);
    return k ? ((__float_as_uint(v) >> 31) << (b - 1)) | k : 0u;
}

// ---------------------------------------------------------------------------
// Encoder, one pass (d = 128V, V in {1, 2, 4, 8}, 16-byte aligned input): one warp
// per bucket; lane L holds the NC = 4V consecutive coordinates [NC L, NC L + NC)
// (one Philox block per 4), computes the norm with the other lanes, and packs its
// NC codes.  When NC*b < 32, G = 32 / (NC b) neighbouring lanes share a word and
// OR their parts together with shuffles.
// ---------------------------------------------------------------------------
template <int V, int B, bool kEF>
__global__ void __launch_bounds__(kBbitBlock) bbit_encode_fast(const float* __restrict__ in, float* __restrict__ ef,
                                                               uint64_t n, uint32_t d, uint64_t seed,
                                                               uint32_t norm_kind, float* norms, uint32_t* codes,
                                                               uint32_t* status) {
    constexpr int NC = 4 * V;
    constexpr uint32_t S = (1u << (B - 1)) - 1u;
    constexpr int kLaneBits = NC * B;  // 8 .. 256
    constexpr int G = kLaneBits >= 32 ? 1 : 32 / kLaneBits;
    constexpr int kLaneWords = kLaneBits >= 32 ? kLaneBits / 32 : 1;
    const int lane = threadIdx.x & 31;
    const uint64_t nb = (n + d - 1) / d;
    const uint64_t gwarps = static_cast<uint64_t>(gridDim.x) * (kBbitBlock / 32);
    const PhiloxKey key{static_cast<uint32_t>(seed), static_cast<uint32_t>(seed >> 32)};
    for (uint64_t bk = static_cast<uint64_t>(blockIdx.x) * (kBbitBlock / 32) + (threadIdx.x >> 5); bk < nb;
         bk += gwarps) {
        const uint64_t base = bk * d;
        const uint32_t m = static_cast<uint32_t>(min(static_cast<uint64_t>(d), n - base));
        const uint32_t first = static_cast<uint32_t>(lane) * NC;
        float ev[kEF ? NC : 1];  // error feedback: the memory of these coordinates
        if constexpr (kEF) ef_load<V>(ef + base, first, m, ev);
        float x[NC];
#pragma unroll
        for (int j = 0; j < V; ++j) {
            const uint32_t i = first + 4 * j;
            float4 q = make_float4(0.f, 0.f, 0.f, 0.f);
            if (i + 4 <= m) {
                q = __ldg(reinterpret_cast<const float4*>(in + base + i));
            } else if (i < m) {  // the ragged last bucket
                q.x = in[base + i];
                if (i + 1 < m) q.y = in[base + i + 1];
                if (i + 2 < m) q.z = in[base + i + 2];
            }
            x[4 * j + 0] = q.x;
            x[4 * j + 1] = q.y;
            x[4 * j + 2] = q.z;
            x[4 * j + 3] = q.w;
        }
        if constexpr (kEF) {  // p = e + g
#pragma unroll
            for (int q = 0; q < NC; ++q) x[q] = __fadd_rn(ev[q], x[q]);
        }
        const float norm = norm_kind == QSGD_NORM_MAX ? warp_bucket_maxnorm<NC>(x) : warp_bucket_norm<NC>(x, true);
        const BucketScale sc = bucket_scale(norm, S, true, status, lane == 0);
        if (lane == 0) norms[bk] = sc.sent;
        uint32_t part[kLaneWords];
#pragma unroll
        for (int w = 0; w < kLaneWords; ++w) part[w] = 0u;
        if (sc.good) {
            const float scale = kEF ? __fdiv_rn(sc.sent, static_cast<float>(S)) : 0.f;
#pragma unroll
            for (int j = 0; j < V; ++j) {
                const uint4 rr = philox4x32_10(((base + first) >> 2) + j, key);
                const uint32_t rw[4] = {rr.x, rr.y, rr.z, rr.w};
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int q = 4 * j + c;
                    const uint32_t code = first + q < m ? bbit_code(x[q], sc.sinv, rw[c], S, B) : 0u;
                    if constexpr (kEF) ev[q] = ef_residual(x[q], code & S, code >> (B - 1), scale);
                    const int bit = q * B;  // offset of the code inside the lane's bits
                    if (kLaneBits >= 32)
                        part[bit / 32] |= code << (32 - B - bit % 32);
                    else
                        part[0] |= code << (kLaneBits - B - bit);
                }
            }
        }
        if constexpr (kEF) {  // the memory keeps p minus what a receiver decodes (p where nothing was sent)
            if (sc.good)
                ef_store<V>(ef + base, first, m, ev);
            else
                ef_store<V>(ef + base, first, m, x);
        }
        // the bucket's codes start on a word: d * b is a multiple of 32
        uint32_t* out = codes + (base * B) / 32;
        const uint32_t mwords = (m * B + 31) / 32;
        if (kLaneBits >= 32) {
#pragma unroll
            for (int w = 0; w < kLaneWords; ++w) {
                const uint32_t ow = static_cast<uint32_t>(lane) * kLaneWords + w;
                if (ow < mwords) out[ow] = part[w];
            }
        } else {
            uint32_t word = part[0] << (32 - kLaneBits * (1 + lane % G));
#pragma unroll
            for (int o = 1; o < G; o <<= 1) word |= __shfl_xor_sync(kAll, word, o);
            const uint32_t ow = static_cast<uint32_t>(lane) / G;
            if (lane % G == 0 && ow < mwords) out[ow] = word;
        }
    }
}

// ---------------------------------------------------------------------------
// Encoder, any shape: bucket norms (one warp per bucket), then one thread per code
// word, which quantises the 32/b coordinates the word holds with their buckets'
// scales (its first coordinate is a multiple of 4: one Philox block per 4).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kBbitBlock) bbit_norms(const float* __restrict__ in, uint64_t n, uint32_t d,
                                                         uint32_t s, uint32_t norm_kind, float* norms,
                                                         uint32_t* status) {
    const int lane = threadIdx.x & 31;
    const uint64_t nb = (n + d - 1) / d;
    const uint64_t gwarps = static_cast<uint64_t>(gridDim.x) * (kBbitBlock / 32);
    for (uint64_t bk = static_cast<uint64_t>(blockIdx.x) * (kBbitBlock / 32) + (threadIdx.x >> 5); bk < nb;
         bk += gwarps) {
        const float* p = in + bk * d;
        const uint64_t m = min(static_cast<uint64_t>(d), n - bk * d);
        if (norm_kind == QSGD_NORM_MAX) {  // uniform in the grid
            const BucketScale sc = bucket_scale(warp_maxnorm(p, m, lane), s, true, status, lane == 0);
            if (lane == 0) norms[bk] = sc.sent;
            continue;
        }
        float ss = 0.f;
        for (uint64_t i = lane; i < m; i += 32) ss = __fmaf_rn(p[i], p[i], ss);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss = __fadd_rn(ss, __shfl_xor_sync(kAll, ss, o));
        float norm = __fsqrt_rn(ss);
        if (needs_rescale(ss) && !isnan(ss)) {  // uniform in the warp
            float mx = 0.f;
            for (uint64_t i = lane; i < m; i += 32) mx = fmaxf(mx, fabsf(p[i]));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kAll, mx, o));
            if (isinf(mx)) {
                norm = mx;
            } else if (mx > 0.f) {
                float unscale;
                const float scale = pow2_scale(mx, unscale);
                float s2 = 0.f;
                for (uint64_t i = lane; i < m; i += 32) {
                    const float y = __fmul_rn(p[i], scale);
                    s2 = __fmaf_rn(y, y, s2);
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) s2 = __fadd_rn(s2, __shfl_xor_sync(kAll, s2, o));
                norm = __fmul_rn(__fsqrt_rn(s2), unscale);
            }
        }
        const BucketScale sc = bucket_scale(norm, s, true, status, lane == 0);
        if (lane == 0) norms[bk] = sc.sent;
    }
}

template <int B>
__global__ void __launch_bounds__(kBbitBlock) bbit_pack(const float* __restrict__ in, uint64_t n, uint32_t d,
                                                        uint64_t seed, const float* __restrict__ norms,
                                                        uint32_t* codes) {
    constexpr uint32_t S = (1u << (B - 1)) - 1u;
    constexpr int PER = 32 / B;  // coordinates per word: 16, 8, 4
    const uint64_t nw = (n * B + 31) / 32;
    const PhiloxKey key{static_cast<uint32_t>(seed), static_cast<uint32_t>(seed >> 32)};
    for (uint64_t w = static_cast<uint64_t>(blockIdx.x) * kBbitBlock + threadIdx.x; w < nw;
         w += static_cast<uint64_t>(gridDim.x) * kBbitBlock) {
        const uint64_t i0 = w * PER;
        uint32_t word = 0u;
        uint64_t bk = i0 / d;
        uint64_t bend = (bk + 1) * d;
        float norm = norms[bk];
        float sinv = norm > 0.f ? __fdiv_rn(__uint2float_rn(S), norm) : 0.f;
#pragma unroll
        for (int j = 0; j < PER / 4; ++j) {
            const uint4 rr = philox4x32_10((i0 >> 2) + j, key);
            const uint32_t rw[4] = {rr.x, rr.y, rr.z, rr.w};
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const uint64_t i = i0 + 4 * j + c;
                if (i >= n) break;
                if (i >= bend) {  // the word crosses into the next bucket
                    bk = i / d;
                    bend = (bk + 1) * d;
                    norm = norms[bk];
                    sinv = norm > 0.f ? __fdiv_rn(__uint2float_rn(S), norm) : 0.f;
                }
                const uint32_t code = norm > 0.f ? bbit_code(in[i], sinv, rw[c], S, B) : 0u;
                word |= code << (32 - B * (1 + 4 * j + c));
            }
        }
        codes[w] = word;
    }
}

// ---------------------------------------------------------------------------
// Decoder: one thread per 4 coordinates (d % 4 == 0, 16-byte aligned output) or
// per coordinate.  BAD_STREAM for a negative or non-finite norm, a non-zero code
// under a zero norm or a zero scale, or a code with sign 1 and k = 0.  The
// accumulating form adds q (+0.0 off the support) to the output: out + q.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float bbit_value(uint32_t code, float norm, float scale, uint32_t s, uint32_t b,
                                            bool& bad) {
    const uint32_t sign = code >> (b - 1);
    const uint32_t k = code & s;
    if (k == 0) {
        bad |= sign != 0;
        return 0.0f;
    }
    bad |= !(norm > 0.f) || !(scale > 0.f);
    const float v = __fmul_rn(scale, __uint2float_rn(k));
    return sign ? -v : v;
}

template <int B, bool kAccumulate>
__global__ void __launch_bounds__(kBbitBlock) bbit_decode_vec(const float* __restrict__ norms,
                                                              const uint32_t* __restrict__ codes, uint64_t n,
                                                              uint32_t d, float* out, uint32_t* status) {
    constexpr uint32_t S = (1u << (B - 1)) - 1u;
    const uint64_t n4 = n / 4;
    bool bad = false;
    for (uint64_t t = static_cast<uint64_t>(blockIdx.x) * kBbitBlock + threadIdx.x; t < n4;
         t += static_cast<uint64_t>(gridDim.x) * kBbitBlock) {
        const uint64_t i0 = 4 * t;
        const float norm = __ldg(norms + i0 / d);
        bad |= !isfinite(norm) || signbit(norm);
        const float scale = __fdiv_rn(norm, __uint2float_rn(S));
        const uint64_t bit = i0 * B;  // 4b bits, inside one word
        const uint32_t w = __ldg(codes + bit / 32);
        const uint32_t bits4 = (w << (bit % 32)) >> (32 - 4 * B);
        float4 v;
        v.x = bbit_value((bits4 >> (3 * B)) & ((1u << B) - 1u), norm, scale, S, B, bad);
        v.y = bbit_value((bits4 >> (2 * B)) & ((1u << B) - 1u), norm, scale, S, B, bad);
        v.z = bbit_value((bits4 >> B) & ((1u << B) - 1u), norm, scale, S, B, bad);
        v.w = bbit_value(bits4 & ((1u << B) - 1u), norm, scale, S, B, bad);
        float4* o = reinterpret_cast<float4*>(out) + t;
        if (kAccumulate) {
            const float4 x = *o;
            v.x = __fadd_rn(x.x, v.x);
            v.y = __fadd_rn(x.y, v.y);
            v.z = __fadd_rn(x.z, v.z);
            v.w = __fadd_rn(x.w, v.w);
        }
        *o = v;
    }
    // the last n % 4 coordinates
    const uint64_t tail = n4 * 4 + static_cast<uint64_t>(blockIdx.x) * kBbitBlock + threadIdx.x;
    if (tail < n && tail < n4 * 4 + 4) {
        const float norm = __ldg(norms + tail / d);
        bad |= !isfinite(norm) || signbit(norm);
        const float scale = __fdiv_rn(norm, __uint2float_rn(S));
        const uint64_t bit = tail * B;
        const uint32_t code = (__ldg(codes + bit / 32) >> (32 - B - bit % 32)) & ((1u << B) - 1u);
        const float q = bbit_value(code, norm, scale, S, B, bad);
        out[tail] = kAccumulate ? __fadd_rn(out[tail], q) : q;
    }
    if (__any_sync(kAll, bad) && (threadIdx.x & 31) == 0) report(status, QSGD_ST_BAD_STREAM);
}

template <int B, bool kAccumulate>
__global__ void __launch_bounds__(kBbitBlock) bbit_decode_scalar(const float* __restrict__ norms,
                                                                 const uint32_t* __restrict__ codes, uint64_t n,
                                                                 uint32_t d, float* out, uint32_t* status) {
    constexpr uint32_t S = (1u << (B - 1)) - 1u;
    bool bad = false;
    for (uint64_t i = static_cast<uint64_t>(blockIdx.x) * kBbitBlock + threadIdx.x; i < n;
         i += static_cast<uint64_t>(gridDim.x) * kBbitBlock) {
        const float norm = __ldg(norms + i / d);
        bad |= !isfinite(norm) || signbit(norm);
        const float scale = __fdiv_rn(norm, __uint2float_rn(S));
        const uint64_t bit = i * B;
        const uint32_t code = (__ldg(codes + bit / 32) >> (32 - B - bit % 32)) & ((1u << B) - 1u);
        const float q = bbit_value(code, norm, scale, S, B, bad);
        out[i] = kAccumulate ? __fadd_rn(out[i], q) : q;
    }
    if (__any_sync(kAll, bad) && (threadIdx.x & 31) == 0) report(status, QSGD_ST_BAD_STREAM);
}

int grid_for(uint64_t items, int per_sm_blocks = 8) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const uint64_t want = (items + kBbitBlock - 1) / kBbitBlock;
    return static_cast<int>(std::max<uint64_t>(1, std::min<uint64_t>(want, static_cast<uint64_t>(sms) * per_sm_blocks)));
}

bool fast_shape(const float* in, const float* ef, uint32_t d) {
    const bool pow2v = d == 128 || d == 256 || d == 512 || d == 1024;
    return pow2v && ((reinterpret_cast<uintptr_t>(in) | reinterpret_cast<uintptr_t>(ef)) & 15u) == 0;
}

template <int B, bool kEF>
cudaError_t launch_bbit_fast(const float* in, float* ef, uint64_t n, uint32_t d, uint64_t seed, uint32_t nk,
                             float* norms, uint32_t* codes, uint32_t* status, cudaStream_t stream) {
    const int grid = grid_for(((n + d - 1) / d) * 32);
    switch (d / 128) {
        case 1: bbit_encode_fast<1, B, kEF><<<grid, kBbitBlock, 0, stream>>>(in, ef, n, d, seed, nk, norms, codes, status); break;
        case 2: bbit_encode_fast<2, B, kEF><<<grid, kBbitBlock, 0, stream>>>(in, ef, n, d, seed, nk, norms, codes, status); break;
        case 4: bbit_encode_fast<4, B, kEF><<<grid, kBbitBlock, 0, stream>>>(in, ef, n, d, seed, nk, norms, codes, status); break;
        default: bbit_encode_fast<8, B, kEF><<<grid, kBbitBlock, 0, stream>>>(in, ef, n, d, seed, nk, norms, codes, status); break;
    }
    return cudaGetLastError();
}

template <int B>
cudaError_t launch_bbit_encode_b(const float* in, float* ef, uint64_t n, uint32_t d, uint64_t seed, uint32_t nk,
                                 float* norms, uint32_t* codes, uint32_t* status, cudaStream_t stream) {
    // one pass: one warp per bucket of d = 128, 256, 512 or 1024, 16-byte aligned input
    if (fast_shape(in, ef, d))
        return ef ? launch_bbit_fast<B, true>(in, ef, n, d, seed, nk, norms, codes, status, stream)
                  : launch_bbit_fast<B, false>(in, ef, n, d, seed, nk, norms, codes, status, stream);
    const uint64_t nb = (n + d - 1) / d;
    bbit_norms<<<grid_for(nb * 32), kBbitBlock, 0, stream>>>(in, n, d, (1u << (B - 1)) - 1u, nk, norms, status);
    bbit_pack<B><<<grid_for((n * B + 31) / 32), kBbitBlock, 0, stream>>>(in, n, d, seed, norms, codes);
    return cudaGetLastError();
}

template <int B, bool kAcc>
cudaError_t launch_bbit_decode_b(const float* norms, const uint32_t* codes, uint64_t n, uint32_t d, float* out,
                                 uint32_t* status, cudaStream_t stream) {
    if (d % 4 == 0 && (reinterpret_cast<uintptr_t>(out) & 15u) == 0)
        bbit_decode_vec<B, kAcc><<<grid_for(n / 4 + 4), kBbitBlock, 0, stream>>>(norms, codes, n, d, out, status);
    else
        bbit_decode_scalar<B, kAcc><<<grid_for(n), kBbitBlock, 0, stream>>>(norms, codes, n, d, out, status);
    return cudaGetLastError();
}

}  // namespace

bool bbit_fast_shape(const float* in, const float* ef, uint32_t d) { return fast_shape(in, ef, d); }

cudaError_t launch_bbit_encode(const float* in, float* ef, uint64_t n, uint32_t d, uint32_t b, uint64_t seed,
                               uint32_t norm_kind, float* norms, uint32_t* codes, uint32_t* status,
                               cudaStream_t stream) {
    if (ef && !fast_shape(in, ef, d)) return cudaErrorInvalidValue;
    switch (b) {
        case 2: return launch_bbit_encode_b<2>(in, ef, n, d, seed, norm_kind, norms, codes, status, stream);
        case 4: return launch_bbit_encode_b<4>(in, ef, n, d, seed, norm_kind, norms, codes, status, stream);
        default: return launch_bbit_encode_b<8>(in, ef, n, d, seed, norm_kind, norms, codes, status, stream);
    }
}

cudaError_t launch_bbit_decode(const float* norms, const uint32_t* codes, uint64_t n, uint32_t d, uint32_t b,
                               float* out, bool accumulate, uint32_t* status, cudaStream_t stream) {
    switch (b) {
        case 2:
            return accumulate ? launch_bbit_decode_b<2, true>(norms, codes, n, d, out, status, stream)
                              : launch_bbit_decode_b<2, false>(norms, codes, n, d, out, status, stream);
        case 4:
            return accumulate ? launch_bbit_decode_b<4, true>(norms, codes, n, d, out, status, stream)
                              : launch_bbit_decode_b<4, false>(norms, codes, n, d, out, status, stream);
        default:
            return accumulate ? launch_bbit_decode_b<8, true>(norms, codes, n, d, out, status, stream)
                              : launch_bbit_decode_b<8, false>(norms, codes, n, d, out, status, stream);
    }
}

}  // namespace qsgd
