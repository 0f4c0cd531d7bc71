// QSGD encoder kernels (sm_100a).
//
// Method: "QSGD (Quantized Stochastic Gradient Descent) with Elias Coding" (AIMech
// curated entry).  Per bucket (claim "QSVRG, non-convex and multi-GPU bucketed
// training", section 3.3 bucketing): the L2 norm, unbiased stochastic rounding of
// every coordinate to one of s+1 levels (definition paragraph), and the Elias-omega
// coding of the tuple (norm, signs, run-length gaps, levels) (definition paragraph;
// claim "Elias coding communication complexity tradeoff", F = 32).
//
// Single pass over the input.  The stream position of every tile comes from a
// prefix scan with decoupled look-back (Merrill & Garland 2016): each tile publishes
// its bit count, then its inclusive prefix; tiles are handed out in order by an
// atomic ticket so every wait is on a tile that is already running.  A tile's bits
// are assembled in shared memory at tile-local offsets and stored with a funnel
// shift once the prefix is known; the one word a tile shares with its predecessor
// is written by the later tile, from the predecessor's published tail word, so
// every output word has exactly one writer and the output needs no clearing.
//
// Two kernels:
//   encode_fast<V>   128 <= d <= 1024, d % 4 == 0, 16-byte aligned input: one warp
//                    per bucket, lane-contiguous 4V coordinates in registers,
//                    8 buckets per tile, persistent CTAs.
//   encode_general   any d and alignment: a norm pre-pass (one warp per bucket),
//                    then tiles of whole buckets (>= 4096 coordinates or one
//                    bucket) streamed in chunks of 1024 coordinates, twice (bit
//                    count, then packing).
#include <cuda_runtime.h>

#include <algorithm>

#include "../../include/qsgd.h"
#include "qsgd_device.cuh"
#include "qsgd_internal.h"

namespace qsgd {
namespace {

constexpr uint32_t kFull = 0xFFFFFFFFu;

__device__ __forceinline__ void report(uint32_t* status, uint32_t bits) { atomicOr(status, bits); }

__device__ __forceinline__ void store_word(const EncodeArgs& a, uint64_t gw, uint32_t v) {
    if (gw < a.cap_words)
        a.words[gw] = v;
    else
        report(a.status, QSGD_ST_OVERFLOW);
}

// Bucket norm and the reciprocal scale s/norm (definition paragraph: the levels
// are s|v_i|/||v||_2).  Degenerate buckets (zero, non-finite, or s/norm beyond
// fp32) are sent as a zero norm with no record.
struct BucketScale {
    float sent;
    float sinv;
    bool good;
};

__device__ __forceinline__ BucketScale bucket_scale(float norm, uint32_t s, bool live,
                                                    uint32_t* status, bool reporter) {
    BucketScale r{0.f, 0.f, false};
    if (!live) return r;
    if (!isfinite(norm)) {
        if (reporter) report(status, QSGD_ST_NONFINITE);
        return r;
    }
    if (norm == 0.f) return r;
    const float sinv = __fdiv_rn(__uint2float_rn(s), norm);
    if (isinf(sinv)) {
        if (reporter) report(status, QSGD_ST_RANGE);
        return r;
    }
    r.sent = norm;
    r.sinv = sinv;
    r.good = true;
    return r;
}

// A plain fp32 sum of squares loses accuracy when squares leave the normal range.
// Such buckets (sum below 2^-60, infinite, or NaN) are recomputed with every
// value multiplied by 2^(127-E), E the exponent field of max|v| (clamped to
// [1, 253]), so the largest scaled value lies in [1, 2); the root is scaled
// back by the exact power of two 2^(E-127).
__device__ __forceinline__ bool needs_rescale(float sumsq) {
    return !(sumsq >= 0x1p-60f) || isinf(sumsq);
}
__device__ __forceinline__ float pow2_scale(float maxabs, float& unscale) {
    uint32_t e = (__float_as_uint(maxabs) >> 23) & 0xFFu;
    e = e < 1u ? 1u : (e > 253u ? 253u : e);
    unscale = __uint_as_float(e << 23);        // 2^(e-127)
    return __uint_as_float((254u - e) << 23);  // 2^(127-e)
}

// Waits (bounded) for the tail word of tile `tile - 1`.
__device__ __forceinline__ bool wait_carry(const EncodeArgs& a, uint32_t tile, uint32_t epoch,
                                           uint32_t& word) {
    const uint64_t* slot = a.carry + (tile - 1);
    for (uint32_t polls = 0;; ++polls) {
        const uint64_t c = ld_acquire(slot);
        if ((c >> 63) != 0 && static_cast<uint32_t>((c >> 32) & kEpochMask) == (epoch & kEpochMask)) {
            word = static_cast<uint32_t>(c);
            return true;
        }
        if (polls > kMaxPolls) return false;
        if ((polls & 63u) == 63u && ld_acquire32(&a.ctrl->abort) != 0) return false;
        __nanosleep(polls < 64 ? 32 : 256);
    }
}

__device__ __forceinline__ void publish_carry(const EncodeArgs& a, uint32_t tile, uint32_t epoch,
                                              uint32_t word) {
    // [63] present, [55:32] epoch, [31:0] the tail word (a zero-filled slot is never "present")
    st_release(a.carry + tile, (uint64_t(1) << 63) | (static_cast<uint64_t>(epoch & kEpochMask) << 32) |
                                   static_cast<uint64_t>(word));
}

__device__ __forceinline__ void abort_all(const EncodeArgs& a) {
    report(a.status, QSGD_ST_LOOKBACK_TIMEOUT);
    atomicExch(&a.ctrl->abort, 1u);
}

// Last CTA out resets the ticket and completion counters and advances the epoch.
__device__ __forceinline__ void cta_exit(ScanControl* ctrl, uint32_t epoch) {
    if (threadIdx.x == 0) {
        __threadfence();
        const uint32_t prev = atomicAdd(&ctrl->done, 1u);
        if (prev == gridDim.x - 1) {
            ctrl->ticket = 0;
            ctrl->done = 0;
            ctrl->abort = 0;
            __threadfence();
            atomicExch(&ctrl->epoch, (epoch + 1) & kEpochMask);
        }
    }
}

// Stores the words of a tile whose bits sit at tile-local offsets in tw[] and
// whose stream prefix is X.  Word q of the tile's global range is
// (tw[q] >> sh) | (tw[q-1] << (32 - sh)), sh = X mod 32.  Word 0 (when sh != 0)
// also holds the predecessor's last bits and is written here after its tail word
// arrives; the tile's own partial last word is published for the successor (or
// stored, for the last tile).
__device__ __forceinline__ void store_tile(const EncodeArgs& a, const uint32_t* tw, uint32_t tile,
                                           uint64_t X, uint64_t tb, uint32_t epoch) {
    const uint32_t sh = static_cast<uint32_t>(X & 31u);
    const uint64_t w0 = X >> 5;
    const uint64_t end = X + tb;
    const uint32_t qe = static_cast<uint32_t>((end >> 5) - w0);
    const bool has_tail = (end & 31u) != 0;
    const uint32_t limit = a.smem_words;
    auto word_at = [&](uint32_t q) -> uint32_t {
        const uint32_t cur = q < limit ? tw[q] : 0u;
        if (sh == 0) return cur;
        const uint32_t prv = (q > 0 && q - 1 < limit) ? tw[q - 1] : 0u;
        return (cur >> sh) | (prv << (32 - sh));
    };
    const int tid = threadIdx.x;
    if (tid == 0 && has_tail) {
        const uint32_t tv = word_at(qe);
        if (tile + 1 == a.ntiles)
            store_word(a, w0 + qe, tv);
        else
            publish_carry(a, tile, epoch, tv);
    }
    for (uint32_t q = (sh ? 1u : 0u) + tid; q < qe; q += kBlock) store_word(a, w0 + q, word_at(q));
    if (tid == 32 && sh != 0) {  // a lane of warp 1, so warp 0's tail publication is not delayed
        uint32_t head;
        if (wait_carry(a, tile, epoch, head))
            store_word(a, w0, head | word_at(0));
        else
            abort_all(a);
    }
}

// ---------------------------------------------------------------------------
// Fast path: one warp per bucket of 128 < d <= 128*V coordinates.
// ---------------------------------------------------------------------------
template <int V>
__global__ void __launch_bounds__(kBlock) encode_fast(const __grid_constant__ EncodeArgs a) {
    extern __shared__ __align__(16) uint32_t smem[];
    uint32_t* tab = smem;
    uint32_t* tw = smem + kOmegaTab;
    __shared__ uint32_t s_tile;
    __shared__ uint32_t s_bits[kWarps];
    __shared__ uint64_t s_off[kWarps + 1];
    __shared__ uint64_t s_prefix;
    __shared__ int s_ok;

    constexpr int NC = 4 * V;  // coordinates per lane
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    omega_table_fill(tab, tid, kBlock);
    const uint32_t epoch = *reinterpret_cast<volatile uint32_t*>(&a.ctrl->epoch);
    const PhiloxKey key{a.key0, a.key1};

    for (;;) {
        if (tid == 0) s_tile = atomicAdd(&a.ctrl->ticket, 1u);
        for (uint32_t i = tid; i < a.smem_words; i += kBlock) tw[i] = 0u;
        __syncthreads();
        const uint32_t tile = s_tile;
        if (tile >= a.ntiles) break;

        const uint64_t b = static_cast<uint64_t>(tile) * kWarps + warp;
        const bool live = b < a.nb;
        const uint64_t base = b * a.d;
        const uint32_t m = live ? static_cast<uint32_t>(min(static_cast<uint64_t>(a.d), a.n - base)) : 0u;
        const uint32_t first = lane * NC;  // first bucket-local coordinate of this lane

        // --- load: 4V consecutive coordinates per lane --------------------
        float x[NC];
#pragma unroll
        for (int j = 0; j < V; ++j) {
            const uint32_t i = first + 4 * j;
            if (i + 4 <= m) {
                const float4 q = __ldg(reinterpret_cast<const float4*>(a.in + base + i));
                x[4 * j + 0] = q.x;
                x[4 * j + 1] = q.y;
                x[4 * j + 2] = q.z;
                x[4 * j + 3] = q.w;
            } else {
#pragma unroll
                for (int c = 0; c < 4; ++c) x[4 * j + c] = (i + c < m) ? __ldg(a.in + base + i + c) : 0.f;
            }
        }

        // --- bucket norm: per-lane FMA chain, then a butterfly (identical in all lanes)
        float ss = 0.f;
#pragma unroll
        for (int q = 0; q < NC; ++q) ss = __fmaf_rn(x[q], x[q], ss);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss = __fadd_rn(ss, __shfl_xor_sync(kFull, ss, o));
        float norm = __fsqrt_rn(ss);
        if (live && needs_rescale(ss) && !isnan(ss)) {  // uniform in the warp
            float mx = 0.f;
#pragma unroll
            for (int q = 0; q < NC; ++q) mx = fmaxf(mx, fabsf(x[q]));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, o));
            if (isinf(mx)) {
                norm = mx;
            } else if (mx > 0.f) {
                float unscale;
                const float scale = pow2_scale(mx, unscale);
                float s2 = 0.f;
#pragma unroll
                for (int q = 0; q < NC; ++q) {
                    const float y = __fmul_rn(x[q], scale);
                    s2 = __fmaf_rn(y, y, s2);
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) s2 = __fadd_rn(s2, __shfl_xor_sync(kFull, s2, o));
                norm = __fmul_rn(__fsqrt_rn(s2), unscale);
            }
        }
        const BucketScale sc = bucket_scale(norm, a.s, live, a.status, lane == 0);
        if (!sc.good) {
#pragma unroll
            for (int q = 0; q < NC; ++q) x[q] = 0.f;
        }

        // --- stochastic rounding: one Philox block per 4 coordinates --------
        uint32_t kq[NC];  // level | sign << 31
        const uint64_t g0 = base + first;  // a multiple of 4
#pragma unroll
        for (int j = 0; j < V; ++j) {
            const uint4 r = philox4x32_10((g0 >> 2) + j, key);
            const uint32_t rw[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float v = x[4 * j + c];
                kq[4 * j + c] = quantize_level(v, sc.sinv, rw[c], a.s) | (__float_as_uint(v) & 0x80000000u);
            }
        }

        // --- gaps: previous non-zero before this lane (exclusive max-scan) --
        int last = -1;
#pragma unroll
        for (int q = 0; q < NC; ++q)
            if (kq[q] & 0x7FFFFFFFu) last = static_cast<int>(first) + q;
        int incl = last;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(kFull, incl, o);
            if (lane >= o) incl = max(incl, t);
        }
        int prev0 = __shfl_up_sync(kFull, incl, 1);
        if (lane == 0) prev0 = -1;

        // --- code lengths: omega(gap) + sign + omega(k) per record ----------
        uint32_t bits = 0;
        {
            int prev = prev0;
#pragma unroll
            for (int q = 0; q < NC; ++q) {
                const uint32_t k = kq[q] & 0x7FFFFFFFu;
                if (k) {
                    const int i = static_cast<int>(first) + q;
                    bits += omega_len(tab, static_cast<uint32_t>(i - prev)) + 1u + omega_len(tab, k);
                    prev = i;
                }
            }
        }
        uint32_t inclb = bits;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t t = __shfl_up_sync(kFull, inclb, o);
            if (lane >= o) inclb += t;
        }
        const uint32_t total = __shfl_sync(kFull, inclb, 31);
        const uint32_t exclb = inclb - bits;
        if (lane == 0) s_bits[warp] = live ? 32u + total : 0u;
        __syncthreads();

        // --- tile aggregate: publish it (tile 0: the inclusive prefix) ------
        if (tid == 0) {
            uint64_t acc = 0;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) {
                s_off[w] = acc;
                acc += s_bits[w];
            }
            s_off[kWarps] = acc;
            st_release(a.desc + tile, make_desc(epoch, tile == 0 ? kStatePrefix : kStateAggregate, acc));
        }
        __syncthreads();

        // --- pack the bucket at its tile-local offset ----------------------
        if (live) {
            const uint64_t bstart = s_off[warp];
            if (lane == 0) {
                const uint32_t nbits = __float_as_uint(sc.sent);
                const uint32_t w = static_cast<uint32_t>(bstart >> 5), sh = static_cast<uint32_t>(bstart & 31u);
                atomicOr(&tw[w], nbits >> sh);
                if (sh) atomicOr(&tw[w + 1], nbits << (32 - sh));
            }
            BitPacker pk;
            pk.start(tw, a.smem_words, bstart + 32u + exclb);
            bool ok = true;
            int prev = prev0;
#pragma unroll
            for (int q = 0; q < NC; ++q) {
                const uint32_t k = kq[q] & 0x7FFFFFFFu;
                if (k) {
                    const int i = static_cast<int>(first) + q;
                    uint64_t gc, kc;
                    uint32_t gl, kl;
                    omega_code(tab, static_cast<uint32_t>(i - prev), gc, gl);
                    omega_code(tab, k, kc, kl);
                    prev = i;
                    ok &= pk.put((gc << 1) | (kq[q] >> 31), gl + 1u);
                    ok &= pk.put(kc, kl);
                }
            }
            ok &= pk.flush();
            if (!ok) report(a.status, QSGD_ST_OVERFLOW);
        }
        __syncthreads();

        // --- look-back (warp 0) -------------------------------------------
        if (warp == 0) {
            uint64_t excl = 0;
            bool ok = true;
            if (tile > 0) ok = lookback(a.desc, tile, epoch, &a.ctrl->abort, excl);
            if (lane == 0) {
                if (!ok)
                    abort_all(a);
                else if (tile > 0)
                    st_release(a.desc + tile, make_desc(epoch, kStatePrefix, excl + s_off[kWarps]));
                s_prefix = excl;
                s_ok = ok;
            }
        }
        __syncthreads();

        // --- offsets header and words -------------------------------------
        if (s_ok) {
            const uint64_t X = s_prefix;
            if (tid < kWarps) {
                const uint64_t bb = static_cast<uint64_t>(tile) * kWarps + tid;
                if (bb < a.nb) a.offsets[bb] = X + s_off[tid];
            }
            if (tid == kWarps && tile + 1 == a.ntiles) a.offsets[a.nb] = X + s_off[kWarps];
            store_tile(a, tw, tile, X, s_off[kWarps], epoch);
        }
        __syncthreads();
    }
    cta_exit(a.ctrl, epoch);
}

// ---------------------------------------------------------------------------
// General path.
// ---------------------------------------------------------------------------

// One warp per bucket: norm and s/norm into the workspace.
__global__ void __launch_bounds__(kBlock) encode_norms(const __grid_constant__ EncodeArgs a) {
    const int lane = threadIdx.x & 31;
    const uint64_t warps = static_cast<uint64_t>(gridDim.x) * kWarps;
    for (uint64_t b = (static_cast<uint64_t>(blockIdx.x) * kBlock + threadIdx.x) >> 5; b < a.nb; b += warps) {
        const uint64_t base = b * a.d;
        const uint64_t m = min(static_cast<uint64_t>(a.d), a.n - base);
        float ss = 0.f;
        for (uint64_t i = lane; i < m; i += 32) {
            const float v = __ldg(a.in + base + i);
            ss = __fmaf_rn(v, v, ss);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss = __fadd_rn(ss, __shfl_xor_sync(kFull, ss, o));
        float norm = __fsqrt_rn(ss);
        if (needs_rescale(ss) && !isnan(ss)) {  // uniform in the warp
            float mx = 0.f;
            for (uint64_t i = lane; i < m; i += 32) mx = fmaxf(mx, fabsf(__ldg(a.in + base + i)));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, o));
            if (isinf(mx)) {
                norm = mx;
            } else if (mx > 0.f) {
                float unscale;
                const float scale = pow2_scale(mx, unscale);
                float s2 = 0.f;
                for (uint64_t i = lane; i < m; i += 32) {
                    const float y = __fmul_rn(__ldg(a.in + base + i), scale);
                    s2 = __fmaf_rn(y, y, s2);
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) s2 = __fadd_rn(s2, __shfl_xor_sync(kFull, s2, o));
                norm = __fmul_rn(__fsqrt_rn(s2), unscale);
            }
        }
        const BucketScale sc = bucket_scale(norm, a.s, true, a.status, lane == 0);
        if (lane == 0) a.norms[b] = make_float2(sc.sent, sc.good ? sc.sinv : 0.f);
    }
}

// Block-wide scans for kBlock threads.
struct BlockScratch {
    int64_t i64[kWarps];
    uint32_t u32[kWarps];
};

// Exclusive max-scan of x with `carry` as the value before thread 0; returns the
// exclusive value and sets `all` to the maximum over carry and every x.
__device__ __forceinline__ int64_t block_excl_max(int64_t x, int64_t carry, BlockScratch& sc,
                                                  int64_t& all) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int64_t incl = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int64_t t = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl = max(incl, t);
    }
    if (lane == 31) sc.i64[warp] = incl;
    __syncthreads();
    int64_t before = carry;
    for (int w = 0; w < warp; ++w) before = max(before, sc.i64[w]);
    all = carry;
    for (int w = 0; w < kWarps; ++w) all = max(all, sc.i64[w]);
    int64_t excl = __shfl_up_sync(kFull, incl, 1);
    excl = lane == 0 ? before : max(before, excl);
    __syncthreads();
    return excl;
}

__device__ __forceinline__ uint32_t block_excl_sum(uint32_t x, BlockScratch& sc, uint32_t& total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t incl = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t t = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += t;
    }
    if (lane == 31) sc.u32[warp] = incl;
    __syncthreads();
    uint32_t before = 0;
    total = 0;
    for (int w = 0; w < kWarps; ++w) {
        if (w < warp) before += sc.u32[w];
        total += sc.u32[w];
    }
    __syncthreads();
    return before + incl - x;
}

// The four coordinates of one thread in one chunk, quantised.
struct Quad {
    uint32_t kq[4];      // level | sign << 31
    uint32_t start[4];   // 1 when the coordinate opens its bucket
    uint64_t bstart[4];  // global index of its bucket's first coordinate
    uint64_t bucket[4];
    float sent[4];
    bool valid[4];
};

__device__ __forceinline__ void quantize_quad(const EncodeArgs& a, uint64_t i0, uint64_t c0,
                                              uint64_t c1, uint64_t b0, PhiloxKey key, Quad& qd) {
    const uint4 r = philox4x32_10(i0 >> 2, key);
    const uint32_t rw[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const uint64_t i = i0 + c;
        qd.valid[c] = i >= c0 && i < c1;
        qd.kq[c] = 0;
        qd.start[c] = 0;
        qd.bstart[c] = 0;
        qd.bucket[c] = 0;
        qd.sent[c] = 0.f;
        if (!qd.valid[c]) continue;
        const uint32_t rel = static_cast<uint32_t>(i - c0);  // < buckets_per_tile * d <= 2^31
        const uint64_t bl = rel / a.d;
        const uint64_t b = b0 + bl;
        const float2 ns = a.norms[b];
        const float v = __ldg(a.in + i);
        qd.bucket[c] = b;
        qd.bstart[c] = b * a.d;
        qd.start[c] = (i == qd.bstart[c]) ? 1u : 0u;
        qd.sent[c] = ns.x;
        const uint32_t k = (ns.y != 0.f) ? quantize_level(v, ns.y, rw[c], a.s) : 0u;
        qd.kq[c] = k | (__float_as_uint(v) & 0x80000000u);
    }
}

__global__ void __launch_bounds__(kBlock) encode_general(const __grid_constant__ EncodeArgs a) {
    extern __shared__ __align__(16) uint32_t smem[];
    uint32_t* tab = smem;
    uint32_t* buf = smem + kOmegaTab;
    __shared__ uint32_t s_tile;
    __shared__ BlockScratch s_scr;
    __shared__ uint64_t s_prefix;
    __shared__ int s_ok;
    __shared__ uint32_t s_pending;  // partial last word carried between chunks
    __shared__ uint32_t s_head;     // own bits of the tile's first word when it is shared

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    omega_table_fill(tab, tid, kBlock);
    const uint32_t epoch = *reinterpret_cast<volatile uint32_t*>(&a.ctrl->epoch);
    const PhiloxKey key{a.key0, a.key1};

    for (;;) {
        if (tid == 0) s_tile = atomicAdd(&a.ctrl->ticket, 1u);
        __syncthreads();
        const uint32_t tile = s_tile;
        if (tile >= a.ntiles) break;
        const uint64_t b0 = static_cast<uint64_t>(tile) * a.buckets_per_tile;
        const uint64_t b1 = min(a.nb, b0 + a.buckets_per_tile);
        const uint64_t c0 = b0 * a.d;
        const uint64_t c1 = min(a.n, b1 * a.d);
        const uint64_t cbase = c0 & ~uint64_t(3);

        // --- pass 1: bit count of the tile --------------------------------
        uint64_t tb = 0;
        int64_t carry_prev = -1;
        for (uint64_t cb = cbase; cb < c1; cb += kChunk) {
            Quad qd;
            quantize_quad(a, cb + 4ull * tid, c0, c1, b0, key, qd);
            int64_t last = -1;
#pragma unroll
            for (int c = 0; c < 4; ++c)
                if (qd.kq[c] & 0x7FFFFFFFu) last = static_cast<int64_t>(cb + 4ull * tid + c);
            int64_t all;
            int64_t prev = block_excl_max(last, carry_prev, s_scr, all);
            carry_prev = all;
            uint32_t bits = 0;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                if (!qd.valid[c]) continue;
                const int64_t i = static_cast<int64_t>(cb + 4ull * tid + c);
                if (qd.start[c]) bits += 32u;
                const uint32_t k = qd.kq[c] & 0x7FFFFFFFu;
                if (k) {
                    const int64_t p = max(prev, static_cast<int64_t>(qd.bstart[c]) - 1);
                    bits += omega_len(tab, static_cast<uint64_t>(i - p)) + 1u + omega_len(tab, k);
                    prev = i;
                }
            }
            uint32_t total;
            block_excl_sum(bits, s_scr, total);
            tb += total;
        }
        if (tid == 0)
            st_release(a.desc + tile, make_desc(epoch, tile == 0 ? kStatePrefix : kStateAggregate, tb));

        // --- look-back ------------------------------------------------------
        if (warp == 0) {
            uint64_t excl = 0;
            bool ok = true;
            if (tile > 0) ok = lookback(a.desc, tile, epoch, &a.ctrl->abort, excl);
            if (lane == 0) {
                if (!ok)
                    abort_all(a);
                else if (tile > 0)
                    st_release(a.desc + tile, make_desc(epoch, kStatePrefix, excl + tb));
                s_prefix = excl;
                s_ok = ok;
                s_pending = 0;
                s_head = 0;
            }
        }
        __syncthreads();
        if (!s_ok) {
            __syncthreads();
            continue;
        }
        const uint64_t X = s_prefix;
        const uint64_t head_word = X >> 5;
        const bool head_shared = (X & 31u) != 0;

        // --- pass 2: pack chunk by chunk at global alignment ----------------
        uint64_t pos = X;  // global bit where the next chunk starts
        carry_prev = -1;
        for (uint64_t cb = cbase; cb < c1; cb += kChunk) {
            Quad qd;
            quantize_quad(a, cb + 4ull * tid, c0, c1, b0, key, qd);
            int64_t last = -1;
#pragma unroll
            for (int c = 0; c < 4; ++c)
                if (qd.kq[c] & 0x7FFFFFFFu) last = static_cast<int64_t>(cb + 4ull * tid + c);
            int64_t all;
            const int64_t prev_in = block_excl_max(last, carry_prev, s_scr, all);
            carry_prev = all;
            uint32_t bits = 0;
            {
                int64_t prev = prev_in;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    if (!qd.valid[c]) continue;
                    const int64_t i = static_cast<int64_t>(cb + 4ull * tid + c);
                    if (qd.start[c]) bits += 32u;
                    const uint32_t k = qd.kq[c] & 0x7FFFFFFFu;
                    if (k) {
                        const int64_t p = max(prev, static_cast<int64_t>(qd.bstart[c]) - 1);
                        bits += omega_len(tab, static_cast<uint64_t>(i - p)) + 1u + omega_len(tab, k);
                        prev = i;
                    }
                }
            }
            uint32_t total;
            const uint32_t excl = block_excl_sum(bits, s_scr, total);
            if (total == 0) continue;  // uniform: every thread sees the same total
            const uint64_t w0 = pos >> 5;
            const uint32_t lead = static_cast<uint32_t>(pos & 31u);
            const uint32_t nwords = (lead + total + 31u) >> 5;
            for (uint32_t q = tid; q < nwords; q += kBlock) buf[q] = (q == 0 && lead) ? s_pending : 0u;
            __syncthreads();
            {
                BitPacker pk;
                pk.start(buf, a.smem_words, lead + excl);
                bool ok = true;
                int64_t prev = prev_in;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    if (!qd.valid[c]) continue;
                    const int64_t i = static_cast<int64_t>(cb + 4ull * tid + c);
                    if (qd.start[c]) {
                        a.offsets[qd.bucket[c]] = ((w0 + pk.word) << 5) + pk.nacc;
                        ok &= pk.put(__float_as_uint(qd.sent[c]), 32);
                    }
                    const uint32_t k = qd.kq[c] & 0x7FFFFFFFu;
                    if (k) {
                        const int64_t p = max(prev, static_cast<int64_t>(qd.bstart[c]) - 1);
                        uint64_t gc, kc;
                        uint32_t gl, kl;
                        omega_code(tab, static_cast<uint64_t>(i - p), gc, gl);
                        omega_code(tab, k, kc, kl);
                        prev = i;
                        ok &= pk.put(gc, gl);
                        ok &= pk.put(qd.kq[c] >> 31, 1);
                        ok &= pk.put(kc, kl);
                    }
                }
                ok &= pk.flush();
                if (!ok) report(a.status, QSGD_ST_OVERFLOW);
            }
            __syncthreads();
            const uint64_t end = pos + total;
            const bool last_complete = (end & 31u) == 0;
            const uint32_t nfinal = last_complete ? nwords : nwords - 1;
            for (uint32_t q = tid; q < nfinal; q += kBlock) {
                const uint64_t gw = w0 + q;
                if (gw == head_word && head_shared)
                    s_head = buf[q];
                else
                    store_word(a, gw, buf[q]);
            }
            __syncthreads();
            if (tid == 0) s_pending = last_complete ? 0u : buf[nwords - 1];
            pos = end;
            __syncthreads();
        }

        // --- tail word, shared head word, end of the header ----------------
        if (tid == 0) {
            const uint64_t end = X + tb;
            if (end & 31u) {
                if (tile + 1 == a.ntiles)
                    store_word(a, end >> 5, s_pending);
                else
                    publish_carry(a, tile, epoch, s_pending);
            }
            if (tile + 1 == a.ntiles) a.offsets[a.nb] = end;
            if (head_shared) {
                uint32_t head;
                if (wait_carry(a, tile, epoch, head))
                    store_word(a, head_word, head | s_head);
                else
                    abort_all(a);
            }
        }
        __syncthreads();
    }
    cta_exit(a.ctrl, epoch);
}

template <int V>
cudaError_t launch_fast(const EncodeArgs& a, cudaStream_t stream) {
    const size_t smem = (kOmegaTab + a.smem_words) * sizeof(uint32_t);
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_set[dev]) {
        cudaFuncSetAttribute(encode_fast<V>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
        attr_set[dev] = true;
    }
    int sms = 0, per_sm = 0;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, encode_fast<V>, kBlock, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const uint64_t grid = std::min<uint64_t>(a.ntiles, static_cast<uint64_t>(sms) * per_sm);
    encode_fast<V><<<static_cast<unsigned>(grid), kBlock, smem, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_encode(EncodeArgs a, bool fast_path, cudaStream_t stream) {
    if (fast_path) {
        const uint32_t v = (a.d + 127) / 128;
        if (v <= 1) return launch_fast<1>(a, stream);
        if (v <= 2) return launch_fast<2>(a, stream);
        if (v <= 4) return launch_fast<4>(a, stream);
        return launch_fast<8>(a, stream);
    }
    int dev = 0, sms = 0, per_sm = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    // norms pre-pass: one warp per bucket
    {
        const uint64_t blocks = std::min<uint64_t>((a.nb + kWarps - 1) / kWarps, static_cast<uint64_t>(sms) * 64);
        encode_norms<<<static_cast<unsigned>(blocks), kBlock, 0, stream>>>(a);
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    const size_t smem = (kOmegaTab + a.smem_words) * sizeof(uint32_t);
    static bool attr_set[64] = {};
    if (dev < 64 && !attr_set[dev]) {
        cudaFuncSetAttribute(encode_general, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
        attr_set[dev] = true;
    }
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, encode_general, kBlock, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const uint64_t grid = std::min<uint64_t>(a.ntiles, static_cast<uint64_t>(sms) * per_sm);
    encode_general<<<static_cast<unsigned>(grid), kBlock, smem, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace qsgd
