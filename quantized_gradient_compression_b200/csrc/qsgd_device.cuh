// Device building blocks of the QSGD codec (sm_100a).
//
// Method: "QSGD (Quantized Stochastic Gradient Descent) with Elias Coding" (AIMech
// curated entry), definition paragraph and the claim "Elias coding communication
// complexity tradeoff".  Random source: Philox4x32-10 (Salmon, Moraes, Dror, Shaw,
// "Parallel Random Numbers: As Easy as 1, 2, 3", SC'11).  Integer code: Elias omega
// (Elias 1975).  The library is compiled with -fmad=false and every rounding-relevant
// fp32 operation below is an explicit _rn intrinsic.
#pragma once

#include <cstdint>

#include "../../include/qsgd.h"
#include "qsgd_limits.h"

namespace qsgd {

// ---------------------------------------------------------------------------
// Philox4x32-10.  One call yields the random words of four consecutive
// coordinates 4j..4j+3 (counter (lo32(j), hi32(j), 0, 0), key = the seed).
// ---------------------------------------------------------------------------
struct PhiloxKey {
    uint32_t k0, k1;
};

__device__ __forceinline__ uint4 philox4x32_10(uint64_t j, PhiloxKey key) {
    uint32_t c0 = static_cast<uint32_t>(j);
    uint32_t c1 = static_cast<uint32_t>(j >> 32);
    uint32_t c2 = 0u, c3 = 0u;
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        // round key: the seed advanced r times by the Weyl constants
        const uint32_t k0 = key.k0 + static_cast<uint32_t>(r) * 0x9E3779B9u;
        const uint32_t k1 = key.k1 + static_cast<uint32_t>(r) * 0xBB67AE85u;
        // S-box: two 32x32 -> 64 products; the high halves are xored with the
        // other counter words and the round key.
        const uint64_t pa = static_cast<uint64_t>(c0) * 0xD2511F53u;
        const uint64_t pb = static_cast<uint64_t>(c2) * 0xCD9E8D57u;
        c0 = static_cast<uint32_t>(pb >> 32) ^ c1 ^ k0;
        c2 = static_cast<uint32_t>(pa >> 32) ^ c3 ^ k1;
        c1 = static_cast<uint32_t>(pb);
        c3 = static_cast<uint32_t>(pa);
    }
    return make_uint4(c0, c1, c2, c3);
}

// ---------------------------------------------------------------------------
// Quantiser of one coordinate (definition paragraph):
//   t = |v| * (s/||v||), l = floor(t), p = t - l, k = l + [u < p], clamped to s.
// floor(t) comes from one round-down add: for 0 <= t < 2^23 the sum t + 2^23 lies
// in [2^23, 2^24), where fp32 spacing is 1, so rounding it down gives exactly
// 2^23 + floor(t); its low mantissa bits are floor(t) and subtracting 2^23 back is
// exact.  p = t - floor(t) is exact (Sterbenz for t >= 1, trivially below).
// u = floor(r / 2^9) * 2^-23 is built exactly as (1 + u) - 1.
// Returns k; the sign is handled by the caller.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t quantize_level(float v, float sinv, uint32_t r, uint32_t s) {
    const float t = __fmul_rn(fabsf(v), sinv);
    const float f = __fadd_rd(t, 8388608.0f);                 // 2^23 + floor(t)
    const uint32_t l = __float_as_uint(f) - 0x4B000000u;      // floor(t)
    const float p = __fsub_rn(t, __fsub_rn(f, 8388608.0f));   // exact
    const float u = __fsub_rn(__uint_as_float(0x3F800000u | (r >> 9)), 1.0f);
    const uint32_t k = l + (u < p ? 1u : 0u);
    return k < s ? k : s;
}

// ---------------------------------------------------------------------------
// Bucket norm and the reciprocal scale s/norm (definition paragraph: the levels
// are s|v_i|/||v||_2).  Degenerate buckets (zero, non-finite, or s/norm beyond
// fp32) are sent as a zero norm with no level.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void report(uint32_t* status, uint32_t bits) { atomicOr(status, bits); }

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

// Norm of a bucket held by one warp, NC values per lane in registers: a per-lane
// FMA chain and a butterfly (the same value in all lanes), with the rescaled form
// when the squares leave the normal range.  `live` is uniform in the warp.
template <int NC>
__device__ __forceinline__ float warp_bucket_norm(const float (&x)[NC], bool live) {
    constexpr uint32_t kAll = 0xFFFFFFFFu;
    float ss = 0.f;
#pragma unroll
    for (int q = 0; q < NC; ++q) ss = __fmaf_rn(x[q], x[q], ss);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss = __fadd_rn(ss, __shfl_xor_sync(kAll, ss, o));
    float norm = __fsqrt_rn(ss);
    if (live && needs_rescale(ss) && !isnan(ss)) {  // uniform in the warp
        float mx = 0.f;
#pragma unroll
        for (int q = 0; q < NC; ++q) mx = fmaxf(mx, fabsf(x[q]));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kAll, mx, o));
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
            for (int o = 16; o > 0; o >>= 1) s2 = __fadd_rn(s2, __shfl_xor_sync(kAll, s2, o));
            norm = __fmul_rn(__fsqrt_rn(s2), unscale);
        }
    }
    return norm;
}

// Max-norm max_i |v_i| of a bucket held by one warp (NC values per lane): the
// scale of the QSGDinf variant.  NaN when any value is NaN, so that the bucket is
// non-finite as under the L2 norm.  Exact: no rounding.
template <int NC>
__device__ __forceinline__ float warp_bucket_maxnorm(const float (&x)[NC]) {
    constexpr uint32_t kAll = 0xFFFFFFFFu;
    float mx = 0.f;
    bool nan = false;
#pragma unroll
    for (int q = 0; q < NC; ++q) {
        nan |= isnan(x[q]);
        mx = fmaxf(mx, fabsf(x[q]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kAll, mx, o));
    return __any_sync(kAll, nan) ? __uint_as_float(0x7FC00000u) : mx;
}

// The same over m values at p, read by one warp (lanes take every 32nd value).
__device__ __forceinline__ float warp_maxnorm(const float* p, uint64_t m, int lane) {
    constexpr uint32_t kAll = 0xFFFFFFFFu;
    float mx = 0.f;
    bool nan = false;
    for (uint64_t i = lane; i < m; i += 32) {
        const float v = __ldg(p + i);
        nan |= isnan(v);
        mx = fmaxf(mx, fabsf(v));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kAll, mx, o));
    return __any_sync(kAll, nan) ? __uint_as_float(0x7FC00000u) : mx;
}

// ---------------------------------------------------------------------------
// Error-feedback memory ("Sparsified SGD with Memory", abstract: the compressor
// keeps what it did not send and adds it to the next gradient).  One lane's NC = 4V
// coordinates [first, first + NC) of a bucket of m values at p: loads give zeros
// past m, stores write nothing past m.  The memory is read once and written once
// per step, so both stream past L1 (.cs).  p + first is 16-byte aligned.
// ---------------------------------------------------------------------------
template <int V>
__device__ __forceinline__ void ef_load(const float* p, uint32_t first, uint32_t m, float (&v)[4 * V]) {
#pragma unroll
    for (int j = 0; j < V; ++j) {
        const uint32_t i = first + 4 * j;
        float4 q = make_float4(0.f, 0.f, 0.f, 0.f);
        if (i + 4 <= m) {
            q = __ldcs(reinterpret_cast<const float4*>(p + i));
        } else if (i < m) {
            q.x = __ldcs(p + i);
            if (i + 1 < m) q.y = __ldcs(p + i + 1);
            if (i + 2 < m) q.z = __ldcs(p + i + 2);
        }
        v[4 * j + 0] = q.x;
        v[4 * j + 1] = q.y;
        v[4 * j + 2] = q.z;
        v[4 * j + 3] = q.w;
    }
}

template <int V>
__device__ __forceinline__ void ef_store(float* p, uint32_t first, uint32_t m, const float (&v)[4 * V]) {
#pragma unroll
    for (int j = 0; j < V; ++j) {
        const uint32_t i = first + 4 * j;
        if (i + 4 <= m) {
            __stcs(reinterpret_cast<float4*>(p + i), make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]));
        } else if (i < m) {
            __stcs(p + i, v[4 * j]);
            if (i + 1 < m) __stcs(p + i + 1, v[4 * j + 1]);
            if (i + 2 < m) __stcs(p + i + 2, v[4 * j + 2]);
        }
    }
}

// The memory left by one coordinate p = e + g sent as level k (sign `neg`) of step
// `scale` = fl(norm / s): p minus the value a receiver decodes, fl(scale * k) with
// the sign applied last; p itself when no record was sent.
__device__ __forceinline__ float ef_residual(float p, uint32_t k, bool neg, float scale) {
    if (k == 0u) return p;
    const float q = __fmul_rn(scale, __uint2float_rn(k));
    return __fsub_rn(p, neg ? -q : q);
}

// ---------------------------------------------------------------------------
// Elias omega code of N >= 1 (Elias 1975): start from "0"; while N > 1, put the
// binary form of N in front and continue with bitlength(N) - 1.  Returned as a
// right-aligned value read MSB-first, and its length in bits.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void omega_compute(uint64_t N, uint64_t& code, uint32_t& len) {
    code = 0;
    len = 1;
    while (N > 1) {
        const uint32_t b = 64u - static_cast<uint32_t>(__clzll(static_cast<long long>(N)));
        code |= N << len;
        len += b;
        N = b - 1;
    }
}

// Table of omega codes for N < kOmegaTab: entry = (code << 8) | len (entry 0 is
// unused).  Built at compile time by the same rule as omega_compute.
struct alignas(16) OmegaTable {  // read with 16-byte loads
    uint32_t v[kOmegaTab];
};
constexpr OmegaTable make_omega_table() {
    OmegaTable t{};
    for (int N = 0; N < kOmegaTab; ++N) {
        uint64_t n = N ? static_cast<uint64_t>(N) : 1u;
        uint64_t code = 0;
        uint32_t len = 1;
        while (n > 1) {
            uint32_t b = 0;
            for (uint64_t x = n; x; x >>= 1) ++b;
            code |= n << len;
            len += b;
            n = b - 1;
        }
        t.v[N] = (static_cast<uint32_t>(code) << 8) | len;
    }
    return t;
}
__device__ const OmegaTable kOmegaTableGlobal = make_omega_table();

// Copies the table into shared memory (16-byte loads).
__device__ __forceinline__ void omega_table_fill(uint32_t* tab, int tid, int nthreads) {
    const uint4* src = reinterpret_cast<const uint4*>(kOmegaTableGlobal.v);
    uint4* dst = reinterpret_cast<uint4*>(tab);
    for (int i = tid; i < kOmegaTab / 4; i += nthreads) dst[i] = src[i];
}

// Whole records omega(gap) | sign | omega(k) for gap < 64 and k < 16, indexed by
// gap << 5 | k << 1 | sign: entry = code << 5 | length (length <= 20 bits).
struct alignas(16) RecordTable {  // read with 16-byte loads
    uint32_t v[kRecordTab];
};
constexpr RecordTable make_record_table() {
    RecordTable t{};
    const OmegaTable om = make_omega_table();
    for (uint32_t gap = 1; gap < 64; ++gap)
        for (uint32_t k = 1; k < 16; ++k)
            for (uint32_t sign = 0; sign < 2; ++sign) {
                const uint32_t ge = om.v[gap], ke = om.v[k];
                const uint32_t kl = ke & 0xFFu;
                const uint32_t code = ((((ge >> 8) << 1) | sign) << kl) | (ke >> 8);
                const uint32_t len = (ge & 0xFFu) + 1u + kl;
                t.v[(gap << 5) | (k << 1) | sign] = (code << 5) | len;
            }
    return t;
}
__device__ const RecordTable kRecordTableGlobal = make_record_table();

__device__ __forceinline__ void record_table_fill(uint32_t* tab, int tid, int nthreads) {
    const uint4* src = reinterpret_cast<const uint4*>(kRecordTableGlobal.v);
    uint4* dst = reinterpret_cast<uint4*>(tab);
    for (int i = tid; i < kRecordTab / 4; i += nthreads) dst[i] = src[i];
}

// Omega code of N >= 1 from the global table (N < kOmegaTab) or computed.
__device__ __forceinline__ void omega_code_global(uint64_t N, uint64_t& code, uint32_t& len) {
    if (N < kOmegaTab) {
        const uint32_t e = __ldg(&kOmegaTableGlobal.v[N]);
        code = e >> 8;
        len = e & 0xFFu;
        return;
    }
    omega_compute(N, code, len);
}

// N < kOmegaTab known by the caller
__device__ __forceinline__ uint32_t omega_len_fast(const uint32_t* tab, uint32_t N) { return tab[N] & 0xFFu; }

__device__ __forceinline__ uint32_t omega_len(const uint32_t* tab, uint64_t N) {
    if (N < kOmegaTab) return tab[N] & 0xFFu;
    uint64_t code;
    uint32_t len;
    omega_compute(N, code, len);
    return len;
}

__device__ __forceinline__ void omega_code(const uint32_t* tab, uint64_t N, uint64_t& code,
                                           uint32_t& len) {
    if (N < kOmegaTab) {
        const uint32_t e = tab[N];
        code = e >> 8;
        len = e & 0xFFu;
        return;
    }
    omega_compute(N, code, len);
}

// ---------------------------------------------------------------------------
// MSB-first bit packing into a zero-filled shared word buffer.  A lane keeps up
// to 31 pending bits; full words are OR-ed into the buffer (neighbouring lanes
// may share a word, so every write is an atomic OR).
// ---------------------------------------------------------------------------
struct BitPacker {
    uint64_t acc;    // pending bits, right-aligned
    uint32_t nacc;   // number of pending bits (< 32 between calls)
    uint32_t word;   // index of the word the pending bits start in
    uint32_t* buf;
    uint32_t limit;  // number of words in buf

    __device__ __forceinline__ void start(uint32_t* b, uint32_t lim, uint64_t bitpos) {
        buf = b;
        limit = lim;
        word = static_cast<uint32_t>(bitpos >> 5);
        nacc = static_cast<uint32_t>(bitpos & 31u);  // leading bits owned by earlier writers
        acc = 0;
    }
    __device__ __forceinline__ bool emit(uint32_t w) {
        if (word >= limit) return false;
        if (w) atomicOr(&buf[word], w);
        ++word;
        return true;
    }
    // Appends len <= 32 bits.
    __device__ __forceinline__ bool put32(uint32_t code, uint32_t len) {
        acc = (acc << len) | code;
        nacc += len;
        if (nacc >= 32) {
            nacc -= 32;
            return emit(static_cast<uint32_t>(acc >> nacc));
        }
        return true;
    }
    __device__ __forceinline__ bool put(uint64_t code, uint32_t len) {
        bool ok = true;
        if (len > 32) {
            ok = put32(static_cast<uint32_t>(code >> 32), len - 32);
            len = 32;
        }
        return put32(static_cast<uint32_t>(code), len) && ok;
    }
    __device__ __forceinline__ bool flush() {
        if (nacc == 0) return true;
        return emit(static_cast<uint32_t>(acc << (32 - nacc)));
    }
};

// ---------------------------------------------------------------------------
// MSB-first packing of one lane's records into its private strip of shared
// memory (word j at base[32 j]; the strips of a warp interleave, so the lanes'
// stores fall in distinct banks).  32-bit state: the partial word and its fill.
// ---------------------------------------------------------------------------
struct LanePacker {
    uint32_t* base;
    uint32_t cur;   // partial word, filled from the top
    uint32_t used;  // bits in cur (0..31)
    uint32_t nw;    // words stored
    // Appends the len (1..32) low bits of code.
    __device__ __forceinline__ void put(uint32_t code, uint32_t len) {
        const uint32_t x = code << (32u - len);  // left-aligned record
        const uint32_t filled = cur | (x >> used);
        const uint32_t tot = used + len;
        const bool full = tot >= 32u;
        if (full) base[32u * nw] = filled;
        nw += full ? 1u : 0u;
        // leftover bits of the record start the next word (none when tot == 32)
        const uint32_t rest = (tot > 32u) ? (x << (32u - used)) : 0u;
        cur = full ? rest : filled;
        used = tot & 31u;
    }
    __device__ __forceinline__ void finish() {
        if (used) base[32u * nw] = cur;
    }
    __device__ __forceinline__ uint32_t bits() const { return 32u * nw + used; }
};

// ---------------------------------------------------------------------------
// Inter-CTA scan state (single-pass prefix scan with decoupled look-back,
// Merrill & Garland 2016).  A descriptor packs [63:40] epoch, [39:38] state,
// [37:0] value.  Descriptors from an earlier call (other epoch) read as "not
// ready", so the workspace needs no clearing between calls.
// ---------------------------------------------------------------------------
constexpr uint64_t kStateAggregate = 1;
constexpr uint64_t kStatePrefix = 2;
constexpr uint64_t kValueMask = (uint64_t(1) << 38) - 1;
constexpr uint32_t kEpochMask = 0xFFFFFFu;

__device__ __forceinline__ uint64_t make_desc(uint32_t epoch, uint64_t state, uint64_t value) {
    return (static_cast<uint64_t>(epoch & kEpochMask) << 40) | (state << 38) | (value & kValueMask);
}
__device__ __forceinline__ uint32_t desc_epoch(uint64_t d) { return static_cast<uint32_t>(d >> 40); }
__device__ __forceinline__ uint64_t desc_state(uint64_t d) { return (d >> 38) & 3u; }
__device__ __forceinline__ uint64_t desc_value(uint64_t d) { return d & kValueMask; }

__device__ __forceinline__ void st_release(uint64_t* p, uint64_t v) {
    asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ uint64_t ld_acquire(const uint64_t* p) {
    uint64_t v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ uint64_t ld_relaxed(const uint64_t* p) {
    uint64_t v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ uint32_t ld_acquire32(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Control block at the start of the workspace.
struct ScanControl {
    uint32_t ticket;  // next tile to hand out
    uint32_t done;    // CTAs that have finished
    uint32_t epoch;   // call counter, advanced by the last CTA
    uint32_t abort;   // set when a bounded wait ran out
    uint32_t pad[12];
};
static_assert(sizeof(ScanControl) == 64, "control block is one 64-byte line");

// Per-tile state in the workspace besides the scan descriptor (which lives in its
// own contiguous array, so that descriptor pairs can be copied 16 bytes at a time).
struct TileState {
    uint64_t slot;   // slot of the word shared with the previous tile
    uint64_t round;  // fast path: RP(r), the stream position after round r (entry r)
};
static_assert(sizeof(TileState) == 16, "tile state is two words");

// Warp-cooperative look-back for tile `tile` (> 0).  All 32 lanes call it; every
// lane returns the exclusive prefix.  Returns false (and leaves the prefix
// undefined) when the bounded wait ran out or another tile aborted.
__device__ __forceinline__ bool lookback(const uint64_t* desc, uint32_t tile, uint32_t epoch,
                                         const uint32_t* abort_flag, uint64_t& exclusive) {
    const int lane = threadIdx.x & 31;
    uint64_t sum = 0;
    int64_t window_end = static_cast<int64_t>(tile) - 1;  // highest predecessor in the window
    uint32_t polls = 0;
    while (window_end >= 0) {
        const int64_t idx = window_end - lane;
        uint64_t d = 0;
        uint64_t st = kStatePrefix;  // lanes past tile 0 act as a zero prefix
        uint64_t val = 0;
        if (idx >= 0) {
            d = ld_acquire(&desc[idx]);
            st = (desc_epoch(d) == (epoch & kEpochMask)) ? desc_state(d) : 0;
            val = desc_value(d);
        }
        const uint32_t not_ready = __ballot_sync(0xFFFFFFFFu, st == 0);
        const uint32_t have_prefix = __ballot_sync(0xFFFFFFFFu, st == kStatePrefix);
        // first lane (nearest predecessor) holding a prefix
        const int first_p = have_prefix ? __ffs(have_prefix) - 1 : 32;
        const uint32_t upto = first_p == 32 ? 0xFFFFFFFFu : ((2u << first_p) - 1u);
        if (not_ready & upto) {
            if (++polls > kMaxPolls) return false;
            if ((polls & 63u) == 0 && ld_acquire32(abort_flag) != 0) return false;
            __nanosleep(polls < 64 ? 32 : 256);
            continue;
        }
        uint64_t contrib = (lane <= first_p) ? val : 0;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) contrib += __shfl_xor_sync(0xFFFFFFFFu, contrib, o);
        sum += contrib;
        if (first_p < 32) break;
        window_end -= 32;
    }
    exclusive = sum;
    return true;
}

}  // namespace qsgd
