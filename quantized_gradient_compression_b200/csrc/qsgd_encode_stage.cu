// QSGD encoder in two launches: a bucket coder and a stream compaction (sm_100a).
//
// Method: "QSGD (Quantized Stochastic Gradient Descent) with Elias Coding" (AIMech
// curated entry).  Per bucket (claim "QSVRG, non-convex and multi-GPU bucketed
// training", section 3.3 bucketing): the L2 norm, unbiased stochastic rounding of
// every coordinate to one of s+1 levels (definition paragraph), and the Elias-omega
// coding of the tuple (norm, signs, run-length gaps, levels) (definition paragraph;
// claim "Elias coding communication complexity tradeoff", F = 32).
//
// 1. code_buckets: one warp per bucket, no warp waits for another.  The warp reads
//    its bucket with coalesced 16-byte loads (lane L holds float4 L + 32j), computes
//    the norm, draws one Philox block per four coordinates, quantises, and writes the
//    bucket's bits (norm, then the records in index order) into the bucket's own
//    slot of a staging area in the workspace, at bucket-local bit offsets, together
//    with the bucket's bit count.  A slot holds the bucket's largest possible size.
// 2. compact_stream: a CTA of 512 threads per tile of 256 buckets scans the bit
//    counts (a block scan and a decoupled look-back over the tiles, Merrill &
//    Garland 2016, reading 512 predecessors at a time), writes the offsets header,
//    and moves every bucket's bits to their stream position with funnel shifts, 8 to
//    32 lanes per bucket.  An output word belongs to the bucket that holds its first
//    bit; that bucket's warp also reads the first bits of the next bucket, so every
//    word has exactly one writer and the output needs no clearing.
// The staging costs two extra passes over the compressed bytes (a few percent of
// the input bytes) and buys an encoder with no inter-CTA waits in its long kernel.
#include <cuda_runtime.h>

#include <algorithm>

#include "../../include/qsgd.h"
#include "qsgd_device.cuh"
#include "qsgd_internal.h"

namespace qsgd {
namespace {

constexpr uint32_t kAll = 0xFFFFFFFFu;

// Whole records omega(gap) | sign | omega(k) for gap < 64 and k < 32, indexed by
// gap << 6 | k << 1 | sign: entry = code << 5 | length (length <= 24 bits).  Gap 0
// holds the record without its gap, sign | omega(k); k = 0 entries are empty.
struct alignas(16) RecordTable64 {  // read with 16-byte loads
    uint32_t v[kRecordTab64];
};
constexpr RecordTable64 make_record_table64() {
    RecordTable64 t{};
    const OmegaTable om = make_omega_table();
    for (uint32_t k = 1; k < 32; ++k)
        for (uint32_t sign = 0; sign < 2; ++sign) {
            const uint32_t ke = om.v[k];
            const uint32_t kl = ke & 0xFFu;
            t.v[(k << 1) | sign] = (((sign << kl) | (ke >> 8)) << 5) | (1u + kl);
        }
    for (uint32_t gap = 1; gap < 64; ++gap)
        for (uint32_t k = 1; k < 32; ++k)
            for (uint32_t sign = 0; sign < 2; ++sign) {
                const uint32_t ge = om.v[gap], ke = om.v[k];
                const uint32_t kl = ke & 0xFFu;
                const uint32_t code = ((((ge >> 8) << 1) | sign) << kl) | (ke >> 8);
                const uint32_t len = (ge & 0xFFu) + 1u + kl;
                t.v[(gap << 6) | (k << 1) | sign] = (code << 5) | len;
            }
    return t;
}
__device__ const RecordTable64 kRecordTable64Global = make_record_table64();

// Philox4x32-10 of counter (j, 0, 0, 0) with the round keys precomputed on the host
// (rk[2r], rk[2r+1] = the seed advanced r times by the Weyl constants).  The
// counter's high words are zero because j = i / 4 < 2^32 for every coordinate.
__device__ __forceinline__ uint4 philox_rk(uint32_t j, const uint32_t* rk) {
    uint32_t c0 = j, c1 = 0u, c2 = 0u, c3 = 0u;
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        const uint64_t pa = static_cast<uint64_t>(c0) * 0xD2511F53u;
        const uint64_t pb = static_cast<uint64_t>(c2) * 0xCD9E8D57u;
        c0 = static_cast<uint32_t>(pb >> 32) ^ c1 ^ rk[2 * r];
        c2 = static_cast<uint32_t>(pa >> 32) ^ c3 ^ rk[2 * r + 1];
        c1 = static_cast<uint32_t>(pb);
        c3 = static_cast<uint32_t>(pa);
    }
    return make_uint4(c0, c1, c2, c3);
}

// The level k = min(floor(t) + [u < p], s) of one coordinate, t = fl(|v| sinv),
// p = t - floor(t), u = floor(r / 2^9) 2^-23 (definition paragraph; fp32 order of
// the wire format).  Exact rewrite of the comparison: with f = RD(t + 2^23) =
// 2^23 + floor(t) (exact for 0 <= t < 2^23), the sum t + (2^23 + 1 - f) is exactly
// 1 + p, and 1 + u lies on the fp32 grid of [1, 2); so u < p holds exactly when
// 1 + u < RU(1 + p).
__device__ __forceinline__ uint32_t level_of(float v, float sinv, uint32_t r, uint32_t s) {
    const float t = __fmul_rn(fabsf(v), sinv);
    const float f = __fadd_rd(t, 8388608.0f);
    const float w = __fadd_ru(t, __fsub_rn(8388609.0f, f));
    const float u1 = __uint_as_float(0x3F800000u | (r >> 9));
    const uint32_t k = (__float_as_uint(f) - 0x4B000000u) + (u1 < w ? 1u : 0u);
    return k < s ? k : s;
}

// ORs the len (1..32) low bits of code, MSB-first, into the zeroed bit buffer at
// bit position pos.
__device__ __forceinline__ void put_bits(uint32_t* buf, uint32_t pos, uint32_t code, uint32_t len) {
    const uint32_t w = pos >> 5, sh = pos & 31u;
    const uint64_t v = static_cast<uint64_t>(code) << (64u - len - sh);
    atomicOr(&buf[w], static_cast<uint32_t>(v >> 32));
    if (static_cast<uint32_t>(v) != 0u) atomicOr(&buf[w + 1], static_cast<uint32_t>(v));
}

// The same for len (1..64) bits.
__device__ __forceinline__ void put_bits64(uint32_t* buf, uint32_t pos, uint64_t code, uint32_t len) {
    if (len > 32) {
        put_bits(buf, pos, static_cast<uint32_t>(code >> 32), len - 32);
        pos += len - 32;
        len = 32;
    }
    put_bits(buf, pos, static_cast<uint32_t>(code), len);
}

// Appends len (0..31) bits of code, right-aligned, to the 96-bit register string
// (w2:w1:w0), right-aligned too.
__device__ __forceinline__ void string_append(uint32_t& w0, uint32_t& w1, uint32_t& w2, uint32_t code, uint32_t len) {
    w2 = __funnelshift_l(w1, w2, len);
    w1 = __funnelshift_l(w0, w1, len);
    w0 = (w0 << len) | code;
}

// ORs the right-aligned nbits (1..96) bits of the register string (w2:w1:w0) into the
// zeroed bit buffer at bit position pos: left-aligned in 96 bits, then at most four
// word atomics.
__device__ __forceinline__ void string_or(uint32_t* buf, uint32_t pos, uint32_t w0, uint32_t w1, uint32_t w2,
                                          uint32_t nbits) {
    const uint32_t sa = 96u - nbits, bsh = sa & 31u, wsh = sa >> 5;
    const uint32_t t2 = __funnelshift_l(w1, w2, bsh), t1 = __funnelshift_l(w0, w1, bsh), t0 = w0 << bsh;
    const uint32_t L0 = wsh == 0 ? t2 : wsh == 1 ? t1 : t0;
    const uint32_t L1 = wsh == 0 ? t1 : wsh == 1 ? t0 : 0u;
    const uint32_t L2 = wsh == 0 ? t0 : 0u;
    const uint32_t wp = pos >> 5, sh = pos & 31u;
    const uint32_t nw = (sh + nbits + 31u) >> 5;  // 1..4
    atomicOr(&buf[wp], L0 >> sh);
    if (nw > 1) atomicOr(&buf[wp + 1], __funnelshift_r(L1, L0, sh));
    if (nw > 2) atomicOr(&buf[wp + 2], __funnelshift_r(L2, L1, sh));
    if (nw > 3) atomicOr(&buf[wp + 3], __funnelshift_r(0u, L2, sh));
}

// Stores one lane's 4V values (float4 L + 32j of a bucket of m values at p) with
// streaming stores; nothing past m is written.
template <int V>
__device__ __forceinline__ void store_lane(float* p, int lane, uint32_t m, const float (&v)[4 * V]) {
#pragma unroll
    for (int j = 0; j < V; ++j) {
        const uint32_t i = 4u * (static_cast<uint32_t>(lane) + 32u * j);
        if (i + 4 <= m) {
            __stcs(reinterpret_cast<float4*>(p + i), make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]));
        } else if (i < m) {
            __stcs(p + i, v[4 * j]);
            if (i + 1 < m) __stcs(p + i + 1, v[4 * j + 1]);
            if (i + 2 < m) __stcs(p + i + 2, v[4 * j + 2]);
        }
    }
}

// One record of the short form (s <= 31): the whole-record table for gap < 64, the
// omega table otherwise (gap <= d <= 1024); code right-aligned, <= 30 bits.
__device__ __forceinline__ void short_record(const uint32_t* rtab, const uint32_t* otab, uint32_t gap, uint32_t kv,
                                             uint32_t& code, uint32_t& len) {
    if (gap < 64u) {
        const uint32_t e = rtab[(gap << 6) | __funnelshift_l(kv, kv, 1)];
        code = e >> 5;
        len = e & 31u;
    } else {
        const uint32_t ge = otab[gap], ke = otab[kv & 0x7FFFFFFFu];
        const uint32_t kl = ke & 0xFFu;
        code = ((((ge >> 8) << 1) | (kv >> 31)) << kl) | (ke >> 8);
        len = (ge & 0xFFu) + 1u + kl;
    }
}

// Loads one lane's NC = 4V consecutive values [q0, q0 + NC) of a bucket of m values
// at p (streaming; zeros past m).
template <int V>
__device__ __forceinline__ void load_contig(const float* p, uint32_t q0, uint32_t m, float (&x)[4 * V]) {
#pragma unroll
    for (int j = 0; j < V; ++j) {
        const uint32_t i = q0 + 4u * j;
        float4 q = make_float4(0.f, 0.f, 0.f, 0.f);
        if (i + 4 <= m) {
            q = __ldcs(reinterpret_cast<const float4*>(p + i));
        } else if (i < m) {
            q.x = p[i];
            if (i + 1 < m) q.y = p[i + 1];
            if (i + 2 < m) q.z = p[i + 2];
        }
        x[4 * j + 0] = q.x;
        x[4 * j + 1] = q.y;
        x[4 * j + 2] = q.z;
        x[4 * j + 3] = q.w;
    }
}

// Stores one lane's NC consecutive values [q0, q0 + NC) (streaming; nothing past m).
template <int V>
__device__ __forceinline__ void store_contig(float* p, uint32_t q0, uint32_t m, const float (&v)[4 * V]) {
#pragma unroll
    for (int j = 0; j < V; ++j) {
        const uint32_t i = q0 + 4u * j;
        if (i + 4 <= m) {
            __stcs(reinterpret_cast<float4*>(p + i), make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]));
        } else if (i < m) {
            __stcs(p + i, v[4 * j]);
            if (i + 1 < m) __stcs(p + i + 1, v[4 * j + 1]);
            if (i + 2 < m) __stcs(p + i + 2, v[4 * j + 2]);
        }
    }
}

// ---------------------------------------------------------------------------
// 1a. Bucket coder for s <= 31 (records <= 30 bits).  Lane L holds the NC = 4V
// consecutive coordinates [NC L, NC L + NC) of its bucket, so a bucket is one run:
// one gap chain over the lanes (a ballot and a shuffle) and one scan of the lanes'
// bit counts.  A lane appends its records to a 96-bit register string as it codes
// them and ORs the string into the bucket buffer once its position is known.  A
// bucket where some lane needs more than 96 bits is placed record by record.
// ---------------------------------------------------------------------------
// Codes one chunk of a bucket for the short coder: lane L holds the values x[] (p,
// for error feedback) of the NC = 4V consecutive coordinates lo + NC L + c; their
// global index is base + that.  carry: the bucket-local index of the last record
// before the chunk (-1 before the first); pos: the bucket-local bit where the chunk's
// records start.  Both advance past the chunk.  The chunk's bits are ORed into the
// zeroed bucket buffer.
template <int V, bool kEF>
__device__ __forceinline__ void code_chunk(const StageArgs& a, const uint32_t* rtab, const uint32_t* otab, uint32_t* buf,
                                           float (&x)[4 * V], float (&ev)[kEF ? 4 * V : 1], const BucketScale& sc,
                                           uint64_t base, uint32_t lo, uint32_t m, int lane, int32_t& carry,
                                           uint32_t& pos) {
    constexpr int NC = 4 * V;
    const uint32_t q0 = lo + static_cast<uint32_t>(NC * lane);  // bucket-local index of x[0]
    const uint32_t lanes_below = (1u << lane) - 1u;
    // --- levels: one Philox block per four coordinates ---------------------------------
    uint32_t kq[NC];  // level | sign << 31
    const uint32_t j0 = static_cast<uint32_t>((base + q0) >> 2);
#pragma unroll
    for (int j = 0; j < V; ++j) {
        const uint4 r = philox_rk(j0 + j, a.rk);
        const uint32_t rw[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const float v = x[4 * j + c];
            kq[4 * j + c] = level_of(v, sc.sinv, rw[c], a.s) | (__float_as_uint(v) & 0x80000000u);
        }
    }
    if constexpr (kEF) {  // the memory keeps p minus what a receiver decodes
        if (sc.good) {
            const float scale = __fdiv_rn(sc.sent, __uint2float_rn(a.s));
#pragma unroll
            for (int q = 0; q < NC; ++q) ev[q] = ef_residual(x[q], kq[q] & 0x7FFFFFFFu, kq[q] >> 31, scale);
            store_contig<V>(a.ef + base, q0, m, ev);
        }
    }
    // --- gap chain: the last record before this lane's coordinates ------------------------
    uint32_t nzm = 0;
#pragma unroll
    for (int c = 0; c < NC; ++c) nzm |= ((kq[c] & 0x7FFFFFFFu) != 0u ? 1u : 0u) << c;
    const int32_t last = nzm ? static_cast<int32_t>(q0 + 31u - __clz(nzm)) : -1;
    const uint32_t any = __ballot_sync(kAll, nzm != 0u);
    const uint32_t B = any & lanes_below;
    const int32_t pv = __shfl_sync(kAll, last, B ? 31 - __clz(B) : 0);
    const int32_t prev_in = B ? pv : carry;
    const int32_t top = __shfl_sync(kAll, last, any ? 31 - __clz(any) : 0);
    carry = any ? top : carry;
    // --- the lane's records, appended to (w2:w1:w0), right-aligned: every record from the
    // whole-record table, the lane's first one without its gap (the gaps inside a lane
    // are below 64); that gap's omega code goes in front at the end -----------------------
    uint32_t w0 = 0, w1 = 0, w2 = 0, nbits = 0;
    {
        const uint32_t cf = nzm ? static_cast<uint32_t>(__ffs(nzm) - 1) : 0u;
        uint32_t prev = q0 + cf;
#pragma unroll
        for (int c = 0; c < NC; ++c) {
            const uint32_t kv = kq[c];
            const uint32_t kr = __funnelshift_l(kv, kv, 1);  // k << 1 | sign
            // below the lane's first record the gap wraps, but k = 0 there: an empty entry
            const uint32_t e = rtab[(((q0 + c - prev) << 6) | kr) & (kRecordTab64 - 1)];
            const uint32_t len = e & 31u;
            string_append(w0, w1, w2, e >> 5, len);
            nbits += len;
            prev = kr > 1u ? q0 + c : prev;
        }
        if (nzm) {  // omega(gap of the first record) in front of the string
            const uint32_t gap = static_cast<uint32_t>(static_cast<int32_t>(q0 + cf) - prev_in);
            uint32_t gl, gc;
            if (gap < static_cast<uint32_t>(kOmegaTab)) {
                const uint32_t ge = otab[gap];
                gl = ge & 0xFFu;
                gc = ge >> 8;
            } else {  // gap <= d <= 16384: omega code of at most 22 bits
                uint64_t c64;
                omega_compute(gap, c64, gl);
                gc = static_cast<uint32_t>(c64);
            }
            if (nbits + gl <= 96u) {
                const uint32_t sh = nbits & 31u;  // gc lands at bit nbits
                const uint32_t glo = sh ? gc << sh : gc, ghi = sh ? gc >> (32u - sh) : 0u;
                if (nbits < 32u) {
                    w0 |= glo;
                    w1 |= ghi;
                } else if (nbits < 64u) {
                    w1 |= glo;
                    w2 |= ghi;
                } else {
                    w2 |= glo;
                }
            }
            nbits += gl;
        }
    }
    // --- the lane's first bit: scan of the bit counts --------------------------------------
    uint32_t incl = nbits;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t t = __shfl_up_sync(kAll, incl, o);
        if (lane >= o) incl += t;
    }
    const uint32_t P = pos + incl - nbits;
    pos += __shfl_sync(kAll, incl, 31);
    if (!__any_sync(kAll, nbits > 96u)) {
        if (nbits != 0u) string_or(buf, P, w0, w1, w2, nbits);
    } else {  // some lane's string is longer than 96 bits: record by record
        int32_t prev = prev_in;
        uint32_t p = P;
#pragma unroll
        for (int c = 0; c < NC; ++c) {
            const uint32_t kv = kq[c];
            if ((kv & 0x7FFFFFFFu) != 0u) {
                const uint32_t gap = static_cast<uint32_t>(static_cast<int32_t>(q0 + c) - prev);
                prev = static_cast<int32_t>(q0 + c);
                if (gap < static_cast<uint32_t>(kOmegaTab)) {
                    uint32_t code, len;
                    short_record(rtab, otab, gap, kv, code, len);
                    put_bits(buf, p, code, len);
                    p += len;
                } else {  // a gap past the omega table: its code, then sign | omega(k)
                    uint64_t gcode;
                    uint32_t glen;
                    omega_compute(gap, gcode, glen);
                    put_bits64(buf, p, gcode, glen);
                    p += glen;
                    const uint32_t ke = otab[kv & 0x7FFFFFFFu];
                    const uint32_t kl = ke & 0xFFu;
                    put_bits(buf, p, ((kv >> 31) << kl) | (ke >> 8), 1u + kl);
                    p += 1u + kl;
                }
            }
        }
    }
}

// ---------------------------------------------------------------------------
// 1a. Bucket coder for s <= 31 (records of up to 30 bits, plus a first gap up to d).
// Lane L holds NC = 4V consecutive coordinates of a chunk of 128V, so a chunk is one
// run: one gap chain over the lanes (a ballot and a shuffle) and one scan of the
// lanes' bit counts.  A lane appends its records to a 96-bit register string as it
// codes them and ORs the string into the bucket buffer once its position is known; a
// chunk where some lane needs more than 96 bits is placed record by record.  A bucket
// of one chunk keeps its values in registers; a longer one (d > 128V) is read twice:
// for its norm, then chunk by chunk for its records.
// ---------------------------------------------------------------------------
template <int V, bool kEF>
__global__ void __launch_bounds__(kStageBlock, (V <= 4 ? 4 : 2)) code_buckets_short(const __grid_constant__ StageArgs a) {
    extern __shared__ __align__(16) uint32_t smem[];
    constexpr int NC = 4 * V;
    constexpr uint32_t kChunkCoords = 128u * V;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint32_t* const otab = smem;                                                  // omega table
    uint32_t* const rtab = smem + kOmegaTab;                                      // record table
    uint32_t* const buf = smem + kOmegaTab + kRecordTab64 + warp * a.buf_words;   // this warp's bucket bits
    omega_table_fill(otab, tid, kStageBlock);
    {
        const uint4* src = reinterpret_cast<const uint4*>(kRecordTable64Global.v);
        for (int i = tid; i < kRecordTab64 / 4; i += kStageBlock) reinterpret_cast<uint4*>(rtab)[i] = src[i];
    }
    for (uint32_t i = lane; i < a.buf_words; i += 32) buf[i] = 0u;
    {  // the compaction's scan state for this call: cleared here, before it runs
        const uint64_t gt = static_cast<uint64_t>(blockIdx.x) * kStageBlock + tid;
        for (uint64_t i = gt; i < a.ntiles; i += static_cast<uint64_t>(gridDim.x) * kStageBlock) a.cdesc[i] = 0;
    }
    __syncthreads();

    const uint32_t d = a.d;
    const uint32_t ql = static_cast<uint32_t>(NC * lane);  // lane offset inside a chunk
    const uint64_t gwarps = static_cast<uint64_t>(gridDim.x) * kStageWarps;
    for (uint64_t b = static_cast<uint64_t>(blockIdx.x) * kStageWarps + warp; b < a.nb; b += gwarps) {
        const uint64_t base = b * d;
        const uint32_t m = static_cast<uint32_t>(min(static_cast<uint64_t>(d), a.n - base));
        float x[NC];
        float ev[kEF ? NC : 1];
        int32_t carry = -1;
        uint32_t pos = 32u;
        if (m <= kChunkCoords) {
            // --- one chunk: the values stay in registers ---------------------------------
            load_contig<V>(a.in + base, ql, m, x);
            if constexpr (kEF) {  // p = e + g
                load_contig<V>(a.ef + base, ql, m, ev);
#pragma unroll
                for (int q = 0; q < NC; ++q) x[q] = __fadd_rn(ev[q], x[q]);
            }
            const float norm =
                a.norm_kind == QSGD_NORM_MAX ? warp_bucket_maxnorm<NC>(x) : warp_bucket_norm<NC>(x, true);
            const BucketScale sc = bucket_scale(norm, a.s, true, a.status, lane == 0);
            if (!sc.good) {  // sent as a zero bucket; the memory keeps p
                if constexpr (kEF) store_contig<V>(a.ef + base, ql, m, x);
#pragma unroll
                for (int q = 0; q < NC; ++q) x[q] = 0.f;
            }
            code_chunk<V, kEF>(a, rtab, otab, buf, x, ev, sc, base, 0u, m, lane, carry, pos);
            if (lane == 0) buf[0] = __float_as_uint(sc.sent);
        } else {
            // --- several chunks: the norm over the whole bucket first ---------------------
            float ss = 0.f, mx = 0.f;
            bool nan = false;
            for (uint32_t lo = 0; lo < m; lo += kChunkCoords) {
                load_contig<V>(a.in + base, lo + ql, m, x);
                if constexpr (kEF) {
                    load_contig<V>(a.ef + base, lo + ql, m, ev);
#pragma unroll
                    for (int q = 0; q < NC; ++q) x[q] = __fadd_rn(ev[q], x[q]);
                }
#pragma unroll
                for (int q = 0; q < NC; ++q) {
                    ss = __fmaf_rn(x[q], x[q], ss);
                    mx = fmaxf(mx, fabsf(x[q]));
                    nan |= isnan(x[q]);
                }
            }
            float norm;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                ss = __fadd_rn(ss, __shfl_xor_sync(kAll, ss, o));
                mx = fmaxf(mx, __shfl_xor_sync(kAll, mx, o));
            }
            if (a.norm_kind == QSGD_NORM_MAX) {
                norm = __any_sync(kAll, nan) ? __uint_as_float(0x7FC00000u) : mx;
            } else {
                norm = __fsqrt_rn(ss);
                if (needs_rescale(ss) && !isnan(ss)) {  // uniform in the warp
                    if (isinf(mx)) {
                        norm = mx;
                    } else if (mx > 0.f) {  // squares outside the normal range: scaled by a power of two
                        float unscale;
                        const float scale = pow2_scale(mx, unscale);
                        float s2 = 0.f;
                        for (uint32_t lo = 0; lo < m; lo += kChunkCoords) {
                            load_contig<V>(a.in + base, lo + ql, m, x);
                            if constexpr (kEF) {
                                load_contig<V>(a.ef + base, lo + ql, m, ev);
#pragma unroll
                                for (int q = 0; q < NC; ++q) x[q] = __fadd_rn(ev[q], x[q]);
                            }
#pragma unroll
                            for (int q = 0; q < NC; ++q) {
                                const float y = __fmul_rn(x[q], scale);
                                s2 = __fmaf_rn(y, y, s2);
                            }
                        }
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1) s2 = __fadd_rn(s2, __shfl_xor_sync(kAll, s2, o));
                        norm = __fmul_rn(__fsqrt_rn(s2), unscale);
                    }
                }
            }
            const BucketScale sc = bucket_scale(norm, a.s, true, a.status, lane == 0);
            // --- then chunk by chunk: levels and records ------------------------------------
            for (uint32_t lo = 0; lo < m; lo += kChunkCoords) {
                load_contig<V>(a.in + base, lo + ql, m, x);
                if constexpr (kEF) {
                    load_contig<V>(a.ef + base, lo + ql, m, ev);
#pragma unroll
                    for (int q = 0; q < NC; ++q) x[q] = __fadd_rn(ev[q], x[q]);
                }
                if (!sc.good) {  // sent as a zero bucket; the memory keeps p
                    if constexpr (kEF) store_contig<V>(a.ef + base, lo + ql, m, x);
#pragma unroll
                    for (int q = 0; q < NC; ++q) x[q] = 0.f;
                }
                code_chunk<V, kEF>(a, rtab, otab, buf, x, ev, sc, base, lo, m, lane, carry, pos);
            }
            if (lane == 0) buf[0] = __float_as_uint(sc.sent);
        }
        __syncwarp();
        // --- the bucket's bits into its staging slot; the buffer cleared again -----------
        const uint32_t total = pos;
        uint32_t* const slot = a.stage + b * a.slot_words;
        const uint32_t nw = (total + 31u) >> 5;
        for (uint32_t i = lane; i < nw; i += 32) {
            slot[i] = buf[i];
            buf[i] = 0u;
        }
        if (lane == 0) a.bits[b] = total;
        __syncwarp();
    }
}

// ---------------------------------------------------------------------------
// 1b. Bucket coder for s > 31 (d <= 1024): lane L holds the float4s L + 32j of its
// bucket, coded run by run (run j is coordinates [128j, 128j + 128)).  Every record
// is omega(gap) | sign from the omega table, then omega(k) from the omega table (or
// computed for k >= 2048), up to 18 + 1 + 34 bits.  A lane appends its run's records
// to a 96-bit register string and ORs it into the bucket buffer once its position is
// known; a run where some lane's string is longer, or a level's code longer than 31
// bits, is placed record by record.
// ---------------------------------------------------------------------------
template <int V, bool kEF>
__global__ void __launch_bounds__(kStageBlock) code_buckets(const __grid_constant__ StageArgs a) {
    extern __shared__ __align__(16) uint32_t smem[];
    constexpr int NC = 4 * V;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint32_t* const otab = smem;                                    // omega table
    uint32_t* const buf = smem + kOmegaTab + warp * a.buf_words;    // this warp's bucket bits
    omega_table_fill(otab, tid, kStageBlock);
    for (uint32_t i = lane; i < a.buf_words; i += 32) buf[i] = 0u;
    // the compaction's scan state for this call: cleared here, before it runs
    {
        const uint64_t gt = static_cast<uint64_t>(blockIdx.x) * kStageBlock + tid;
        for (uint64_t i = gt; i < a.ntiles; i += static_cast<uint64_t>(gridDim.x) * kStageBlock) a.cdesc[i] = 0;
    }
    __syncthreads();

    const uint32_t d = a.d;
    const uint64_t gwarps = static_cast<uint64_t>(gridDim.x) * kStageWarps;
    for (uint64_t b = static_cast<uint64_t>(blockIdx.x) * kStageWarps + warp; b < a.nb; b += gwarps) {
        const uint64_t base = b * d;
        const uint32_t m = static_cast<uint32_t>(min(static_cast<uint64_t>(d), a.n - base));
        // --- the bucket: lane L holds float4 f = L + 32j (coordinates 4f..4f+3) ----
        float x[NC];
        float ev[kEF ? NC : 1];
#pragma unroll
        for (int j = 0; j < V; ++j) {
            const uint32_t i = 4u * (static_cast<uint32_t>(lane) + 32u * j);
            float4 q = make_float4(0.f, 0.f, 0.f, 0.f);
            float4 e = make_float4(0.f, 0.f, 0.f, 0.f);
            if (i + 4 <= m) {
                q = __ldcs(reinterpret_cast<const float4*>(a.in + base + i));
                if constexpr (kEF) e = __ldcs(reinterpret_cast<const float4*>(a.ef + base + i));
            } else if (i < m) {  // the ragged end of the last bucket
                q.x = a.in[base + i];
                if (i + 1 < m) q.y = a.in[base + i + 1];
                if (i + 2 < m) q.z = a.in[base + i + 2];
                if constexpr (kEF) {
                    e.x = a.ef[base + i];
                    if (i + 1 < m) e.y = a.ef[base + i + 1];
                    if (i + 2 < m) e.z = a.ef[base + i + 2];
                }
            }
            x[4 * j + 0] = q.x;
            x[4 * j + 1] = q.y;
            x[4 * j + 2] = q.z;
            x[4 * j + 3] = q.w;
            if constexpr (kEF) {
                ev[4 * j + 0] = e.x;
                ev[4 * j + 1] = e.y;
                ev[4 * j + 2] = e.z;
                ev[4 * j + 3] = e.w;
            }
        }
        if constexpr (kEF) {  // p = e + g
#pragma unroll
            for (int q = 0; q < NC; ++q) x[q] = __fadd_rn(ev[q], x[q]);
        }
        const float norm = a.norm_kind == QSGD_NORM_MAX ? warp_bucket_maxnorm<NC>(x) : warp_bucket_norm<NC>(x, true);
        const BucketScale sc = bucket_scale(norm, a.s, true, a.status, lane == 0);
        if (!sc.good) {  // sent as a zero bucket; the memory keeps p
            if constexpr (kEF) store_lane<V>(a.ef + base, lane, m, x);
#pragma unroll
            for (int q = 0; q < NC; ++q) x[q] = 0.f;
        }
        // --- levels: one Philox block per float4 ----------------------------------
        uint32_t kq[NC];  // level | sign << 31
        const uint32_t j0 = static_cast<uint32_t>(base >> 2) + static_cast<uint32_t>(lane);
#pragma unroll
        for (int j = 0; j < V; ++j) {
            const uint4 r = philox_rk(j0 + 32u * j, a.rk);
            const uint32_t rw[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float v = x[4 * j + c];
                kq[4 * j + c] = level_of(v, sc.sinv, rw[c], a.s) | (__float_as_uint(v) & 0x80000000u);
            }
        }
        if constexpr (kEF) {  // the memory keeps p minus what a receiver decodes
            if (sc.good) {
                const float scale = __fdiv_rn(sc.sent, __uint2float_rn(a.s));
#pragma unroll
                for (int q = 0; q < NC; ++q) ev[q] = ef_residual(x[q], kq[q] & 0x7FFFFFFFu, kq[q] >> 31, scale);
                store_lane<V>(a.ef + base, lane, m, ev);
            }
        }
        // --- records, run by run: run j is coordinates [128j, 128j + 128) ----------
        if (lane == 0) buf[0] = __float_as_uint(sc.sent);
        uint32_t pos = 32u;      // bucket-local bit where the current run starts
        int32_t carry = -1;      // last record's index before the current run
#pragma unroll
        for (int j = 0; j < V; ++j) {
            const uint32_t qb = 4u * (static_cast<uint32_t>(lane) + 32u * j);
            uint32_t m4 = 0;
#pragma unroll
            for (int c = 0; c < 4; ++c) m4 |= ((kq[4 * j + c] & 0x7FFFFFFFu) != 0u ? 1u : 0u) << c;
            const int32_t last = m4 ? static_cast<int32_t>(qb + 31u - __clz(m4)) : -1;
            const uint32_t B = __ballot_sync(kAll, m4 != 0u);
            const uint32_t lower = B & ((1u << lane) - 1u);
            const int32_t pv = __shfl_sync(kAll, last, lower ? 31 - __clz(lower) : 0);
            const int32_t prev_in = lower ? pv : carry;
            carry = B ? __shfl_sync(kAll, last, 31 - __clz(B)) : carry;
            // the lane's records of this run, appended to the register string while
            // every piece is at most 31 bits
            uint32_t w0 = 0, w1 = 0, w2 = 0, lbits = 0;
            bool fits = true;
            {
                int32_t prev = prev_in;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const uint32_t kv = kq[4 * j + c];
                    const uint32_t k = kv & 0x7FFFFFFFu;
                    if (k != 0u) {
                        const uint32_t gap = static_cast<uint32_t>(static_cast<int32_t>(qb + c) - prev);
                        prev = static_cast<int32_t>(qb + c);
                        const uint32_t ge = otab[gap];  // gap <= d <= 1024
                        const uint32_t glen = (ge & 0xFFu) + 1u;
                        string_append(w0, w1, w2, ((ge >> 8) << 1) | (kv >> 31), glen);
                        uint64_t kcode;
                        uint32_t klen;
                        if (k < static_cast<uint32_t>(kOmegaTab)) {
                            const uint32_t ke = otab[k];
                            kcode = ke >> 8;
                            klen = ke & 0xFFu;
                        } else {
                            omega_compute(k, kcode, klen);
                        }
                        fits = fits && klen <= 31u;
                        string_append(w0, w1, w2, static_cast<uint32_t>(kcode), klen <= 31u ? klen : 0u);
                        lbits += glen + klen;
                    }
                }
            }
            // the lane's first bit in the run: exclusive scan of the lane lengths
            uint32_t incl = lbits;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t t = __shfl_up_sync(kAll, incl, o);
                if (lane >= o) incl += t;
            }
            const uint32_t p0 = pos + incl - lbits;
            if (!__any_sync(kAll, !fits || lbits > 96u)) {
                if (lbits != 0u) string_or(buf, p0, w0, w1, w2, lbits);
            } else {  // some lane's string is longer than 96 bits: record by record
                int32_t prev = prev_in;
                uint32_t p = p0;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const uint32_t kv = kq[4 * j + c];
                    const uint32_t k = kv & 0x7FFFFFFFu;
                    if (k != 0u) {
                        const uint32_t gap = static_cast<uint32_t>(static_cast<int32_t>(qb + c) - prev);
                        prev = static_cast<int32_t>(qb + c);
                        const uint32_t ge = otab[gap];
                        const uint32_t glen = (ge & 0xFFu) + 1u;
                        put_bits(buf, p, ((ge >> 8) << 1) | (kv >> 31), glen);
                        p += glen;
                        uint64_t kcode;
                        uint32_t klen;
                        if (k < static_cast<uint32_t>(kOmegaTab)) {
                            const uint32_t ke = otab[k];
                            kcode = ke >> 8;
                            klen = ke & 0xFFu;
                        } else {
                            omega_compute(k, kcode, klen);
                        }
                        put_bits64(buf, p, kcode, klen);
                        p += klen;
                    }
                }
            }
            pos += __shfl_sync(kAll, incl, 31);
        }
        __syncwarp();
        // --- the bucket's bits into its staging slot; the buffer cleared again -----
        uint32_t* const slot = a.stage + b * a.slot_words;
        const uint32_t nw = (pos + 31u) >> 5;
        for (uint32_t i = lane; i < nw; i += 32) {
            slot[i] = buf[i];
            buf[i] = 0u;
        }
        if (lane == 0) a.bits[b] = pos;
        __syncwarp();
    }
}

// The last compaction CTA out returns the control block to its resting state (ticket
// and completion count zero, no abort), which every encoder of the library expects
// at the start of a call on this workspace.
__device__ __forceinline__ void release_control(ScanControl* ctrl) {
    if (threadIdx.x == 0) {
        __threadfence();
        if (atomicAdd(&ctrl->done, 1u) == gridDim.x - 1) {
            ctrl->ticket = 0;
            ctrl->abort = 0;
            __threadfence();
            atomicExch(&ctrl->done, 0u);
        }
    }
}

// ---------------------------------------------------------------------------
// 2. Compaction: offsets header and the stream at its final bit positions.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kCompactThreads, 2) compact_stream(const __grid_constant__ StageArgs a) {
    constexpr int kWarps = kCompactThreads / 32;
    extern __shared__ __align__(16) uint32_t smem[];  // the tile's staged words (gather)
    __shared__ uint32_t s_R[kCompactBlock];
    __shared__ uint32_t s_L[kCompactBlock];
    __shared__ uint32_t s_RW[kCompactBlock + 1];
    __shared__ uint32_t s_tile;
    __shared__ uint64_t s_X;
    __shared__ int s_ok;
    __shared__ uint32_t s_first;
    __shared__ uint64_t s_part[kWarps];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) s_tile = atomicAdd(&a.ctrl->ticket, 1u);  // tiles in scheduling order
    __syncthreads();
    const uint64_t tile = s_tile;
    const uint64_t b0 = tile * kCompactBlock;
    const uint64_t b = b0 + tid;
    const uint32_t L = tid < kCompactBlock && b < a.nb ? a.bits[b] : 0u;
    // one block scan of two counts at once: the bucket's bits (low half; a tile is at
    // most 256 * 2^21 bits, far below 2^32) and its staged words in whole 16-byte
    // units (high half: a slot starts 16-byte aligned, so its words are gathered 16
    // bytes a copy, up to three words past the bucket's last)
    const uint32_t NW = ((L + 127u) >> 7) << 2;
    const uint64_t pair = static_cast<uint64_t>(NW) << 32 | L;
    uint64_t pincl = pair;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint64_t t = __shfl_up_sync(kAll, pincl, o);
        if (lane >= o) pincl += t;
    }
    if (lane == 31) s_part[warp] = pincl;
    if (tid < kCompactBlock) s_L[tid] = L;
    __syncthreads();
    uint64_t pbefore = 0, ptotal = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
        const uint64_t x = s_part[w];
        pbefore += w < warp ? x : 0u;
        ptotal += x;
    }
    const uint32_t total = static_cast<uint32_t>(ptotal);
    const uint32_t excl = static_cast<uint32_t>(pbefore + pincl - pair);
    if (tid == 0) st_release(&a.cdesc[tile], make_desc(0, tile == 0 ? kStatePrefix : kStateAggregate, total));
    if (tid < kCompactBlock) s_R[tid] = excl;  // tile-relative start of each bucket
    const uint32_t wincl = static_cast<uint32_t>((pbefore + pincl) >> 32), wtotal = static_cast<uint32_t>(ptotal >> 32);
    const uint32_t wbefore = wincl - NW;
    if (tid <= kCompactBlock) s_RW[tid] = wbefore;  // tile-relative first staged word; s_RW[kCompactBlock] = wtotal
    // (the 16-byte copies need 16-byte aligned slots: a workspace laid out otherwise
    // takes the direct copy)
    const bool gather = wtotal <= kCompactSmemWords && (a.slot_words & 3u) == 0u &&
                        (reinterpret_cast<uintptr_t>(a.stage) & 15u) == 0u;
    const uint32_t nt = static_cast<uint32_t>(min(static_cast<uint64_t>(kCompactBlock), a.nb - b0));
    __syncthreads();
    if (gather) {
        // gG lanes per bucket (4, 8, 16 or 32: the fewest that cover the tile's mean
        // count of 16-byte units), each lane one unit a pass
        const uint32_t mc = (wtotal / 4u + nt - 1u) / nt;
        const uint32_t gG = mc <= 4u ? 4u : mc <= 8u ? 8u : mc <= 16u ? 16u : 32u;
        const uint32_t gsub = static_cast<uint32_t>(lane) / gG, gl = static_cast<uint32_t>(lane) % gG;
        for (uint32_t i = static_cast<uint32_t>(warp) * (32u / gG) + gsub; i < nt; i += kWarps * (32u / gG)) {
            const uint32_t nw4 = ((s_L[i] + 127u) >> 7) << 2, rw = s_RW[i];
            const uint32_t* src0 = a.stage + (b0 + i) * a.slot_words;
            for (uint32_t k = 4u * gl; k < nw4; k += 4u * gG) {
                const uint32_t saddr = static_cast<uint32_t>(__cvta_generic_to_shared(smem + rw + k));
                const uint32_t* src = src0 + k;
                asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(saddr), "l"(src) : "memory");
            }
        }
        asm volatile("cp.async.commit_group;\n" ::: "memory");
    }
    // look-back by the whole CTA: thread i reads the descriptor of tile (window end -
    // i), so one read covers kCompactThreads predecessors; the nearest one holding its
    // inclusive prefix ends the walk, and every tile between must have published its
    // bit count.  Bounded: an abort or kMaxPolls empty reads end it with an error.
    uint64_t Xacc = 0;
    bool ok = true;
    if (tile > 0) {
        int64_t wend = static_cast<int64_t>(tile) - 1;
        uint32_t polls = 0;
        while (wend >= 0) {
            const int64_t idx = wend - tid;
            uint64_t st = kStatePrefix, val = 0;  // threads past tile 0 act as a zero prefix
            if (idx >= 0) {
                const uint64_t dsc = ld_acquire(&a.cdesc[idx]);
                st = desc_state(dsc);
                val = desc_value(dsc);
            }
            // nearest prefix: the smallest thread index holding one
            if (tid == 0) s_first = kCompactThreads;
            __syncthreads();
            if (st == kStatePrefix) atomicMin(&s_first, static_cast<uint32_t>(tid));
            __syncthreads();
            const uint32_t first = s_first;
            const bool wait_here = st == 0 && static_cast<uint32_t>(tid) <= first;
            if (__syncthreads_or(wait_here)) {
                ++polls;  // the same count in every thread
                const bool give_up =
                    polls > kMaxPolls || (tid == 0 && (polls & 63u) == 0 && ld_acquire32(&a.ctrl->abort) != 0);
                if (__syncthreads_or(give_up)) {
                    ok = false;
                    break;
                }
                __nanosleep(polls < 64 ? 32 : 256);
                continue;
            }
            // the window's sum up to (and with) the nearest prefix
            uint64_t c = static_cast<uint32_t>(tid) <= first ? val : 0;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(kAll, c, o);
            if (lane == 0) s_part[warp] = c;
            __syncthreads();
#pragma unroll
            for (int w = 0; w < kWarps; ++w) Xacc += s_part[w];
            __syncthreads();
            if (first < kCompactThreads) break;
            wend -= kCompactThreads;
        }
        if (tid == 0 && ok) st_release(&a.cdesc[tile], make_desc(0, kStatePrefix, Xacc + total));
    }
    if (tid == 0) {
        s_X = Xacc;
        s_ok = ok;
        if (!ok) {
            report(a.status, QSGD_ST_LOOKBACK_TIMEOUT);
            atomicExch(&a.ctrl->abort, 1u);
        }
    }
    __syncthreads();
    if (!s_ok) {
        if (gather) asm volatile("cp.async.wait_all;\n" ::: "memory");  // no copy outlives the CTA
        release_control(a.ctrl);
        return;
    }
    const uint64_t X = s_X;
    if (tid < kCompactBlock) {
        const uint64_t F = X + excl;
        if (b < a.nb) a.offsets[b] = F;
        if (b + 1 == a.nb) a.offsets[a.nb] = F + L;
    }
    if (gather) {
        asm volatile("cp.async.wait_all;\n" ::: "memory");
        __syncthreads();
    }
    // G lanes per bucket (G = 4 below 16 words a bucket on the tile's mean, else 8: a
    // quarter of the lanes that would cover a mean bucket at once, so that one setup
    // serves several words a lane), over the
    // output words whose first bit lies in the bucket: word k is bits [delta + 32 k,
    // + 32) of the bucket's staged bits, delta the distance from the bucket's start to
    // the next word boundary; a word that runs past the bucket's end takes the first
    // bits of the next bucket (always >= 32 bits, so one word of it suffices).  Every
    // output word has exactly one writer.
    const uint32_t mean_words = total / (32u * nt);
    const uint32_t G = mean_words < 16u ? 4u : 8u;
    const uint32_t per_warp = 32u / G, sub = static_cast<uint32_t>(lane) / G, sl = static_cast<uint32_t>(lane) % G;
    const uint32_t step = kWarps * per_warp;
    if (gather) {  // the words are in shared memory
        for (uint32_t i = static_cast<uint32_t>(warp) * per_warp + sub; i < nt; i += step) {
            const uint32_t Lb = s_L[i], rw = s_RW[i];
            const uint64_t F = X + s_R[i];
            const uint64_t wf = (F + 31u) >> 5;
            const uint32_t cnt = static_cast<uint32_t>(((F + Lb + 31u) >> 5) - wf);
            const uint32_t delta = static_cast<uint32_t>((wf << 5) - F);
            const uint32_t nw = (Lb + 31u) >> 5;
            // the next bucket's first word, for the word that runs past this one's end
            const uint32_t hd = i + 1 < nt ? smem[s_RW[i + 1]]
                                : b0 + i + 1 < a.nb ? a.stage[(b0 + i + 1) * a.slot_words] : 0u;
            for (uint32_t k = sl; k < cnt; k += G) {
                const uint32_t r = delta + 32u * k;  // bucket-relative bit of the word (< Lb)
                const uint32_t a0 = smem[rw + k];
                const uint32_t a1 = k + 1 < nw ? smem[rw + k + 1] : 0u;
                uint32_t v = __funnelshift_l(a1, a0, delta);
                if (r + 32u > Lb) v |= hd >> (Lb - r);  // 1 <= Lb - r <= 31
                const uint64_t w = wf + k;
                if (w < a.cap_words)
                    a.words[w] = v;
                else
                    report(a.status, QSGD_ST_OVERFLOW);
            }
        }
        release_control(a.ctrl);
        return;
    }
    // four buckets at a time and two words a lane of each, all loaded before any is
    // stored, so that their loads are in flight together
    constexpr int kU = 4, kC = 2;
    for (uint32_t i0 = static_cast<uint32_t>(warp) * per_warp + sub; i0 < nt; i0 += kU * step) {
        uint32_t Lb[kU], hd[kU];
        uint64_t F[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const uint32_t i = i0 + static_cast<uint32_t>(u) * step;
            Lb[u] = hd[u] = 0u;
            F[u] = 0u;
            if (i < nt) {
                Lb[u] = s_L[i];
                F[u] = X + s_R[i];
                // the next bucket's first word, for the word that runs past this one's end
                if (b0 + i + 1 < a.nb) hd[u] = a.stage[(b0 + i + 1) * a.slot_words];
            }
        }
        for (uint32_t kb = sl;; kb += kC * G) {
            uint32_t a0[kU][kC], a1[kU][kC];
            bool more = false;
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const uint64_t wf = (F[u] + 31u) >> 5;
                const uint32_t cnt = static_cast<uint32_t>(((F[u] + Lb[u] + 31u) >> 5) - wf);
                const uint32_t nw = (Lb[u] + 31u) >> 5;
                const uint32_t* src = a.stage + (b0 + i0 + static_cast<uint32_t>(u) * step) * a.slot_words;
#pragma unroll
                for (int c = 0; c < kC; ++c) {
                    const uint32_t k = kb + static_cast<uint32_t>(c) * G;
                    a0[u][c] = k < cnt ? src[k] : 0u;
                    a1[u][c] = k + 1 < nw && k < cnt ? src[k + 1] : 0u;
                }
                more = more || kb + kC * G < cnt;
            }
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const uint64_t wf = (F[u] + 31u) >> 5;
                const uint32_t cnt = static_cast<uint32_t>(((F[u] + Lb[u] + 31u) >> 5) - wf);
                const uint32_t delta = static_cast<uint32_t>((wf << 5) - F[u]);
#pragma unroll
                for (int c = 0; c < kC; ++c) {
                    const uint32_t k = kb + static_cast<uint32_t>(c) * G;
                    if (k < cnt) {
                        const uint32_t r = delta + 32u * k;  // bucket-relative bit of the word (< Lb)
                        uint32_t v = __funnelshift_l(a1[u][c], a0[u][c], delta);
                        if (r + 32u > Lb[u]) v |= hd[u] >> (Lb[u] - r);  // 1 <= Lb - r <= 31
                        const uint64_t w = wf + k;
                        if (w < a.cap_words)
                            a.words[w] = v;
                        else
                            report(a.status, QSGD_ST_OVERFLOW);
                    }
                }
            }
            if (!more) break;
        }
    }
    release_control(a.ctrl);
}

// One instance per kernel, so that each kernel gets its own shared-memory attribute.
template <auto kernel>
cudaError_t launch_coder(const StageArgs& a, cudaStream_t stream) {
    const size_t smem = stage_smem_bytes(a.s, a.buf_words);
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_set[dev]) {
        cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
        attr_set[dev] = true;
    }
    int sms = 0, per_sm = 0;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kStageBlock, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const uint64_t want = (a.nb + kStageWarps - 1) / kStageWarps;
    const uint64_t grid = std::max<uint64_t>(1, std::min<uint64_t>(want, static_cast<uint64_t>(sms) * per_sm));
    kernel<<<static_cast<unsigned>(grid), kStageBlock, smem, stream>>>(a);
    return cudaGetLastError();
}

template <int V, bool kShort, bool kEF>
cudaError_t launch_code(const StageArgs& a, cudaStream_t stream) {
    if constexpr (kShort)
        return launch_coder<code_buckets_short<V, kEF>>(a, stream);
    else
        return launch_coder<code_buckets<V, kEF>>(a, stream);
}

template <int V>
cudaError_t launch_code_v(const StageArgs& a, cudaStream_t stream) {
    const bool sh = a.s <= kStageShortMaxS;
    if (a.ef) return sh ? launch_code<V, true, true>(a, stream) : launch_code<V, false, true>(a, stream);
    return sh ? launch_code<V, true, false>(a, stream) : launch_code<V, false, false>(a, stream);
}

}  // namespace

cudaError_t launch_encode_stage(const StageArgs& a, cudaStream_t stream) {
    cudaError_t e;
    switch (stage_v(a.d)) {
        case 1: e = launch_code_v<1>(a, stream); break;
        case 2: e = launch_code_v<2>(a, stream); break;
        case 4: e = launch_code_v<4>(a, stream); break;
        default: e = launch_code_v<8>(a, stream); break;
    }
    if (e != cudaSuccess) return e;
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_set[dev]) {
        cudaFuncSetAttribute(compact_stream, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kCompactSmemWords * sizeof(uint32_t)));
        attr_set[dev] = true;
    }
    compact_stream<<<static_cast<unsigned>(a.ntiles), kCompactThreads, kCompactSmemWords * sizeof(uint32_t), stream>>>(a);
    return cudaGetLastError();
}

}  // namespace qsgd
