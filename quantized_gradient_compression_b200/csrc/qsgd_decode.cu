// QSGD decoders for the shapes the row decoders do not take, and the several-stream
// kernel (sm_100a).
//
// Method: "QSGD (Quantized Stochastic Gradient Descent) with Elias Coding" (AIMech
// curated entry).  The definition paragraph calls the coding "lossless prefix
// coding" of the tuple (||v||_2, signs, run-length gaps, levels k_i); the decoder
// inverts it and evaluates Q_s(v)_i = ||v||_2 * sgn(v_i) * k_i / s as
// fl(fl(norm / s) * k), sign last, +0.0 off the support.  A receiver in
// "distributed data-parallel optimization" (same paragraph) sums the decoded
// streams of its peers: out_i <- out_i + q^0_i + ... + q^{K-1}_i in stream order.
//
// Layout of the work: buckets are independent prefix-code streams located by the
// offsets header, so each lane of a warp parses one bucket.  The decoded values of
// a segment of coordinates of each of the warp's 32 buckets are scattered into a
// shared-memory staging tile (zero-filled, or loaded from the output for
// decode-accumulate) and the tile is written back.  A record is normally decoded
// with one lookup of its first 12 bits in a shared-memory table of complete
// records; longer records take a bit-serial path.  Every read is bounded by the
// bucket's [offsets[b], offsets[b+1]) range and by the stream length.
//   - decode_warp: any shape (d % 4 != 0, unaligned output), up to 16 streams a
//     launch, each lane's per-stream state in shared memory.
//   - decode_multi: two or more streams (and the mean) with d % 4 == 0, d <= 4096,
//     s < 1024 and an aligned output, a warp per stream, side by side; the row
//     decoders' side-by-side kernel takes d <= 1024 with s <= 127.
// The launch routing (launch_decode) sends one stream with d <= 1024, and several
// streams with d <= 1024 and s <= 127, to the row decoders, and d > 1024 to the
// large-bucket decoder (qsgd_decode_rows.cu).
#include <cuda_runtime.h>

#include <algorithm>

#include "../../include/qsgd.h"
#include "qsgd_device.cuh"
#include "qsgd_internal.h"
#include "qsgd_tables.cuh"

namespace qsgd {
namespace {

constexpr int kLut = kLutSize;

// Record table entry for a 12-bit window: [4:0] record length (0: not complete in
// 12 bits, or k > s), [5] the window holds a complete record with k > s, [15:6] gap,
// [25:16] k, [31] sign.  Computed at compile time for every level (within 12 bits,
// gap <= 15 and k <= 15); the copy into shared memory marks levels above s.
struct alignas(16) RecordLut {  // read with 16-byte loads
    uint32_t v[kLutSize];
};
constexpr RecordLut make_record_lut() {
    RecordLut t{};
    for (uint32_t w = 0; w < static_cast<uint32_t>(kLutSize); ++w) {
        int pos = 0;
        uint32_t gap = 0, k = 0, e = 0;
        if (window_omega(w, kLutBits, pos, gap) && pos < kLutBits) {
            const uint32_t sign = (w >> (kLutBits - 1 - pos)) & 1u;
            ++pos;
            if (window_omega(w, kLutBits, pos, k)) e = static_cast<uint32_t>(pos) | (gap << 6) | (k << 16) | (sign << 31);
        }
        t.v[w] = e;
    }
    return t;
}
__device__ const RecordLut kRecordLutGlobal = make_record_lut();

__device__ __forceinline__ void record_lut_fill(uint32_t* lut, uint32_t s, int tid, int nthreads) {
    const uint4* src = reinterpret_cast<const uint4*>(kRecordLutGlobal.v);
    for (int i = tid; i < kLutSize / 4; i += nthreads) {
        uint4 q = src[i];
        uint32_t* e = &q.x;
#pragma unroll
        for (int j = 0; j < 4; ++j)
            if ((e[j] & 31u) != 0u && ((e[j] >> 16) & 1023u) > s) e[j] = 32u;  // a level above s
        reinterpret_cast<uint4*>(lut)[i] = q;
    }
}

// MSB-first reader of one bucket with a 64-bit cache.  `pos` is the bit position
// of the cache's first unconsumed bit; bits at or past `end` are never used.
struct Reader {
    const uint32_t* w;
    uint64_t num_words;
    uint64_t pos;
    uint64_t end;
    uint64_t cache;     // 64 stream bits starting at bit 32 * cword
    uint64_t cword;     // word index of the cache's first word
    __device__ __forceinline__ uint32_t word(uint64_t i) const { return i < num_words ? __ldg(w + i) : 0u; }
    __device__ __forceinline__ void init(uint64_t p) {
        pos = p;
        cword = p >> 5;
        cache = (static_cast<uint64_t>(word(cword)) << 32) | word(cword + 1);
    }
    // next 32 bits at pos (zeros past the stream)
    __device__ __forceinline__ uint32_t peek32() {
        uint32_t off = static_cast<uint32_t>(pos - (cword << 5));
        if (off >= 32) {  // advance the cache by one word
            cache = (cache << 32) | word(cword + 2);
            ++cword;
            off -= 32;
        }
        return static_cast<uint32_t>((cache << off) >> 32);
    }
    __device__ __forceinline__ uint64_t left() const { return end - pos; }
    // bit-serial omega (any length up to 2^32 - 1)
    __device__ __forceinline__ bool omega(uint32_t& N) {
        uint32_t v = 1;
        for (;;) {
            if (pos >= end) return false;
            const uint32_t bit = peek32() >> 31;
            ++pos;
            if (bit == 0) {
                N = v;
                return true;
            }
            if (v > 31 || left() < v) return false;
            const uint32_t rest = peek32() >> (32 - v);
            pos += v;
            v = (1u << v) | rest;
        }
    }
};

// One decoded record: index within the bucket and signed level.
struct Record {
    uint32_t idx;   // bucket-local index; 0xFFFFFFFF when the bucket has no more records
    uint32_t k;
    uint32_t sign;
};

// Decodes the next record of `r`, or marks the end.  Returns false on a
// malformed stream (the bucket is then finished).
__device__ __forceinline__ bool next_record(Reader& r, const uint32_t* lut, uint32_t m, uint32_t s,
                                            uint32_t& next, Record& rec) {
    if (r.pos >= r.end) {
        rec.idx = 0xFFFFFFFFu;
        return true;
    }
    const uint32_t w = r.peek32();
    const uint32_t e = lut[w >> (32 - kLutBits)];
    const uint32_t len = e & 31u;
    uint32_t gap, k, sign;
    if (len != 0 && len <= r.left()) {
        r.pos += len;
        gap = (e >> 6) & 1023u;
        k = (e >> 16) & 1023u;
        sign = e >> 31;
    } else {
        if (!r.omega(gap)) return false;
        if (r.pos >= r.end) return false;
        sign = r.peek32() >> 31;
        ++r.pos;
        if (!r.omega(k) || k > s) return false;
    }
    if (static_cast<uint64_t>(next) + gap - 1 >= m) return false;
    rec.idx = next + gap - 1;
    rec.k = k;
    rec.sign = sign;
    next = rec.idx + 1;
    return true;
}

constexpr int kSeg = 64;                 // coordinates per bucket per staging round
constexpr int kStride = kSeg + 4;        // padded row (floats) of the staging tile
constexpr int kDecWarps = kDecodeBlock / 32;

// Per-lane state of one stream of one bucket between staging rounds (24 bytes):
// reader position, next free index, the pending record (index, level | sign << 30
// | malformed << 31) and the bucket's scale norm/s.
struct LaneStream {
    uint64_t pos;
    uint32_t next;
    uint32_t idx;
    uint32_t kflags;
    float scale;
};
static_assert(sizeof(LaneStream) == 24, "compact stream state");

__device__ __forceinline__ Record pending(const LaneStream& ls) {
    return Record{ls.idx, ls.kflags & 0x3FFFFFFFu, (ls.kflags >> 30) & 1u};
}
__device__ __forceinline__ void set_pending(LaneStream& ls, const Record& r, bool bad) {
    ls.idx = bad ? 0xFFFFFFFFu : r.idx;
    ls.kflags = (r.k & 0x3FFFFFFFu) | (r.sign << 30) | (bad ? 0x80000000u : 0u);
}

template <bool kAccumulate>
__global__ void __launch_bounds__(kDecodeBlock) decode_warp(const __grid_constant__ DecodeArgs a) {
    extern __shared__ __align__(16) uint32_t smem[];
    uint32_t* lut = smem;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    float* stage = reinterpret_cast<float*>(smem + kLut) + warp * 32 * kStride;
    LaneStream* lstate = reinterpret_cast<LaneStream*>(smem + kLut + kDecWarps * 32 * kStride) +
                         (warp * 32 + lane) * a.K;
    record_lut_fill(lut, a.s, tid, kDecodeBlock);
    __syncthreads();

    const uint64_t ngroups = (a.nb + 31) / 32;
    const uint64_t gwarps = static_cast<uint64_t>(gridDim.x) * kDecWarps;
    for (uint64_t g = static_cast<uint64_t>(blockIdx.x) * kDecWarps + warp; g < ngroups; g += gwarps) {
        const uint64_t b = g * 32 + lane;  // this lane's bucket
        const bool live = b < a.nb;
        const uint64_t base = b * a.d;
        const uint32_t m = live ? static_cast<uint32_t>(min(static_cast<uint64_t>(a.d), a.n - base)) : 0u;
        bool any_bad = false;

        // open every stream of this lane's bucket: header checks and the norm
        for (int j = 0; j < a.K; ++j) {
            LaneStream ls{0, 0, 0xFFFFFFFFu, 0, 0.f};
            Record rec{0xFFFFFFFFu, 0, 0};
            bool bad = false;
            if (live) {
                const StreamRef st = a.streams[j];
                const uint64_t begin = st.offsets[b];
                const uint64_t end = st.offsets[b + 1];
                if (!(end >= begin && end - begin >= 32 && end <= st.num_words * 32)) {
                    bad = true;
                } else {
                    Reader r{st.words, st.num_words, 0, end, 0, 0};
                    r.init(begin);
                    const uint32_t nbits = r.peek32();
                    r.pos += 32;
                    const float norm = __uint_as_float(nbits);
                    if (nbits == 0) {
                        bad = r.pos != end;
                    } else if (!(isfinite(norm) && norm > 0.f)) {
                        bad = true;
                    } else {
                        ls.scale = __fdiv_rn(norm, __uint2float_rn(a.s));
                        // a scale that rounds to zero carries no records (wire format)
                        bad = !(ls.scale > 0.f) ? r.pos != end : !next_record(r, lut, m, a.s, ls.next, rec);
                    }
                    ls.pos = r.pos;
                }
            }
            set_pending(ls, rec, bad);
            any_bad |= bad;
            lstate[j] = ls;
        }

        for (uint32_t lo = 0; lo < a.d; lo += kSeg) {
            // --- fill the staging tile: zeros, or the current output ----------
            if (kAccumulate) {
                for (int r = 0; r < 32; ++r) {
                    const uint64_t bb = g * 32 + r;
                    if (bb >= a.nb) break;
                    const uint32_t mm = static_cast<uint32_t>(min(static_cast<uint64_t>(a.d), a.n - bb * a.d));
                    for (uint32_t c = lane; c < kSeg; c += 32) {
                        const uint32_t i = lo + c;
                        float v = 0.f;
                        if (i < mm) {
                            v = a.out[bb * a.d + i];
                            if (a.first_group) v = __fadd_rn(v, 0.0f);  // -0.0 + (+0.0) = +0.0
                        }
                        stage[r * kStride + c] = v;
                    }
                }
            } else {
                for (int q = lane; q < 32 * kStride / 4; q += 32)
                    reinterpret_cast<float4*>(stage)[q] = make_float4(0.f, 0.f, 0.f, 0.f);
            }
            __syncwarp();

            // --- scatter this segment's records of every stream, in order ------
            const uint32_t hi = lo + kSeg;
            float* row = stage + lane * kStride;
            for (int j = 0; j < a.K; ++j) {
                LaneStream ls = lstate[j];
                if (ls.idx < hi) {
                    const StreamRef st = a.streams[j];
                    Reader r{st.words, st.num_words, 0, st.offsets[b + 1], 0, 0};
                    r.init(ls.pos);
                    Record rec = pending(ls);
                    bool bad = false;
                    while (rec.idx < hi) {
                        float val = __fmul_rn(ls.scale, __uint2float_rn(rec.k));
                        if (rec.sign) val = -val;
                        float* dst = row + (rec.idx - lo);
                        *dst = kAccumulate ? __fadd_rn(*dst, val) : val;
                        if (!next_record(r, lut, m, a.s, ls.next, rec)) {
                            bad = true;
                            break;
                        }
                    }
                    ls.pos = r.pos;
                    set_pending(ls, rec, bad);
                    any_bad |= bad;
                    lstate[j] = ls;
                }
            }
            __syncwarp();

            // --- write the tile back: row r is bucket g*32 + r -----------------
            const uint32_t seg_len = min(static_cast<uint32_t>(kSeg), a.d - lo);
            if ((a.d & 3u) == 0 && (reinterpret_cast<uintptr_t>(a.out) & 15u) == 0) {
                // 16-byte stores: kSeg/4 per row
                constexpr int kVec = kSeg / 4;
                for (int q = lane; q < 32 * kVec; q += 32) {
                    const int r = q / kVec, c4 = (q % kVec) * 4;
                    const uint64_t bb = g * 32 + r;
                    if (bb >= a.nb || static_cast<uint32_t>(c4) >= seg_len) continue;
                    const uint32_t mm = static_cast<uint32_t>(min(static_cast<uint64_t>(a.d), a.n - bb * a.d));
                    const uint32_t i = lo + c4;
                    if (i + 4 <= mm) {
                        *reinterpret_cast<float4*>(a.out + bb * a.d + i) =
                            *reinterpret_cast<const float4*>(stage + r * kStride + c4);
                    } else {
                        for (int t = 0; t < 4; ++t)
                            if (i + t < mm) a.out[bb * a.d + i + t] = stage[r * kStride + c4 + t];
                    }
                }
            } else {
                for (int r = 0; r < 32; ++r) {
                    const uint64_t bb = g * 32 + r;
                    if (bb >= a.nb) break;
                    const uint32_t mm = static_cast<uint32_t>(min(static_cast<uint64_t>(a.d), a.n - bb * a.d));
                    for (uint32_t c = lane; c < seg_len; c += 32)
                        if (lo + c < mm) a.out[bb * a.d + lo + c] = stage[r * kStride + c];
                }
            }
            __syncwarp();
        }
        if (any_bad) atomicOr(a.status, QSGD_ST_BAD_STREAM);
    }
}

// ---------------------------------------------------------------------------
// Bit reader and record step of the several-stream kernel (d % 4 == 0,
// d <= kMultiMaxD, s < 1024, 16-byte aligned output).
//
// Reader: a 64-bit left-aligned bit buffer -- the next unread bits of the bucket
// are the top `valid` bits of `buf` (valid >= 32 after every refill) -- plus the
// next stream word `nx`, loaded one word ahead.  `left` counts the bits of the
// bucket not yet consumed; a record that would run past the bucket end is only
// detected when the bucket ends (the staging writes stay inside the segment by
// construction), so the common path has no per-record bounds checks.
// ---------------------------------------------------------------------------
constexpr uint32_t kMultiMaxD = 4096;
constexpr uint32_t kFullMask = 0xFFFFFFFFu;

struct BitBuf {
    const uint32_t* base;  // word holding the bucket's first bit
    uint32_t wi;           // next word to fetch, relative to base
    uint32_t wlim;         // words available from base to the end of the stream
    uint64_t buf;
    uint32_t valid;
    uint32_t nx;
    uint32_t left;
    __device__ __forceinline__ uint32_t fetch() {
        const uint32_t w = wi < wlim ? __ldg(base + wi) : 0u;
        ++wi;
        return w;
    }
    __device__ __forceinline__ void init(const uint32_t* words, uint64_t num_words, uint64_t begin, uint32_t nbits) {
        const uint64_t w0 = begin >> 5;
        base = words + w0;
        wlim = static_cast<uint32_t>(min(num_words - w0, static_cast<uint64_t>(0xFFFFFFFFu)));
        wi = 0;
        const uint32_t a0 = fetch(), a1 = fetch();
        nx = fetch();
        const uint32_t sh = static_cast<uint32_t>(begin & 31u);
        buf = ((static_cast<uint64_t>(a0) << 32) | a1) << sh;
        valid = 64u - sh;
        left = nbits;
        refill();
    }
    __device__ __forceinline__ void refill() {
        if (valid < 32u) {
            buf |= static_cast<uint64_t>(nx) << (32u - valid);
            valid += 32u;
            nx = fetch();
        }
    }
    // consumes n <= 32 bits
    __device__ __forceinline__ void consume(uint32_t n) {
        buf <<= n;
        valid -= n;
        left -= n;
        refill();
    }
    __device__ __forceinline__ uint32_t top(uint32_t n) const { return static_cast<uint32_t>(buf >> (64u - n)); }
    // bit-serial omega for codes the record table does not hold
    __device__ __forceinline__ bool omega(uint32_t& N) {
        uint32_t v = 1;
        for (;;) {
            if (left == 0) return false;
            const uint32_t bit = static_cast<uint32_t>(buf >> 63);
            consume(1);
            if (bit == 0) {
                N = v;
                return true;
            }
            if (v > 31 || left < v) return false;
            const uint32_t rest = top(v);
            consume(v);
            v = (1u << v) | rest;
        }
    }
};

// The decoders' loops end by construction (each step consumes at least one bit of a
// bounded range); kLoopGuard is a second, explicit bound that marks the bucket bad.
constexpr uint32_t kLoopGuard = 1u << 20;
constexpr uint32_t kNoRecord = 0xFFFFFFFFu;  // no record left in the bucket
constexpr uint32_t kParked = 0xFFFFFFFEu;    // the next record needs the bit-serial path

// Next record through the table: its bucket-local index and value bits, or
// kParked when the record is longer than the table's window, or kNoRecord at the
// end of the bucket.  A record that overruns the bucket leaves `left` negative,
// which the end-of-bucket check reports.
__device__ __forceinline__ void table_next(BitBuf& r, const uint32_t* lut, float scale, uint32_t& next,
                                           uint32_t& idx, uint32_t& vbits) {
    if (static_cast<int32_t>(r.left) <= 0) {
        idx = kNoRecord;
        return;
    }
    const uint32_t e = lut[static_cast<uint32_t>(r.buf >> (64 - kLutBits))];
    const uint32_t len = e & 31u;
    if (len == 0) {
        idx = kParked;
        return;
    }
    r.consume(len);
    next += (e >> 6) & 1023u;
    idx = next - 1;
    vbits = __float_as_uint(__fmul_rn(scale, __uint2float_rn((e >> 16) & 1023u))) | (e & 0x80000000u);
}

// The record at the reader through the bit-serial path.  Returns false on a
// malformed record.
__device__ __forceinline__ bool slow_next(BitBuf& r, uint32_t s, float scale, uint32_t& next, uint32_t& idx,
                                       uint32_t& vbits) {
    uint32_t gap, k;
    if (!r.omega(gap) || r.left == 0 || gap > 0xFFFFu) return false;
    const uint32_t sign = static_cast<uint32_t>(r.buf >> 63) << 31;
    r.consume(1);
    if (!r.omega(k) || k > s) return false;
    next += gap;
    idx = next - 1;
    vbits = __float_as_uint(__fmul_rn(scale, __uint2float_rn(k))) | sign;
    return true;
}

// ---------------------------------------------------------------------------
// Decode-accumulate and mean of several streams in one launch.
//
// The one-stream decoder leaves about ten warps on an SM, each one chain of
// dependent table lookups, so K streams decoded one launch after another wait K
// times on that latency and move the output 2K times.  Here the kMultiWarps warps of
// a CTA decode side by side: with W = min(K, kMultiWarps) streams to a chunk, the CTA
// takes G = kMultiWarps / W groups of 32 buckets at once, and warp w decodes stream
// c * W + (w mod W) of chunk c for group w div W into its own staging tile.  Each
// stream puts at most one value on a coordinate, so a tile holds q_j (+0 off the
// support).  After each segment the CTA adds a group's tiles onto the output in
// stream order, every coordinate and every stream:
//   out <- ((out + q_cW) + q_cW+1) + ...
// which is the decode-accumulate order.  With start_zero the first chunk starts from
// +0 instead of the output; with div != 0 the last chunk divides the sum by div (the
// mean of the streams).  The output is read and written once per chunk.  Segments
// are 32 columns wide, so that four CTAs fit on an SM.
// ---------------------------------------------------------------------------
constexpr int kMultiWarps = 8;
constexpr int kMultiBlock = 32 * kMultiWarps;
constexpr int kMSeg = 32;              // coordinates per bucket per staging round
constexpr int kMStride = kMSeg + 4;    // padded row (floats) of a staging tile

__global__ void __launch_bounds__(kMultiBlock) decode_multi(const __grid_constant__ DecodeArgs a) {
    extern __shared__ __align__(16) uint32_t smem[];
    uint32_t* lut = smem;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    float* const tiles = reinterpret_cast<float*>(smem + kLut);
    float* const stage = tiles + warp * 32 * kMStride;
    float* const row = stage + lane * kMStride;
    record_lut_fill(lut, a.s, tid, kMultiBlock);
    __syncthreads();
    const float fs = __uint2float_rn(a.s);
    const uint32_t d = a.d;
    const uint64_t ngroups = (a.nb + 31) / 32;
    const int W = min(a.K, kMultiWarps);  // streams to a chunk
    const int G = kMultiWarps / W;        // groups a CTA takes at once
    const int gi = warp / W;              // this warp's group of the G (G when idle)
    const int wj = warp - gi * W;         // this warp's stream within a chunk
    for (uint64_t g0 = static_cast<uint64_t>(blockIdx.x) * G; g0 < ngroups; g0 += static_cast<uint64_t>(gridDim.x) * G) {
        const uint64_t g = g0 + gi;
        const uint64_t b = g * 32 + lane;
        const bool live = gi < G && b < a.nb;
        const uint32_t m = live ? static_cast<uint32_t>(min(static_cast<uint64_t>(d), a.n - b * d)) : 0u;
        for (int c0 = 0; c0 < a.K; c0 += W) {
            const int nt = min(W, a.K - c0);              // streams in this chunk
            const bool mine = gi < G && g < ngroups && wj < nt;  // uniform in the warp
            const bool last_chunk = c0 + nt == a.K;
            // --- open this lane's bucket of stream c0 + wj ----------------------
            bool bad = false;
            BitBuf r;
            r.left = 0;
            float scale = 0.f;
            if (mine && live) {
                const StreamRef st = a.streams[c0 + wj];
                const uint64_t begin = st.offsets[b];
                const uint64_t end = st.offsets[b + 1];
                if (!(end >= begin && end - begin >= 32 && end <= st.num_words * 32 && end - begin < (1ull << 30))) {
                    bad = true;
                } else {
                    r.init(st.words, st.num_words, begin, static_cast<uint32_t>(end - begin));
                    const uint32_t nbits = r.top(32);
                    r.consume(32);
                    const float norm = __uint_as_float(nbits);
                    if (nbits == 0) {
                        bad = r.left != 0;
                        r.left = 0;
                    } else if (!(isfinite(norm) && norm > 0.f)) {
                        bad = true;
                        r.left = 0;
                    } else {
                        scale = __fdiv_rn(norm, fs);
                        if (!(scale > 0.f) && r.left != 0) {  // a zero scale carries no records
                            bad = true;
                            r.left = 0;
                        }
                    }
                }
            }
            uint32_t next = 0, pidx = kNoRecord, pval = 0;
            if (mine && !bad) table_next(r, lut, scale, next, pidx, pval);
            for (uint32_t lo = 0; lo < d; lo += kMSeg) {
                if (mine) {
                    // --- this stream's values of the segment into a zeroed tile ----
                    for (int q = lane; q < 32 * kMStride / 4; q += 32)
                        reinterpret_cast<float4*>(stage)[q] = make_float4(0.f, 0.f, 0.f, 0.f);
                    __syncwarp();
                    const uint32_t hi = lo + kMSeg;
                    for (uint32_t it = 0;; ++it) {
                        const bool place = pidx < hi;
                        if (it == kLoopGuard) {
                            bad = true;
                            pidx = kNoRecord;
                        }
                        if (__any_sync(kFullMask, place) && it < kLoopGuard) {
                            if (place) {
                                row[pidx - lo] = __uint_as_float(pval);
                                table_next(r, lut, scale, next, pidx, pval);
                            }
                        } else if (__any_sync(kFullMask, pidx == kParked)) {
                            if (pidx == kParked && !slow_next(r, a.s, scale, next, pidx, pval)) {
                                bad = true;
                                pidx = kNoRecord;
                            }
                        } else {
                            break;
                        }
                    }
                }
                __syncthreads();  // every tile of the chunk holds its segment
                // --- the CTA adds each group's tiles onto the output in stream order
                for (int q = tid; q < G * 32 * (kMSeg / 4); q += kMultiBlock) {
                    const int qg = q / (32 * (kMSeg / 4));
                    const int qr = q - qg * (32 * (kMSeg / 4));
                    const uint32_t rr = static_cast<uint32_t>(qr) / (kMSeg / 4);
                    const uint32_t cc = (static_cast<uint32_t>(qr) % (kMSeg / 4)) * 4;
                    const uint64_t bb = (g0 + qg) * 32 + rr;
                    const uint32_t mm = bb < a.nb ? static_cast<uint32_t>(min(static_cast<uint64_t>(d), a.n - bb * d)) : 0u;
                    const uint32_t c = lo + cc;
                    if (c >= mm) continue;
                    float* gp = a.out + bb * d + c;
                    const bool whole = c + 4 <= mm;
                    float v[4] = {0.f, 0.f, 0.f, 0.f};
                    if (!(a.start_zero && c0 == 0)) {
                        if (whole) {
                            const float4 o = *reinterpret_cast<const float4*>(gp);
                            v[0] = o.x;
                            v[1] = o.y;
                            v[2] = o.z;
                            v[3] = o.w;
                        } else {  // c < mm <= c + 3
                            v[0] = gp[0];
                            if (c + 1 < mm) v[1] = gp[1];
                            if (c + 2 < mm) v[2] = gp[2];
                        }
                    }
                    for (int t = 0; t < nt; ++t) {
                        const float4 w = *reinterpret_cast<const float4*>(tiles + ((qg * W + t) * 32 + rr) * kMStride + cc);
                        v[0] = __fadd_rn(v[0], w.x);
                        v[1] = __fadd_rn(v[1], w.y);
                        v[2] = __fadd_rn(v[2], w.z);
                        v[3] = __fadd_rn(v[3], w.w);
                    }
                    if (last_chunk && a.div != 0.f) {
#pragma unroll
                        for (int e = 0; e < 4; ++e) v[e] = __fdiv_rn(v[e], a.div);
                    }
                    if (whole) {
                        *reinterpret_cast<float4*>(gp) = make_float4(v[0], v[1], v[2], v[3]);
                    } else {
                        gp[0] = v[0];
                        if (c + 1 < mm) gp[1] = v[1];
                        if (c + 2 < mm) gp[2] = v[2];
                    }
                }
                __syncthreads();  // the tiles are free for the next segment
            }
            // every record index below m, and the bucket consumed exactly
            if (mine && live && !bad && (next > m || r.left != 0 || pidx != kNoRecord)) bad = true;
            if (mine && bad) atomicOr(a.status, QSGD_ST_BAD_STREAM);
        }
    }
}

cudaError_t launch_multi(const DecodeArgs& a, cudaStream_t stream) {
    const size_t smem = kLut * sizeof(uint32_t) + static_cast<size_t>(kMultiWarps) * 32 * kMStride * sizeof(float);
    static bool attr_set[64] = {};
    int dev = 0, sms = 0, per_sm = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_set[dev]) {
        cudaFuncSetAttribute(decode_multi, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
        attr_set[dev] = true;
    }
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_multi, kMultiBlock, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const uint64_t G = static_cast<uint64_t>(kMultiWarps / std::min(a.K, kMultiWarps));  // groups a CTA takes at once
    const uint64_t sets = ((a.nb + 31) / 32 + G - 1) / G;
    const uint64_t blocks = std::min<uint64_t>(sets, static_cast<uint64_t>(sms) * per_sm);
    decode_multi<<<static_cast<unsigned>(blocks), kMultiBlock, smem, stream>>>(a);
    return cudaGetLastError();
}

template <bool kAccumulate>
cudaError_t launch(const DecodeArgs& a, cudaStream_t stream) {
    const size_t smem = kLut * sizeof(uint32_t) + static_cast<size_t>(kDecWarps) * 32 * kStride * sizeof(float) +
                        static_cast<size_t>(kDecodeBlock) * a.K * sizeof(LaneStream);
    static bool attr_set[64] = {};
    int dev = 0, sms = 0, per_sm = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_set[dev]) {
        cudaFuncSetAttribute(decode_warp<kAccumulate>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
        attr_set[dev] = true;
    }
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_warp<kAccumulate>,
                                                                  kDecodeBlock, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const uint64_t groups = (a.nb + 31) / 32;
    const uint64_t blocks = std::min<uint64_t>((groups + kDecWarps - 1) / kDecWarps,
                                               static_cast<uint64_t>(sms) * per_sm);
    decode_warp<kAccumulate><<<static_cast<unsigned>(blocks), kDecodeBlock, smem, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace

bool decode_multi_shape(uint32_t d, uint32_t s, const float* out) {
    return d % 4 == 0 && d <= kMultiMaxD && s < 1024 && (reinterpret_cast<uintptr_t>(out) & 15u) == 0;
}

cudaError_t launch_decode(const DecodeArgs& a, bool accumulate, cudaStream_t stream) {
    if (a.nb == 0) return cudaSuccess;
    const bool multi = decode_multi_shape(a.d, a.s, a.out);
    // the row decoders when the shape allows: one stream staged as codes; several
    // streams (and the mean) parsed side by side as byte codes (s <= 127), or added
    // onto fp32 tiles in stream order where the several-stream kernel below, which
    // decodes the streams side by side, does not take the levels (s >= 1024)
    if (decode_rows_shape(a.d, a.s, a.out)) {
        if (a.K == 1 && !a.start_zero && a.div == 0.f) return launch_decode_rows(a, accumulate, stream);
        if (a.s <= kRowsMaxS8 && (accumulate || a.start_zero)) return launch_decode_rows_side(a, stream);
        if (!multi) return launch_decode_rows_multi(a, stream);
    }
    // the mean in one pass: streams decoded side by side, the sum divided at the end
    if (a.start_zero || a.div != 0.f) return multi ? launch_multi(a, stream) : cudaErrorInvalidValue;
    // buckets larger than the rows: a fill of the output, then the records
    if (decode_sparse_shape(a.d, a.out)) return launch_decode_sparse(a, accumulate, stream);
    // several streams on the rows' shapes: decoded side by side, the output moved once
    if (multi && accumulate && a.K >= 2) return launch_multi(a, stream);
    // every other shape (d % 4 != 0, an unaligned output): one warp per 32 buckets
    return accumulate ? launch<true>(a, stream) : launch<false>(a, stream);
}

}  // namespace qsgd
