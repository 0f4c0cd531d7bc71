// QSGD row decoders: one stream staged as level codes, several streams parsed side by
// side or added onto fp32 tiles, and large buckets (sm_100a).
//
// Method: "QSGD (Quantized Stochastic Gradient Descent) with Elias Coding" (AIMech
// curated entry).  The definition paragraph calls the coding "lossless prefix
// coding" of the tuple (||v||_2, signs, run-length gaps, levels k_i); the decoder
// inverts it and evaluates Q_s(v)_i = ||v||_2 * sgn(v_i) * k_i / s as
// fl(fl(norm / s) * k), sign last, +0.0 off the support.  Decode-accumulate (a
// receiver in "distributed data-parallel optimization", same paragraph) adds the
// decoded stream onto the output: out_i <- fl(out_i + q_i).
//
// One stream: each lane of a warp parses one bucket (buckets are independent
// prefix-code streams located by the offsets header), 32 consecutive buckets to a
// warp, and stores each record's code at its index in its bucket's row of a zeroed
// staging area in shared memory; no lane waits for another while parsing.  The warp
// then converts the rows to fp32 and writes each bucket with coalesced 16-byte
// stores (decode-accumulate first reads the output, which a prefetch to L2 issued
// before the parse has brought in).
//   - decode_rows (s <= 127): byte codes sign << 7 | k in whole rows of d codes;
//     records through a table of the whole records at the start of a 12-bit window
//     (up to two per entry), two lookups a step.
//   - decode_rows_ring (127 < s <= 32767, where nearly every coordinate has a
//     record): 16-bit codes sign << 15 | k in a ring of two 128-column segments per
//     row, written back segment by segment (half the shared memory of whole rows,
//     twice the warps); records through a table of omega codes, one lookup for the
//     gap and one for the level.
// Several streams (decode-accumulate, K >= 2, and the mean):
//   - decode_rows_side (s <= 127): a warp a stream, the streams of a chunk side by
//     side in one CTA, each parsed as decode_rows does into a ring of byte codes; the
//     CTA adds a segment's values onto the output in stream order once every warp has
//     passed it.
//   - decode_rows_multi (larger s where the other several-stream kernel does not
//     take the levels): the streams one after another onto an fp32 tile.
// Longer records take a bit-serial path.
#include <cuda_runtime.h>

#include <algorithm>

#include "../../include/qsgd.h"
#include "qsgd_device.cuh"
#include "qsgd_internal.h"
#include "qsgd_tables.cuh"

namespace qsgd {
namespace {

constexpr uint32_t kWarpAll = 0xFFFFFFFFu;
constexpr uint32_t kParseGuard = 1u << 20;  // a second, explicit bound of the parse loop

// MSB-first reader of one bucket over two stream words: the next unread bits are
// the top bits of funnelshift(nx, cur, off) (0 <= off < 32); `left` counts the bits
// of the bucket not yet consumed (negative, as int32, after a record that overran).
// kAhead: one more word held, loaded a word ahead of its use (the large-bucket
// decoders, whose few warps per SM wait on each refill otherwise).
template <bool kAhead>
struct RowReaderT {
    const uint32_t* base;  // word holding the bucket's first bit
    uint32_t wi;           // next word to fetch, relative to base
    uint32_t wlim;         // words available from base to the end of the stream
    uint32_t cur, nx, nx2, off;
    int32_t left;
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
        cur = fetch();
        nx = fetch();
        if (kAhead) nx2 = fetch();
        off = static_cast<uint32_t>(begin & 31u);
        left = static_cast<int32_t>(nbits);
    }
    __device__ __forceinline__ uint32_t peek() const { return __funnelshift_l(nx, cur, off); }
    __device__ __forceinline__ void advance(uint32_t n) {  // n <= 32
        off += n;
        left -= static_cast<int32_t>(n);
        if (off >= 32u) {
            cur = nx;
            if (kAhead) {
                nx = nx2;
                nx2 = fetch();
            } else {
                nx = fetch();
            }
            off -= 32u;
        }
    }
    __device__ __forceinline__ bool omega(uint32_t& N) {  // bit-serial, any length up to 2^32 - 1
        uint32_t v = 1;
        for (;;) {
            if (left <= 0) return false;
            const uint32_t bit = peek() >> 31;
            advance(1);
            if (bit == 0) {
                N = v;
                return true;
            }
            if (v > 31 || left < static_cast<int32_t>(v)) return false;
            const uint32_t rest = peek() >> (32 - v);
            advance(v);
            v = (1u << v) | rest;
        }
    }
};
using RowReader = RowReaderT<false>;

// The 16-bit ring decoder's reader: the bucket's stream words pass through a ring of
// eight words a lane in shared memory, refilled four words at a time with cp.async
// while the lane parses the other four.  (That kernel's shared memory leaves L1 little
// room, so a word loaded straight from the stream waits on L2 at every refill.)  Same
// bit order and interface as RowReaderT.
struct StagedReader {
    const uint32_t* base;  // word holding the bucket's first bit
    uint32_t* sbuf;        // this lane's eight words (word w in slot w mod 8)
    uint32_t wi;           // next word to read, relative to base
    uint32_t wlim;         // words available from base to the end of the stream
    uint32_t cur, nx, off;
    int32_t left;
    // words w0 .. w0 + 3 into their slots (zeros past the stream), one commit group
    __device__ __forceinline__ void copy_half(uint32_t w0) {
#pragma unroll
        for (uint32_t i = 0; i < 4u; ++i) {
            const uint32_t w = w0 + i;
            uint32_t* const dst = sbuf + (w & 7u);
            if (w < wlim) {
                const uint32_t saddr = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
                const uint32_t* const src = base + w;
                asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(saddr), "l"(src) : "memory");
            } else {
                *dst = 0u;
            }
        }
        asm volatile("cp.async.commit_group;\n" ::: "memory");
    }
    __device__ __forceinline__ uint32_t fetch() {
        if ((wi & 3u) == 0u) {  // entering a half: its words have landed; refill the half just left
            asm volatile("cp.async.wait_all;\n" ::: "memory");
            copy_half(wi + 4u);
        }
        const uint32_t w = sbuf[wi & 7u];
        ++wi;
        return w;
    }
    __device__ __forceinline__ void init(const uint32_t* words, uint64_t num_words, uint64_t begin, uint32_t nbits) {
        asm volatile("cp.async.wait_all;\n" ::: "memory");  // no copy of an earlier bucket is still landing
        const uint64_t w0 = begin >> 5;
        base = words + w0;
        wlim = static_cast<uint32_t>(min(num_words - w0, static_cast<uint64_t>(0xFFFFFFFFu)));
        copy_half(0u);
        copy_half(4u);
        asm volatile("cp.async.wait_all;\n" ::: "memory");
        cur = sbuf[0];
        nx = sbuf[1];
        wi = 2;
        off = static_cast<uint32_t>(begin & 31u);
        left = static_cast<int32_t>(nbits);
    }
    __device__ __forceinline__ uint32_t peek() const { return __funnelshift_l(nx, cur, off); }
    __device__ __forceinline__ void advance(uint32_t n) {  // n <= 32
        off += n;
        left -= static_cast<int32_t>(n);
        if (off >= 32u) {
            cur = nx;
            nx = fetch();
            off -= 32u;
        }
    }
    __device__ __forceinline__ bool omega(uint32_t& N) {  // bit-serial, any length up to 2^32 - 1
        uint32_t v = 1;
        for (;;) {
            if (left <= 0) return false;
            const uint32_t bit = peek() >> 31;
            advance(1);
            if (bit == 0) {
                N = v;
                return true;
            }
            if (v > 31 || left < static_cast<int32_t>(v)) return false;
            const uint32_t rest = peek() >> (32 - v);
            advance(v);
            v = (1u << v) | rest;
        }
    }
};

// A record the table does not hold, bit by bit: false when it is malformed (its gap
// beyond the bucket length d, or its level beyond s).
template <class Reader>
__device__ __forceinline__ bool slow_record(Reader& r, uint32_t s, uint32_t d, uint32_t& gap, uint32_t& sign,
                                            uint32_t& k) {
    if (!r.omega(gap) || r.left <= 0 || gap > d) return false;
    sign = r.peek() >> 31;
    r.advance(1);
    return r.omega(k) && k <= s;
}

// A row code: sign << 7 | k in a byte (s <= 127) or sign << 15 | k in 16 bits.
template <class T>
__device__ __forceinline__ T row_code(uint32_t sign, uint32_t k) {
    return static_cast<T>((sign << (8 * sizeof(T) - 1)) | k);
}
// The output of bucket bb as lane `lane` reads it in the write-back: float4 i is
// coordinates 4 (lane + 32 i) .. + 3, zeros past the bucket's end.
template <int V>
__device__ __forceinline__ void load_row(const DecodeArgs& a, uint64_t bb, int lane, float4 (&o)[V]) {
    const uint32_t mm = static_cast<uint32_t>(min(static_cast<uint64_t>(a.d), a.n - bb * a.d));
    const float* gp = a.out + bb * a.d;
#pragma unroll
    for (int i = 0; i < V; ++i) {
        const uint32_t c = 4u * (static_cast<uint32_t>(lane) + 32u * i);
        o[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (c + 4 <= mm) {
            o[i] = __ldcs(reinterpret_cast<const float4*>(gp + c));
        } else if (c < mm) {
            o[i].x = gp[c];
            if (c + 1 < mm) o[i].y = gp[c + 1];
            if (c + 2 < mm) o[i].z = gp[c + 2];
        }
    }
}

// One parse step through the whole-record table (byte codes): up to two table
// entries, each up to two records.  The 32 bits at the cursor hold both 12-bit
// windows (the first entry's records take at most 12 bits, so a step moves at most
// 60 columns); a record is taken only when it ends inside the bucket.  A record
// longer than the window whose gap's code fits it goes through near_long_record
// (gap <= 63, k <= 15 and k <= s; at most 63 columns).  put(index, code) stores a
// record's code (sign << 7 | k) at its bucket-local index.  Returns false, having
// read nothing, when the record at the cursor is neither (far_record takes it).
template <class Reader, class Put>
__device__ __forceinline__ bool rows_table_step(Reader& r, const uint32_t* lut, const uint8_t* klut, uint32_t s,
                                                uint32_t& next, const Put& put) {
    const uint32_t w = r.peek();
    const uint32_t e = lut[w >> (32 - kLutBits)];
    const uint32_t len1 = e & 15u;
    if (len1 == 0u) {
        uint32_t gap = 0, code = 0;
        const uint32_t len = near_long_record(w, e, klut, gap, code);
        if (len == 0u || (code & 0x7Fu) > s) return false;
        next += gap;
        put(next - 1u, code);
        r.advance(len);
        return true;
    }
    const uint32_t len2 = (e >> 4) & 15u;
    const bool two = static_cast<int32_t>(len2) <= r.left;
    uint32_t used = two ? len2 : len1;
    next += (e >> 8) & 15u;
    put(next - 1u, (e >> 16) & 0xFFu);
    const uint32_t c2 = e >> 24;
    if (two && c2 != 0u) {
        next += (e >> 12) & 15u;
        put(next - 1u, c2);
    }
    if (two) {
        const uint32_t f = lut[(w << used) >> (32 - kLutBits)];
        const uint32_t flen1 = f & 15u;
        if (flen1 != 0u && static_cast<int32_t>(used + flen1) <= r.left) {
            const uint32_t flen2 = (f >> 4) & 15u;
            const bool ftwo = static_cast<int32_t>(used + flen2) <= r.left;
            next += (f >> 8) & 15u;
            put(next - 1u, (f >> 16) & 0xFFu);
            const uint32_t fc2 = f >> 24;
            if (ftwo && fc2 != 0u) {
                next += (f >> 12) & 15u;
                put(next - 1u, fc2);
            }
            used += ftwo ? flen2 : flen1;
        }
    }
    r.advance(used);
    return true;
}

// A record the table step does not take: far_long_record (gap < 2^16, k <= 15),
// else bit by bit.  Returns false when it is malformed (gap beyond d, level beyond
// s); else its gap, sign and level, the reader past it.
template <class Reader>
__device__ __forceinline__ bool far_record(Reader& r, const uint8_t* plut, const uint8_t* klut, uint32_t s,
                                           uint32_t d, uint32_t& gap, uint32_t& sign, uint32_t& k) {
    uint32_t code = 0;
    const uint32_t len = far_long_record(r.peek(), plut, klut, gap, code);
    if (len != 0u && (code & 0x7Fu) <= s) {
        r.advance(len);
        sign = code >> 7;
        k = code & 0x7Fu;
        return true;
    }
    return slow_record(r, s, d, gap, sign, k);
}

template <int V, bool kAcc>
__global__ void __launch_bounds__(32 * kRowsMaxWarps) decode_rows(const __grid_constant__ DecodeArgs a,
                                                                   uint32_t stride_w) {
    extern __shared__ __align__(16) uint32_t smem[];
    uint32_t* const lut = smem;
    uint8_t* const klut = reinterpret_cast<uint8_t*>(smem + kLutSize);
    uint8_t* const plut = reinterpret_cast<uint8_t*>(smem + kLutSize + kKLutWords);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int W = blockDim.x >> 5;
    uint32_t* const rows = smem + kLutSize + kSmallLutWords + static_cast<uint32_t>(warp) * 32u * stride_w;
    uint8_t* const myrow = reinterpret_cast<uint8_t*>(rows + static_cast<uint32_t>(lane) * stride_w);
    rows_lut_fill(lut, a.s, tid, blockDim.x);
    k_lut_fill(klut, tid, blockDim.x);
    p_lut_fill(plut, tid, blockDim.x);
    __syncthreads();
    const StreamRef st = a.streams[0];
    const float fs = __uint2float_rn(a.s);
    const uint32_t d = a.d;
    const uint64_t ngroups = (a.nb + 31) / 32;
    for (uint64_t g = blockIdx.x + static_cast<uint64_t>(gridDim.x) * warp; g < ngroups;
         g += static_cast<uint64_t>(gridDim.x) * W) {
        const uint64_t b = g * 32 + lane;
        const bool live = b < a.nb;
        const uint32_t m = live ? static_cast<uint32_t>(min(static_cast<uint64_t>(d), a.n - b * d)) : 0u;
        if constexpr (kAcc) {  // bring the group's output into L2 while the records are parsed
            const float* gp = a.out + g * 32 * d;
            const uint64_t gbytes = 4 * (min(a.n, (g + 1) * 32 * d) - g * 32 * d);
            for (uint64_t off = static_cast<uint64_t>(lane) * 128; off < gbytes; off += 32 * 128)
                asm volatile("prefetch.global.L2 [%0];" ::"l"(reinterpret_cast<const char*>(gp) + off));
        }
        // zero the warp's rows (32 * stride_w words, a multiple of four)
        for (uint32_t q = lane; q < 8u * stride_w; q += 32)
            reinterpret_cast<uint4*>(rows)[q] = make_uint4(0u, 0u, 0u, 0u);
        // open this lane's bucket: header checks and the norm
        bool bad = false;
        RowReader r;
        r.left = 0;
        float scale = 0.f;
        if (live) {
            const uint64_t begin = st.offsets[b];
            const uint64_t end = st.offsets[b + 1];
            if (!(end >= begin && end - begin >= 32 && end <= st.num_words * 32 && end - begin < (1ull << 30))) {
                bad = true;
            } else {
                r.init(st.words, st.num_words, begin, static_cast<uint32_t>(end - begin));
                const uint32_t nbits = r.peek();
                r.advance(32);
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
        __syncwarp();
        // --- parse: every record's code into the lane's row -------------------------
        uint32_t next = 0;  // bucket-local index after the last record
        if (bad) r.left = 0;
        for (uint32_t it = 0; __any_sync(kWarpAll, r.left > 0); ++it) {
            if (it == kParseGuard) {
                bad = bad || r.left > 0;
                break;
            }
            if (r.left > 0) {
                const auto put = [&](uint32_t idx, uint32_t code) { myrow[min(idx, d)] = static_cast<uint8_t>(code); };
                if (!rows_table_step(r, lut, klut, a.s, next, put)) {
                    uint32_t gap = 0, sign = 0, k = 0;
                    if (far_record(r, plut, klut, a.s, d, gap, sign, k)) {
                        next += gap;
                        put(next - 1u, row_code<uint8_t>(sign, k));
                    } else {
                        bad = true;
                        r.left = 0;
                    }
                }
            }
        }
        // every record index below m, and the bucket consumed exactly (a record that
        // overran leaves left negative; an index past m lands in the row's padding)
        if (live && !bad && (next > m || r.left != 0)) bad = true;
        __syncwarp();
        // --- write the rows back: row rr is bucket g*32 + rr -----------------------
        // (decode-accumulate reads the next row's output before it stores this row's,
        // so that two rows of loads are in flight)
        const int nrows = static_cast<int>(min(static_cast<uint64_t>(32), a.nb - g * 32));
        float4 cur[kAcc ? V : 1], nxt[kAcc ? V : 1];
        if constexpr (kAcc) load_row<V>(a, g * 32, lane, cur);
        for (int rr = 0; rr < nrows; ++rr) {
            const uint64_t bb = g * 32 + rr;
            const float sc = __shfl_sync(kWarpAll, scale, rr);
            if constexpr (kAcc) {
                if (rr + 1 < nrows) load_row<V>(a, bb + 1, lane, nxt);
            }
            const uint32_t mm = static_cast<uint32_t>(min(static_cast<uint64_t>(d), a.n - bb * d));
            const uint32_t* rowp = rows + static_cast<uint32_t>(rr) * stride_w;
            float* gp = a.out + bb * d;
#pragma unroll
            for (int i = 0; i < V; ++i) {
                const uint32_t q = static_cast<uint32_t>(lane) + 32u * i;
                const uint32_t c = 4u * q;
                if (c < mm) {
                    uint32_t code[4];
                    const uint32_t w = rowp[q];
#pragma unroll
                    for (int j = 0; j < 4; ++j) code[j] = ((w >> (8 * j)) & 0x7Fu) | (((w >> (8 * j)) & 0x80u) << 24);
                    float v[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        // code[j] = k | sign << 31: k as fp32 through the 2^23 offset (exact
                        // for k < 2^23), times the step, the sign last
                        const float kf = __fsub_rn(__uint_as_float(0x4B000000u | (code[j] & 0x7FFFFFFFu)), 8388608.0f);
                        v[j] = __uint_as_float(__float_as_uint(__fmul_rn(sc, kf)) | (code[j] & 0x80000000u));
                    }
                    if constexpr (kAcc) {
                        v[0] = __fadd_rn(cur[i].x, v[0]);
                        v[1] = __fadd_rn(cur[i].y, v[1]);
                        v[2] = __fadd_rn(cur[i].z, v[2]);
                        v[3] = __fadd_rn(cur[i].w, v[3]);
                    }
                    if (c + 4 <= mm) {
                        __stcs(reinterpret_cast<float4*>(gp + c), make_float4(v[0], v[1], v[2], v[3]));
                    } else {
                        for (uint32_t j = 0; j < 4 && c + j < mm; ++j) gp[c + j] = v[j];
                    }
                }
            }
            if constexpr (kAcc) {
#pragma unroll
                for (int i = 0; i < V; ++i) cur[i] = nxt[i];
            }
        }
        if (bad) atomicOr(a.status, QSGD_ST_BAD_STREAM);
        __syncwarp();
    }
}

// Segments and the ring of codes: the warp decodes its 32 buckets kRSeg columns at a
// time and writes each segment back as soon as every lane has parsed past it, so
// the output stores of one segment overlap the parse of the next.  A row holds two
// segments of codes (column c at ring slot c mod kRRing): while segment [lo, hi) is
// parsed, a record may land up to kRSeg columns past hi (a step of table records
// moves at most 60 columns, one omega-table record 63), which is the next segment's
// half.  A bit-serial record further ahead is held in registers until its segment.
#ifndef QSGD_ROWS_SEG
#define QSGD_ROWS_SEG 128
#endif
constexpr uint32_t kRSeg = QSGD_ROWS_SEG;
constexpr uint32_t kRRing = 2 * kRSeg;
static_assert(kRSeg == 64 || (kRSeg % 128 == 0 && kRSeg >= 128), "a segment is half a warp's or whole float4 columns");
constexpr uint32_t kRLanesPerRow = kRSeg / 4 < 32 ? kRSeg / 4 : 32;  // lanes on one row of a segment
constexpr uint32_t kRRowsPerPass = 32 / kRLanesPerRow;               // rows a warp writes at once
constexpr int kRVec = kRSeg / 128 > 0 ? static_cast<int>(kRSeg / 128) : 1;  // float4 per lane per row
constexpr int kRBatch = 8;  // passes whose output is loaded together

template <bool kAcc>
__global__ void __launch_bounds__(32 * kRowsMaxWarps) decode_rows_ring(const __grid_constant__ DecodeArgs a,
                                                                   uint32_t stride_w) {
    extern __shared__ __align__(16) uint32_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int W = blockDim.x >> 5;
    uint32_t* const rows = smem + kLutSize + static_cast<uint32_t>(warp) * 32u * stride_w;
    uint16_t* const myrow = reinterpret_cast<uint16_t*>(rows + static_cast<uint32_t>(lane) * stride_w);
    // this lane's ring of stream words (after every warp's rows)
    uint32_t* const sbuf = smem + kLutSize + static_cast<uint32_t>(W) * 32u * stride_w + static_cast<uint32_t>(tid) * 8u;
    // the omega table, looked up for the gap and then for the level
    uint16_t* const olut = reinterpret_cast<uint16_t*>(smem);
    omega_lut_fill(olut, tid, blockDim.x);
    __syncthreads();
    const StreamRef st = a.streams[0];
    const float fs = __uint2float_rn(a.s);
    const uint32_t d = a.d;
    const uint64_t ngroups = (a.nb + 31) / 32;
    for (uint64_t g = blockIdx.x + static_cast<uint64_t>(gridDim.x) * warp; g < ngroups;
         g += static_cast<uint64_t>(gridDim.x) * W) {
        const uint64_t b = g * 32 + lane;
        const bool live = b < a.nb;
        const uint32_t m = live ? static_cast<uint32_t>(min(static_cast<uint64_t>(d), a.n - b * d)) : 0u;
        const int nrows = static_cast<int>(min(static_cast<uint64_t>(32), a.nb - g * 32));
        if constexpr (kAcc) {  // bring the group's output into L2 while the records are parsed
            const float* gp = a.out + g * 32 * d;
            const uint64_t gbytes = 4 * (min(a.n, (g + 1) * 32 * d) - g * 32 * d);
            for (uint64_t off = static_cast<uint64_t>(lane) * 128; off < gbytes; off += 32 * 128)
                asm volatile("prefetch.global.L2 [%0];" ::"l"(reinterpret_cast<const char*>(gp) + off));
        }
        // zero the warp's rows (32 * stride_w words, a multiple of four)
        for (uint32_t q = lane; q < 8u * stride_w; q += 32)
            reinterpret_cast<uint4*>(rows)[q] = make_uint4(0u, 0u, 0u, 0u);
        // open this lane's bucket: header checks and the norm
        bool bad = false;
        StagedReader r;
        r.sbuf = sbuf;
        r.left = 0;
        float scale = 0.f;
        if (live) {
            const uint64_t begin = st.offsets[b];
            const uint64_t end = st.offsets[b + 1];
            if (!(end >= begin && end - begin >= 32 && end <= st.num_words * 32 && end - begin < (1ull << 30))) {
                bad = true;
            } else {
                r.init(st.words, st.num_words, begin, static_cast<uint32_t>(end - begin));
                const uint32_t nbits = r.peek();
                r.advance(32);
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
        if (bad) r.left = 0;
        __syncwarp();
        uint32_t next = 0;            // bucket-local index after the last record
        bool pend = false;            // a bit-serial record beyond the ring, held here
        uint32_t pidx = 0, pcode = 0;
        uint32_t it = 0;              // parse steps over the whole bucket (an explicit bound)
        for (uint32_t lo = 0; lo < d; lo += kRSeg) {
            const uint32_t hi = lo + kRSeg;
            if (pend && pidx < hi + kRSeg) {
                myrow[pidx & (kRRing - 1u)] = static_cast<uint16_t>(pcode);
                pend = false;
            }
            // --- parse until every lane has passed column hi (or ended) ---------------
            for (;; ++it) {
                const bool act = r.left > 0 && !pend && next < hi;
                if (!__any_sync(kWarpAll, act)) break;
                if (it >= kParseGuard) {  // never reached by a well-formed stream
                    if (act) {
                        bad = true;
                        r.left = 0;
                    }
                    continue;
                }
                if (!act) continue;
                // one record a step: omega(gap) (<= 12 bits), the sign, omega(k) (<= 12
                // bits) from the 32 bits at the cursor; k <= 63 < s, so no level check
                const uint32_t w = r.peek();
                const uint32_t ge = olut[w >> (32 - kLutBits)];
                const uint32_t gl = ge & 15u;
                const uint32_t w2 = w << gl;
                const uint32_t ke = olut[(w2 << 1) >> (32 - kLutBits)];
                const uint32_t kl = ke & 15u;
                if (gl != 0u && kl != 0u) {
                    next += ge >> 4;
                    myrow[min(next - 1u, d) & (kRRing - 1u)] = row_code<uint16_t>(w2 >> 31, ke >> 4);
                    r.advance(gl + 1u + kl);
                    continue;
                }
                // a record the table does not hold, bit by bit
                uint32_t gap = 0, sign = 0, k = 0;
                if (slow_record(r, a.s, a.d, gap, sign, k)) {
                    next += gap;
                    const uint32_t idx = min(next - 1u, d);
                    if (idx >= hi + kRSeg) {
                        pend = true;
                        pidx = idx;
                        pcode = row_code<uint16_t>(sign, k);
                    } else {
                        myrow[idx & (kRRing - 1u)] = row_code<uint16_t>(sign, k);
                    }
                } else {
                    bad = true;
                    r.left = 0;
                }
            }
            __syncwarp();
            // --- write back columns [lo, hi) of the 32 rows, and clear them ----------
            // (kRRowsPerPass rows a pass, kRLanesPerRow lanes a row; decode-accumulate
            // loads the output of kRBatch passes at a time, so that their loads are in
            // flight together)
            const uint32_t wsub = static_cast<uint32_t>(lane) / kRLanesPerRow;
            const uint32_t wcol = static_cast<uint32_t>(lane) % kRLanesPerRow;
            for (int r0 = 0; r0 < nrows; r0 += kRBatch * static_cast<int>(kRRowsPerPass)) {
                float4 o[kAcc ? kRBatch * kRVec : 1];
                if constexpr (kAcc) {
#pragma unroll
                    for (int t = 0; t < kRBatch; ++t) {
                        const int rr = r0 + t * static_cast<int>(kRRowsPerPass) + static_cast<int>(wsub);
                        const uint64_t bb = g * 32 + rr;
                        const uint32_t mm = rr < nrows ? static_cast<uint32_t>(min(static_cast<uint64_t>(d), a.n - bb * d)) : 0u;
                        const float* gp = a.out + bb * d;
#pragma unroll
                        for (int i = 0; i < kRVec; ++i) {
                            const uint32_t c = lo + 4u * (wcol + kRLanesPerRow * i);
                            float4& x = o[t * kRVec + i];
                            x = make_float4(0.f, 0.f, 0.f, 0.f);
                            if (c + 4 <= mm) {
                                x = __ldcs(reinterpret_cast<const float4*>(gp + c));
                            } else if (c < mm) {
                                x.x = gp[c];
                                if (c + 1 < mm) x.y = gp[c + 1];
                                if (c + 2 < mm) x.z = gp[c + 2];
                            }
                        }
                    }
                }
#pragma unroll
                for (int t = 0; t < kRBatch; ++t) {
                    const int rr = r0 + t * static_cast<int>(kRRowsPerPass) + static_cast<int>(wsub);
                    const float sc = __shfl_sync(kWarpAll, scale, rr & 31);
                    if (rr >= nrows) continue;
                    const uint64_t bb = g * 32 + rr;
                    const uint32_t mm = static_cast<uint32_t>(min(static_cast<uint64_t>(d), a.n - bb * d));
                    uint32_t* const rowp = rows + static_cast<uint32_t>(rr) * stride_w;
                    float* const gp = a.out + bb * d;
#pragma unroll
                    for (int i = 0; i < kRVec; ++i) {
                        const uint32_t c = lo + 4u * (wcol + kRLanesPerRow * i);
                        if (c < mm) {
                            const uint32_t q = (c & (kRRing - 1u)) >> 2;  // four codes
                            const uint2 w = reinterpret_cast<const uint2*>(rowp)[q];
                            reinterpret_cast<uint2*>(rowp)[q] = make_uint2(0u, 0u);
                            uint32_t code[4];
                            code[0] = (w.x & 0x7FFFu) | ((w.x & 0x8000u) << 16);
                            code[1] = (w.x >> 16 & 0x7FFFu) | (w.x & 0x80000000u);
                            code[2] = (w.y & 0x7FFFu) | ((w.y & 0x8000u) << 16);
                            code[3] = (w.y >> 16 & 0x7FFFu) | (w.y & 0x80000000u);
                            float v[4];
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                // code[j] = k | sign << 31: k as fp32 through the 2^23
                                // offset (exact for k < 2^23), times the step, the sign last
                                const float kf = __fsub_rn(__uint_as_float(0x4B000000u | (code[j] & 0x7FFFFFFFu)), 8388608.0f);
                                v[j] = __uint_as_float(__float_as_uint(__fmul_rn(sc, kf)) | (code[j] & 0x80000000u));
                            }
                            if constexpr (kAcc) {
                                const float4& x = o[t * kRVec + i];
                                v[0] = __fadd_rn(x.x, v[0]);
                                v[1] = __fadd_rn(x.y, v[1]);
                                v[2] = __fadd_rn(x.z, v[2]);
                                v[3] = __fadd_rn(x.w, v[3]);
                            }
                            if (c + 4 <= mm) {
                                __stcs(reinterpret_cast<float4*>(gp + c), make_float4(v[0], v[1], v[2], v[3]));
                            } else {
                                for (uint32_t j = 0; j < 4 && c + j < mm; ++j) gp[c + j] = v[j];
                            }
                        }
                    }
                }
            }
            __syncwarp();
        }
        // every record index below m, and the bucket consumed exactly (a record that
        // overran leaves left negative; one past m, or never placed, fails too)
        if (live && !bad && (next > m || r.left != 0 || pend)) bad = true;
        if (bad) atomicOr(a.status, QSGD_ST_BAD_STREAM);
        __syncwarp();
    }
    asm volatile("cp.async.wait_all;\n" ::: "memory");  // no copy outlives the CTA
}

// ---------------------------------------------------------------------------
// Several streams (decode-accumulate and the mean), K <= 16 to a launch.
//
// A warp takes 32 buckets (lane = bucket) and walks their columns in segments of
// kMSeg.  For every segment it holds an fp32 tile of the 32 buckets' columns in
// shared memory (the output + 0, or +0 for the first launch of a mean), decodes
// stream 0's records of the segment and adds each value onto the tile, then stream
// 1's, and so on: every coordinate gets its adds in stream order, the order of
// decode-accumulate, and a stream adds nothing off its support.  The tile is then
// written back (divided by K in the last launch of a mean).  Between segments each
// stream's parse state (reader, next index, the record read past the segment, the
// bucket's scale) waits in shared memory.  Records are read through the omega table,
// once for the gap and once for the level, so gaps and levels up to 63 take two
// lookups; others take the bit-serial path.
// ---------------------------------------------------------------------------
constexpr int kMSeg = 64;          // columns per segment
constexpr int kMTile = kMSeg + 1;  // tile row stride (odd: lanes' rows on different banks)
constexpr uint32_t kNoPend = 0xFFFFFFFFu;

// Parse state of one stream of one bucket, kept in registers while the stream is
// decoded and in shared memory (one array per field, [stream][lane]) in between.
struct MsReader {
    uint64_t wabs;  // absolute index of the next word to fetch
    uint32_t cur, nx, off;
    int32_t left;
    uint32_t next;  // bucket-local index after the last record
    uint32_t pidx;  // a record read past the segment: its index (kNoPend: none) ...
    float pval;     // ... and value
    float scale;
};
struct MsState {  // [field][stream][lane]
    uint32_t v[10][kMaxStreamsPerLaunch][32];
};
__device__ __forceinline__ void ms_save(MsState& S, int j, int lane, const MsReader& r) {
    S.v[0][j][lane] = static_cast<uint32_t>(r.wabs);
    S.v[1][j][lane] = static_cast<uint32_t>(r.wabs >> 32);
    S.v[2][j][lane] = r.cur;
    S.v[3][j][lane] = r.nx;
    S.v[4][j][lane] = r.off;
    S.v[5][j][lane] = static_cast<uint32_t>(r.left);
    S.v[6][j][lane] = r.next;
    S.v[7][j][lane] = r.pidx;
    S.v[8][j][lane] = __float_as_uint(r.pval);
    S.v[9][j][lane] = __float_as_uint(r.scale);
}
__device__ __forceinline__ void ms_load(const MsState& S, int j, int lane, MsReader& r) {
    r.wabs = S.v[0][j][lane] | (static_cast<uint64_t>(S.v[1][j][lane]) << 32);
    r.cur = S.v[2][j][lane];
    r.nx = S.v[3][j][lane];
    r.off = S.v[4][j][lane];
    r.left = static_cast<int32_t>(S.v[5][j][lane]);
    r.next = S.v[6][j][lane];
    r.pidx = S.v[7][j][lane];
    r.pval = __uint_as_float(S.v[8][j][lane]);
    r.scale = __uint_as_float(S.v[9][j][lane]);
}
__device__ __forceinline__ uint32_t ms_fetch(const StreamRef& st, uint64_t& wabs) {
    const uint32_t w = wabs < st.num_words ? __ldg(st.words + wabs) : 0u;
    ++wabs;
    return w;
}
__device__ __forceinline__ void ms_advance(MsReader& r, const StreamRef& st, uint32_t n) {  // n <= 32
    r.off += n;
    r.left -= static_cast<int32_t>(n);
    if (r.off >= 32u) {
        r.cur = r.nx;
        r.nx = ms_fetch(st, r.wabs);
        r.off -= 32u;
    }
}
__device__ __forceinline__ uint32_t ms_peek(const MsReader& r) { return __funnelshift_l(r.nx, r.cur, r.off); }
__device__ __forceinline__ bool ms_omega(MsReader& r, const StreamRef& st, uint32_t& N) {
    uint32_t v = 1;
    for (;;) {
        if (r.left <= 0) return false;
        const uint32_t bit = ms_peek(r) >> 31;
        ms_advance(r, st, 1);
        if (bit == 0) {
            N = v;
            return true;
        }
        if (v > 31 || r.left < static_cast<int32_t>(v)) return false;
        const uint32_t rest = ms_peek(r) >> (32 - v);
        ms_advance(r, st, v);
        v = (1u << v) | rest;
    }
}

__global__ void __launch_bounds__(32 * kRowsMaxWarps) decode_rows_multi(const __grid_constant__ DecodeArgs a) {
    extern __shared__ __align__(16) uint32_t smem[];
    uint16_t* const olut = reinterpret_cast<uint16_t*>(smem);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int W = blockDim.x >> 5;
    char* const wbase = reinterpret_cast<char*>(smem) + kLutSize * sizeof(uint16_t) +
                        static_cast<size_t>(warp) * (sizeof(MsState) + 32 * kMTile * sizeof(float));
    MsState& S = *reinterpret_cast<MsState*>(wbase);
    float* const tile = reinterpret_cast<float*>(wbase + sizeof(MsState));
    float* const myrow = tile + lane * kMTile;
    omega_lut_fill(olut, tid, blockDim.x);
    __syncthreads();
    const float fs = __uint2float_rn(a.s);
    const uint32_t d = a.d;
    const int K = a.K;
    const uint64_t ngroups = (a.nb + 31) / 32;
    for (uint64_t g = blockIdx.x + static_cast<uint64_t>(gridDim.x) * warp; g < ngroups;
         g += static_cast<uint64_t>(gridDim.x) * W) {
        const uint64_t b = g * 32 + lane;
        const bool live = b < a.nb;
        const uint32_t m = live ? static_cast<uint32_t>(min(static_cast<uint64_t>(d), a.n - b * d)) : 0u;
        const int nrows = static_cast<int>(min(static_cast<uint64_t>(32), a.nb - g * 32));
        bool bad = false;
        // --- open this lane's bucket in every stream --------------------------------
        for (int j = 0; j < K; ++j) {
            const StreamRef st = a.streams[j];
            MsReader r{0, 0, 0, 0, 0, 0, kNoPend, 0.f, 0.f};
            if (live) {
                const uint64_t begin = st.offsets[b];
                const uint64_t end = st.offsets[b + 1];
                if (!(end >= begin && end - begin >= 32 && end <= st.num_words * 32 && end - begin < (1ull << 30))) {
                    bad = true;
                } else {
                    r.wabs = begin >> 5;
                    r.cur = ms_fetch(st, r.wabs);
                    r.nx = ms_fetch(st, r.wabs);
                    r.off = static_cast<uint32_t>(begin & 31u);
                    r.left = static_cast<int32_t>(end - begin);
                    const uint32_t nbits = ms_peek(r);
                    ms_advance(r, st, 32);
                    const float norm = __uint_as_float(nbits);
                    if (nbits == 0) {
                        bad = bad || r.left != 0;
                        r.left = 0;
                    } else if (!(isfinite(norm) && norm > 0.f)) {
                        bad = true;
                        r.left = 0;
                    } else {
                        r.scale = __fdiv_rn(norm, fs);
                        if (!(r.scale > 0.f) && r.left != 0) {  // a zero scale carries no records
                            bad = true;
                            r.left = 0;
                        }
                    }
                }
            }
            ms_save(S, j, lane, r);
        }
        for (uint32_t lo = 0; lo < d; lo += kMSeg) {
            const uint32_t hi = lo + kMSeg;
            const uint32_t ncols = min(static_cast<uint32_t>(kMSeg), d - lo);
            // --- the tile: the output + 0 (canonical zeros), or +0 ---------------------
            for (int rr = 0; rr < nrows; ++rr) {
                const uint64_t bb = g * 32 + rr;
                const uint32_t mm = static_cast<uint32_t>(min(static_cast<uint64_t>(d), a.n - bb * d));
                const float* gp = a.out + bb * d + lo;
#pragma unroll
                for (int c0 = 0; c0 < kMSeg; c0 += 32) {
                    const uint32_t c = static_cast<uint32_t>(c0 + lane);
                    float v = 0.f;
                    if (!a.start_zero && c < ncols && lo + c < mm) v = __fadd_rn(gp[c], 0.0f);
                    tile[rr * kMTile + c] = v;
                }
            }
            __syncwarp();
            // --- the streams, in order --------------------------------------------------
            for (int j = 0; j < K; ++j) {
                const StreamRef st = a.streams[j];
                MsReader r;
                ms_load(S, j, lane, r);
                if (r.pidx < hi) {
                    myrow[r.pidx - lo] = __fadd_rn(myrow[r.pidx - lo], r.pval);
                    r.pidx = kNoPend;
                }
                for (uint32_t it = 0; it < kParseGuard; ++it) {
                    const bool act = r.pidx == kNoPend && r.left > 0;
                    if (!__any_sync(kWarpAll, act)) break;
                    if (act) {
                        uint32_t gap = 0, k = 0, sign = 0;
                        bool ok = false;
                        const uint32_t w = ms_peek(r);
                        const uint32_t ge = olut[w >> (32 - kLutBits)];
                        const uint32_t gl = ge & 15u;
                        const uint32_t w2 = w << gl;
                        const uint32_t ke = olut[(w2 << 1) >> (32 - kLutBits)];
                        const uint32_t kl = ke & 15u;
                        if (gl != 0u && kl != 0u && (ke >> 4) <= a.s) {
                            gap = ge >> 4;
                            k = ke >> 4;
                            sign = w2 >> 31;
                            ms_advance(r, st, gl + 1u + kl);
                            ok = r.left >= 0;
                        } else if (ms_omega(r, st, gap) && r.left > 0 && gap <= 0xFFFFu) {
                            sign = ms_peek(r) >> 31;
                            ms_advance(r, st, 1);
                            ok = ms_omega(r, st, k) && k <= a.s;
                        }
                        const uint32_t idx = r.next + gap - 1u;
                        if (!ok || idx >= m) {
                            bad = true;
                            r.left = 0;
                        } else {
                            r.next = idx + 1u;
                            const float q = __fmul_rn(r.scale, __uint2float_rn(k));
                            const float val = sign ? -q : q;
                            if (idx < hi) {
                                myrow[idx - lo] = __fadd_rn(myrow[idx - lo], val);
                            } else {
                                r.pidx = idx;
                                r.pval = val;
                            }
                        }
                    }
                }
                ms_save(S, j, lane, r);
            }
            __syncwarp();
            // --- the tile back to the output --------------------------------------------
            const bool last = a.div != 0.f;
            for (int rr = 0; rr < nrows; ++rr) {
                const uint64_t bb = g * 32 + rr;
                const uint32_t mm = static_cast<uint32_t>(min(static_cast<uint64_t>(d), a.n - bb * d));
                float* gp = a.out + bb * d + lo;
#pragma unroll
                for (int c0 = 0; c0 < kMSeg; c0 += 32) {
                    const uint32_t c = static_cast<uint32_t>(c0 + lane);
                    if (c < ncols && lo + c < mm) {
                        const float v = tile[rr * kMTile + c];
                        gp[c] = last ? __fdiv_rn(v, a.div) : v;
                    }
                }
            }
            __syncwarp();
        }
        // every stream's bucket consumed exactly, every index below m
        for (int j = 0; j < K && live && !bad; ++j) {
            MsReader r;
            ms_load(S, j, lane, r);
            if (r.left != 0 || r.next > m || r.pidx != kNoPend) bad = true;
        }
        if (bad) atomicOr(a.status, QSGD_ST_BAD_STREAM);
        __syncwarp();
    }
}

// ---------------------------------------------------------------------------
// Several streams side by side, byte codes (decode-accumulate with K >= 2 and the
// mean of K >= 1 streams, s <= 127).
//
// The kSideWarps warps of a CTA take W = min(K, kSideWarps) streams at a time (a
// chunk) and G = kSideWarps / W groups of 32 buckets: warp w parses stream
// c0 + (w mod W) of group w div W, a bucket a lane, into a ring of byte codes
// (sign << 7 | k) of two kSSeg-column segments a row, with the whole-record table (up
// to two records a lookup, two lookups a step).  Once every lane of every warp has
// passed a segment, the CTA adds the chunk's values there onto the output, each
// coordinate in stream order: v = out + 0 (+0 for the first chunk of a mean), then
// v = v + q_j for every stream j of the chunk, v / div in the last chunk of a mean.
// The first add makes a -0.0 output +0.0 as the first stream's add would; after it
// adding a zero code's +0 leaves v as it is, as the sum in stream order does.  The
// add clears the codes it reads for the ring's next turn; the output is read and
// written once per chunk.  A step of table records moves at most 60 columns, so the
// records of a lane still short of the segment's end land in the ring; a longer
// record further ahead waits in registers until its segment.  Segments of 64 columns keep a CTA at 51 KB of
// shared memory; three CTAs an SM (76 registers a thread) measured faster than four
// (64 registers, with spills) or two (segments of 128 columns).
// ---------------------------------------------------------------------------
#ifndef QSGD_SIDE_SEG
#define QSGD_SIDE_SEG 64
#endif
constexpr int kSideWarps = 8;
constexpr uint32_t kSSeg = QSGD_SIDE_SEG;         // columns a segment
constexpr uint32_t kSRing = 2 * kSSeg;            // codes (bytes) a ring row
constexpr uint32_t kSStride = kSRing / 4 + 1;     // words a ring row: 1 mod 32, rows on different banks
constexpr uint32_t kSSegWords = kSSeg / 4;        // words of a row's segment
constexpr uint32_t kSRowsPerWarp = 32 / kSSegWords;  // rows a warp's 32 threads add at once
// (a step of table records moves at most 60 columns)
static_assert(kSSeg == 64 || kSSeg == 128, "a segment holds a step of records and a warp whole rows");
static_assert((32 * kSSegWords) % (2 * 32 * kSideWarps) == 0, "a group's items come in pairs a thread");

// The value of one byte code (sign << 7 | k) of a bucket with step sc: fl(sc * k),
// the sign last.
__device__ __forceinline__ float side_value(uint32_t code, float sc) {
    const float kf = __fsub_rn(__uint_as_float(0x4B000000u | (code & 0x7Fu)), 8388608.0f);
    return __uint_as_float(__float_as_uint(__fmul_rn(sc, kf)) | ((code & 0x80u) << 24));
}

#ifndef QSGD_SIDE_MINB
#define QSGD_SIDE_MINB 3
#endif
__global__ void __launch_bounds__(32 * kSideWarps, QSGD_SIDE_MINB) decode_rows_side(const __grid_constant__ DecodeArgs a) {
    extern __shared__ __align__(16) uint32_t smem[];
    constexpr int kThreads = 32 * kSideWarps;
    uint32_t* const lut = smem;
    uint8_t* const klut = reinterpret_cast<uint8_t*>(smem + kLutSize);
    uint8_t* const plut = reinterpret_cast<uint8_t*>(smem + kLutSize + kKLutWords);
    float* const s_scale = reinterpret_cast<float*>(smem + kLutSize + kSmallLutWords);  // [warp][lane]
    uint32_t* const rings = smem + kLutSize + kSmallLutWords + kThreads;                // [warp][row][kSStride]
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint8_t* const myrow = reinterpret_cast<uint8_t*>(rings + static_cast<uint32_t>(tid) * kSStride);
    rows_lut_fill(lut, a.s, tid, kThreads);
    k_lut_fill(klut, tid, kThreads);
    p_lut_fill(plut, tid, kThreads);
    for (uint32_t q = static_cast<uint32_t>(tid); q < kThreads * kSStride; q += kThreads) rings[q] = 0u;
    __syncthreads();
    const float fs = __uint2float_rn(a.s);
    const uint32_t d = a.d;
    const uint64_t ngroups = (a.nb + 31) / 32;
    const int W = min(a.K, kSideWarps);  // streams to a chunk
    const int G = kSideWarps / W;        // groups a CTA takes at once
    const int gi = warp / W;             // this warp's group of the G (G when idle)
    const int wj = warp - gi * W;        // this warp's stream within a chunk
    for (uint64_t g0 = static_cast<uint64_t>(blockIdx.x) * G; g0 < ngroups; g0 += static_cast<uint64_t>(gridDim.x) * G) {
        const uint64_t g = g0 + gi;
        const uint64_t b = g * 32 + lane;
        const bool live = gi < G && b < a.nb;
        const uint32_t m = live ? static_cast<uint32_t>(min(static_cast<uint64_t>(d), a.n - b * d)) : 0u;
        for (int c0 = 0; c0 < a.K; c0 += W) {
            const int nt = min(W, a.K - c0);                     // streams in this chunk
            const bool mine = gi < G && g < ngroups && wj < nt;  // uniform in the warp
            const bool from_zero = a.start_zero && c0 == 0;
            const bool divide = c0 + nt == a.K && a.div != 0.f;
            if (c0 == 0 && !from_zero) {  // bring the groups' output into L2 while the records are parsed
                const uint64_t i0 = g0 * 32 * d, i1 = min(a.n, (g0 + G) * 32 * d);
                const char* const gpb = reinterpret_cast<const char*>(a.out + i0);
                for (uint64_t off = static_cast<uint64_t>(tid) * 128; off < 4 * (i1 - i0); off += kThreads * 128)
                    asm volatile("prefetch.global.L2 [%0];" ::"l"(gpb + off));
            }
            // --- open this lane's bucket of stream c0 + wj: header checks, the norm ----
            bool bad = false;
            RowReader r;
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
                    const uint32_t nbits = r.peek();
                    r.advance(32);
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
            if (bad) r.left = 0;
            s_scale[tid] = scale;
            uint32_t next = 0;  // bucket-local index after the last record
            bool pend = false;  // a bit-serial record beyond the ring, held here
            uint32_t pidx = 0, pcode = 0;
            uint32_t it = 0;  // parse steps over the whole bucket (an explicit bound)
            // a table step's record into the ring (it lies less than 64 columns past the
            // segment's end)
            const auto put = [&](uint32_t idx, uint32_t code) { myrow[idx & (kSRing - 1u)] = static_cast<uint8_t>(code); };
            for (uint32_t lo = 0; lo < d; lo += kSSeg) {
                const uint32_t hi = lo + kSSeg;
                if (mine) {
                    if (pend && pidx < hi + kSSeg) {
                        put(pidx, pcode);
                        pend = false;
                    }
                    // --- parse until every lane has passed column hi (or ended) -------
                    for (;; ++it) {
                        const bool act = r.left > 0 && !pend && next < hi;
                        if (!__any_sync(kWarpAll, act)) break;
                        if (it >= kParseGuard) {  // never reached by a well-formed stream
                            if (act) {
                                bad = true;
                                r.left = 0;
                            }
                            continue;
                        }
                        if (!act || rows_table_step(r, lut, klut, a.s, next, put)) continue;
                        // a longer record; held here when it lies past the ring (the lane
                        // then waits for its segment)
                        uint32_t gap = 0, sign = 0, k = 0;
                        if (far_record(r, plut, klut, a.s, d, gap, sign, k)) {
                            next += gap;
                            const uint32_t idx = min(next - 1u, d);
                            if (idx >= hi + kSSeg) {
                                pend = true;
                                pidx = idx;
                                pcode = row_code<uint8_t>(sign, k);
                            } else {
                                put(idx, row_code<uint8_t>(sign, k));
                            }
                        } else {
                            bad = true;
                            r.left = 0;
                        }
                    }
                }
                __syncthreads();  // every warp's codes of [lo, hi) are in its ring, the scales too
                // --- the chunk's values of [lo, hi) onto the output, in stream order ---
                const uint32_t slot0 = (lo & (kSRing - 1u)) >> 2;  // the segment's first word in a ring row
                // two items (four coordinates of a row) a thread at a time, both outputs
                // loaded before either is added; a warp's threads take rows i and
                // i + 32 / kSRowsPerWarp, whose ring words lie on different banks
                for (uint32_t q0 = static_cast<uint32_t>(tid); q0 < static_cast<uint32_t>(G) * 32u * kSSegWords;
                     q0 += 2u * kThreads) {
                    uint32_t c[2], mm[2], row0[2], sc0[2];
                    float* gp[2];
                    float v[2][4];
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const uint32_t q = q0 + static_cast<uint32_t>(u) * kThreads;
                        const uint32_t qg = q / (32u * kSSegWords);
                        const uint32_t qi = q % (32u * kSSegWords);
                        const uint32_t cw = qi % kSSegWords;
                        const uint32_t rr = qi / 32u + (qi % 32u) / kSSegWords * (32u / kSRowsPerWarp);
                        const uint64_t bb = (g0 + qg) * 32 + rr;
                        c[u] = lo + 4u * cw;
                        mm[u] = bb < a.nb ? static_cast<uint32_t>(min(static_cast<uint64_t>(d), a.n - bb * d)) : 0u;
                        gp[u] = a.out + bb * d + c[u];
                        row0[u] = (qg * static_cast<uint32_t>(W) * 32u + rr) * kSStride + slot0 + cw;
                        sc0[u] = qg * static_cast<uint32_t>(W) * 32u + rr;
#pragma unroll
                        for (int e = 0; e < 4; ++e) v[u][e] = 0.f;
                        if (c[u] < mm[u] && !from_zero) {
                            if (c[u] + 4 <= mm[u]) {
                                const float4 o = *reinterpret_cast<const float4*>(gp[u]);
                                v[u][0] = o.x;
                                v[u][1] = o.y;
                                v[u][2] = o.z;
                                v[u][3] = o.w;
                            } else {  // c < mm <= c + 3
                                v[u][0] = gp[u][0];
                                if (c[u] + 1 < mm[u]) v[u][1] = gp[u][1];
                                if (c[u] + 2 < mm[u]) v[u][2] = gp[u][2];
                            }
                        }
                    }
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
#pragma unroll
                        for (int e = 0; e < 4; ++e) v[u][e] = __fadd_rn(v[u][e], 0.f);  // -0.0 -> +0.0, as a first add of +0
                        for (int t = 0; t < nt; ++t) {
                            uint32_t* const p = rings + row0[u] + static_cast<uint32_t>(t) * 32u * kSStride;
                            const uint32_t w = *p;
                            *p = 0u;
                            const float sc = s_scale[sc0[u] + static_cast<uint32_t>(t) * 32u];
#pragma unroll
                            for (int e = 0; e < 4; ++e) v[u][e] = __fadd_rn(v[u][e], side_value(w >> (8 * e), sc));
                        }
                        if (c[u] >= mm[u]) continue;
                        if (divide) {
#pragma unroll
                            for (int e = 0; e < 4; ++e) v[u][e] = __fdiv_rn(v[u][e], a.div);
                        }
                        if (c[u] + 4 <= mm[u]) {
                            *reinterpret_cast<float4*>(gp[u]) = make_float4(v[u][0], v[u][1], v[u][2], v[u][3]);
                        } else {
                            gp[u][0] = v[u][0];
                            if (c[u] + 1 < mm[u]) gp[u][1] = v[u][1];
                            if (c[u] + 2 < mm[u]) gp[u][2] = v[u][2];
                        }
                    }
                }
                __syncthreads();  // the ring's words of [lo, hi) are clear again
            }
            // every record index below m, the bucket consumed exactly, nothing held back
            if (mine && live && !bad && (next > m || r.left != 0 || pend)) bad = true;
            if (mine && bad) atomicOr(a.status, QSGD_ST_BAD_STREAM);
            // a malformed bucket may have left codes past its segments: clear the ring
            if (__syncthreads_or(mine && bad)) {
                for (uint32_t q = static_cast<uint32_t>(tid); q < kThreads * kSStride; q += kThreads) rings[q] = 0u;
                __syncthreads();
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Large buckets (d > 1024).  The outputs of such gradients are mostly zeros (a 60 M
// coordinate gradient in buckets of 8192 at s = 1: 0.107 bits a coordinate), so
// writing the output carries the traffic and the records are few.  The output is first written whole with 16-byte stores where it is
// aligned: zeros (decode), or the output + 0 (decode-accumulate; +0 turns -0.0 into
// +0.0 as the add of a zero term does).  Then one lane a bucket parses the bucket of
// every stream in order and stores each record's value (decode) or adds it
// (accumulate) at its coordinate.
//   - decode: sparse_fill over the whole output (every SM, no barrier), then
//     sparse_records, a lane a bucket;
//   - decode-accumulate: decode_sparse_acc, a CTA a group of kSparseGroup buckets, its
//     threads adding +0 to the group's output and, after a CTA barrier, lane L of
//     warp 0 parsing bucket L of the group, whose output the CTA has just brought
//     into L2.
// ---------------------------------------------------------------------------

// The records of bucket b of every stream onto its output row (the row written
// before): a record's value is stored, or added with kAcc.  Returns false when a
// stream's bucket is malformed.
template <bool kAcc>
__device__ __forceinline__ bool sparse_bucket(const DecodeArgs& a, const uint32_t* lut, const uint8_t* plut,
                                              const uint8_t* klut, uint64_t b) {
    const float fs = __uint2float_rn(a.s);
    const uint32_t m = static_cast<uint32_t>(min(static_cast<uint64_t>(a.d), a.n - b * a.d));
    float* const row = a.out + b * a.d;
    bool bad = false;
    for (int j = 0; j < a.K; ++j) {
        const StreamRef st = a.streams[j];
        const uint64_t begin = st.offsets[b];
        const uint64_t end = st.offsets[b + 1];
        if (!(end >= begin && end - begin >= 32 && end <= st.num_words * 32 && end - begin < (1ull << 31))) {
            bad = true;
            continue;
        }
        RowReaderT<true> r;
        r.init(st.words, st.num_words, begin, static_cast<uint32_t>(end - begin));
        const uint32_t nbits = r.peek();
        r.advance(32);
        const float norm = __uint_as_float(nbits);
        float scale = 0.f;
        if (nbits == 0) {
            bad = bad || r.left != 0;
            continue;
        } else if (!(isfinite(norm) && norm > 0.f)) {
            bad = true;
            continue;
        }
        scale = __fdiv_rn(norm, fs);
        if (!(scale > 0.f) && r.left != 0) {  // a zero scale carries no records
            bad = true;
            continue;
        }
        uint32_t next = 0;
        // the records: up to two table entries a step, each up to two records
        // (a second record or entry only when it ends inside the bucket)
        bool ok = true;
        auto put = [&](uint32_t gap, uint32_t sign, uint32_t k) {
            next += gap;
            if (next > m) {
                ok = false;
                return;
            }
            const float q = __fmul_rn(scale, __uint2float_rn(k));
            const float v = sign ? -q : q;
            row[next - 1] = kAcc ? __fadd_rn(row[next - 1], v) : v;
        };
        for (uint32_t it = 0; r.left > 0 && ok; ++it) {
            if (it >= kParseGuard) {
                ok = false;
                break;
            }
            const uint32_t w = r.peek();
            const uint32_t e = lut[w >> (32 - kLutBits)];
            const uint32_t len1 = e & 15u;
            if (len1 == 0u) {  // a record longer than the window
                // (such buckets are sparse: the gap's code is mostly past the window)
                uint32_t gap = 0, code = 0, sign = 0, k = 0;
                uint32_t len = far_long_record(w, plut, klut, gap, code);
                if (len == 0u) len = near_long_record(w, e, klut, gap, code);
                if (len != 0u && (code & 0x7Fu) <= a.s) {
                    r.advance(len);
                    sign = code >> 7;
                    k = code & 0x7Fu;
                } else if (!slow_record(r, a.s, a.d, gap, sign, k)) {
                    ok = false;
                    break;
                }
                put(gap, sign, k);
                continue;
            }
            const uint32_t len2 = (e >> 4) & 15u;
            const bool two = static_cast<int32_t>(len2) <= r.left;
            uint32_t used = two ? len2 : len1;
            put((e >> 8) & 15u, (e >> 23) & 1u, (e >> 16) & 0x7Fu);  // table codes: sign << 7 | k
            const uint32_t c2 = e >> 24;
            if (ok && two && c2 != 0u) put((e >> 12) & 15u, c2 >> 7, c2 & 0x7Fu);
            if (ok && two) {
                const uint32_t f = lut[(w << used) >> (32 - kLutBits)];
                const uint32_t flen1 = f & 15u;
                if (flen1 != 0u && static_cast<int32_t>(used + flen1) <= r.left) {
                    const uint32_t flen2 = (f >> 4) & 15u;
                    const bool ftwo = static_cast<int32_t>(used + flen2) <= r.left;
                    put((f >> 8) & 15u, (f >> 23) & 1u, (f >> 16) & 0x7Fu);
                    const uint32_t fc2 = f >> 24;
                    if (ok && ftwo && fc2 != 0u) put((f >> 12) & 15u, fc2 >> 7, fc2 & 0x7Fu);
                    used += ftwo ? flen2 : flen1;
                }
            }
            r.advance(used);
        }
        if (!ok) bad = true;
        if (r.left != 0) bad = true;
    }
    return !bad;
}

// Writes out[c0, c1) (out 16-byte aligned): zeros, or out + 0 with kAcc; thread t of
// nthreads takes every nthreads-th float4 of the aligned body.
template <bool kAcc>
__device__ __forceinline__ void sparse_fill_range(float* out, uint64_t c0, uint64_t c1, uint64_t t, uint64_t nthreads) {
    const uint64_t head = min(c1, (c0 + 3) & ~uint64_t(3));  // aligned start of the body
    const uint64_t tail = max(head, c1 & ~uint64_t(3));
    for (uint64_t i = c0 + t; i < head; i += nthreads) out[i] = kAcc ? __fadd_rn(out[i], 0.0f) : 0.0f;
    for (uint64_t i = tail + t; i < c1; i += nthreads) out[i] = kAcc ? __fadd_rn(out[i], 0.0f) : 0.0f;
    for (uint64_t i = head + 4 * t; i < tail; i += 4 * nthreads) {
        float4* p4 = reinterpret_cast<float4*>(out + i);
        if constexpr (kAcc) {
            float4 v = *p4;
            v.x = __fadd_rn(v.x, 0.0f);
            v.y = __fadd_rn(v.y, 0.0f);
            v.z = __fadd_rn(v.z, 0.0f);
            v.w = __fadd_rn(v.w, 0.0f);
            *p4 = v;
        } else {
            __stcs(p4, make_float4(0.f, 0.f, 0.f, 0.f));
        }
    }
}

// The decode's fill: zeros over the whole output.
__global__ void __launch_bounds__(kSparseBlock) sparse_fill(float* out, uint64_t n) {
    sparse_fill_range<false>(out, 0, n, static_cast<uint64_t>(blockIdx.x) * kSparseBlock + threadIdx.x,
                             static_cast<uint64_t>(gridDim.x) * kSparseBlock);
}

// The decode's records: lanes 0 .. kSparseRecLanes - 1 of every warp take a bucket
// each (fewer chains a warp, so less of the warp's time goes to paths that only
// some of its lanes take, and more warps an SM to hide each chain's latency).
__global__ void __launch_bounds__(kSparseRecBlock) sparse_records(const __grid_constant__ DecodeArgs a) {
    __shared__ __align__(16) uint32_t lut[kLutSize];
    __shared__ __align__(16) uint8_t plut[1 << kPLutBits];
    __shared__ __align__(16) uint8_t klut[1 << kKLutBits];
    rows_lut_fill(lut, a.s, threadIdx.x, kSparseRecBlock);
    p_lut_fill(plut, threadIdx.x, kSparseRecBlock);
    k_lut_fill(klut, threadIdx.x, kSparseRecBlock);
    __syncthreads();
    const uint32_t lane = threadIdx.x & 31u;
    const uint64_t b = static_cast<uint64_t>(blockIdx.x) * kSparseRecBuckets + (threadIdx.x >> 5) * kSparseRecLanes + lane;
    if (lane < kSparseRecLanes && b < a.nb && !sparse_bucket<false>(a, lut, plut, klut, b))
        atomicOr(a.status, QSGD_ST_BAD_STREAM);
}

// Decode-accumulate: a CTA a group of kSparseGroup buckets, the fill by all its
// threads, then the records by lanes 0 .. kSparseGroup - 1 of warp 0.
__global__ void __launch_bounds__(kSparseBlock) decode_sparse_acc(const __grid_constant__ DecodeArgs a) {
    __shared__ __align__(16) uint32_t lut[kLutSize];
    __shared__ __align__(16) uint8_t plut[1 << kPLutBits];
    __shared__ __align__(16) uint8_t klut[1 << kKLutBits];
    const int tid = threadIdx.x;
    rows_lut_fill(lut, a.s, tid, kSparseBlock);
    p_lut_fill(plut, tid, kSparseBlock);
    k_lut_fill(klut, tid, kSparseBlock);
    __syncthreads();
    const uint64_t d = a.d;
    const uint64_t ngroups = (a.nb + kSparseGroup - 1) / kSparseGroup;
    for (uint64_t g = blockIdx.x; g < ngroups; g += gridDim.x) {
        sparse_fill_range<true>(a.out, g * kSparseGroup * d, min(a.n, (g + 1) * kSparseGroup * d),
                                static_cast<uint64_t>(tid), kSparseBlock);
        __syncthreads();
        const uint64_t b = g * kSparseGroup + static_cast<uint64_t>(tid);
        if (tid < kSparseGroup && b < a.nb && !sparse_bucket<true>(a, lut, plut, klut, b))
            atomicOr(a.status, QSGD_ST_BAD_STREAM);
        __syncthreads();
    }
}

// Words of one row of byte codes: d codes and a padding code (where an index past the
// bucket is parked), rounded to 1 mod 32 so that consecutive rows start on different
// banks.
uint32_t rows_stride_words(uint32_t d) {
    const uint32_t need = (d + 1 + 3) / 4;
    return ((need + 30) / 32) * 32 + 1;
}
// Words of one row of the ring of 16-bit codes: kRRing codes, even (the write-back
// reads 8 bytes a lane) and 2 mod 32.
constexpr uint32_t ring_stride_words() { return kRRing * 2 / 4 + 2; }

// One CTA per SM, its warps one group each where the groups allow: every SM busy.
template <class Kernel>
cudaError_t launch_row_kernel(Kernel kernel, bool& attr_done, const DecodeArgs& a, uint32_t stride, cudaStream_t stream,
                              size_t extra_per_warp = 0) {
    int dev = 0, sms = 0, optin = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    const size_t per_warp = static_cast<size_t>(32) * stride * sizeof(uint32_t) + extra_per_warp;
    // the record table and the small tables (the ring kernel uses the first half of
    // the record table's room for its omega table, and the small tables' not at all)
    const size_t lut_bytes = static_cast<size_t>(kLutSize + kSmallLutWords) * sizeof(uint32_t);
    const int W_fit = static_cast<int>(std::min<size_t>(kRowsMaxWarps, (static_cast<size_t>(optin) - lut_bytes - 1024) / per_warp));
    if (W_fit < 1) return cudaErrorInvalidConfiguration;
    const uint64_t groups = (a.nb + 31) / 32;
    const int W = static_cast<int>(std::max<uint64_t>(1, std::min<uint64_t>(W_fit, (groups + sms - 1) / sms)));
    const size_t smem = lut_bytes + W * per_warp;
    if (!attr_done) {
        cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
        attr_done = true;
    }
    const uint64_t blocks = std::max<uint64_t>(1, std::min<uint64_t>(static_cast<uint64_t>(sms), (groups + W - 1) / W));
    kernel<<<static_cast<unsigned>(blocks), 32 * W, smem, stream>>>(a, stride);
    return cudaGetLastError();
}

template <int V, bool kAcc>
cudaError_t launch_rows_v(const DecodeArgs& a, cudaStream_t stream) {
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    bool scratch = false;
    return launch_row_kernel(decode_rows<V, kAcc>, dev < 64 ? attr_set[dev] : scratch, a, rows_stride_words(a.d), stream);
}

template <bool kAcc>
cudaError_t launch_rows_ring(const DecodeArgs& a, cudaStream_t stream) {
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    bool scratch = false;
    return launch_row_kernel(decode_rows_ring<kAcc>, dev < 64 ? attr_set[dev] : scratch, a, ring_stride_words(), stream,
                             32 * 8 * sizeof(uint32_t));
}

template <bool kAcc>
cudaError_t launch_rows_bytes(const DecodeArgs& a, cudaStream_t stream) {
    switch (fast_v(a.d)) {
        case 1: return launch_rows_v<1, kAcc>(a, stream);
        case 2: return launch_rows_v<2, kAcc>(a, stream);
        case 4: return launch_rows_v<4, kAcc>(a, stream);
        default: return launch_rows_v<8, kAcc>(a, stream);
    }
}

cudaError_t launch_rows_multi(const DecodeArgs& a, cudaStream_t stream) {
    int dev = 0, sms = 0, optin = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    const size_t per_warp = sizeof(MsState) + 32 * kMTile * sizeof(float);
    const size_t luts = kLutSize * sizeof(uint16_t);
    const int W_fit = static_cast<int>(std::min<size_t>(kRowsMaxWarps, (static_cast<size_t>(optin) - luts - 1024) / per_warp));
    if (W_fit < 1) return cudaErrorInvalidConfiguration;
    const uint64_t groups = (a.nb + 31) / 32;
    const int W = static_cast<int>(std::max<uint64_t>(1, std::min<uint64_t>(W_fit, (groups + sms - 1) / sms)));
    const size_t smem = luts + W * per_warp;
    static bool attr_set[64] = {};
    if (dev < 64 && !attr_set[dev]) {
        cudaFuncSetAttribute(decode_rows_multi, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
        attr_set[dev] = true;
    }
    const uint64_t blocks = std::max<uint64_t>(1, std::min<uint64_t>(static_cast<uint64_t>(sms), (groups + W - 1) / W));
    decode_rows_multi<<<static_cast<unsigned>(blocks), 32 * W, smem, stream>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_rows_side(const DecodeArgs& a, cudaStream_t stream) {
    constexpr int kThreads = 32 * kSideWarps;
    const size_t smem =
        (static_cast<size_t>(kLutSize) + kSmallLutWords + kThreads + static_cast<size_t>(kThreads) * kSStride) * sizeof(uint32_t);
    static bool attr_set[64] = {};
    int dev = 0, sms = 0, per_sm = 0;
    cudaGetDevice(&dev);
    if (dev >= 64 || !attr_set[dev]) {
        cudaFuncSetAttribute(decode_rows_side, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        if (dev < 64) attr_set[dev] = true;
    }
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_rows_side, kThreads, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const uint64_t G = static_cast<uint64_t>(kSideWarps / std::min(a.K, kSideWarps));  // groups a CTA takes at once
    const uint64_t sets = ((a.nb + 31) / 32 + G - 1) / G;
    const uint64_t blocks = std::max<uint64_t>(1, std::min<uint64_t>(sets, static_cast<uint64_t>(sms) * per_sm));
    decode_rows_side<<<static_cast<unsigned>(blocks), kThreads, smem, stream>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_sparse(const DecodeArgs& a, bool accumulate, cudaStream_t stream) {
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (!accumulate) {  // the fill over every SM, then a lane a bucket
        const uint64_t fill_threads = (a.n + 3) / 4;
        const uint64_t fill_blocks = std::max<uint64_t>(
            1, std::min<uint64_t>((fill_threads + kSparseBlock - 1) / kSparseBlock, static_cast<uint64_t>(sms) * 8));
        sparse_fill<<<static_cast<unsigned>(fill_blocks), kSparseBlock, 0, stream>>>(a.out, a.n);
        const uint64_t rec_blocks = (a.nb + kSparseRecBuckets - 1) / kSparseRecBuckets;
        sparse_records<<<static_cast<unsigned>(rec_blocks), kSparseRecBlock, 0, stream>>>(a);
        return cudaGetLastError();
    }
    const uint64_t groups = (a.nb + kSparseGroup - 1) / kSparseGroup;
    const uint64_t blocks = std::max<uint64_t>(1, std::min<uint64_t>(groups, static_cast<uint64_t>(sms) * 8));
    decode_sparse_acc<<<static_cast<unsigned>(blocks), kSparseBlock, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace

bool decode_sparse_shape(uint32_t d, const float* out) {
    return d > kRowsMaxD && (reinterpret_cast<uintptr_t>(out) & 15u) == 0;
}

cudaError_t launch_decode_sparse(const DecodeArgs& a, bool accumulate, cudaStream_t stream) {
    return launch_sparse(a, accumulate, stream);
}

bool decode_rows_shape(uint32_t d, uint32_t s, const float* out) {
    return d % 4 == 0 && d >= 4 && d <= kRowsMaxD && s <= kRowsMaxS && (reinterpret_cast<uintptr_t>(out) & 15u) == 0;
}

cudaError_t launch_decode_rows_multi(const DecodeArgs& a, cudaStream_t stream) { return launch_rows_multi(a, stream); }

cudaError_t launch_decode_rows_side(const DecodeArgs& a, cudaStream_t stream) { return launch_rows_side(a, stream); }

cudaError_t launch_decode_rows(const DecodeArgs& a, bool accumulate, cudaStream_t stream) {
    if (a.s <= kRowsMaxS8) return accumulate ? launch_rows_bytes<true>(a, stream) : launch_rows_bytes<false>(a, stream);
    return accumulate ? launch_rows_ring<true>(a, stream) : launch_rows_ring<false>(a, stream);
}

}  // namespace qsgd
