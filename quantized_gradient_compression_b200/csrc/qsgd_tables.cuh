// Decoding tables of the record decoders, computed at compile time and copied into
// shared memory by every CTA that uses them (sm_100a).  Included by the decoders'
// sources; everything here has internal linkage.
//
// Method: "QSGD (Quantized Stochastic Gradient Descent) with Elias Coding" (AIMech
// curated entry): each record of a bucket is omega(gap) | sign | omega(k), MSB-first
// (definition paragraph: Elias recursive codes of the run-length gaps and levels).
#pragma once

#include <cstdint>

namespace qsgd {
namespace {

constexpr int kLutBits = 12;
constexpr int kLutSize = 1 << kLutBits;

// Decoding tables, computed at compile time and copied into shared memory by every
// CTA.  Both read windows MSB-first; a window is the next 12 bits of the stream.

// One omega code from the top of an n-bit window w, starting at bit pos (MSB = 0).
constexpr bool window_omega(uint32_t w, int nbits, int& pos, uint32_t& value) {
    uint32_t v = 1;
    for (;;) {
        if (pos >= nbits) return false;
        const uint32_t bit = (w >> (nbits - 1 - pos)) & 1u;
        ++pos;
        if (bit == 0) {
            value = v;
            return true;
        }
        if (pos + static_cast<int>(v) > nbits) return false;
        const uint32_t rest = (w >> (nbits - pos - v)) & ((1u << v) - 1u);
        pos += v;
        v = (1u << v) | rest;
    }
}

// One whole record (omega(gap) | sign | omega(k)) at bit pos of a 12-bit window: its
// gap, code sign << 7 | k and the bit after it.  Within 12 bits, gap <= 15 and k <= 15.
constexpr bool window_record(uint32_t w, int& pos, uint32_t& gap, uint32_t& code) {
    uint32_t k = 0;
    if (!window_omega(w, kLutBits, pos, gap) || pos >= kLutBits) return false;
    const uint32_t sign = (w >> (kLutBits - 1 - pos)) & 1u;
    ++pos;
    if (!window_omega(w, kLutBits, pos, k)) return false;
    code = (sign << 7) | k;
    return true;
}

// The whole records at the start of a 12-bit window, up to two: [3:0] length of the
// first, [7:4] length of both (the first's when there is no second), [11:8] first
// gap, [15:12] second gap, [23:16] first code, [31:24] second code (0: none; a code
// is never 0, since k >= 1).  A window that holds no whole record has [3:0] = 0 and,
// when the gap's omega code fits the window, [7:4] its length and [13:8] the gap
// (<= 63, as every omega code of at most 12 bits): near_long_record reads the sign
// and the level after it.  For s >= 15 the table is the same for every s; a smaller s
// drops the records with k > s when the table is copied (rows_lut_fill).
struct alignas(16) RowsLut {  // read with 16-byte loads
    uint32_t v[kLutSize];
};
constexpr RowsLut make_rows_lut() {
    RowsLut t{};
    for (uint32_t w = 0; w < static_cast<uint32_t>(kLutSize); ++w) {
        int pos = 0;
        uint32_t g1 = 0, c1 = 0, e = 0;
        if (window_record(w, pos, g1, c1)) {
            const int len1 = pos;
            uint32_t g2 = 0, c2 = 0;
            int len2 = len1;
            if (!window_record(w, len2, g2, c2)) {
                g2 = 0;
                c2 = 0;
                len2 = len1;
            }
            e = static_cast<uint32_t>(len1) | (static_cast<uint32_t>(len2) << 4) | (g1 << 8) | (g2 << 12) |
                (c1 << 16) | (c2 << 24);
        } else {
            int gpos = 0;
            uint32_t gap = 0;
            if (window_omega(w, kLutBits, gpos, gap)) e = (static_cast<uint32_t>(gpos) << 4) | (gap << 8);
        }
        t.v[w] = e;
    }
    return t;
}
__device__ const RowsLut kRowsLutGlobal = make_rows_lut();

// The omega code of a level at the top of a 7-bit window: [3:0] length (0: longer
// than 7 bits), [7:4] value (<= 15, as every code of at most 7 bits).
constexpr int kKLutBits = 7;
constexpr int kKLutWords = (1 << kKLutBits) / 4;  // its size in shared memory, in words
struct alignas(16) KLut {  // read with 16-byte loads
    uint8_t v[1 << kKLutBits];
};
constexpr KLut make_k_lut() {
    KLut t{};
    for (uint32_t w = 0; w < (1u << kKLutBits); ++w) {
        int pos = 0;
        uint32_t val = 0;
        t.v[w] = window_omega(w, kKLutBits, pos, val) ? static_cast<uint8_t>(static_cast<uint32_t>(pos) | (val << 4)) : 0;
    }
    return t;
}
__device__ const KLut kKLutGlobal = make_k_lut();
__device__ __forceinline__ void k_lut_fill(uint8_t* klut, int tid, int nthreads) {
    const uint4* src = reinterpret_cast<const uint4*>(kKLutGlobal.v);
    for (int i = tid; i < (1 << kKLutBits) / 16; i += nthreads) reinterpret_cast<uint4*>(klut)[i] = src[i];
}

// The start of an omega code (a gap) at the top of a 7-bit window, read group by
// group (v = 1; a 1 bit starts a group of v + 1 bits that becomes v; a 0 bit ends
// the code with value v):
//   [7] = 0: the code ends inside the window: [6:3] value, [2:0] length - 1;
//   [7] = 1: a group of v + 1 <= 16 bits starts at bit p of the window (every group
//            before it inside): [6:3] v, [2:0] p.  After that group, a 0 bit ends the
//            code (values below 2^16); a 1 bit would start another group;
//   0xFF:    neither (a group longer than 16 bits, or an earlier group running past
//            the window with v > 15).
constexpr int kPLutBits = 7;
constexpr int kPLutWords = (1 << kPLutBits) / 4;  // its size in shared memory, in words
struct alignas(16) PLut {  // read with 16-byte loads
    uint8_t v[1 << kPLutBits];
};
constexpr PLut make_p_lut() {
    PLut t{};
    for (uint32_t w = 0; w < (1u << kPLutBits); ++w) {
        uint32_t v = 1;
        int pos = 0;
        uint8_t e = 0xFF;
        while (pos < kPLutBits) {
            if (((w >> (kPLutBits - 1 - pos)) & 1u) == 0) {  // the code ends: value v
                e = static_cast<uint8_t>((v << 3) | static_cast<uint32_t>(pos));
                break;
            }
            const int glen = static_cast<int>(v) + 1;
            if (pos + glen > kPLutBits) {  // the group runs past the window
                if (glen <= 16) e = static_cast<uint8_t>(0x80u | (v << 3) | static_cast<uint32_t>(pos));
                break;
            }
            v = (w >> (kPLutBits - pos - glen)) & ((1u << glen) - 1u);
            pos += glen;
        }
        t.v[w] = e;
    }
    return t;
}
__device__ const PLut kPLutGlobal = make_p_lut();
// The level table and the gap-prefix table, one after the other in shared memory.
constexpr int kSmallLutWords = kKLutWords + kPLutWords;

// The omega code at the top of a 12-bit window: [3:0] length (0: longer than 12
// bits), [9:4] value (<= 63, as every code of at most 12 bits).
struct alignas(16) OmegaLut {  // read with 16-byte loads
    uint16_t v[kLutSize];
};
constexpr OmegaLut make_omega_lut() {
    OmegaLut t{};
    for (uint32_t w = 0; w < static_cast<uint32_t>(kLutSize); ++w) {
        int pos = 0;
        uint32_t val = 0;
        t.v[w] = window_omega(w, kLutBits, pos, val) ? static_cast<uint16_t>(static_cast<uint32_t>(pos) | (val << 4)) : 0;
    }
    return t;
}
__device__ const OmegaLut kOmegaLutGlobal = make_omega_lut();

// The record table for levels up to s, in shared memory (16-byte loads).
__device__ __forceinline__ void rows_lut_fill(uint32_t* lut, uint32_t s, int tid, int nthreads) {
    const uint4* src = reinterpret_cast<const uint4*>(kRowsLutGlobal.v);
    for (int i = tid; i < kLutSize / 4; i += nthreads) {
        uint4 q = src[i];
        if (s < 15u) {
            uint32_t* e = &q.x;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                if (((e[j] >> 16) & 0x7Fu) > s)
                    e[j] = 0u;  // the first record's level is beyond s: bit-serial path
                else if ((e[j] >> 24 & 0x7Fu) > s)
                    e[j] = (e[j] & 0x00FF0F0Fu) | ((e[j] & 15u) << 4);  // keep the first record only
            }
        }
        reinterpret_cast<uint4*>(lut)[i] = q;
    }
}
__device__ __forceinline__ void p_lut_fill(uint8_t* plut, int tid, int nthreads) {
    const uint4* src = reinterpret_cast<const uint4*>(kPLutGlobal.v);
    for (int i = tid; i < (1 << kPLutBits) / 16; i += nthreads) reinterpret_cast<uint4*>(plut)[i] = src[i];
}

// The sign and level after a gap code of gl bits at the top of w: code = sign << 7 | k
// with the level's code through kKLut (k <= 15).  Returns the record's length
// (gl + 1 + the level's), 0 when the level's code is longer than 7 bits.
__device__ __forceinline__ uint32_t record_tail(uint32_t w, uint32_t gl, const uint8_t* klut, uint32_t& code) {
    const uint32_t kc = klut[(w << (gl + 1u)) >> (32 - kKLutBits)];
    const uint32_t kl = kc & 15u;
    if (kl == 0u) return 0;
    code = (((w << gl) >> 31) << 7) | (kc >> 4);
    return gl + 1u + kl;
}

// A record at the top of the 32 bits w that the whole-record table does not hold (its
// entry e has [3:0] = 0), when the gap's code fits the table's window (gap <= 63,
// from e) and k <= 15.  Returns its length (at most 24 bits), with gap and code =
// sign << 7 | k; 0 otherwise.
__device__ __forceinline__ uint32_t near_long_record(uint32_t w, uint32_t e, const uint8_t* klut, uint32_t& gap,
                                                     uint32_t& code) {
    const uint32_t gl = (e >> 4) & 15u;  // bits of the gap's code
    if (gl == 0u) return 0;
    gap = (e >> 8) & 63u;
    return record_tail(w, gl, klut, code);
}

// A record at the top of w whose gap's code is longer than the table's window but
// whose gap is below 2^16, with k <= 15: the gap through kPLut (the one group that
// runs past its 7-bit window, then the terminating 0 bit), then the sign and the
// level.  Such a record takes at most 31 bits.  Returns its length, 0 otherwise (the
// bit-serial path takes it).
__device__ __forceinline__ uint32_t far_long_record(uint32_t w, const uint8_t* plut, const uint8_t* klut,
                                                    uint32_t& gap, uint32_t& code) {
    const uint32_t pe = plut[w >> (32 - kPLutBits)];
    if (pe == 0xFFu || !(pe & 0x80u)) return 0;  // (a code ending inside 7 bits fits the table's window)
    const uint32_t v = (pe >> 3) & 15u, p = pe & 7u;
    gap = (w << p) >> (31u - v);                    // the group of v + 1 bits at p
    const uint32_t gl = p + v + 2u;                 // the group and the 0 after it
    if (((w << (gl - 1u)) >> 31) != 0u) return 0;   // another group: a gap of 2^16 or more
    return record_tail(w, gl, klut, code);
}

__device__ __forceinline__ void omega_lut_fill(uint16_t* olut, int tid, int nthreads) {
    const uint4* src = reinterpret_cast<const uint4*>(kOmegaLutGlobal.v);
    for (int i = tid; i < kLutSize / 8; i += nthreads) reinterpret_cast<uint4*>(olut)[i] = src[i];
}

}  // namespace
}  // namespace qsgd
