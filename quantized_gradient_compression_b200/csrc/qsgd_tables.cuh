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
// (<= 63, as every omega code of at most 12 bits); the sign and the level follow it
// (the level through kKLut).  For s >= 15 the table is the same for every s; a
// smaller s drops the records with k > s when the table is copied (rows_lut_fill).
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
__device__ __forceinline__ void omega_lut_fill(uint16_t* olut, int tid, int nthreads) {
    const uint4* src = reinterpret_cast<const uint4*>(kOmegaLutGlobal.v);
    for (int i = tid; i < kLutSize / 8; i += nthreads) reinterpret_cast<uint4*>(olut)[i] = src[i];
}

}  // namespace
}  // namespace qsgd
