// Limits and launch constants of the QSGD library (host and device).
#pragma once

#include <cstdint>

namespace qsgd {

constexpr uint64_t kMaxN = uint64_t(1) << 34;
constexpr uint64_t kMaxD = uint64_t(1) << 31;
constexpr uint32_t kMaxS = 1u << 22;          // keeps t = |v| s/||v|| below 2^23
constexpr uint64_t kMaxStreamBits = (uint64_t(1) << 38) - 1;  // scan descriptor value field

constexpr int kOmegaTab = 2048;               // omega code table entries (N < 2048)
constexpr int kRecordTab = 2048;              // record table: gap < 64, k < 16, sign
constexpr int kRecordTab64 = 4096;            // record table of the bucket coder: gap < 64, k < 32, sign
constexpr uint32_t kMaxPolls = 1u << 22;      // bound of every spin wait (~1 s)

constexpr int kBlock = 256;                   // threads per CTA, every encode kernel
constexpr int kWarps = kBlock / 32;
constexpr uint32_t kFastMinD = 128;           // warp-per-bucket path: 128 <= d <= 1024,
constexpr uint32_t kFastMaxD = 1024;          //   d % 4 == 0, 16-byte aligned input,
constexpr uint32_t kFastMaxS = (1u << 21) - 1;  //   s < 2^21 (a record list entry is 32 bits)
constexpr uint32_t kChunk = 4 * kBlock;       // coordinates per chunk of the general path
constexpr uint32_t kGeneralTileCoords = 4096; // general path: buckets per tile = max(1, 4096/d)

// Fast encoder: warps per CTA (one bucket each per tile) and the CTAs per SM the
// register budget is sized for (64 registers a thread at 32 warps per SM).
#ifndef QSGD_FAST_WARPS
#define QSGD_FAST_WARPS 16
#endif
#ifndef QSGD_FAST_MIN_BLOCKS
#define QSGD_FAST_MIN_BLOCKS (32 / QSGD_FAST_WARPS)
#endif
constexpr int kFastWarps = QSGD_FAST_WARPS;
constexpr int kFastBlock = 32 * kFastWarps;
// Fast encoder pipeline: a CTA gathers the prefix of (and stores) the tile it coded
// enc_depth(V) iterations earlier, with enc_depth(V) + 1 tile buffers (V = float4s
// per lane).  Depth 1 by default: depth 2 (QSGD_ENC_DEPTH=2, for V <= 4) measured
// the same on the 25.6 M coordinate gradient at d = 512.  V = 8 always uses depth 1,
// so that its larger tiles leave room
// for two CTAs per SM.
#ifndef QSGD_ENC_DEPTH
#define QSGD_ENC_DEPTH 1
#endif
__host__ __device__ constexpr int enc_depth(unsigned v) { return v <= 4 ? QSGD_ENC_DEPTH : 1; }
constexpr int kFastMinBlocks = QSGD_FAST_MIN_BLOCKS;

// Two-launch encoder (bucket coder + compaction): d % 4 == 0, 4 <= d <= 1024 (or
// 16384 for s <= 31), 16-byte aligned input; one warp per bucket, kStageWarps warps
// per CTA; the compaction takes a tile of kCompactBlock buckets per CTA of
// kCompactThreads threads.  Whole-record table for s <= 31.
constexpr int kStageWarps = 8;
constexpr int kStageBlock = 32 * kStageWarps;
#ifndef QSGD_COMPACT_BLOCK
#define QSGD_COMPACT_BLOCK 256
#endif
constexpr int kCompactBlock = QSGD_COMPACT_BLOCK;
constexpr int kCompactThreads = 2 * kCompactBlock;
// A tile whose staged words fit in this many words of shared memory is gathered
// there while the compaction's look-back runs; a larger one is read from the
// staging slots directly.
#ifndef QSGD_COMPACT_SMEM_WORDS
#define QSGD_COMPACT_SMEM_WORDS 16384
#endif
constexpr uint32_t kCompactSmemWords = QSGD_COMPACT_SMEM_WORDS;
constexpr uint32_t kStageMinD = 4;
constexpr uint32_t kStageMaxD = 1024;        // s > 31: one chunk of 128V coordinates per bucket
constexpr uint32_t kStageShortMaxD = 16384;  // s <= 31: buckets of several 512-coordinate chunks
constexpr uint32_t kStageShortMaxS = 31;

// One-stream decoder with byte codes staged in whole bucket rows: d % 4 == 0,
// 4 <= d <= 1024, s <= 32767 (a code is sign << 7 | k in a byte, or sign << 15 | k
// in 16 bits above s = 127), 16-byte aligned output; up to
// kRowsMaxWarps warps (32 buckets each) to a CTA, as many as the shared memory holds.
constexpr int kRowsMaxWarps = 16;
constexpr uint32_t kRowsMaxD = 1024;
constexpr uint32_t kRowsMaxS8 = 127;     // byte codes up to here, 16-bit codes above
constexpr uint32_t kRowsMaxS = 32767;

// Large-bucket decoder (d > kRowsMaxD, 16-byte aligned output): a CTA fills the
// output of 32 buckets, then one lane per bucket stores the records.
constexpr int kSparseBlock = 256;
constexpr int kSparseGroup = 8;     // buckets a CTA of the large-bucket decode-accumulate takes at once
#ifndef QSGD_SPARSE_REC_LANES
#define QSGD_SPARSE_REC_LANES 4
#endif
constexpr int kSparseRecBlock = 256;                      // threads a CTA of the large-bucket decode's records
constexpr int kSparseRecLanes = QSGD_SPARSE_REC_LANES;    // lanes of a warp there that take a bucket
constexpr int kSparseRecBuckets = kSparseRecBlock / 32 * kSparseRecLanes;  // buckets a CTA

constexpr int kDecodeBlock = 128;
constexpr int kMaxStreamsPerLaunch = 16;  // decode-accumulate streams per launch

}  // namespace qsgd
