// Limits and launch constants of the QSGD library (host and device).
#pragma once

#include <cstdint>

namespace qsgd {

constexpr uint64_t kMaxN = uint64_t(1) << 34;
constexpr uint64_t kMaxD = uint64_t(1) << 31;
constexpr uint32_t kMaxS = 1u << 22;          // keeps t = |v| s/||v|| below 2^23
constexpr uint64_t kMaxStreamBits = (uint64_t(1) << 38) - 1;  // scan descriptor value field

constexpr int kOmegaTab = 1024;               // shared-memory omega table entries
constexpr uint32_t kMaxPolls = 1u << 22;      // bound of every spin wait (~1 s)

constexpr int kBlock = 256;                   // threads per CTA, every encode kernel
constexpr int kWarps = kBlock / 32;
constexpr uint32_t kFastMinD = 128;           // warp-per-bucket path: 128 <= d <= 1024,
constexpr uint32_t kFastMaxD = 1024;          //   d % 4 == 0, 16-byte aligned input
constexpr uint32_t kChunk = 4 * kBlock;       // coordinates per chunk of the general path
constexpr uint32_t kGeneralTileCoords = 4096; // general path: buckets per tile = max(1, 4096/d)

constexpr int kDecodeBlock = 128;
constexpr int kMaxStreamsPerLaunch = 64;

}  // namespace qsgd
