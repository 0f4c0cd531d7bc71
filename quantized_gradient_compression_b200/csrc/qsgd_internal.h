// Library-internal declarations shared by the host API and the kernel files.
#pragma once

#include <cuda_runtime_api.h>

#include <cstddef>
#include <cstdint>

#include "qsgd_limits.h"

namespace qsgd {

struct ScanControl;
struct TileState;

// Workspace layout of the one-pass encoders: [0, 256) ScanControl; from 256 the tile
// scan descriptors (uint64 per tile, the count rounded up to an even number); then
// TileState per tile (shared-word slot, round prefix).  Every entry carries the
// call's epoch.  The host zeroes the entries before every one-pass launch, because
// the two-launch encoder keeps staging data in the same bytes, and data there can
// look like a descriptor of any epoch.
struct WorkspaceLayout {
    size_t desc_off, tiles_off, total;
    uint64_t max_tiles;
};
WorkspaceLayout workspace_layout(uint64_t n, uint32_t d);

struct EncodeArgs {
    const float* in;
    uint64_t n;
    uint32_t d;
    uint32_t s;
    uint32_t key0, key1;
    uint32_t* words;
    uint64_t cap_words;
    uint64_t* offsets;
    uint32_t* status;
    ScanControl* ctrl;
    uint64_t* tdesc;  // scan descriptor per tile (16-byte aligned)
    TileState* ts;
    uint64_t nb;
    uint64_t ntiles;
    uint32_t buckets_per_tile;
    uint32_t smem_words;  // words of the per-tile (or per-chunk) bit buffer
    uint32_t norm_kind;   // QSGD_NORM_L2 or QSGD_NORM_MAX
    float* ef;            // error-feedback memory fused into the fast encoder, or null
};

// Chooses the kernel, sets the launch shape and enqueues it.  Returns a CUDA
// error code (cudaSuccess on success).
cudaError_t launch_encode(EncodeArgs a, bool fast_path, cudaStream_t stream);

// Dynamic shared memory of the general encoder: omega table | chunk buffer |
// (norm, s/norm) of the tile's buckets.
inline size_t general_smem_bytes(uint32_t smem_words, uint32_t buckets_per_tile) {
    return (static_cast<size_t>(kOmegaTab) + ((smem_words + 1) & ~1u) + 2 * static_cast<size_t>(buckets_per_tile)) *
           sizeof(uint32_t);
}

// Float4s per lane of the fast encoder for bucket size d (a power of two >= d/128).
inline uint32_t fast_v(uint32_t d) {
    const uint32_t v = (d + 127) / 128;
    return v <= 1 ? 1 : v <= 2 ? 2 : v <= 4 ? 4 : 8;
}
// Words of one lane's private bit strip in the fast encoder: 4V records of at
// most 30 bits (s <= 31) or 18 + 1 + 32 bits (larger s), plus one.
__host__ __device__ inline constexpr uint32_t fast_lane_words(uint32_t V, bool short_records) {
    return (4 * V * (short_records ? 30u : 51u) + 31u) / 32u + 1u;
}
// Dynamic shared memory of the fast encoder: record table | one tile of input
// (kFastWarps * 128V floats; also the warps' record lists) | kEncBufs tile buffers |
// the lane strips.
inline size_t fast_smem_bytes(uint32_t d, uint32_t s, uint32_t smem_words) {
    const uint32_t v = fast_v(d);
    return (static_cast<size_t>(kRecordTab) + static_cast<size_t>(kFastWarps) * 128 * v +
            static_cast<size_t>(enc_depth(v) + 1) * smem_words +
            static_cast<size_t>(kFastWarps) * 32 * fast_lane_words(v, s <= 31)) *
           sizeof(uint32_t);
}

// Two-launch encoder (qsgd_encode_stage.cu): the bucket coder writes every bucket's
// bits into its own staging slot and its bit count; the compaction scans the counts
// and writes the offsets header and the stream.
struct StageArgs {
    const float* in;
    float* ef;            // error-feedback memory fused into the bucket coder, or null
    uint64_t n;
    uint32_t d, s, norm_kind;
    uint32_t rk[20];      // Philox round keys: the seed advanced r times by the Weyl constants
    uint64_t nb;
    uint32_t slot_words;  // staging words per bucket (its largest size)
    uint32_t buf_words;   // shared-memory words of one warp's bucket buffer
    uint32_t* stage;      // nb * slot_words
    uint32_t* bits;       // nb bucket sizes in bits
    uint32_t* status;
    uint32_t* words;
    uint64_t cap_words;
    uint64_t* offsets;
    ScanControl* ctrl;
    uint64_t* cdesc;      // compaction scan descriptor per tile of kCompactBlock buckets
    uint64_t ntiles;
};

// Workspace of the two-launch encoder: [0, 256) control block; the compaction's
// descriptors; the bucket sizes; the staging slots.
struct StageLayout {
    size_t desc_off, bits_off, stage_off, total;
    uint64_t ntiles;
    uint32_t slot_words;
};
StageLayout stage_layout(uint64_t n, uint32_t d, uint32_t s);

// Float4s per lane of the bucket coder (a power of two >= d/128; 4 for buckets of
// several 512-coordinate chunks).
inline uint32_t stage_v(uint32_t d) { return d <= 1024 ? fast_v(d) : 4; }
// Dynamic shared memory of the bucket coder: omega table | record table (s <= 31) |
// one bucket buffer per warp.
inline size_t stage_smem_bytes(uint32_t s, uint32_t buf_words) {
    return (static_cast<size_t>(kOmegaTab) + (s <= kStageShortMaxS ? kRecordTab64 : 0) +
            static_cast<size_t>(kStageWarps) * buf_words) *
           sizeof(uint32_t);
}
// Whether the two-launch encoder takes (d, s) (alignment aside): the shapes above,
// with one bucket buffer per warp within the shared memory.
bool stage_shape(uint32_t d, uint32_t s);
cudaError_t launch_encode_stage(const StageArgs& a, cudaStream_t stream);

// The encode entry behind qsgd_encode_ex and qsgd_encode_ef (d_ef null or the
// memory).  strict: the workspace must hold qsgd_encode_workspace_bytes; otherwise
// the one-pass encoders run when the two-launch layout does not fit.
int encode_entry(const float* d_in, float* d_ef, uint64_t n, uint32_t d, uint32_t s, uint64_t seed,
                 uint32_t norm_kind, uint32_t* d_words, uint64_t words_capacity, uint64_t* d_offsets, void* d_ws,
                 size_t ws_bytes, uint32_t* d_status, cudaStream_t stream, bool strict);
// Workspace of the one-pass encoders alone (their scan state).
size_t min_encode_workspace_bytes(uint64_t n, uint32_t d, uint32_t s);

struct StreamRef {
    const uint32_t* words;
    uint64_t num_words;
    const uint64_t* offsets;
};

struct DecodeArgs {
    StreamRef streams[kMaxStreamsPerLaunch];
    int K;
    uint64_t n;
    uint32_t d;
    uint32_t s;
    uint64_t nb;
    float* out;
    uint32_t* status;
    int first_group;  // decode-accumulate: this launch holds stream 0
    int start_zero;   // several-stream kernel: the sum starts from +0, not from out
    float div;        // several-stream kernel: divide the finished sum by div (0: no)
};

cudaError_t launch_decode(const DecodeArgs& a, bool accumulate, cudaStream_t stream);
// The one-stream decoder with whole rows staged as byte codes (qsgd_decode_rows.cu).
bool decode_rows_shape(uint32_t d, uint32_t s, const float* out);
cudaError_t launch_decode_rows(const DecodeArgs& a, bool accumulate, cudaStream_t stream);
// Several streams (decode-accumulate and the mean) on the same shapes (qsgd_decode_rows.cu):
// added onto fp32 tiles one stream after another (any s), or parsed side by side as
// byte codes (s <= 127).
cudaError_t launch_decode_rows_multi(const DecodeArgs& a, cudaStream_t stream);
cudaError_t launch_decode_rows_side(const DecodeArgs& a, cudaStream_t stream);
// Buckets larger than the row decoders take (qsgd_decode_rows.cu): decode and
// decode-accumulate (K <= 16 streams to a launch, in order).
bool decode_sparse_shape(uint32_t d, const float* out);
cudaError_t launch_decode_sparse(const DecodeArgs& a, bool accumulate, cudaStream_t stream);
// Whether the several-stream kernel (decode_multi, which start_zero / div need)
// takes this shape.
bool decode_multi_shape(uint32_t d, uint32_t s, const float* out);

// Fixed-width b-bit variant (b in {2, 4, 8}, checked by the caller).
cudaError_t launch_bbit_encode(const float* in, float* ef, uint64_t n, uint32_t d, uint32_t b, uint64_t seed,
                               uint32_t norm_kind, float* norms, uint32_t* codes, uint32_t* status,
                               cudaStream_t stream);
// Whether launch_bbit_encode fuses error feedback for this shape (else ef must be null).
bool bbit_fast_shape(const float* in, const float* ef, uint32_t d);

// out[i] <- fl(out[i] / K): the last step of the mean of K streams (qsgd_mean.cu).
cudaError_t launch_div(float* out, uint64_t n, uint32_t K, cudaStream_t stream);

// Error feedback for the shapes the fused encoders do not take (qsgd_ef.cu):
// e <- e + g; then, after the encoder has read p from e, the residual passes.
cudaError_t launch_ef_add(const float* g, float* e, uint64_t n, cudaStream_t stream);
cudaError_t launch_ef_residual(float* e, const uint32_t* words, uint64_t cap_words, const uint64_t* offsets,
                               uint64_t n, uint32_t d, uint32_t s, uint64_t seed, cudaStream_t stream);
cudaError_t launch_bbit_ef_residual(float* e, const float* norms, const uint32_t* codes, uint64_t n, uint32_t d,
                                    uint32_t b, cudaStream_t stream);
cudaError_t launch_bbit_decode(const float* norms, const uint32_t* codes, uint64_t n, uint32_t d, uint32_t b,
                               float* out, bool accumulate, uint32_t* status, cudaStream_t stream);

// Omega code length on the host (for the size bound).
uint32_t omega_len_host(uint64_t N);

}  // namespace qsgd
