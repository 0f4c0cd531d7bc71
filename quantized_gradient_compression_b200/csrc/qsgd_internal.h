// Library-internal declarations shared by the host API and the kernel files.
#pragma once

#include <cuda_runtime_api.h>

#include <cstddef>
#include <cstdint>

#include "qsgd_limits.h"

namespace qsgd {

struct ScanControl;

// Workspace layout (all offsets 256-byte aligned):
//   [0, 64)          ScanControl
//   desc[ntiles]     uint64 scan descriptors
//   carry[ntiles]    uint64 tail-word slots (1 << 63 | epoch << 32 | word)
//   norms[nb]        float2 (sent norm, s/norm) of the general path
struct WorkspaceLayout {
    size_t desc_off, carry_off, norms_off, total;
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
    uint64_t* desc;
    uint64_t* carry;
    float2* norms;     // general path only
    uint64_t nb;
    uint64_t ntiles;
    uint32_t buckets_per_tile;
    uint32_t smem_words;  // words of the per-tile (or per-chunk) bit buffer
};

// Chooses the kernel, sets the launch shape and enqueues it.  Returns a CUDA
// error code (cudaSuccess on success).
cudaError_t launch_encode(EncodeArgs a, bool fast_path, cudaStream_t stream);

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
};

cudaError_t launch_decode(const DecodeArgs& a, bool accumulate, cudaStream_t stream);

// Omega code length on the host (for the size bound).
uint32_t omega_len_host(uint64_t N);

}  // namespace qsgd
