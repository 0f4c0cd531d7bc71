// Host side of the QSGD C ABI (include/qsgd.h): argument checks, workspace layout,
// kernel selection.  No allocation happens here or anywhere in the library.
#include <cuda_runtime.h>

#include <cstdint>
#include <algorithm>
#include <cstring>

#include "../../include/qsgd.h"
#include "qsgd_device.cuh"
#include "qsgd_internal.h"

namespace qsgd {

uint32_t omega_len_host(uint64_t N) {
    uint32_t len = 1;
    while (N > 1) {
        uint32_t b = 0;
        for (uint64_t x = N; x; x >>= 1) ++b;
        len += b;
        N = b - 1;
    }
    return len;
}

namespace {

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

uint64_t ceil_div(uint64_t a, uint64_t b) { return (a + b - 1) / b; }

bool valid_params(uint64_t n, uint32_t d, uint32_t s) {
    return n <= kMaxN && d >= 1 && static_cast<uint64_t>(d) <= kMaxD && s >= 1 && s <= kMaxS;
}

uint32_t general_buckets_per_tile(uint32_t d) {
    return d >= kGeneralTileCoords ? 1u : kGeneralTileCoords / d;
}

uint64_t max_bits(uint64_t n, uint32_t d, uint32_t s) {
    if (n == 0) return 0;
    const uint64_t nb = ceil_div(n, d);
    const uint64_t per = 2u + omega_len_host(s);
    // (32 + m_b * per) summed over buckets = 32 nb + n * per
    return 32u * nb + n * per;
}

bool fast_eligible(const float* in, uint32_t d, uint32_t s) {
    return d >= kFastMinD && d <= kFastMaxD && d % 4 == 0 && s <= kFastMaxS &&
           (reinterpret_cast<uintptr_t>(in) & 15u) == 0;
}

}  // namespace

WorkspaceLayout workspace_layout(uint64_t n, uint32_t d) {
    WorkspaceLayout L{};
    const uint64_t nb = n ? ceil_div(n, d) : 0;
    // fast path: tiles of kFastWarps buckets; general path: tiles of whole buckets
    const uint64_t per_tile = std::min<uint64_t>(kFastWarps, general_buckets_per_tile(d));
    L.max_tiles = nb ? ceil_div(nb, per_tile) : 0;
    L.desc_off = 256;
    L.tiles_off = L.desc_off + align256(sizeof(uint64_t) * ((L.max_tiles + 1) & ~uint64_t(1)));
    L.total = L.tiles_off + align256(sizeof(TileState) * L.max_tiles);
    return L;
}

bool stage_shape(uint32_t d, uint32_t s) {
    if (d < kStageMinD || d % 4 != 0 || d > (s <= kStageShortMaxS ? kStageShortMaxD : kStageMaxD)) return false;
    const uint64_t slot_bits = 32u + static_cast<uint64_t>(d) * (2u + omega_len_host(s));
    return stage_smem_bytes(s, static_cast<uint32_t>(ceil_div(slot_bits, 32)) + 1u) <= 200 * 1024;
}

StageLayout stage_layout(uint64_t n, uint32_t d, uint32_t s) {
    StageLayout L{};
    const uint64_t nb = n ? ceil_div(n, d) : 0;
    const uint64_t slot_bits = 32u + static_cast<uint64_t>(d) * (2u + omega_len_host(s));
    // a whole number of 16-byte units, so that every slot starts 16-byte aligned
    L.slot_words = static_cast<uint32_t>(ceil_div(ceil_div(slot_bits, 32), 4) * 4);
    L.ntiles = ceil_div(nb, kCompactBlock);
    L.desc_off = 256;
    L.bits_off = L.desc_off + align256(sizeof(uint64_t) * L.ntiles);
    L.stage_off = L.bits_off + align256(sizeof(uint32_t) * nb);
    L.total = L.stage_off + align256(sizeof(uint32_t) * nb * L.slot_words);
    return L;
}

}  // namespace qsgd

using namespace qsgd;

extern "C" {

uint64_t qsgd_num_buckets(uint64_t n, uint32_t d) { return d ? ceil_div(n, d) : 0; }

uint64_t qsgd_max_encoded_words(uint64_t n, uint32_t d, uint32_t s) {
    if (!valid_params(n, d, s)) return 0;
    return ceil_div(max_bits(n, d, s), 32);
}

// Workspace of the one-pass encoders (encode_fast, encode_general) alone: the scan
// state, a few bytes per tile.
static size_t one_pass_workspace_bytes(uint64_t n, uint32_t d, uint32_t s) {
    if (!valid_params(n, d, s)) return 0;
    return workspace_layout(n, d).total;
}

size_t qsgd_encode_workspace_bytes(uint64_t n, uint32_t d, uint32_t s) {
    const size_t one = one_pass_workspace_bytes(n, d, s);
    if (one == 0 || !stage_shape(d, s)) return one;
    return std::max(one, stage_layout(n, d, s).total);
}

int qsgd_workspace_init(void* d_ws, size_t ws_bytes, cudaStream_t stream) {
    if (!d_ws || ws_bytes == 0) return QSGD_ERR_ARG;
    return cudaMemsetAsync(d_ws, 0, ws_bytes, stream) == cudaSuccess ? QSGD_OK : QSGD_ERR_CUDA;
}

}  // extern "C"

namespace {

constexpr int kNothingToDo = -1;  // n == 0: only the end of the header is written (no QSGD_* code is negative)

// Checks the arguments of an encode of d_in and fills the kernel arguments.
// Returns QSGD_OK, kNothingToDo (n == 0, header written) or a QSGD_ERR_* code.
int prepare_encode(const float* d_in, uint64_t n, uint32_t d, uint32_t s, uint64_t seed, uint32_t norm_kind,
                   uint32_t* d_words, uint64_t words_capacity, uint64_t* d_offsets, void* d_ws, size_t ws_bytes,
                   uint32_t* d_status, cudaStream_t stream, EncodeArgs& a, bool& fast) {
    if (norm_kind != QSGD_NORM_L2 && norm_kind != QSGD_NORM_MAX) return QSGD_ERR_ARG;
    if (!valid_params(n, d, s) || !d_offsets || !d_status) return QSGD_ERR_ARG;
    if (max_bits(n, d, s) > kMaxStreamBits) return QSGD_ERR_ARG;
    if ((reinterpret_cast<uintptr_t>(d_offsets) & 7u) != 0 || (reinterpret_cast<uintptr_t>(d_words) & 3u) != 0)
        return QSGD_ERR_ARG;
    if (n == 0) {
        return cudaMemsetAsync(d_offsets, 0, sizeof(uint64_t), stream) == cudaSuccess ? kNothingToDo
                                                                                      : QSGD_ERR_CUDA;
    }
    if (!d_in || !d_words || !d_ws) return QSGD_ERR_ARG;
    if ((reinterpret_cast<uintptr_t>(d_ws) & 255u) != 0) return QSGD_ERR_ARG;
    if (words_capacity < qsgd_max_encoded_words(n, d, s)) return QSGD_ERR_CAPACITY;
    const WorkspaceLayout L = workspace_layout(n, d);
    if (ws_bytes < L.total) return QSGD_ERR_WORKSPACE;

    char* ws = static_cast<char*>(d_ws);
    a = EncodeArgs{};
    a.in = d_in;
    a.n = n;
    a.d = d;
    a.s = s;
    a.key0 = static_cast<uint32_t>(seed);
    a.key1 = static_cast<uint32_t>(seed >> 32);
    a.words = d_words;
    a.cap_words = words_capacity;
    a.offsets = d_offsets;
    a.status = d_status;
    a.norm_kind = norm_kind;
    a.ef = nullptr;
    a.ctrl = reinterpret_cast<ScanControl*>(ws);
    a.tdesc = reinterpret_cast<uint64_t*>(ws + L.desc_off);
    a.ts = reinterpret_cast<TileState*>(ws + L.tiles_off);
    a.nb = ceil_div(n, d);
    const uint32_t wl = 2u + omega_len_host(s);
    // the fast path when its tile fits in shared memory, else the general one
    const uint64_t fast_tile_bits = static_cast<uint64_t>(kFastWarps) * (32u + static_cast<uint64_t>(d) * wl);
    const uint32_t fast_words = static_cast<uint32_t>(std::min<uint64_t>(ceil_div(fast_tile_bits, 32) + 2, 1u << 24));
    fast = fast_eligible(d_in, d, s) && fast_smem_bytes(d, s, fast_words) <= 200 * 1024;
    if (fast) {
        a.buckets_per_tile = kFastWarps;  // one bucket per warp
        a.ntiles = ceil_div(a.nb, kFastWarps);
        a.smem_words = fast_words;
    } else {
        a.buckets_per_tile = general_buckets_per_tile(d);
        a.ntiles = ceil_div(a.nb, a.buckets_per_tile);
        // one chunk: 31 leading bits, kChunk records bounded by the gap argument plus
        // one record whose gap reaches back past the chunk (<= 43 + 1 + |omega(s)|),
        // and a norm for every bucket that starts inside the chunk
        const uint64_t starts = kChunk / d + 2;
        const uint64_t chunk_bits = 31u + static_cast<uint64_t>(kChunk) * wl + 44u + omega_len_host(s) + 32u * starts;
        a.smem_words = static_cast<uint32_t>(ceil_div(chunk_bits, 32) + 2);
    }
    const uint64_t smem_bytes = fast ? fast_smem_bytes(d, s, a.smem_words)
                                     : general_smem_bytes(a.smem_words, a.buckets_per_tile);
    if (smem_bytes > 200 * 1024) return QSGD_ERR_ARG;
    if (a.ntiles > L.max_tiles) return QSGD_ERR_WORKSPACE;
    return QSGD_OK;
}

// Whether [a, a + n) and [b, b + n) share a float.
bool overlaps(const float* a, const float* b, uint64_t n) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    const uint64_t bytes = n * sizeof(float);
    return x < y + bytes && y < x + bytes;
}

}  // namespace

namespace qsgd {

// Fills the two-launch encoder's arguments (after prepare_encode has checked them).
static StageArgs stage_args(const EncodeArgs& e, float* d_ef, uint64_t seed, void* d_ws) {
    const StageLayout L = stage_layout(e.n, e.d, e.s);
    char* ws = static_cast<char*>(d_ws);
    StageArgs a{};
    a.in = e.in;
    a.ef = d_ef;
    a.n = e.n;
    a.d = e.d;
    a.s = e.s;
    a.norm_kind = e.norm_kind;
    const uint32_t k0 = static_cast<uint32_t>(seed), k1 = static_cast<uint32_t>(seed >> 32);
    for (uint32_t r = 0; r < 10; ++r) {
        a.rk[2 * r] = k0 + r * 0x9E3779B9u;
        a.rk[2 * r + 1] = k1 + r * 0xBB67AE85u;
    }
    a.nb = e.nb;
    a.slot_words = L.slot_words;
    a.buf_words = L.slot_words + 1;
    a.stage = reinterpret_cast<uint32_t*>(ws + L.stage_off);
    a.bits = reinterpret_cast<uint32_t*>(ws + L.bits_off);
    a.status = e.status;
    a.words = e.words;
    a.cap_words = e.cap_words;
    a.offsets = e.offsets;
    a.ctrl = reinterpret_cast<ScanControl*>(ws);
    a.cdesc = reinterpret_cast<uint64_t*>(ws + L.desc_off);
    a.ntiles = L.ntiles;
    return a;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// qsgd_encode_ex / qsgd_encode_ef.  d_ef: the error-feedback memory, or null.  With
// `strict`, the workspace must hold qsgd_encode_workspace_bytes; otherwise (the static
// workspace entry point) the two-launch encoder runs when its layout fits, else a
// one-pass encoder.  Every path writes the same stream.
int encode_entry(const float* d_in, float* d_ef, uint64_t n, uint32_t d, uint32_t s, uint64_t seed,
                 uint32_t norm_kind, uint32_t* d_words, uint64_t words_capacity, uint64_t* d_offsets, void* d_ws,
                 size_t ws_bytes, uint32_t* d_status, cudaStream_t stream, bool strict) {
    if (d_ef && n > 0) {
        if (!d_in || ((reinterpret_cast<uintptr_t>(d_in) | reinterpret_cast<uintptr_t>(d_ef)) & 3u) != 0)
            return QSGD_ERR_ARG;
        if (overlaps(d_in, d_ef, n)) return QSGD_ERR_ARG;
    }
    EncodeArgs a;
    bool fast = false;
    int rc = prepare_encode(d_in, n, d, s, seed, norm_kind, d_words, words_capacity, d_offsets, d_ws, ws_bytes,
                            d_status, stream, a, fast);
    if (rc != QSGD_OK) return rc == kNothingToDo ? QSGD_OK : rc;
    if (strict && ws_bytes < qsgd_encode_workspace_bytes(n, d, s)) return QSGD_ERR_WORKSPACE;
    if (stage_shape(d, s) && aligned16(d_in) && (!d_ef || aligned16(d_ef)) &&
        ws_bytes >= stage_layout(n, d, s).total) {
        // two launches: bucket coder (with the memory fused in), compaction
        return launch_encode_stage(stage_args(a, d_ef, seed, d_ws), stream) == cudaSuccess ? QSGD_OK : QSGD_ERR_CUDA;
    }
    // one-pass encoders: their descriptor entries zeroed first (the two-launch encoder
    // may have left staging data in those bytes)
    if (cudaMemsetAsync(static_cast<char*>(d_ws) + 256, 0, workspace_layout(n, d).total - 256, stream) != cudaSuccess)
        return QSGD_ERR_CUDA;
    if (!d_ef) return launch_encode(a, fast, stream) == cudaSuccess ? QSGD_OK : QSGD_ERR_CUDA;
    if (fast && aligned16(d_ef)) {
        // one pass: the fast encoder reads g and e and writes the stream and e
        a.ef = d_ef;
        return launch_encode(a, true, stream) == cudaSuccess ? QSGD_OK : QSGD_ERR_CUDA;
    }
    // three passes: e <- e + g; encode p from e; e <- p - decoded
    rc = prepare_encode(d_ef, n, d, s, seed, norm_kind, d_words, words_capacity, d_offsets, d_ws, ws_bytes, d_status,
                        stream, a, fast);
    if (rc != QSGD_OK) return rc;
    if (launch_ef_add(d_in, d_ef, n, stream) != cudaSuccess) return QSGD_ERR_CUDA;
    if (launch_encode(a, fast, stream) != cudaSuccess) return QSGD_ERR_CUDA;
    return launch_ef_residual(d_ef, d_words, words_capacity, d_offsets, n, d, s, seed, stream) == cudaSuccess
               ? QSGD_OK
               : QSGD_ERR_CUDA;
}

size_t min_encode_workspace_bytes(uint64_t n, uint32_t d, uint32_t s) { return one_pass_workspace_bytes(n, d, s); }

}  // namespace qsgd

extern "C" {

int qsgd_encode_ex(const float* d_in, uint64_t n, uint32_t d, uint32_t s, uint64_t seed, uint32_t norm_kind,
                   uint32_t* d_words, uint64_t words_capacity, uint64_t* d_offsets, void* d_ws, size_t ws_bytes,
                   uint32_t* d_status, cudaStream_t stream) {
    return encode_entry(d_in, nullptr, n, d, s, seed, norm_kind, d_words, words_capacity, d_offsets, d_ws, ws_bytes,
                        d_status, stream, true);
}

int qsgd_encode_ef(const float* d_g, float* d_e, uint64_t n, uint32_t d, uint32_t s, uint64_t seed,
                   uint32_t norm_kind, uint32_t* d_words, uint64_t words_capacity, uint64_t* d_offsets, void* d_ws,
                   size_t ws_bytes, uint32_t* d_status, cudaStream_t stream) {
    if (n > 0 && (!d_g || !d_e)) return QSGD_ERR_ARG;
    return encode_entry(d_g, d_e, n, d, s, seed, norm_kind, d_words, words_capacity, d_offsets, d_ws, ws_bytes,
                        d_status, stream, true);
}

int qsgd_encode(const float* d_in, uint64_t n, uint32_t d, uint32_t s, uint64_t seed, uint32_t* d_words,
                uint64_t words_capacity, uint64_t* d_offsets, void* d_ws, size_t ws_bytes, uint32_t* d_status,
                cudaStream_t stream) {
    return qsgd_encode_ex(d_in, n, d, s, seed, QSGD_NORM_L2, d_words, words_capacity, d_offsets, d_ws, ws_bytes,
                          d_status, stream);
}

// Streams from which the several-stream decode kernel beats one launch per stream
// (measured on B200 at n = 25.6 M, d = 512, s = 16: 2 streams 173 against 263 us,
// 4 streams 269 against 525 us, 8 streams 451 against 1036 us; one stream 209
// against 133 us, so one stream stays on the one-stream kernel).
constexpr int kMultiMinStreams = 2;

static int decode_impl(const uint32_t* const* words, const uint64_t* num_words,
                       const uint64_t* const* offsets, int K, uint64_t n, uint32_t d, uint32_t s,
                       float* d_out, uint32_t* d_status, cudaStream_t stream, bool accumulate,
                       bool mean = false) {
    if (!valid_params(n, d, s) || !d_status || K < 1 || K > 1024) return QSGD_ERR_ARG;
    if (n == 0) return QSGD_OK;
    if (!d_out || !words || !num_words || !offsets) return QSGD_ERR_ARG;
    for (int j = 0; j < K; ++j)
        if (!words[j] || !offsets[j] || (reinterpret_cast<uintptr_t>(offsets[j]) & 7u) != 0)
            return QSGD_ERR_ARG;
    DecodeArgs a{};
    a.n = n;
    a.d = d;
    a.s = s;
    a.nb = ceil_div(n, d);
    a.out = d_out;
    a.status = d_status;
    for (int j0 = 0; j0 < K; j0 += kMaxStreamsPerLaunch) {
        a.K = std::min(K - j0, kMaxStreamsPerLaunch);
        a.first_group = j0 == 0;
        a.start_zero = mean && j0 == 0;  // the mean: the sum starts from +0 ...
        a.div = mean && j0 + a.K == K ? static_cast<float>(K) : 0.f;  // ... and is divided at the end
        for (int j = 0; j < a.K; ++j) {
            a.streams[j].words = words[j0 + j];
            a.streams[j].num_words = num_words[j0 + j];
            a.streams[j].offsets = offsets[j0 + j];
        }
        if (accumulate && !mean && a.K > 1 && a.K < kMultiMinStreams) {
            // a few streams: one launch each, in order
            DecodeArgs o = a;
            o.K = 1;
            for (int j = 0; j < a.K; ++j) {
                o.streams[0] = a.streams[j];
                o.first_group = a.first_group && j == 0;
                if (launch_decode(o, true, stream) != cudaSuccess) return QSGD_ERR_CUDA;
            }
            continue;
        }
        const cudaError_t e = launch_decode(a, accumulate, stream);
        if (e != cudaSuccess) return QSGD_ERR_CUDA;
    }
    return QSGD_OK;
}

int qsgd_decode(const uint32_t* d_words, uint64_t num_words, const uint64_t* d_offsets, uint64_t n,
                uint32_t d, uint32_t s, float* d_out, uint32_t* d_status, cudaStream_t stream) {
    const uint32_t* w[1] = {d_words};
    const uint64_t nw[1] = {num_words};
    const uint64_t* o[1] = {d_offsets};
    return decode_impl(w, nw, o, 1, n, d, s, d_out, d_status, stream, false);
}

int qsgd_decode_mean(const uint32_t* const* h_words, const uint64_t* h_num_words,
                     const uint64_t* const* h_offsets, int K, uint64_t n, uint32_t d, uint32_t s, float* d_out,
                     uint32_t* d_status, cudaStream_t stream) {
    if (!h_words || !h_num_words || !h_offsets || K < 1 || K > 1024) return QSGD_ERR_ARG;
    if (!valid_params(n, d, s) || !d_status) return QSGD_ERR_ARG;
    for (int j = 0; j < K; ++j)  // every stream is checked before the first launch
        if (!h_words[j] || !h_offsets[j] || (reinterpret_cast<uintptr_t>(h_offsets[j]) & 7u) != 0)
            return QSGD_ERR_ARG;
    // the several-stream kernel: sum from +0 in stream order, divided in its last launch
    if (decode_multi_shape(d, s, d_out) && K >= kMultiMinStreams)
        return decode_impl(h_words, h_num_words, h_offsets, K, n, d, s, d_out, d_status, stream, true, true);
    // other shapes and a few streams: stream 0 decoded into d_out, the others added in
    // order, then the division
    int rc = decode_impl(h_words, h_num_words, h_offsets, 1, n, d, s, d_out, d_status, stream, false);
    if (rc != QSGD_OK || n == 0) return rc;
    if (K > 1) {
        rc = decode_impl(h_words + 1, h_num_words + 1, h_offsets + 1, K - 1, n, d, s, d_out, d_status, stream, true);
        if (rc != QSGD_OK) return rc;
    }
    return launch_div(d_out, n, static_cast<uint32_t>(K), stream) == cudaSuccess ? QSGD_OK : QSGD_ERR_CUDA;
}

int qsgd_decode_accumulate(const uint32_t* const* h_words, const uint64_t* h_num_words,
                           const uint64_t* const* h_offsets, int K, uint64_t n, uint32_t d,
                           uint32_t s, float* d_out, uint32_t* d_status, cudaStream_t stream) {
    return decode_impl(h_words, h_num_words, h_offsets, K, n, d, s, d_out, d_status, stream, true);
}

uint64_t qsgd_bbit_code_words(uint64_t n, uint32_t b) { return (n * static_cast<uint64_t>(b) + 31u) / 32u; }

static bool valid_bbit(uint64_t n, uint32_t d, uint32_t b) {
    return (b == 2 || b == 4 || b == 8) && d >= 1 && d <= kMaxD && n <= kMaxN;
}

int qsgd_bbit_encode_ex(const float* d_in, uint64_t n, uint32_t d, uint32_t b, uint64_t seed, uint32_t norm_kind,
                        float* d_norms, uint32_t* d_codes, uint32_t* d_status, cudaStream_t stream) {
    if (!valid_bbit(n, d, b) || !d_status) return QSGD_ERR_ARG;
    if (norm_kind != QSGD_NORM_L2 && norm_kind != QSGD_NORM_MAX) return QSGD_ERR_ARG;
    if (n == 0) return QSGD_OK;
    if (!d_in || !d_norms || !d_codes || (reinterpret_cast<uintptr_t>(d_in) & 3u) != 0 ||
        (reinterpret_cast<uintptr_t>(d_norms) & 3u) != 0 || (reinterpret_cast<uintptr_t>(d_codes) & 3u) != 0)
        return QSGD_ERR_ARG;
    return launch_bbit_encode(d_in, nullptr, n, d, b, seed, norm_kind, d_norms, d_codes, d_status, stream) ==
                   cudaSuccess
               ? QSGD_OK
               : QSGD_ERR_CUDA;
}

int qsgd_bbit_encode_ef(const float* d_g, float* d_e, uint64_t n, uint32_t d, uint32_t b, uint64_t seed,
                        uint32_t norm_kind, float* d_norms, uint32_t* d_codes, uint32_t* d_status,
                        cudaStream_t stream) {
    if (!valid_bbit(n, d, b) || !d_status) return QSGD_ERR_ARG;
    if (norm_kind != QSGD_NORM_L2 && norm_kind != QSGD_NORM_MAX) return QSGD_ERR_ARG;
    if (n == 0) return QSGD_OK;
    if (!d_g || !d_e || !d_norms || !d_codes ||
        ((reinterpret_cast<uintptr_t>(d_g) | reinterpret_cast<uintptr_t>(d_e) | reinterpret_cast<uintptr_t>(d_norms) |
          reinterpret_cast<uintptr_t>(d_codes)) & 3u) != 0)
        return QSGD_ERR_ARG;
    if (overlaps(d_g, d_e, n)) return QSGD_ERR_ARG;
    if (bbit_fast_shape(d_g, d_e, d))  // one pass
        return launch_bbit_encode(d_g, d_e, n, d, b, seed, norm_kind, d_norms, d_codes, d_status, stream) ==
                       cudaSuccess
                   ? QSGD_OK
                   : QSGD_ERR_CUDA;
    // three passes: e <- e + g; encode p from e; e <- p - decoded
    if (launch_ef_add(d_g, d_e, n, stream) != cudaSuccess) return QSGD_ERR_CUDA;
    if (launch_bbit_encode(d_e, nullptr, n, d, b, seed, norm_kind, d_norms, d_codes, d_status, stream) !=
        cudaSuccess)
        return QSGD_ERR_CUDA;
    return launch_bbit_ef_residual(d_e, d_norms, d_codes, n, d, b, stream) == cudaSuccess ? QSGD_OK : QSGD_ERR_CUDA;
}

int qsgd_bbit_encode(const float* d_in, uint64_t n, uint32_t d, uint32_t b, uint64_t seed, float* d_norms,
                     uint32_t* d_codes, uint32_t* d_status, cudaStream_t stream) {
    return qsgd_bbit_encode_ex(d_in, n, d, b, seed, QSGD_NORM_L2, d_norms, d_codes, d_status, stream);
}

int qsgd_bbit_decode(const float* d_norms, const uint32_t* d_codes, uint64_t n, uint32_t d, uint32_t b,
                     float* d_out, uint32_t* d_status, cudaStream_t stream) {
    if (!valid_bbit(n, d, b) || !d_status) return QSGD_ERR_ARG;
    if (n == 0) return QSGD_OK;
    if (!d_norms || !d_codes || !d_out || (reinterpret_cast<uintptr_t>(d_out) & 3u) != 0) return QSGD_ERR_ARG;
    return launch_bbit_decode(d_norms, d_codes, n, d, b, d_out, false, d_status, stream) == cudaSuccess
               ? QSGD_OK
               : QSGD_ERR_CUDA;
}

int qsgd_bbit_decode_accumulate(const float* const* h_norms, const uint32_t* const* h_codes, int K, uint64_t n,
                                uint32_t d, uint32_t b, float* d_out, uint32_t* d_status, cudaStream_t stream) {
    if (!valid_bbit(n, d, b) || !d_status || K < 1 || !h_norms || !h_codes) return QSGD_ERR_ARG;
    if (n == 0) return QSGD_OK;
    if (!d_out || (reinterpret_cast<uintptr_t>(d_out) & 3u) != 0) return QSGD_ERR_ARG;
    for (int j = 0; j < K; ++j)
        if (!h_norms[j] || !h_codes[j]) return QSGD_ERR_ARG;
    // one launch per stream, in order on `stream`: every coordinate's adds run left
    // to right
    for (int j = 0; j < K; ++j)
        if (launch_bbit_decode(h_norms[j], h_codes[j], n, d, b, d_out, true, d_status, stream) != cudaSuccess)
            return QSGD_ERR_CUDA;
    return QSGD_OK;
}

int qsgd_bbit_decode_mean(const float* const* h_norms, const uint32_t* const* h_codes, int K, uint64_t n,
                          uint32_t d, uint32_t b, float* d_out, uint32_t* d_status, cudaStream_t stream) {
    if (!valid_bbit(n, d, b) || !d_status || K < 1 || K > 1024 || !h_norms || !h_codes) return QSGD_ERR_ARG;
    if (n == 0) return QSGD_OK;
    if (!d_out || (reinterpret_cast<uintptr_t>(d_out) & 3u) != 0) return QSGD_ERR_ARG;
    for (int j = 0; j < K; ++j)
        if (!h_norms[j] || !h_codes[j]) return QSGD_ERR_ARG;
    for (int j = 0; j < K; ++j)
        if (launch_bbit_decode(h_norms[j], h_codes[j], n, d, b, d_out, j > 0, d_status, stream) != cudaSuccess)
            return QSGD_ERR_CUDA;
    return launch_div(d_out, n, static_cast<uint32_t>(K), stream) == cudaSuccess ? QSGD_OK : QSGD_ERR_CUDA;
}

const char* qsgd_error_string(int code) {
    switch (code) {
        case QSGD_OK: return "ok";
        case QSGD_ERR_ARG: return "invalid argument";
        case QSGD_ERR_CAPACITY: return "output capacity below qsgd_max_encoded_words";
        case QSGD_ERR_CUDA: return "CUDA runtime error";
        case QSGD_ERR_WORKSPACE: return "workspace below qsgd_encode_workspace_bytes";
        case QSGD_ERR_STATIC_LIMIT:
            return "problem needs more scan state than the fixed device workspace of qsgd_encode_static_ws; "
                   "call qsgd_encode with a caller workspace";
        default: return "unknown error";
    }
}

const char* qsgd_version(void) { return "qsgd-b200 1.0 (wire format v1, sm_100a)"; }

}  // extern "C"
