// qsgd_encode_static_ws: the encoder for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc at the point where they compress a gradient:
// code running inside a caching allocator's own hooks, a communication library's
// progress thread that must not take the allocator lock, or an embedding that only
// hands the codec its input and output buffers.  For them the encoder's scan state
// lives in a fixed array of device memory owned by this library.  The array is a
// file-scope static device variable: every GPU that loads the library holds it
// (kStaticWorkspaceBytes) until the process exits.  Nothing here allocates.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/qsgd.h"
#include "qsgd_internal.h"

namespace {

constexpr size_t kStaticWorkspaceBytes = size_t(4) << 20;  // 4 MiB

// Zero at module load.  The scan state in it tags every entry with the call's
// epoch and the last CTA of each call resets the counters, so it never needs
// clearing between calls.
static __device__ __align__(256) unsigned char g_static_ws[kStaticWorkspaceBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_ws_ptr[kMaxDevices] = {};

// Device address of the array on the current device.  In host code the symbol
// g_static_ws is only a host-side stand-in, so the address is looked up once per
// device with that device current.
int static_ws_address(void** ptr) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return QSGD_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (g_ws_ptr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_ws) != cudaSuccess || p == nullptr) return QSGD_ERR_CUDA;
        g_ws_ptr[dev] = p;
    }
    *ptr = g_ws_ptr[dev];
    return QSGD_OK;
}

}  // namespace

extern "C" {

size_t qsgd_static_workspace_limit(void) { return kStaticWorkspaceBytes; }

int qsgd_encode_static_ws(const float* d_in, uint64_t n, uint32_t d, uint32_t s, uint64_t seed,
                          uint32_t* d_words, uint64_t words_capacity, uint64_t* d_offsets,
                          uint32_t* d_status, cudaStream_t stream) {
    // the one-pass encoders' scan state must fit; the two-launch encoder runs when its
    // staging fits as well
    const size_t need = qsgd::min_encode_workspace_bytes(n, d, s);
    if (need == 0) return QSGD_ERR_ARG;
    if (need > kStaticWorkspaceBytes) return QSGD_ERR_STATIC_LIMIT;
    void* ws = nullptr;
    const int rc = static_ws_address(&ws);
    if (rc != QSGD_OK) return rc;
    return qsgd::encode_entry(d_in, nullptr, n, d, s, seed, QSGD_NORM_L2, d_words, words_capacity, d_offsets, ws,
                              kStaticWorkspaceBytes, d_status, stream, false);
}

}  // extern "C"
