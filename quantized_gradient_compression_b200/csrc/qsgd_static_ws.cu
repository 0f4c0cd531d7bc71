// qsgd_encode_static_ws: the encoder for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc at the point where they compress a gradient:
// code running inside a caching allocator's own hooks, a communication library's
// progress thread that must not take the allocator lock, or an embedding that only
// hands the codec its input and output buffers.  For them the encoder's scan state
// lives in a fixed array of device memory owned by this library.  The array is a
// file-scope static device variable: every GPU that loads the library holds it
// (kStaticWorkspaceBytes) until the process exits.  Nothing here allocates.
#include <cuda.h>
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

// The array's address is cached per device together with the ID of the CUDA context
// it was looked up in: after a cudaDeviceReset the device's next context loads the
// module again, possibly at another address, so a new context ID means a new lookup.
struct CachedAddress {
    unsigned long long ctx_id;
    void* ptr;
};
CachedAddress g_ws[kMaxDevices] = {};

// The current context's ID, through the driver entry points the runtime hands out
// (no link against the driver library).  0 when it cannot be had.
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);
unsigned long long current_context_id() {
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    if (!get_current || !get_id) {
        cudaDriverEntryPointQueryResult q1, q2;
        void* f1 = nullptr;
        void* f2 = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1) != cudaSuccess ||
            cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &q2) != cudaSuccess ||
            q1 != cudaDriverEntryPointSuccess || q2 != cudaDriverEntryPointSuccess || !f1 || !f2)
            return 0;
        get_current = reinterpret_cast<CtxGetCurrentFn>(f1);
        get_id = reinterpret_cast<CtxGetIdFn>(f2);
    }
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

// Device address of the array on the current device.  In host code the symbol
// g_static_ws is only a host-side stand-in, so the address is looked up with the
// device current: once per device and context (twice when the first call comes
// before the runtime has made the device's context current: that lookup makes it
// current, and the next call caches the address under the context's ID).
int static_ws_address(void** ptr) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return QSGD_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    const unsigned long long id = current_context_id();
    if (g_ws[dev].ptr == nullptr || id == 0 || g_ws[dev].ctx_id != id) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_ws) != cudaSuccess || p == nullptr) return QSGD_ERR_CUDA;
        g_ws[dev].ptr = p;
        g_ws[dev].ctx_id = id;
    }
    *ptr = g_ws[dev].ptr;
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
