// Host emulation of the warp-level CUDA features the decoder kernels use, so that
// their exact source can run on a CPU in tests.  Every CUDA thread of a block is a
// std::thread; each warp primitive gathers all 32 lanes of the warp and checks that
// they stand at the same call site (on a GPU, lanes at different primitives
// deadlock; here that is reported as a failure, as is a rendezvous that times out).
#pragma once
#include <algorithm>
#include <atomic>
#include <chrono>
#include <condition_variable>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#define __device__
#define __host__
#define __global__
#define __forceinline__ inline
#define __launch_bounds__(...)
#define __grid_constant__
#define __align__(n) alignas(n)
#define __restrict__

typedef int cudaError_t;
typedef void* cudaStream_t;
enum { cudaSuccess = 0, cudaErrorInvalidConfiguration = 9 };
struct uint4 { uint32_t x, y, z, w; };
struct float4 { float x, y, z, w; };
inline float4 make_float4(float a, float b, float c, float d) { return float4{a, b, c, d}; }
inline uint4 make_uint4(uint32_t a, uint32_t b, uint32_t c, uint32_t d) { return uint4{a, b, c, d}; }
struct dim3e { unsigned x, y, z; };
extern thread_local dim3e threadIdx, blockIdx;
extern dim3e gridDim, blockDim;

template <class T> inline T __ldg(const T* p) { return *p; }
inline uint32_t __funnelshift_l(uint32_t lo, uint32_t hi, uint32_t sh) {
    const uint64_t x = ((static_cast<uint64_t>(hi) << 32) | lo) << (sh & 31u);
    return static_cast<uint32_t>(x >> 32);
}
inline float __fadd_rn(float a, float b) { volatile float r = a + b; return r; }
inline float __fsub_rn(float a, float b) { volatile float r = a - b; return r; }
inline float __fmul_rn(float a, float b) { volatile float r = a * b; return r; }
inline float __fdiv_rn(float a, float b) { volatile float r = a / b; return r; }
inline float __uint2float_rn(uint32_t u) { return static_cast<float>(u); }
inline float __uint_as_float(uint32_t u) { float f; std::memcpy(&f, &u, 4); return f; }
inline uint32_t __float_as_uint(float f) { uint32_t u; std::memcpy(&u, &f, 4); return u; }
using std::isfinite;
using std::min;
using std::max;
inline uint32_t atomicOr(uint32_t* p, uint32_t v) { return __atomic_fetch_or(p, v, __ATOMIC_SEQ_CST); }

// ---- shared memory of the current block --------------------------------
extern unsigned char* g_emu_smem;
inline uint32_t __cvta_generic_to_shared(const void* p) {
    return static_cast<uint32_t>(static_cast<const unsigned char*>(p) - g_emu_smem);
}
inline void emu_cp16(uint32_t dst, const void* src) { std::memcpy(g_emu_smem + dst, src, 16); }

// ---- warp rendezvous ------------------------------------------------------
struct WarpSync {
    std::mutex mu;
    std::condition_variable cv;
    int arrived = 0;
    uint64_t gen = 0;
    int site[32];
    uint64_t val[32];
    uint64_t out[32];
    int live = 32;
};
extern WarpSync* g_warps;
extern std::atomic<int> g_emu_error;
inline void emu_fail(const char* what, int line) {
    if (g_emu_error.exchange(1) == 0) std::fprintf(stderr, "EMU FAILURE: %s (line %d)\n", what, line);
}
// op: 0 any, 1 ballot, 2 max, 3 shfl_down, 4 shfl_up, 5 shfl idx, 6 syncwarp
inline uint64_t emu_warp(int op, int line, uint64_t v, int arg, int width) {
    const int lane = threadIdx.x & 31;
    WarpSync& w = g_warps[threadIdx.x >> 5];
    std::unique_lock<std::mutex> lk(w.mu);
    const uint64_t my_gen = w.gen;
    w.site[lane] = line * 8 + op;
    w.val[lane] = v;
    if (++w.arrived == 32) {
        for (int i = 1; i < 32; ++i)
            if (w.site[i] != w.site[0]) {
                char msg[128];
                std::snprintf(msg, sizeof msg, "lanes at different warp primitives: lane0 site %d, lane%d site %d",
                              w.site[0], i, w.site[i]);
                emu_fail(msg, line);
                break;
            }
        uint64_t any = 0, ballot = 0, mx = 0;
        for (int i = 0; i < 32; ++i) {
            any |= (w.val[i] != 0);
            ballot |= (w.val[i] != 0 ? 1ull : 0ull) << i;
            mx = std::max(mx, w.val[i]);
        }
        for (int i = 0; i < 32; ++i) {
            const int seg = i - (i % width), pos = i % width;
            switch (op) {
                case 0: w.out[i] = any; break;
                case 1: w.out[i] = ballot; break;
                case 2: w.out[i] = mx; break;
                case 3: w.out[i] = (pos + arg < width) ? w.val[i + arg] : w.val[i]; break;
                case 4: w.out[i] = (pos >= arg) ? w.val[i - arg] : w.val[i]; break;
                case 5: w.out[i] = w.val[seg + (arg % width)]; break;
                default: w.out[i] = 0;
            }
        }
        w.arrived = 0;
        ++w.gen;
        w.cv.notify_all();
    } else {
        if (!w.cv.wait_for(lk, std::chrono::seconds(20), [&] { return w.gen != my_gen; })) {
            emu_fail("warp rendezvous timed out (some lanes never arrived)", line);
            std::exit(3);
        }
    }
    return w.out[lane];
}
#define __any_sync(m, p) (emu_warp(0, __LINE__, (p) ? 1 : 0, 0, 32) != 0)
#define __all_sync(m, p) (emu_warp(0, __LINE__, (p) ? 0 : 1, 0, 32) == 0)
#define __ballot_sync(m, p) static_cast<uint32_t>(emu_warp(1, __LINE__, (p) ? 1 : 0, 0, 32))
#define __reduce_max_sync(m, v) static_cast<uint32_t>(emu_warp(2, __LINE__, static_cast<uint32_t>(v), 0, 32))
template <class T> inline T emu_cast(uint64_t x) { T t; std::memcpy(&t, &x, sizeof(T)); return t; }
template <class T> inline uint64_t emu_bits(T v) { uint64_t x = 0; std::memcpy(&x, &v, sizeof(T)); return x; }
#define __shfl_down_sync(m, v, d, ...) emu_cast<decltype(v)>(emu_warp(3, __LINE__, emu_bits(v), (d), emu_width(__VA_ARGS__)))
#define __shfl_up_sync(m, v, d, ...) emu_cast<decltype(v)>(emu_warp(4, __LINE__, emu_bits(v), (d), emu_width(__VA_ARGS__)))
#define __shfl_sync(m, v, s, ...) emu_cast<decltype(v)>(emu_warp(5, __LINE__, emu_bits(v), (s), emu_width(__VA_ARGS__)))
#define __shfl_xor_sync(m, v, x, ...) EMU_NO_XOR
#define __syncwarp(...) ((void)emu_warp(6, __LINE__, 0, 0, 32))
inline int emu_width() { return 32; }
inline int emu_width(int w) { return w; }
void __syncthreads();
