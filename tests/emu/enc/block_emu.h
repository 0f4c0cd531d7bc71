// Host emulation of the CUDA features the encoder kernels use, so that their exact
// source runs on a CPU in tests.  A whole grid runs at once, every CUDA thread a
// std::thread, because the encoder's CTAs hand tiles to one another (a ticket, and
// prefixes that later tiles wait for).  Each block has its own shared memory, warp
// rendezvous and barrier.  A warp primitive gathers all 32 lanes and checks that they
// stand at the same call site; a rendezvous or barrier that waits too long is
// reported as a failure (on a GPU it would hang).
#pragma once
#include <algorithm>
#include <atomic>
#include <cfenv>
#include <chrono>
#include <cmath>
#include <condition_variable>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <memory>
#include <mutex>
#include <thread>
#include <type_traits>
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
enum { cudaSuccess = 0, cudaErrorInvalidConfiguration = 9, cudaErrorInvalidValue = 1 };
struct uint2 { uint32_t x, y; };
struct uint4 { uint32_t x, y, z, w; };
struct float2 { float x, y; };
struct float4 { float x, y, z, w; };
inline float2 make_float2(float a, float b) { return float2{a, b}; }
inline float4 make_float4(float a, float b, float c, float d) { return float4{a, b, c, d}; }
inline uint4 make_uint4(uint32_t a, uint32_t b, uint32_t c, uint32_t d) { return uint4{a, b, c, d}; }
inline uint2 make_uint2(uint32_t a, uint32_t b) { return uint2{a, b}; }
struct dim3e { unsigned x, y, z; };
extern thread_local dim3e threadIdx, blockIdx;
extern dim3e gridDim, blockDim;

// ---- arithmetic with the rounding the names give --------------------------------
inline float __fadd_rn(float a, float b) { volatile float r = a + b; return r; }
inline float __fsub_rn(float a, float b) { volatile float r = a - b; return r; }
inline float __fmul_rn(float a, float b) { volatile float r = a * b; return r; }
inline float __fdiv_rn(float a, float b) { volatile float r = a / b; return r; }
inline float __fsqrt_rn(float a) { volatile float r = std::sqrt(a); return r; }
inline float __fmaf_rn(float a, float b, float c) { volatile float r = std::fma(a, b, c); return r; }
inline float __fadd_rd(float a, float b) {
    const int old = std::fegetround();
    std::fesetround(FE_DOWNWARD);
    volatile float x = a, y = b;
    volatile float r = x + y;
    std::fesetround(old);
    return r;
}
inline float __fadd_ru(float a, float b) {
    const int old = std::fegetround();
    std::fesetround(FE_UPWARD);
    volatile float x = a, y = b;
    volatile float r = x + y;
    std::fesetround(old);
    return r;
}
// the high word of (hi:lo) << (sh mod 32)
inline uint32_t __funnelshift_l(uint32_t lo, uint32_t hi, uint32_t sh) {
    const uint64_t x = (static_cast<uint64_t>(hi) << 32) | lo;
    return static_cast<uint32_t>((x << (sh & 31u)) >> 32);
}
// the low word of (hi:lo) >> (sh mod 32)
inline uint32_t __funnelshift_r(uint32_t lo, uint32_t hi, uint32_t sh) {
    const uint64_t x = (static_cast<uint64_t>(hi) << 32) | lo;
    return static_cast<uint32_t>(x >> (sh & 31u));
}
inline float __uint2float_rn(uint32_t u) { return static_cast<float>(u); }
inline float __uint_as_float(uint32_t u) { float f; std::memcpy(&f, &u, 4); return f; }
inline uint32_t __float_as_uint(float f) { uint32_t u; std::memcpy(&u, &f, 4); return u; }
inline int __clz(uint32_t x) { return x ? __builtin_clz(x) : 32; }
inline int __clzll(uint64_t x) { return x ? __builtin_clzll(x) : 64; }
inline int __ffs(uint32_t x) { return __builtin_ffs(static_cast<int>(x)); }
inline int __popc(uint32_t x) { return __builtin_popcount(x); }
using std::isfinite;
using std::isnan;
using std::isinf;
using std::signbit;
using std::min;
using std::max;

// ---- global memory -------------------------------------------------------------
template <class T> inline T __ldg(const T* p) { return *p; }
template <class T> inline T __ldcs(const T* p) { return *p; }
template <class T> inline void __stcs(T* p, T v) { *p = v; }
inline uint32_t atomicOr(uint32_t* p, uint32_t v) { return __atomic_fetch_or(p, v, __ATOMIC_SEQ_CST); }
inline int atomicOr(int* p, int v) { return __atomic_fetch_or(p, v, __ATOMIC_SEQ_CST); }
inline uint32_t atomicAdd(uint32_t* p, uint32_t v) { return __atomic_fetch_add(p, v, __ATOMIC_SEQ_CST); }
inline unsigned long long atomicAdd(unsigned long long* p, unsigned long long v) {
    return __atomic_fetch_add(p, v, __ATOMIC_SEQ_CST);
}
inline uint32_t atomicMin(uint32_t* p, uint32_t v) {
    uint32_t cur = __atomic_load_n(p, __ATOMIC_SEQ_CST);
    while (v < cur && !__atomic_compare_exchange_n(p, &cur, v, false, __ATOMIC_SEQ_CST, __ATOMIC_SEQ_CST)) {
    }
    return cur;
}
inline uint32_t atomicExch(uint32_t* p, uint32_t v) { return __atomic_exchange_n(p, v, __ATOMIC_SEQ_CST); }
inline unsigned long long atomicCAS(unsigned long long* p, unsigned long long cmp, unsigned long long v) {
    __atomic_compare_exchange_n(p, &cmp, v, false, __ATOMIC_SEQ_CST, __ATOMIC_SEQ_CST);
    return cmp;
}
inline void __threadfence() { __atomic_thread_fence(__ATOMIC_SEQ_CST); }
// host helpers that size grids ask for the device: one B200-sized answer
enum { cudaDevAttrMultiProcessorCount = 16 };
inline cudaError_t cudaGetDevice(int* dev) { *dev = 0; return cudaSuccess; }
inline cudaError_t cudaDeviceGetAttribute(int* v, int, int) { *v = 148; return cudaSuccess; }
inline void __nanosleep(unsigned) { std::this_thread::yield(); }

// ---- one block's state ---------------------------------------------------------
struct WarpSync {
    std::mutex mu;
    std::condition_variable cv;
    int arrived = 0;
    uint64_t gen = 0;
    int site[32];
    int arg[32];
    uint64_t val[32];
    uint64_t out[32];
};
struct BlockCtx {
    std::vector<unsigned char> smem;  // dynamic shared memory
    WarpSync warps[32];
    std::mutex bmu;
    std::condition_variable bcv;
    int arrived = 0;
    uint64_t gen = 0;
    int or_acc = 0, or_out = 0;
    std::mutex smu;  // static shared variables, one per declaration
    std::map<int, std::unique_ptr<unsigned char[]>> statics;
};
extern thread_local BlockCtx* t_blk;
extern std::atomic<int> g_emu_error;
inline void emu_fail(const char* what, int line) {
    if (g_emu_error.exchange(1) == 0) std::fprintf(stderr, "EMU FAILURE: %s (line %d)\n", what, line);
}
template <class T> inline T& emu_shared(int key) {
    std::lock_guard<std::mutex> lk(t_blk->smu);
    auto& slot = t_blk->statics[key];
    if (!slot) {
        slot.reset(new unsigned char[sizeof(T) + 16]);
        std::memset(slot.get(), 0xAB, sizeof(T) + 16);
    }
    return *reinterpret_cast<T*>(slot.get());
}
inline unsigned char* emu_smem() { return t_blk->smem.data(); }
inline uint32_t __cvta_generic_to_shared(const void* p) {
    return static_cast<uint32_t>(static_cast<const unsigned char*>(p) - emu_smem());
}
// cp.async with its source size: the first `src_bytes` bytes copied, the rest zeroed
inline void emu_cp16z(uint32_t dst, const void* src, uint32_t src_bytes) {
    if ((dst & 15u) != 0 || (reinterpret_cast<uintptr_t>(src) & 15u) != 0) emu_fail("cp.async of 16 bytes not 16-byte aligned", __LINE__);
    std::memset(emu_smem() + dst, 0, 16);
    std::memcpy(emu_smem() + dst, src, src_bytes);
}
inline void emu_cp16(uint32_t dst, const void* src) { emu_cp16z(dst, src, 16); }
inline void emu_cp4(uint32_t dst, const void* src) { std::memcpy(emu_smem() + dst, src, 4); }

// op: 0 any, 1 ballot, 4 shfl_up, 5 shfl idx, 6 syncwarp, 7 shfl_xor
inline uint64_t emu_warp(int op, int line, uint64_t v, int arg, int width) {
    const int lane = threadIdx.x & 31;
    WarpSync& w = t_blk->warps[threadIdx.x >> 5];
    std::unique_lock<std::mutex> lk(w.mu);
    const uint64_t my_gen = w.gen;
    w.site[lane] = line * 8 + (op & 7);
    w.val[lane] = v;
    w.arg[lane] = arg;
    if (++w.arrived == 32) {
        for (int i = 1; i < 32; ++i)
            if (w.site[i] != w.site[0]) {
                char msg[128];
                std::snprintf(msg, sizeof msg, "lanes at different warp primitives: lane0 site %d, lane%d site %d",
                              w.site[0], i, w.site[i]);
                emu_fail(msg, line);
                break;
            }
        uint64_t any = 0, ballot = 0;
        for (int i = 0; i < 32; ++i) {
            any |= (w.val[i] != 0);
            ballot |= (w.val[i] != 0 ? 1ull : 0ull) << i;
        }
        for (int i = 0; i < 32; ++i) {
            const int seg = i - (i % width), pos = i % width;
            switch (op) {
                case 0: w.out[i] = any; break;
                case 1: w.out[i] = ballot; break;
                // each lane's own offset, source lane or mask
                case 4: w.out[i] = (pos >= w.arg[i]) ? w.val[i - w.arg[i]] : w.val[i]; break;
                case 5: w.out[i] = w.val[seg + (w.arg[i] % width)]; break;
                case 7: w.out[i] = ((pos ^ w.arg[i]) < width) ? w.val[seg + (pos ^ w.arg[i])] : w.val[i]; break;
                default: w.out[i] = 0;
            }
        }
        w.arrived = 0;
        ++w.gen;
        w.cv.notify_all();
    } else if (!w.cv.wait_for(lk, std::chrono::seconds(60), [&] { return w.gen != my_gen; })) {
        emu_fail("warp rendezvous timed out (some lanes never arrived)", line);
        std::exit(3);
    }
    return w.out[lane];
}
template <class T> inline std::remove_cv_t<T> emu_cast(uint64_t x) {
    std::remove_cv_t<T> t;
    std::memcpy(&t, &x, sizeof(T));
    return t;
}
template <class T> inline uint64_t emu_bits(T v) { uint64_t x = 0; std::memcpy(&x, &v, sizeof(T)); return x; }
inline int emu_width() { return 32; }
inline int emu_width(int w) { return w; }
#define __any_sync(m, p) (emu_warp(0, __LINE__, (p) ? 1 : 0, 0, 32) != 0)
#define __ballot_sync(m, p) static_cast<uint32_t>(emu_warp(1, __LINE__, (p) ? 1 : 0, 0, 32))
#define __shfl_up_sync(m, v, d, ...) emu_cast<decltype(v)>(emu_warp(4, __LINE__, emu_bits(v), (d), emu_width(__VA_ARGS__)))
#define __shfl_sync(m, v, s, ...) emu_cast<decltype(v)>(emu_warp(5, __LINE__, emu_bits(v), (s), emu_width(__VA_ARGS__)))
#define __shfl_xor_sync(m, v, x, ...) emu_cast<decltype(v)>(emu_warp(7, __LINE__, emu_bits(v), (x), emu_width(__VA_ARGS__)))
#define __syncwarp(...) ((void)emu_warp(6, __LINE__, 0, 0, 32))

inline int emu_barrier(int pred) {
    BlockCtx& b = *t_blk;
    std::unique_lock<std::mutex> lk(b.bmu);
    const uint64_t gen = b.gen;
    b.or_acc |= pred ? 1 : 0;
    if (++b.arrived == static_cast<int>(blockDim.x)) {
        b.arrived = 0;
        b.or_out = b.or_acc;
        b.or_acc = 0;
        ++b.gen;
        b.bcv.notify_all();
    } else if (!b.bcv.wait_for(lk, std::chrono::seconds(60), [&] { return b.gen != gen; })) {
        emu_fail("__syncthreads timed out", 0);
        std::exit(3);
    }
    return b.or_out;
}
inline void __syncthreads() { (void)emu_barrier(0); }
inline int __syncthreads_or(int p) { return emu_barrier(p); }
