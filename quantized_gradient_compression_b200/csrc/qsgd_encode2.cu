// Two-pass QSGD encoder for the fast shapes (d = 128 V): an alternative to
// encode_fast, compiled in but off unless QSGD_ENCODER_TWO_PASS is set.
//
// Same stream as encode_fast (the wire format of the definition paragraph of "QSGD
// (Quantized Stochastic Gradient Descent) with Elias Coding", AIMech curated entry),
// in three launches instead of one:
//   A. one warp per bucket: norm, Philox words, levels, the bucket's record list
//      (idx | k << 10 | sign << 31) and its bit count, into a scratch area;
//   S. one CTA: the exclusive scan of the bit counts gives the offsets header; the
//      words two buckets share (a bucket whose first bit is not on a word boundary)
//      are zeroed;
//   C. one warp per bucket: omega-codes the record list, assembles the bucket's
//      bits in shared memory and stores them at its offset (atomic OR on the two
//      words it may share with its neighbours, plain stores elsewhere).
// No tile waits for another tile's prefix; the price is a second pass over the
// records (about 2.2 bytes per coordinate at s = 16) and 4 n bytes of scratch.
#include <cuda_runtime.h>

#include <algorithm>

#include "../../include/qsgd.h"
#include "qsgd_device.cuh"
#include "qsgd_internal.h"

namespace qsgd {
namespace {

constexpr uint32_t kWarpAll = 0xFFFFFFFFu;
constexpr int kE2Warps = 16;
constexpr int kE2Block = 32 * kE2Warps;
constexpr int kScanBlock = 1024;

struct Enc2Args {
    const float* in;
    uint64_t n;
    uint32_t d, s, key0, key1, norm_kind;
    uint64_t nb;
    uint32_t* recs;     // bucket b's records at recs + b d: idx | k << 10 | sign << 31
    uint32_t* nz;       // records per bucket
    uint32_t* bits;     // bits per bucket (32 + its records)
    float* norms;       // sent norm per bucket
    uint64_t* offsets;  // nb + 1
    uint32_t* words;
    uint64_t cap_words;
    uint32_t* status;
    uint32_t bucket_words;  // words of one bucket's staging buffer (its bits, or its record list)
};

// Pass A: one warp per bucket.  Norm, levels, the record list, the bit count.
template <int V>
__global__ void __launch_bounds__(kE2Block) enc2_levels(const __grid_constant__ Enc2Args a) {
    extern __shared__ __align__(16) uint32_t smem[];
    uint32_t* const otab = smem;  // omega code table
    constexpr int NC = 4 * V;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint32_t* const slist = smem + kOmegaTab + warp * 128 * V;  // this warp's record list
    omega_table_fill(otab, tid, kE2Block);
    __syncthreads();
    const PhiloxKey key{a.key0, a.key1};
    const uint64_t gw = static_cast<uint64_t>(gridDim.x) * kE2Warps;
    for (uint64_t b = static_cast<uint64_t>(blockIdx.x) * kE2Warps + warp; b < a.nb; b += gw) {
        const uint64_t base = b * a.d;
        const uint32_t m = static_cast<uint32_t>(min(static_cast<uint64_t>(a.d), a.n - base));
        const uint32_t first = static_cast<uint32_t>(lane) * NC;
        float x[NC];
#pragma unroll
        for (int j = 0; j < V; ++j) {
            const uint32_t i = first + 4 * j;
            float4 q = make_float4(0.f, 0.f, 0.f, 0.f);
            if (i + 4 <= m) {
                q = __ldg(reinterpret_cast<const float4*>(a.in + base + i));
            } else if (i < m) {
                q.x = a.in[base + i];
                if (i + 1 < m) q.y = a.in[base + i + 1];
                if (i + 2 < m) q.z = a.in[base + i + 2];
            }
            x[4 * j + 0] = q.x;
            x[4 * j + 1] = q.y;
            x[4 * j + 2] = q.z;
            x[4 * j + 3] = q.w;
        }
        const float norm = a.norm_kind == QSGD_NORM_MAX ? warp_bucket_maxnorm<NC>(x) : warp_bucket_norm<NC>(x, true);
        const BucketScale sc = bucket_scale(norm, a.s, true, a.status, lane == 0);
        uint32_t kq[NC];
#pragma unroll
        for (int j = 0; j < V; ++j) {
            const uint4 r = philox4x32_10(((base + first) >> 2) + j, key);
            const uint32_t rw[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float v = x[4 * j + c];
                kq[4 * j + c] = sc.good ? (quantize_level(v, sc.sinv, rw[c], a.s) | (__float_as_uint(v) & 0x80000000u))
                                        : 0u;
            }
        }
        // records of this lane, in index order, and the last one's index
        uint32_t cnt = 0;
        int32_t last = -1;
#pragma unroll
        for (int q = 0; q < NC; ++q)
            if (kq[q] & 0x7FFFFFFFu) {
                ++cnt;
                last = static_cast<int32_t>(first + q);
            }
        uint32_t incl = cnt;
        int32_t lmax = last;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t t = __shfl_up_sync(kWarpAll, incl, o);
            const int32_t u = __shfl_up_sync(kWarpAll, lmax, o);
            if (lane >= o) {
                incl += t;
                lmax = max(lmax, u);
            }
        }
        int32_t prev = __shfl_up_sync(kWarpAll, lmax, 1);  // the last record before this lane's
        if (lane == 0) prev = -1;
        uint32_t pos = incl - cnt, lbits = 0;
#pragma unroll
        for (int q = 0; q < NC; ++q) {
            const uint32_t k = kq[q] & 0x7FFFFFFFu;
            if (k) {
                const uint32_t i = first + q;
                slist[pos++] = i | (k << 10) | (kq[q] & 0x80000000u);
                lbits += omega_len(otab, static_cast<uint64_t>(static_cast<int32_t>(i) - prev)) + 1u + omega_len(otab, k);
                prev = static_cast<int32_t>(i);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) lbits += __shfl_xor_sync(kWarpAll, lbits, o);
        const uint32_t nzb = __shfl_sync(kWarpAll, incl, 31);
        __syncwarp();  // the list is complete
        uint32_t* rec = a.recs + base;
        for (uint32_t r = lane; r < nzb; r += 32) rec[r] = slist[r];
        __syncwarp();  // the list is free for the next bucket
        if (lane == 0) {
            a.nz[b] = nzb;
            a.bits[b] = 32u + lbits;
            a.norms[b] = sc.sent;
        }
    }
}

// Pass S: offsets = exclusive scan of the bucket sizes; zero the words that two
// buckets share (their first bit is not on a word boundary).  One CTA.
__global__ void __launch_bounds__(kScanBlock) enc2_scan(const __grid_constant__ Enc2Args a) {
    __shared__ uint64_t s_part[kScanBlock];
    const int tid = threadIdx.x;
    const uint64_t per = (a.nb + kScanBlock - 1) / kScanBlock;
    const uint64_t b0 = min(a.nb, per * tid), b1 = min(a.nb, b0 + per);
    uint64_t sum = 0;
    for (uint64_t b = b0; b < b1; ++b) sum += a.bits[b];
    s_part[tid] = sum;
    __syncthreads();
    // inclusive scan of the partial sums (Hillis-Steele over the block)
    for (int o = 1; o < kScanBlock; o <<= 1) {
        const uint64_t t = tid >= o ? s_part[tid - o] : 0u;
        __syncthreads();
        s_part[tid] += t;
        __syncthreads();
    }
    uint64_t run = s_part[tid] - sum;
    for (uint64_t b = b0; b < b1; ++b) {
        a.offsets[b] = run;
        if ((run & 31u) && (run >> 5) < a.cap_words) a.words[run >> 5] = 0u;
        run += a.bits[b];
    }
    if (tid == kScanBlock - 1) {
        a.offsets[a.nb] = run;
        if ((run & 31u) && (run >> 5) < a.cap_words) a.words[run >> 5] = 0u;
        if (run > a.cap_words * 32) report(a.status, QSGD_ST_OVERFLOW);
    }
}

// Pass C: one warp per bucket.  Code the record list, assemble the bucket's bits
// in shared memory and store them at its offset (atomic OR on the two words it may
// share with its neighbours).
template <int V, bool kShort>
__global__ void __launch_bounds__(kE2Block) enc2_pack(const __grid_constant__ Enc2Args a) {
    extern __shared__ __align__(16) uint32_t smem[];
    uint32_t* const rtab = smem;
    uint32_t* const bufs = smem + kRecordTab;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint32_t* const buf = bufs + warp * a.bucket_words;
    uint32_t* const pb = bufs + kE2Warps * a.bucket_words + warp * 32 * fast_lane_words(V, kShort) + lane;
    record_table_fill(rtab, tid, kE2Block);
    __syncthreads();
    const uint64_t gw = static_cast<uint64_t>(gridDim.x) * kE2Warps;
    for (uint64_t b = static_cast<uint64_t>(blockIdx.x) * kE2Warps + warp; b < a.nb; b += gw) {
        const uint32_t nz = a.nz[b];
        const uint32_t nbits = a.bits[b];
        const uint64_t o = a.offsets[b];
        const uint32_t* grec = a.recs + b * a.d;
        for (uint32_t r = lane; r < nz; r += 32) buf[r] = grec[r];  // the list, staged in buf
        __syncwarp();
        const uint32_t* rec = buf;
        // this lane's run of records into its strip
        LanePacker pk{pb, 0u, 0u, 0u};
        const uint32_t per = (nz + 31) >> 5;
        const uint32_t r0 = min(nz, lane * per), r1 = min(nz, r0 + per);
        uint32_t prev = r0 ? (rec[r0 - 1] & 1023u) : 0xFFFFFFFFu;
        for (uint32_t r = r0; r < r1; ++r) {
            const uint32_t e = rec[r];
            const uint32_t i = e & 1023u;
            const uint32_t k = (e >> 10) & 0x1FFFFFu;
            const uint32_t gap = i - prev;
            prev = i;
            if (gap < 64u && k < 16u) {
                const uint32_t re = rtab[(gap << 5) | (k << 1) | (e >> 31)];
                pk.put(re >> 5, re & 31u);
            } else {
                uint64_t gc, kc;
                uint32_t gl, kl;
                omega_code_global(gap, gc, gl);
                omega_code_global(k, kc, kl);
                pk.put((static_cast<uint32_t>(gc) << 1) | (e >> 31), gl + 1u);
                if (kl > 32) pk.put(static_cast<uint32_t>(kc >> 32), kl - 32u);
                pk.put(static_cast<uint32_t>(kc), kl > 32 ? 32u : kl);
            }
        }
        pk.finish();
        const uint32_t lb = pk.bits();
        __syncwarp();  // every lane has read its run: buf takes the bucket's bits next
        uint32_t incl = lb;
#pragma unroll
        for (int s = 1; s < 32; s <<= 1) {
            const uint32_t t = __shfl_up_sync(kWarpAll, incl, s);
            if (lane >= s) incl += t;
        }
        const uint32_t pos = 32u + incl - lb;  // bucket-local bit of this lane's first record
        // the bucket's bits, word by word, in the warp's buffer
        const uint32_t bw = (nbits + 31) >> 5;
        for (uint32_t j = lane; j < bw; j += 32) buf[j] = 0u;
        __syncwarp();
        if (lane == 0) buf[0] = __float_as_uint(a.norms[b]);
        {
            const uint32_t w = pos >> 5, sh = pos & 31u;
            const uint32_t nsrc = (lb + 31u) >> 5, ndst = (sh + lb + 31u) >> 5;
            uint32_t prv = 0;
            for (uint32_t j = 0; j < ndst; ++j) {
                const uint32_t cur = j < nsrc ? pb[32 * j] : 0u;
                const uint32_t v = sh ? (cur >> sh) | (prv << (32 - sh)) : cur;
                if (v) atomicOr(&buf[w + j], v);
                prv = cur;
            }
        }
        __syncwarp();
        // store at the global offset o
        if (o + nbits > a.cap_words * 32) {
            if (lane == 0) report(a.status, QSGD_ST_OVERFLOW);
        } else {
            const uint64_t g0 = o >> 5;
            const uint32_t sh = static_cast<uint32_t>(o & 31u);
            const uint32_t gw_n = (sh + nbits + 31u) >> 5;  // global words touched
            const bool shared_last = ((o + nbits) & 31u) != 0;
            for (uint32_t j = lane; j < gw_n; j += 32) {
                const uint32_t cur = j < bw ? buf[j] : 0u;
                const uint32_t pre = (j > 0 && j - 1 < bw) ? buf[j - 1] : 0u;
                const uint32_t v = sh ? (cur >> sh) | (pre << (32 - sh)) : cur;
                const bool shared = (j == 0 && sh != 0) || (j + 1 == gw_n && shared_last);
                if (shared)
                    atomicOr(&a.words[g0 + j], v);
                else
                    a.words[g0 + j] = v;
            }
        }
        __syncwarp();  // buf and the strips are reused by the next bucket
    }
}

template <int V>
cudaError_t launch_v(const Enc2Args& a, int grid, cudaStream_t stream) {
    const size_t smem_a = (static_cast<size_t>(kOmegaTab) + static_cast<size_t>(kE2Warps) * 128 * V) * sizeof(uint32_t);
    cudaFuncSetAttribute(enc2_levels<V>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    enc2_levels<V><<<grid, kE2Block, smem_a, stream>>>(a);
    enc2_scan<<<1, kScanBlock, 0, stream>>>(a);
    const bool sh = a.s <= 31;
    const size_t smem = (static_cast<size_t>(kRecordTab) + static_cast<size_t>(kE2Warps) * a.bucket_words +
                         static_cast<size_t>(kE2Warps) * 32 * fast_lane_words(V, sh)) * sizeof(uint32_t);
    if (smem > 200 * 1024) return cudaErrorInvalidValue;
    if (sh) {
        cudaFuncSetAttribute(enc2_pack<V, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
        enc2_pack<V, true><<<grid, kE2Block, smem, stream>>>(a);
    } else {
        cudaFuncSetAttribute(enc2_pack<V, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
        enc2_pack<V, false><<<grid, kE2Block, smem, stream>>>(a);
    }
    return cudaGetLastError();
}

}  // namespace

bool encode2_fits(uint32_t d, uint32_t s) {
    const uint32_t V = fast_v(d);
    const uint64_t bw = std::max<uint64_t>((32u + static_cast<uint64_t>(d) * (2u + omega_len_host(s)) + 31) / 32 + 1, d);
    const uint64_t words_c = kRecordTab + kE2Warps * bw + static_cast<uint64_t>(kE2Warps) * 32 * fast_lane_words(V, s <= 31);
    const uint64_t words_a = kOmegaTab + static_cast<uint64_t>(kE2Warps) * 128 * V;
    return std::max(words_a, words_c) * sizeof(uint32_t) <= 200 * 1024;
}

size_t encode2_scratch_bytes(uint64_t n, uint32_t d) {
    const uint64_t nb = (n + d - 1) / d;
    return sizeof(uint32_t) * (nb * d + 3 * nb) + 256;
}

cudaError_t launch_encode2(const EncodeArgs& e, void* scratch, cudaStream_t stream) {
    Enc2Args a{};
    a.in = e.in;
    a.n = e.n;
    a.d = e.d;
    a.s = e.s;
    a.key0 = e.key0;
    a.key1 = e.key1;
    a.norm_kind = e.norm_kind;
    a.nb = e.nb;
    uint32_t* p = static_cast<uint32_t*>(scratch);
    a.recs = p;
    a.nz = p + e.nb * e.d;
    a.bits = a.nz + e.nb;
    a.norms = reinterpret_cast<float*>(a.bits + e.nb);
    a.offsets = e.offsets;
    a.words = e.words;
    a.cap_words = e.cap_words;
    a.status = e.status;
    // a bucket's bits, or its record list before them
    a.bucket_words = static_cast<uint32_t>(std::max<uint64_t>(
        (32u + static_cast<uint64_t>(e.d) * (2u + omega_len_host(e.s)) + 31) / 32 + 1, e.d));
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const uint64_t want = (e.nb + kE2Warps - 1) / kE2Warps;
    const int grid = static_cast<int>(std::max<uint64_t>(1, std::min<uint64_t>(want, static_cast<uint64_t>(sms) * 4)));
    switch (fast_v(e.d)) {
        case 1: return launch_v<1>(a, grid, stream);
        case 2: return launch_v<2>(a, grid, stream);
        case 4: return launch_v<4>(a, grid, stream);
        default: return launch_v<8>(a, grid, stream);
    }
}

}  // namespace qsgd
