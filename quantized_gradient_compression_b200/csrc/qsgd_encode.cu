// QSGD encoder kernels (sm_100a).
//
// Method: "QSGD (Quantized Stochastic Gradient Descent) with Elias Coding" (AIMech
// curated entry).  Per bucket (claim "QSVRG, non-convex and multi-GPU bucketed
// training", section 3.3 bucketing): the L2 norm, unbiased stochastic rounding of
// every coordinate to one of s+1 levels (definition paragraph), and the Elias-omega
// coding of the tuple (norm, signs, run-length gaps, levels) (definition paragraph;
// claim "Elias coding communication complexity tradeoff", F = 32).
//
// Single pass over the input.  The stream position of every tile comes from a
// prefix scan with decoupled look-back (Merrill & Garland 2016): each tile publishes
// its bit count, then its inclusive prefix; tiles are handed out in order by an
// atomic ticket so every wait is on a tile that is already running.  A tile's bits
// are assembled in shared memory at tile-local offsets and stored with a funnel
// shift once the prefix is known; the one word a tile shares with its predecessor
// is written by the later tile, from the predecessor's published tail word, so
// every output word has exactly one writer and the output needs no clearing.
//
// Two kernels:
//   encode_fast<V>   128 <= d <= 1024, d % 4 == 0, 16-byte aligned input: one warp
//                    per bucket, lane-contiguous 4V coordinates in registers,
//                    8 buckets per tile, persistent CTAs.
//   encode_general   any d and alignment: a norm pre-pass (one warp per bucket),
//                    then tiles of whole buckets (>= 4096 coordinates or one
//                    bucket) streamed in chunks of 1024 coordinates, twice (bit
//                    count, then packing).
#include <cuda_runtime.h>

#include <algorithm>

#include "../../include/qsgd.h"
#include "qsgd_device.cuh"
#include "qsgd_internal.h"

namespace qsgd {
namespace {

constexpr uint32_t kFull = 0xFFFFFFFFu;

__device__ __forceinline__ void store_word(const EncodeArgs& a, uint64_t gw, uint32_t v) {
    if (gw < a.cap_words)
        a.words[gw] = v;
    else
        report(a.status, QSGD_ST_OVERFLOW);
}

__device__ __forceinline__ void abort_all(const EncodeArgs& a) {
    report(a.status, QSGD_ST_LOOKBACK_TIMEOUT);
    atomicExch(&a.ctrl->abort, 1u);
}

// Last CTA out resets the ticket and completion counters and advances the epoch.
__device__ __forceinline__ void cta_exit(ScanControl* ctrl, uint32_t epoch) {
    if (threadIdx.x == 0) {
        __threadfence();
        const uint32_t prev = atomicAdd(&ctrl->done, 1u);
        if (prev == gridDim.x - 1) {
            ctrl->ticket = 0;
            ctrl->done = 0;
            ctrl->abort = 0;
            __threadfence();
            atomicExch(&ctrl->epoch, (epoch + 1) & kEpochMask);
        }
    }
}

// ---------------------------------------------------------------------------
// Fast path (128 <= d <= 128*V, d % 4 == 0, s < 2^21, 16-byte aligned input).
//
// Tiles of kFastWarps consecutive buckets, one bucket per warp; lane L codes the 4V
// consecutive coordinates [4VL, 4VL+4V) of its bucket.  CTAs draw tiles from an
// atomic ticket, in order.  Stream positions come from a two-level scan that never
// walks a chain: rounds are C consecutive tickets (C = grid size); a tile publishes
// its bit count A(t) as soon as it is known, and its exclusive prefix is the
// previous round's total RP(r-1) plus the sum of A over its round's earlier tiles,
// read in parallel; the round's last tile publishes RP(r).  A tile only waits on
// tiles with smaller tickets, which are held by running CTAs.  Each CTA codes its
// next tile into the second of two tile buffers before it waits for the current
// tile's prefix, and copies the input of the tile after that into shared memory
// with cp.async while it works.  The one word two neighbouring tiles share is
// merged through a slot: whichever tile comes second writes it, nobody waits.
// ---------------------------------------------------------------------------
struct TileSlot {
    uint32_t bits[kFastWarps];  // bits of each bucket of the tile
    uint64_t total;         // bits of the tile
};

// Slot of the word shared by tiles t-1 and t: [63:40] epoch, [32] present,
// [31:0] the first writer's bits.  The second writer ORs its bits in and stores
// the word; a zero-filled slot or one from an earlier call reads as empty.
__device__ __forceinline__ void merge_shared_word(const EncodeArgs& a, uint64_t* slot, uint64_t gw,
                                                  uint32_t bits, uint32_t epoch) {
    const uint64_t mine = (static_cast<uint64_t>(epoch & kEpochMask) << 40) | (uint64_t(1) << 32) | bits;
    uint64_t cur = ld_acquire(slot);
    for (int attempt = 0; attempt < 4; ++attempt) {
        if (static_cast<uint32_t>(cur >> 40) == (epoch & kEpochMask) && ((cur >> 32) & 1u)) {
            store_word(a, gw, bits | static_cast<uint32_t>(cur));
            return;
        }
        const unsigned long long prev = atomicCAS(reinterpret_cast<unsigned long long*>(slot),
                                                  static_cast<unsigned long long>(cur),
                                                  static_cast<unsigned long long>(mine));
        if (prev == cur) return;  // first: the other tile writes the word
        cur = prev;
    }
    abort_all(a);  // unreachable with two writers per slot
}

// Copies the input of tile t into `xin` (cp.async, 16 bytes per copy).  Lane L of
// warp w takes float4 j of its coordinates to slot L*V + (j ^ swz(L)), so that the
// later 16-byte reads (lane L, slot j) fall in distinct bank groups.
template <int V>
__device__ __forceinline__ void prefetch_tile(const EncodeArgs& a, uint64_t t, float4* xin) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint64_t b = t * kFastWarps + warp;
    // a group is committed in every case, so that the waits can count groups
    if (t >= a.ntiles || b >= a.nb) {
        asm volatile("cp.async.commit_group;\n" ::: "memory");
        return;
    }
    const uint64_t base = b * a.d;
    const uint32_t m = static_cast<uint32_t>(min(static_cast<uint64_t>(a.d), a.n - base));
    const uint32_t swz = (static_cast<uint32_t>(lane) * V / 8) & (V - 1);
    float4* dst = xin + warp * 32 * V + lane * V;
#pragma unroll
    for (int j = 0; j < V; ++j) {
        const uint32_t i = lane * 4 * V + 4 * j;
        const uint32_t avail = i < m ? min(16u, (m - i) * 4u) : 0u;
        const uint32_t saddr = static_cast<uint32_t>(__cvta_generic_to_shared(dst + (j ^ swz)));
        const float* src = a.in + base + (i < m ? i : 0);
        if (avail == 16u)
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(saddr), "l"(src) : "memory");
        else  // the ragged end of the last bucket: zero-filled past m
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(saddr), "l"(src), "r"(avail)
                         : "memory");
    }
    asm volatile("cp.async.commit_group;\n" ::: "memory");
}

// Codes tile t into tbuf (tile-local bit offsets) and publishes A(t).  On entry
// the tile's input is in flight into xin.  Two CTA barriers.
template <int V, bool kShort, bool kEF>
__device__ __forceinline__ void code_tile(const EncodeArgs& a, uint64_t t, const uint32_t* t_after_slot, const uint32_t* rtab,
                                          uint32_t* tbuf, uint32_t* pb, float4* xin, TileSlot& slot,
                                          uint32_t epoch) {
    // tbuf holds the bits of the tile coded two tiles ago (slot.total, set by that
    // tile): clear the words it used
    const uint32_t dirty = min(a.smem_words, static_cast<uint32_t>((slot.total + 31) >> 5) + 2u);
    constexpr int NC = 4 * V;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint64_t b = t * kFastWarps + warp;
    const bool live = b < a.nb;
    const uint64_t base = b * a.d;
    const uint32_t first = lane * NC;  // first bucket-local coordinate of this lane

    // error feedback: the memory of this lane's coordinates, loaded before the wait
    const uint32_t mlen = live ? static_cast<uint32_t>(min(static_cast<uint64_t>(a.d), a.n - base)) : 0u;
    float ev[kEF ? NC : 1];
    if constexpr (kEF) ef_load<V>(a.ef + base, first, mlen, ev);

    asm volatile("cp.async.wait_all;\n" ::: "memory");  // the tile's input
    __syncthreads();  // B0: the tile's input has landed; every warp is done with tbuf's last tile
    // clear the words tbuf's last tile used (nothing writes tbuf before B1)
    for (uint32_t i = tid; i < dirty; i += kFastBlock) tbuf[i] = 0u;

    // --- input from shared memory ------------------------------------------
    float x[NC];
    {
        const uint32_t swz = (static_cast<uint32_t>(lane) * V / 8) & (V - 1);
        const float4* src = xin + warp * 32 * V + lane * V;
#pragma unroll
        for (int j = 0; j < V; ++j) {
            const float4 q = live ? src[j ^ swz] : make_float4(0.f, 0.f, 0.f, 0.f);
            x[4 * j + 0] = q.x;
            x[4 * j + 1] = q.y;
            x[4 * j + 2] = q.z;
            x[4 * j + 3] = q.w;
        }
    }
    if constexpr (kEF) {  // p = e + g
#pragma unroll
        for (int q = 0; q < NC; ++q) x[q] = __fadd_rn(ev[q], x[q]);
    }

    // --- bucket norm: per-lane FMA chain, butterfly (same value in all lanes) --
    const float norm = a.norm_kind == QSGD_NORM_MAX ? warp_bucket_maxnorm<NC>(x) : warp_bucket_norm<NC>(x, live);
    const BucketScale sc = bucket_scale(norm, a.s, live, a.status, lane == 0);
    if (!sc.good) {
        if constexpr (kEF) ef_store<V>(a.ef + base, first, mlen, x);  // nothing sent: the memory keeps p
#pragma unroll
        for (int q = 0; q < NC; ++q) x[q] = 0.f;
    }

    // --- stochastic rounding: one Philox block per 4 coordinates ------------
    uint32_t kq[NC];  // level | sign << 31
    const uint64_t g0 = base + first;  // a multiple of 4
    const PhiloxKey key{a.key0, a.key1};
#pragma unroll
    for (int j = 0; j < V; ++j) {
        const uint4 r = philox4x32_10((g0 >> 2) + j, key);
        const uint32_t rw[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const float v = x[4 * j + c];
            kq[4 * j + c] = quantize_level(v, sc.sinv, rw[c], a.s) | (__float_as_uint(v) & 0x80000000u);
        }
    }
    if constexpr (kEF) {  // the memory keeps p minus what a receiver decodes
        if (sc.good) {
            const float scale = __fdiv_rn(sc.sent, __uint2float_rn(a.s));
#pragma unroll
            for (int q = 0; q < NC; ++q) ev[q] = ef_residual(x[q], kq[q] & 0x7FFFFFFFu, kq[q] >> 31, scale);
            ef_store<V>(a.ef + base, first, mlen, ev);
        }
    }

    // --- compact the bucket's non-zeros into the warp's record list, which
    // reuses this warp's slice of the input buffer (free once x is in registers);
    // entry = index | k << 10 | sign << 31, in index order ---------------------
    uint32_t* const rec = reinterpret_cast<uint32_t*>(xin + warp * 32 * V);
    uint32_t cnt = 0;
#pragma unroll
    for (int q = 0; q < NC; ++q) cnt += (kq[q] & 0x7FFFFFFFu) != 0u;
    uint32_t incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t tt = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += tt;
    }
    const uint32_t nz = __shfl_sync(kFull, incl, 31);
    {
        uint32_t pos = incl - cnt;
#pragma unroll
        for (int q = 0; q < NC; ++q) {
            if (kq[q] & 0x7FFFFFFFu) {
                rec[pos] = (first + q) | ((kq[q] & 0x7FFFFFFFu) << 10) | (kq[q] & 0x80000000u);
                ++pos;
            }
        }
    }
    __syncwarp();

    // --- records omega(gap) | sign | omega(k) of a contiguous run, packed
    // MSB-first into this lane's private strip (word j at pb[32 j + lane]) ----
    LanePacker pk{pb + lane, 0u, 0u, 0u};
    {
        const uint32_t per = (nz + 31) >> 5;
        const uint32_t r0 = min(nz, lane * per), r1 = min(nz, r0 + per);
        uint32_t prev = r0 ? (rec[r0 - 1] & 1023u) : 0xFFFFFFFFu;  // -1 before the first
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
    }
    const uint32_t nbits = pk.bits();
    uint32_t inclb = nbits;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t tt = __shfl_up_sync(kFull, inclb, o);
        if (lane >= o) inclb += tt;
    }
    const uint32_t exclb = inclb - nbits;
    if (lane == 31) slot.bits[warp] = live ? 32u + inclb : 0u;
    __syncthreads();  // B1: bucket sizes known; the input buffer is free
    prefetch_tile<V>(a, *t_after_slot, xin);  // the ticket was stored before B0
    // tile-local start of this warp's bucket and the tile's size (kFastWarps-lane scan)
    uint32_t bsc = lane < kFastWarps ? slot.bits[lane] : 0u;
#pragma unroll
    for (int o = 1; o < kFastWarps; o <<= 1) {
        const uint32_t tt = __shfl_up_sync(kFull, bsc, o);
        if (lane >= o) bsc += tt;
    }
    const uint64_t tb = __shfl_sync(kFull, bsc, kFastWarps - 1);
    const uint64_t bstart = warp ? __shfl_sync(kFull, bsc, warp - 1) : 0u;
    if (tid == 0) {
        st_release(&a.tdesc[t], make_desc(epoch, kStateAggregate, tb));
        slot.total = tb;
    }

    // --- move the bits to their tile-local offsets ----------------------------
    if (live) {
        if (lane == 0) {
            const uint32_t nb32 = __float_as_uint(sc.sent);
            const uint32_t w = static_cast<uint32_t>(bstart >> 5), sh = static_cast<uint32_t>(bstart & 31u);
            atomicOr(&tbuf[w], nb32 >> sh);
            if (sh) atomicOr(&tbuf[w + 1], nb32 << (32 - sh));
        }
        const uint32_t pos = static_cast<uint32_t>(bstart) + 32u + exclb;  // first bit of this lane's records
        const uint32_t w = pos >> 5, sh = pos & 31u;
        const uint32_t nsrc = (nbits + 31u) >> 5;         // words in the strip
        const uint32_t ndst = (sh + nbits + 31u) >> 5;    // words touched in the tile buffer
        if (w + ndst > a.smem_words) {
            report(a.status, QSGD_ST_OVERFLOW);
        } else {
            uint32_t prv = 0;
            for (uint32_t j = 0; j < ndst; ++j) {
                const uint32_t cur = j < nsrc ? pb[32 * j + lane] : 0u;
                const uint32_t v = sh ? (cur >> sh) | (prv << (32 - sh)) : cur;
                if (v) atomicOr(&tbuf[w + j], v);
                prv = cur;
            }
        }
    }
    __syncwarp();
}

// Exclusive prefix of tile t = r*C + c: RP(r-2) + the bit counts A of every tile
// of round r-1 + those of round r's tiles before c, all read in parallel.  The A
// values are published when tiles are coded, well before they are needed, and
// RP(r-2) one round earlier, so the wait is normally empty.  One CTA barrier;
// every thread returns the same value.  `acc` is a zeroed shared accumulator;
// false when a bounded wait ran out (or another CTA aborted).
__device__ __forceinline__ bool wait_value(const uint64_t* p, uint64_t state, uint32_t epoch,
                                           const uint32_t* abort_flag, uint64_t& value) {
    for (uint32_t polls = 0;; ++polls) {
        const uint64_t d = ld_acquire(p);
        if (desc_epoch(d) == (epoch & kEpochMask) && desc_state(d) == state) {
            value = desc_value(d);
            return true;
        }
        if (polls > kMaxPolls || ((polls & 63u) == 63u && ld_acquire32(abort_flag) != 0)) return false;
        __nanosleep(polls < 16 ? 64 : 512);
    }
}

// Exclusive prefix of tile t = r*C + c: RP(r-2) + the bit counts A of every tile
// of round r-1 + those of round r's tiles before c, all read in parallel.  The A
// values are published when tiles are coded, normally well before they are needed,
// and RP(r-2) one round earlier.  One CTA barrier; every thread returns the same
// value.  `acc` is a zeroed shared accumulator; false when a bounded wait ran out
// (or another CTA aborted).
__device__ __forceinline__ bool gather_prefix(const EncodeArgs& a, uint32_t r, uint32_t C, uint32_t c,
                                              uint32_t epoch, unsigned long long* acc, int* bad,
                                              uint64_t& prefix) {
    const int tid = threadIdx.x, lane = tid & 31;
    uint64_t sum = 0;
    bool ok = true;
    // tiles [t_lo, t_hi): all of round r-1 and round r up to c; the values are
    // the data, so relaxed loads suffice
    const uint64_t t_lo = r >= 1 ? static_cast<uint64_t>(r - 1) * C : 0;
    const uint64_t t_hi = static_cast<uint64_t>(r) * C + c;
    for (uint64_t i = t_lo + tid; i < t_hi; i += kFastBlock) {
        uint64_t d = ld_relaxed(&a.tdesc[i]);
        if (!(desc_epoch(d) == (epoch & kEpochMask) && desc_state(d) == kStateAggregate)) {
            uint64_t v = 0;
            ok = ok && wait_value(&a.tdesc[i], kStateAggregate, epoch, &a.ctrl->abort, v);
            d = v;
        } else {
            d = desc_value(d);
        }
        sum += d;
    }
    if (tid == kFastBlock - 1 && r >= 2 && ok) {
        uint64_t v = 0;
        ok = wait_value(&a.ts[r - 2].round, kStatePrefix, epoch, &a.ctrl->abort, v);
        sum += v;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(kFull, sum, o);
    if (!ok) atomicOr(bad, 1);
    if (lane == 0 && sum) atomicAdd(acc, static_cast<unsigned long long>(sum));
    __syncthreads();  // Bg
    prefix = *acc;
    return *bad == 0;
}

// Writes tile t (bits at tile-local offsets in tbuf, stream prefix X, tb bits):
// offsets header, the words it owns alone, and its share of the words it shares
// with the neighbouring tiles.
__device__ __forceinline__ void store_tile(const EncodeArgs& a, const uint32_t* tbuf, const TileSlot& slot,
                                           uint64_t t, uint64_t X, uint64_t tb, uint32_t epoch) {
    const int tid = threadIdx.x;
    const uint32_t sh = static_cast<uint32_t>(X & 31u);
    const uint64_t w0 = X >> 5;
    const uint64_t end = X + tb;
    const uint32_t qe = static_cast<uint32_t>((end >> 5) - w0);
    const uint32_t limit = a.smem_words;
    auto word_at = [&](uint32_t q) -> uint32_t {
        const uint32_t cur = q < limit ? tbuf[q] : 0u;
        if (sh == 0) return cur;
        const uint32_t prv = (q > 0 && q - 1 < limit) ? tbuf[q - 1] : 0u;
        return (cur >> sh) | (prv << (32 - sh));
    };
    if (tid < 32) {
        uint32_t v = tid < kFastWarps ? slot.bits[tid] : 0u;
#pragma unroll
        for (int o = 1; o < kFastWarps; o <<= 1) {
            const uint32_t tt = __shfl_up_sync(kFull, v, o);
            if (tid >= o) v += tt;
        }
        const uint64_t bb = t * kFastWarps + tid;
        if (tid < kFastWarps && bb < a.nb) a.offsets[bb] = X + v - slot.bits[tid];
    }
    if (tid == 0 && (end & 31u) != 0) {
        if (t + 1 == a.ntiles)
            store_word(a, w0 + qe, word_at(qe));
        else
            merge_shared_word(a, &a.ts[t + 1].slot, w0 + qe, word_at(qe), epoch);
    }
    if (tid == 32) {
        if (t + 1 == a.ntiles) a.offsets[a.nb] = end;
        if (sh != 0) merge_shared_word(a, &a.ts[t].slot, w0, word_at(0), epoch);
    }
    for (uint32_t q = (sh ? 1u : 0u) + tid; q < qe; q += kFastBlock) store_word(a, w0 + q, word_at(q));
}

template <int V, bool kShort, bool kEF>
__global__ void __launch_bounds__(kFastBlock, (V <= 4 ? kFastMinBlocks : 1)) encode_fast(const __grid_constant__ EncodeArgs a) {
    constexpr int kEncDepth = enc_depth(V);
    constexpr int kEncBufs = kEncDepth + 1;
    extern __shared__ __align__(16) uint32_t smem[];
    __shared__ TileSlot s_slot[kEncBufs];
    __shared__ unsigned long long s_acc[2];
    __shared__ int s_bad;
    __shared__ uint32_t s_ticket[kEncDepth + 1];  // the first tickets; then [it & 1] each iteration
    const int tid = threadIdx.x;
    uint32_t* const rtab = smem;                                                 // record table
    float4* const xin = reinterpret_cast<float4*>(smem + kRecordTab);           // kFastWarps * 128V floats
    uint32_t* const tbuf0 = smem + kRecordTab + kFastWarps * 128 * V;           // kEncBufs tile buffers
    uint32_t* const pb = tbuf0 + kEncBufs * a.smem_words + (tid >> 5) * 32 * fast_lane_words(V, kShort);  // lane strips
    record_table_fill(rtab, tid, kFastBlock);
    const uint32_t epoch = *reinterpret_cast<volatile uint32_t*>(&a.ctrl->epoch);
    const uint32_t C = gridDim.x;
    if (tid == 0) {
#pragma unroll
        for (int j = 0; j <= kEncDepth; ++j) s_ticket[j] = atomicAdd(&a.ctrl->ticket, 1u);
        s_acc[0] = s_acc[1] = 0;
        s_bad = 0;
#pragma unroll
        for (int j = 0; j < kEncBufs; ++j) s_slot[j].total = static_cast<uint64_t>(a.smem_words) * 32;  // clear all at first use
    }
    __syncthreads();
    // Prologue: code the first kEncDepth tiles (each coding starts the input copy of
    // the next ticket at its B1).  held[] are the coded tiles not yet stored, oldest
    // first; tile number q (in coding order) lives in buffer q mod kEncBufs.
    uint64_t held[kEncDepth];
    prefetch_tile<V>(a, s_ticket[0], xin);
#pragma unroll
    for (int j = 0; j < kEncDepth; ++j) {
        held[j] = s_ticket[j];
        if (held[j] < a.ntiles)
            code_tile<V, kShort, kEF>(a, held[j], &s_ticket[j + 1], rtab, tbuf0 + j * a.smem_words, pb, xin, s_slot[j], epoch);
    }
    uint64_t tn = s_ticket[kEncDepth];
    __syncthreads();  // every thread has read s_ticket before the loop reuses it
    // Per iteration: draw the ticket tnn; code tile tn (its B1 starts the input copy
    // of tnn; B0 publishes tnn); gather the prefix of the oldest coded tile and store
    // it.  CTA barriers: B0 and B1 inside the coding, Bg inside the gather.  Coding
    // runs kEncDepth tiles ahead of storing, so the tiles a gather waits for have had
    // kEncDepth iterations to publish their sizes.
    for (uint32_t it = 0; held[0] < a.ntiles; ++it) {
        if (tid == 0) s_ticket[it & 1] = atomicAdd(&a.ctrl->ticket, 1u);
        const uint64_t t = held[0];
        const uint32_t bs = it % kEncBufs;                // buffer of t
        const uint32_t bn = (it + kEncDepth) % kEncBufs;  // buffer for tn
        const uint32_t r = static_cast<uint32_t>(t) / C;
        const uint32_t c = static_cast<uint32_t>(t) - r * C;
        if (tn < a.ntiles)
            code_tile<V, kShort, kEF>(a, tn, &s_ticket[it & 1], rtab, tbuf0 + bn * a.smem_words, pb, xin, s_slot[bn], epoch);
        else
            __syncthreads();  // orders the ticket, the accumulator reset and store_tile
        const uint64_t tnn = s_ticket[it & 1];
        const uint64_t tb = s_slot[bs].total;
        uint64_t X = 0;
        const bool ok = gather_prefix(a, r, C, c, epoch, &s_acc[it & 1], &s_bad, X);
        if (tid == 0) s_acc[(it + 1) & 1] = 0;  // the next iteration's accumulator
        if (!ok) {
            if (tid == 0) abort_all(a);
        } else {
            if (tid == 0 && ((c + 1 == C) || (t + 1 == a.ntiles)))
                st_release(&a.ts[r].round, make_desc(epoch, kStatePrefix, X + tb));
            store_tile(a, tbuf0 + bs * a.smem_words, s_slot[bs], t, X, tb, epoch);
        }
#pragma unroll
        for (int j = 0; j + 1 < kEncDepth; ++j) held[j] = held[j + 1];
        held[kEncDepth - 1] = tn;
        tn = tnn;
    }
    asm volatile("cp.async.wait_all;\n" ::: "memory");
    __syncthreads();
    cta_exit(a.ctrl, epoch);
}

// ---------------------------------------------------------------------------
// General path.
// ---------------------------------------------------------------------------

// Norm of `m` values starting at p, by one warp (lanes take every 32nd value, then
// a butterfly); the rescaled form when the squares leave the normal range.
__device__ __forceinline__ float warp_norm(const float* p, uint64_t m, int lane) {
    float ss = 0.f;
    for (uint64_t i = lane; i < m; i += 32) {
        const float v = __ldg(p + i);
        ss = __fmaf_rn(v, v, ss);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss = __fadd_rn(ss, __shfl_xor_sync(kFull, ss, o));
    float norm = __fsqrt_rn(ss);
    if (needs_rescale(ss) && !isnan(ss)) {  // uniform in the warp
        float mx = 0.f;
        for (uint64_t i = lane; i < m; i += 32) mx = fmaxf(mx, fabsf(__ldg(p + i)));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, o));
        if (isinf(mx)) {
            norm = mx;
        } else if (mx > 0.f) {
            float unscale;
            const float scale = pow2_scale(mx, unscale);
            float s2 = 0.f;
            for (uint64_t i = lane; i < m; i += 32) {
                const float y = __fmul_rn(__ldg(p + i), scale);
                s2 = __fmaf_rn(y, y, s2);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) s2 = __fadd_rn(s2, __shfl_xor_sync(kFull, s2, o));
            norm = __fmul_rn(__fsqrt_rn(s2), unscale);
        }
    }
    return norm;
}

// Norm of one large bucket by the whole CTA: thread i takes every kBlock-th value,
// then a butterfly per warp and the warp sums in order (deterministic).
__device__ __forceinline__ float block_norm(const float* p, uint64_t m, float* red) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    auto block_sum = [&](float x) -> float {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) x = __fadd_rn(x, __shfl_xor_sync(kFull, x, o));
        __syncthreads();
        if (lane == 0) red[warp] = x;
        __syncthreads();
        float tot = 0.f;
        for (int w = 0; w < kWarps; ++w) tot = __fadd_rn(tot, red[w]);
        return tot;
    };
    auto block_max = [&](float x) -> float {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(kFull, x, o));
        __syncthreads();
        if (lane == 0) red[warp] = x;
        __syncthreads();
        float mx = 0.f;
        for (int w = 0; w < kWarps; ++w) mx = fmaxf(mx, red[w]);
        return mx;
    };
    float ss = 0.f;
    for (uint64_t i = tid; i < m; i += kBlock) {
        const float v = __ldg(p + i);
        ss = __fmaf_rn(v, v, ss);
    }
    ss = block_sum(ss);
    float norm = __fsqrt_rn(ss);
    if (needs_rescale(ss) && !isnan(ss)) {  // uniform in the block
        float mx = 0.f;
        for (uint64_t i = tid; i < m; i += kBlock) mx = fmaxf(mx, fabsf(__ldg(p + i)));
        mx = block_max(mx);
        if (isinf(mx)) {
            norm = mx;
        } else if (mx > 0.f) {
            float unscale;
            const float scale = pow2_scale(mx, unscale);
            float s2 = 0.f;
            for (uint64_t i = tid; i < m; i += kBlock) {
                const float y = __fmul_rn(__ldg(p + i), scale);
                s2 = __fmaf_rn(y, y, s2);
            }
            s2 = block_sum(s2);
            norm = __fmul_rn(__fsqrt_rn(s2), unscale);
        }
    }
    return norm;
}

// Max-norm of m values at p by the whole CTA (NaN if any value is NaN).
__device__ __forceinline__ float block_maxnorm(const float* p, uint64_t m, float* red) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    float mx = 0.f;
    bool nan = false;
    for (uint64_t i = tid; i < m; i += kBlock) {
        const float v = __ldg(p + i);
        nan |= isnan(v);
        mx = fmaxf(mx, fabsf(v));
    }
    if (__syncthreads_or(nan)) return __uint_as_float(0x7FC00000u);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, o));
    if (lane == 0) red[warp] = mx;
    __syncthreads();
    float tot = 0.f;
    for (int w = 0; w < kWarps; ++w) tot = fmaxf(tot, red[w]);
    __syncthreads();  // red is reused by the next call
    return tot;
}

// Block-wide scans for kBlock threads.
struct BlockScratch {
    int64_t i64[kWarps];
    uint32_t u32[kWarps];
};

// Exclusive max-scan of x with `carry` as the value before thread 0; returns the
// exclusive value and sets `all` to the maximum over carry and every x.
__device__ __forceinline__ int64_t block_excl_max(int64_t x, int64_t carry, BlockScratch& sc,
                                                  int64_t& all) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int64_t incl = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int64_t t = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl = max(incl, t);
    }
    if (lane == 31) sc.i64[warp] = incl;
    __syncthreads();
    int64_t before = carry;
    for (int w = 0; w < warp; ++w) before = max(before, sc.i64[w]);
    all = carry;
    for (int w = 0; w < kWarps; ++w) all = max(all, sc.i64[w]);
    int64_t excl = __shfl_up_sync(kFull, incl, 1);
    excl = lane == 0 ? before : max(before, excl);
    __syncthreads();
    return excl;
}

__device__ __forceinline__ uint32_t block_excl_sum(uint32_t x, BlockScratch& sc, uint32_t& total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t incl = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t t = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += t;
    }
    if (lane == 31) sc.u32[warp] = incl;
    __syncthreads();
    uint32_t before = 0;
    total = 0;
    for (int w = 0; w < kWarps; ++w) {
        if (w < warp) before += sc.u32[w];
        total += sc.u32[w];
    }
    __syncthreads();
    return before + incl - x;
}

// The four coordinates of one thread in one chunk, quantised.
struct Quad {
    uint32_t kq[4];      // level | sign << 31
    uint32_t start[4];   // 1 when the coordinate opens its bucket
    uint64_t bstart[4];  // global index of its bucket's first coordinate
    uint64_t bucket[4];
    float sent[4];
    bool valid[4];
};

__device__ __forceinline__ void quantize_quad(const EncodeArgs& a, uint64_t i0, uint64_t c0,
                                              uint64_t c1, uint64_t b0, PhiloxKey key, const float2* norms,
                                              Quad& qd) {
    const uint4 r = philox4x32_10(i0 >> 2, key);
    const uint32_t rw[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const uint64_t i = i0 + c;
        qd.valid[c] = i >= c0 && i < c1;
        qd.kq[c] = 0;
        qd.start[c] = 0;
        qd.bstart[c] = 0;
        qd.bucket[c] = 0;
        qd.sent[c] = 0.f;
        if (!qd.valid[c]) continue;
        const uint32_t rel = static_cast<uint32_t>(i - c0);  // < buckets_per_tile * d <= 2^31
        const uint64_t bl = rel / a.d;
        const uint64_t b = b0 + bl;
        const float2 ns = norms[bl];
        const float v = __ldg(a.in + i);
        qd.bucket[c] = b;
        qd.bstart[c] = b * a.d;
        qd.start[c] = (i == qd.bstart[c]) ? 1u : 0u;
        qd.sent[c] = ns.x;
        const uint32_t k = (ns.y != 0.f) ? quantize_level(v, ns.y, rw[c], a.s) : 0u;
        qd.kq[c] = k | (__float_as_uint(v) & 0x80000000u);
    }
}

__global__ void __launch_bounds__(kBlock) encode_general(const __grid_constant__ EncodeArgs a) {
    extern __shared__ __align__(16) uint32_t smem[];
    uint32_t* tab = smem;
    uint32_t* buf = smem + kOmegaTab;
    float2* s_norms = reinterpret_cast<float2*>(smem + kOmegaTab + ((a.smem_words + 1) & ~1u));  // (norm, s/norm)
    __shared__ float s_red[kWarps];
    __shared__ uint32_t s_tile;
    __shared__ BlockScratch s_scr;
    __shared__ uint64_t s_prefix;
    __shared__ int s_ok;
    __shared__ uint32_t s_pending;  // partial last word carried between chunks
    __shared__ uint32_t s_head;     // own bits of the tile's first word when it is shared

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    omega_table_fill(tab, tid, kBlock);
    const uint32_t epoch = *reinterpret_cast<volatile uint32_t*>(&a.ctrl->epoch);
    const PhiloxKey key{a.key0, a.key1};

    for (;;) {
        if (tid == 0) s_tile = atomicAdd(&a.ctrl->ticket, 1u);
        __syncthreads();
        const uint32_t tile = s_tile;
        if (tile >= a.ntiles) break;
        const uint64_t b0 = static_cast<uint64_t>(tile) * a.buckets_per_tile;
        const uint64_t b1 = min(a.nb, b0 + a.buckets_per_tile);
        const uint64_t c0 = b0 * a.d;
        const uint64_t c1 = min(a.n, b1 * a.d);
        const uint64_t cbase = c0 & ~uint64_t(3);

        // --- bucket norms into shared memory -------------------------------
        if (b1 - b0 == 1) {
            const uint64_t m = c1 - c0;
            const float norm = a.norm_kind == QSGD_NORM_MAX ? block_maxnorm(a.in + c0, m, s_red)
                                                            : block_norm(a.in + c0, m, s_red);
            const BucketScale sc = bucket_scale(norm, a.s, true, a.status, tid == 0);
            if (tid == 0) s_norms[0] = make_float2(sc.sent, sc.good ? sc.sinv : 0.f);
        } else {
            for (uint64_t bl = warp; bl < b1 - b0; bl += kWarps) {
                const uint64_t base = (b0 + bl) * a.d;
                const uint64_t m = min(static_cast<uint64_t>(a.d), a.n - base);
                const float norm = a.norm_kind == QSGD_NORM_MAX ? warp_maxnorm(a.in + base, m, lane)
                                                                : warp_norm(a.in + base, m, lane);
                const BucketScale sc = bucket_scale(norm, a.s, true, a.status, lane == 0);
                if (lane == 0) s_norms[bl] = make_float2(sc.sent, sc.good ? sc.sinv : 0.f);
            }
        }
        __syncthreads();

        // --- pass 1: bit count of the tile --------------------------------
        uint64_t tb = 0;
        int64_t carry_prev = -1;
        for (uint64_t cb = cbase; cb < c1; cb += kChunk) {
            Quad qd;
            quantize_quad(a, cb + 4ull * tid, c0, c1, b0, key, s_norms, qd);
            int64_t last = -1;
#pragma unroll
            for (int c = 0; c < 4; ++c)
                if (qd.kq[c] & 0x7FFFFFFFu) last = static_cast<int64_t>(cb + 4ull * tid + c);
            int64_t all;
            int64_t prev = block_excl_max(last, carry_prev, s_scr, all);
            carry_prev = all;
            uint32_t bits = 0;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                if (!qd.valid[c]) continue;
                const int64_t i = static_cast<int64_t>(cb + 4ull * tid + c);
                if (qd.start[c]) bits += 32u;
                const uint32_t k = qd.kq[c] & 0x7FFFFFFFu;
                if (k) {
                    const int64_t p = max(prev, static_cast<int64_t>(qd.bstart[c]) - 1);
                    bits += omega_len(tab, static_cast<uint64_t>(i - p)) + 1u + omega_len(tab, k);
                    prev = i;
                }
            }
            uint32_t total;
            block_excl_sum(bits, s_scr, total);
            tb += total;
        }
        if (tid == 0)
            st_release(&a.tdesc[tile], make_desc(epoch, tile == 0 ? kStatePrefix : kStateAggregate, tb));

        // --- look-back ------------------------------------------------------
        if (warp == 0) {
            uint64_t excl = 0;
            bool ok = true;
            if (tile > 0) ok = lookback(a.tdesc, tile, epoch, &a.ctrl->abort, excl);
            if (lane == 0) {
                if (!ok)
                    abort_all(a);
                else if (tile > 0)
                    st_release(&a.tdesc[tile], make_desc(epoch, kStatePrefix, excl + tb));
                s_prefix = excl;
                s_ok = ok;
                s_pending = 0;
                s_head = 0;
            }
        }
        __syncthreads();
        if (!s_ok) {
            __syncthreads();
            continue;
        }
        const uint64_t X = s_prefix;
        const uint64_t head_word = X >> 5;
        const bool head_shared = (X & 31u) != 0;

        // --- pass 2: pack chunk by chunk at global alignment ----------------
        uint64_t pos = X;  // global bit where the next chunk starts
        carry_prev = -1;
        for (uint64_t cb = cbase; cb < c1; cb += kChunk) {
            Quad qd;
            quantize_quad(a, cb + 4ull * tid, c0, c1, b0, key, s_norms, qd);
            int64_t last = -1;
#pragma unroll
            for (int c = 0; c < 4; ++c)
                if (qd.kq[c] & 0x7FFFFFFFu) last = static_cast<int64_t>(cb + 4ull * tid + c);
            int64_t all;
            const int64_t prev_in = block_excl_max(last, carry_prev, s_scr, all);
            carry_prev = all;
            uint32_t bits = 0;
            {
                int64_t prev = prev_in;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    if (!qd.valid[c]) continue;
                    const int64_t i = static_cast<int64_t>(cb + 4ull * tid + c);
                    if (qd.start[c]) bits += 32u;
                    const uint32_t k = qd.kq[c] & 0x7FFFFFFFu;
                    if (k) {
                        const int64_t p = max(prev, static_cast<int64_t>(qd.bstart[c]) - 1);
                        bits += omega_len(tab, static_cast<uint64_t>(i - p)) + 1u + omega_len(tab, k);
                        prev = i;
                    }
                }
            }
            uint32_t total;
            const uint32_t excl = block_excl_sum(bits, s_scr, total);
            if (total == 0) continue;  // uniform: every thread sees the same total
            const uint64_t w0 = pos >> 5;
            const uint32_t lead = static_cast<uint32_t>(pos & 31u);
            const uint32_t nwords = (lead + total + 31u) >> 5;
            for (uint32_t q = tid; q < nwords; q += kBlock) buf[q] = (q == 0 && lead) ? s_pending : 0u;
            __syncthreads();
            {
                BitPacker pk;
                pk.start(buf, a.smem_words, lead + excl);
                bool ok = true;
                int64_t prev = prev_in;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    if (!qd.valid[c]) continue;
                    const int64_t i = static_cast<int64_t>(cb + 4ull * tid + c);
                    if (qd.start[c]) {
                        a.offsets[qd.bucket[c]] = ((w0 + pk.word) << 5) + pk.nacc;
                        ok &= pk.put(__float_as_uint(qd.sent[c]), 32);
                    }
                    const uint32_t k = qd.kq[c] & 0x7FFFFFFFu;
                    if (k) {
                        const int64_t p = max(prev, static_cast<int64_t>(qd.bstart[c]) - 1);
                        uint64_t gc, kc;
                        uint32_t gl, kl;
                        omega_code(tab, static_cast<uint64_t>(i - p), gc, gl);
                        omega_code(tab, k, kc, kl);
                        prev = i;
                        ok &= pk.put(gc, gl);
                        ok &= pk.put(qd.kq[c] >> 31, 1);
                        ok &= pk.put(kc, kl);
                    }
                }
                ok &= pk.flush();
                if (!ok) report(a.status, QSGD_ST_OVERFLOW);
            }
            __syncthreads();
            const uint64_t end = pos + total;
            const bool last_complete = (end & 31u) == 0;
            const uint32_t nfinal = last_complete ? nwords : nwords - 1;
            for (uint32_t q = tid; q < nfinal; q += kBlock) {
                const uint64_t gw = w0 + q;
                if (gw == head_word && head_shared)
                    s_head = buf[q];
                else
                    store_word(a, gw, buf[q]);
            }
            __syncthreads();
            if (tid == 0) s_pending = last_complete ? 0u : buf[nwords - 1];
            pos = end;
            __syncthreads();
        }

        // --- tail word, shared head word, end of the header ----------------
        if (tid == 0) {
            const uint64_t end = X + tb;
            if (end & 31u) {
                if (tile + 1 == a.ntiles)
                    store_word(a, end >> 5, s_pending);
                else
                    merge_shared_word(a, &a.ts[tile + 1].slot, end >> 5, s_pending, epoch);
            }
            if (tile + 1 == a.ntiles) a.offsets[a.nb] = end;
            if (head_shared) merge_shared_word(a, &a.ts[tile].slot, head_word, s_head, epoch);
        }
        __syncthreads();
    }
    cta_exit(a.ctrl, epoch);
}

template <int V, bool kShort, bool kEF>
cudaError_t launch_fast(const EncodeArgs& a, cudaStream_t stream) {
    const size_t smem = fast_smem_bytes(a.d, a.s, a.smem_words);
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_set[dev]) {
        cudaFuncSetAttribute(encode_fast<V, kShort, kEF>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
        attr_set[dev] = true;
    }
    int sms = 0, per_sm = 0;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, encode_fast<V, kShort, kEF>, kFastBlock, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const uint64_t grid = std::min<uint64_t>(a.ntiles, static_cast<uint64_t>(sms) * per_sm);
    encode_fast<V, kShort, kEF><<<static_cast<unsigned>(grid), kFastBlock, smem, stream>>>(a);
    return cudaGetLastError();
}

template <int V>
cudaError_t launch_fast_v(const EncodeArgs& a, cudaStream_t stream) {
    if (a.ef) return a.s <= 31 ? launch_fast<V, true, true>(a, stream) : launch_fast<V, false, true>(a, stream);
    return a.s <= 31 ? launch_fast<V, true, false>(a, stream) : launch_fast<V, false, false>(a, stream);
}

}  // namespace

cudaError_t launch_encode(EncodeArgs a, bool fast_path, cudaStream_t stream) {
    if (fast_path) {
        switch (fast_v(a.d)) {
            case 1: return launch_fast_v<1>(a, stream);
            case 2: return launch_fast_v<2>(a, stream);
            case 4: return launch_fast_v<4>(a, stream);
            default: return launch_fast_v<8>(a, stream);
        }
    }
    int dev = 0, sms = 0, per_sm = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const size_t smem = general_smem_bytes(a.smem_words, a.buckets_per_tile);
    static bool attr_set[64] = {};
    if (dev < 64 && !attr_set[dev]) {
        cudaFuncSetAttribute(encode_general, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
        attr_set[dev] = true;
    }
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, encode_general, kBlock, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const uint64_t grid = std::min<uint64_t>(a.ntiles, static_cast<uint64_t>(sms) * per_sm);
    encode_general<<<static_cast<unsigned>(grid), kBlock, smem, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace qsgd
