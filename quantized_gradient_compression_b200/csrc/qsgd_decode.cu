// QSGD decoder and decode-accumulate kernels (sm_100a).
//
// Method: "QSGD (Quantized Stochastic Gradient Descent) with Elias Coding" (AIMech
// curated entry).  The definition paragraph calls the coding "lossless prefix
// coding" of the tuple (||v||_2, signs, run-length gaps, levels k_i); the decoder
// inverts it and evaluates Q_s(v)_i = ||v||_2 * sgn(v_i) * k_i / s as
// fl(fl(norm / s) * k), sign last, +0.0 off the support.  A receiver in
// "distributed data-parallel optimization" (same paragraph) sums the decoded
// streams of its peers: out_i <- out_i + q^0_i + ... + q^{K-1}_i in stream order.
//
// Buckets are independent prefix-code streams located by the offsets header, so
// every bucket is parsed by its own thread; every read is bounded by the
// bucket's [offsets[b], offsets[b+1]) range and by the stream length.
#include <cuda_runtime.h>

#include "../../include/qsgd.h"
#include "qsgd_device.cuh"
#include "qsgd_internal.h"

namespace qsgd {
namespace {

// MSB-first reader over [pos, end) of a word array of num_words words.
struct BitReader {
    const uint32_t* w;
    uint64_t num_words;
    uint64_t pos;
    uint64_t end;

    __device__ __forceinline__ uint32_t peek32() const {
        const uint64_t wi = pos >> 5;
        const uint32_t sh = static_cast<uint32_t>(pos & 31u);
        const uint32_t hi = wi < num_words ? __ldg(w + wi) : 0u;
        const uint32_t lo = wi + 1 < num_words ? __ldg(w + wi + 1) : 0u;
        return sh ? (hi << sh) | (lo >> (32 - sh)) : hi;
    }
    // Reads 1 <= nbits <= 32 bits; false if they pass `end`.
    __device__ __forceinline__ bool read(uint32_t nbits, uint32_t& v) {
        if (end - pos < nbits) return false;
        v = peek32() >> (32 - nbits);
        pos += nbits;
        return true;
    }
    // Elias omega: a 0 ends the code; a 1 starts a group of (value + 1) bits whose
    // value becomes the next length.  Values above 2^32 - 1 are rejected.
    __device__ __forceinline__ bool omega(uint32_t& N) {
        uint32_t value = 1;
        for (;;) {
            uint32_t bit;
            if (!read(1, bit)) return false;
            if (bit == 0) {
                N = value;
                return true;
            }
            if (value > 31) return false;
            uint32_t rest;
            if (!read(value, rest)) return false;
            value = (1u << value) | rest;
        }
    }
};

template <bool kAccumulate>
__global__ void __launch_bounds__(kDecodeBlock) decode_buckets(const __grid_constant__ DecodeArgs a) {
    const uint64_t b = static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (b >= a.nb) return;
    const uint64_t base = b * a.d;
    const uint32_t m = static_cast<uint32_t>(min(static_cast<uint64_t>(a.d), a.n - base));
    float* out = a.out + base;
    const float fs = __uint2float_rn(a.s);
    if (kAccumulate && a.first_group) {
        // out + (+0.0): a coordinate off every support turns -0.0 into +0.0, as the
        // dense sum does; every other value is unchanged.
        for (uint32_t i = 0; i < m; ++i) out[i] = __fadd_rn(out[i], 0.0f);
    }
    for (int j = 0; j < a.K; ++j) {
        const StreamRef st = a.streams[j];
        const uint64_t begin = st.offsets[b];
        const uint64_t end = st.offsets[b + 1];
        bool bad = !(end >= begin && end - begin >= 32 && end <= st.num_words * 32);
        uint32_t cur = 0;  // next coordinate not yet written (plain decode)
        if (!bad) {
            BitReader br{st.words, st.num_words, begin, end};
            uint32_t nbits = 0;
            br.read(32, nbits);
            const float norm = __uint_as_float(nbits);
            if (nbits == 0) {
                bad = br.pos != end;
            } else if (!(isfinite(norm) && norm > 0.f)) {
                bad = true;
            } else {
                const float scale = __fdiv_rn(norm, fs);
                uint32_t next = 0;  // index of the previous record + 1
                while (br.pos < end) {
                    uint32_t gap, sign, k;
                    if (!br.omega(gap) || static_cast<uint64_t>(next) + gap - 1 >= m) {
                        bad = true;
                        break;
                    }
                    const uint32_t idx = next + gap - 1;
                    if (!br.read(1, sign) || !br.omega(k) || k > a.s) {
                        bad = true;
                        break;
                    }
                    float val = __fmul_rn(scale, __uint2float_rn(k));
                    if (sign) val = -val;
                    if (kAccumulate) {
                        out[idx] = __fadd_rn(out[idx], val);
                    } else {
                        for (; cur < idx; ++cur) out[cur] = 0.0f;
                        out[idx] = val;
                        cur = idx + 1;
                    }
                    next = idx + 1;
                }
            }
        }
        if (bad) atomicOr(a.status, QSGD_ST_BAD_STREAM);
        if (!kAccumulate)
            for (; cur < m; ++cur) out[cur] = 0.0f;
    }
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs& a, bool accumulate, cudaStream_t stream) {
    const uint64_t blocks = (a.nb + kDecodeBlock - 1) / kDecodeBlock;
    if (blocks == 0) return cudaSuccess;
    if (accumulate)
        decode_buckets<true><<<static_cast<unsigned>(blocks), kDecodeBlock, 0, stream>>>(a);
    else
        decode_buckets<false><<<static_cast<unsigned>(blocks), kDecodeBlock, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace qsgd
