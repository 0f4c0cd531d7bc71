/*
 * qsgd.h -- C ABI of the B200 (sm_100a) QSGD gradient codec.
 *
 * The method is the one of the page "QSGD (Quantized Stochastic Gradient Descent)
 * with Elias Coding" (AIMech curated entry):
 *   - definition paragraph: Q_s(v)_i = ||v||_2 * sgn(v_i) * xi_i(v, s), where
 *     xi_i = (l_i + 1)/s with probability p_i = s|v_i|/||v||_2 - l_i, else l_i/s,
 *     l_i = floor(s|v_i|/||v||_2); the sparse tuple (||v||_2, signs, run-length
 *     gaps, levels k_i = s*xi_i) is sent with Elias recursive (omega) codes;
 *   - claim "Elias coding communication complexity tradeoff": F = 32 bits for the
 *     norm, index gaps between non-zeros, levels k_i in {1..s};
 *   - claim "QSVRG, non-convex and multi-GPU bucketed training": d-block
 *     bucketing, each bucket quantised with its own norm;
 *   - definition paragraph ("distributed data-parallel optimization"): a receiver
 *     decodes its peers' streams and sums them.
 *
 * Wire format (the same one the test oracle implements, independently):
 *   bucket b = coordinates [b*d, min(n,(b+1)*d)); per bucket: 32 raw bits of the
 *   fp32 norm, then per coordinate with k >= 1 in ascending index:
 *   omega(gap) || sign (1 = negative) || omega(k); gap = i - prev, prev = -1 at the
 *   bucket start.  Bits MSB-first within uint32 words; buckets back to back.
 *   offsets[b] = first bit of bucket b; offsets[nb] = total bits.
 *   Random source: u_i = floor(r_i / 2^9) * 2^-23 with r_i word (i mod 4) of
 *   Philox4x32-10(counter = (lo32(i/4), hi32(i/4), 0, 0), key = (lo32(seed),
 *   hi32(seed))), i the global coordinate index.  Quantiser arithmetic in fp32,
 *   round-to-nearest-even: sinv = s / norm (once per bucket), t = |v_i| * sinv,
 *   l = floor(t), p = t - l, k = min(l + [u_i < p], s).  Decoder: fl(fl(norm/s)*k),
 *   sign applied last, +0.0 off the support.
 *
 * Conventions for every call below:
 *   - "d_" pointers are device pointers on the current CUDA device; "h_" pointers
 *     are host pointers.  The caller owns every buffer.  The library allocates no
 *     memory.
 *   - All work is enqueued on `stream` (0 = legacy default stream) and the call
 *     returns without synchronising.
 *   - The return value (qsgd_err) reports argument and launch errors found on the
 *     host.  Data-dependent conditions found on the device are OR-ed into the
 *     device word *d_status (QSGD_ST_* bits); the caller zeroes it beforehand and
 *     reads it after synchronising.  d_status may not be NULL.
 *   - Limits: 0 <= n <= 2^34, 1 <= d <= 2^31, 1 <= s <= 2^22, and the size bound
 *     of the stream (qsgd_max_encoded_words * 32) below 2^38 bits.
 *   - Kernels never trap and never wait without a bound.
 */
#ifndef QSGD_H
#define QSGD_H

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define QSGD_API __attribute__((visibility("default")))
#else
#define QSGD_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Host return codes. */
typedef enum {
    QSGD_OK = 0,
    QSGD_ERR_ARG = 1,       /* a pointer, size or parameter out of range */
    QSGD_ERR_CAPACITY = 2,  /* output buffer smaller than qsgd_max_encoded_words */
    QSGD_ERR_CUDA = 3,      /* a CUDA runtime call or kernel launch failed */
    QSGD_ERR_WORKSPACE = 4,   /* workspace smaller than qsgd_encode_workspace_bytes */
    QSGD_ERR_STATIC_LIMIT = 5 /* qsgd_encode_static_ws: the problem needs more scan state than
                                 the library's fixed device workspace */
} qsgd_err;

/* Device status bits, OR-ed into *d_status. */
enum {
    QSGD_ST_NONFINITE = 1,        /* encode: a bucket's norm is not finite; sent as zero */
    QSGD_ST_BAD_STREAM = 2,       /* decode: malformed bucket (see qsgd_decode) */
    QSGD_ST_LOOKBACK_TIMEOUT = 4, /* encode: a bounded wait ran out; output invalid */
    QSGD_ST_OVERFLOW = 8,         /* encode: a write would pass words_capacity */
    QSGD_ST_RANGE = 16            /* encode: norm > 0 but s/norm overflows fp32; sent as zero */
};

/* Bucket scale of the encoders' _ex forms.  QSGD_NORM_L2 is the definition
 * paragraph's ||v||_2 (what qsgd_encode and qsgd_bbit_encode use).  QSGD_NORM_MAX is
 * max_i |v_i|, the QSGDinf heuristic that the NUQSGD abstract names (no formula on
 * the page: the name gives the norm); a NaN in a bucket makes it non-finite.  The
 * scale is sent in the norm field, so the decoders are the same for both. */
enum { QSGD_NORM_L2 = 0, QSGD_NORM_MAX = 1 };

/* Number of buckets, ceil(n / d) (0 when d == 0). */
QSGD_API uint64_t qsgd_num_buckets(uint64_t n, uint32_t d);

/* Worst-case stream size in 32-bit words: ceil(sum_b (32 + m_b*(2 + |omega(s)|)) / 32)
 * with m_b the length of bucket b.  A record of gap g costs at most g*(2+|omega(s)|)
 * bits and the gaps of a bucket sum to at most m_b.  Returns 0 for invalid d or s. */
QSGD_API uint64_t qsgd_max_encoded_words(uint64_t n, uint32_t d, uint32_t s);

/* Bytes of device workspace qsgd_encode (and _ex, _ef) needs for (n, d, s).  The
 * workspace holds, for the shapes the two-launch encoder takes (d % 4 == 0,
 * 4 <= d <= 1024, or d <= 16384 for s <= 31, 16-byte aligned input): a control
 * block, one scan descriptor per 256 buckets, each bucket's bit count and a staging
 * slot per bucket of the bucket's largest possible size; for the other shapes, the
 * scan state of the one-pass encoder (control block, tile descriptors, tail words,
 * per-bucket norms for large buckets).  The size is the larger of the two, so one
 * workspace serves every encoder for (n, d, s).  It must be zero-filled once before
 * its first use (qsgd_workspace_init); every encode leaves it ready for the next
 * one, whichever encoder ran before.  One workspace must not be used by two encodes
 * that may run at the same time.  A call that returned an error after enqueueing
 * work (QSGD_ERR_CUDA) may leave it mid-call: zero-fill it again before reusing it. */
QSGD_API size_t qsgd_encode_workspace_bytes(uint64_t n, uint32_t d, uint32_t s);

/* Zero-fills a workspace (cudaMemsetAsync on `stream`). */
QSGD_API int qsgd_workspace_init(void* d_ws, size_t ws_bytes, cudaStream_t stream);

/* Encoder: QSGD-quantises d_in[0..n) bucket by bucket and writes the Elias-omega
 * stream.  (Definition paragraph and the two claims cited above.)
 *   d_in            fp32[n], any alignment (16-byte alignment with d % 4 == 0 and
 *                   d within the limits above takes the two-launch encoder: a
 *                   bucket coder into the staging slots, then a compaction that
 *                   scans the bit counts and moves the bits to their offsets)
 *   seed            Philox key of the stochastic rounding
 *   d_words         uint32[words_capacity]; words past ceil(offsets[nb]/32) are
 *                   not written
 *   words_capacity  must be >= qsgd_max_encoded_words(n, d, s), else QSGD_ERR_CAPACITY
 *   d_offsets       uint64[nb+1] (bit offsets, see above); 8-byte aligned
 *   d_ws, ws_bytes  workspace of at least qsgd_encode_workspace_bytes(n, d, s)
 *   d_status        NONFINITE / RANGE per degenerate bucket (sent as 32 zero bits),
 *                   LOOKBACK_TIMEOUT or OVERFLOW if the output is not valid.
 * The stream is a deterministic function of (d_in, n, d, s, seed). */
QSGD_API int qsgd_encode(const float* d_in, uint64_t n, uint32_t d, uint32_t s, uint64_t seed,
                uint32_t* d_words, uint64_t words_capacity, uint64_t* d_offsets,
                void* d_ws, size_t ws_bytes, uint32_t* d_status, cudaStream_t stream);

/* qsgd_encode with the bucket scale chosen by norm_kind (QSGD_NORM_L2 or
 * QSGD_NORM_MAX, else QSGD_ERR_ARG).  Under QSGD_NORM_MAX the sent norm is exactly
 * max_i |v_i|, and the largest value of a bucket gets level s whenever
 * fl(max * fl(s / max)) rounds to s. */
QSGD_API int qsgd_encode_ex(const float* d_in, uint64_t n, uint32_t d, uint32_t s, uint64_t seed,
                            uint32_t norm_kind, uint32_t* d_words, uint64_t words_capacity,
                            uint64_t* d_offsets, void* d_ws, size_t ws_bytes, uint32_t* d_status,
                            cudaStream_t stream);

/* Error feedback around the Elias codec ("Sparsified SGD with Memory", abstract: the
 * compressor keeps what it did not send in memory and adds it to the next gradient).
 * Per coordinate, p = fl(e + g); the stream is qsgd_encode_ex of p (same d, s, seed,
 * norm_kind, words, offsets, workspace and status rules); then e becomes
 * fl(p - q), where q is the value qsgd_decode gives the coordinate.  Where no record
 * was sent (q = +0), e keeps p bit for bit.  The learning rate is the caller's: scale
 * g first.
 *   d_g  [n] fp32, device, read only.
 *   d_e  [n] fp32, device, read and overwritten.  It must not overlap d_g
 *        (QSGD_ERR_ARG).  Both are 4-byte aligned.
 * The encode is one fused kernel when the fast encoder takes the shape and both
 * arrays are 16-byte aligned.  Otherwise it is three kernels: e <- e + g, the encoder
 * on e, and a pass that subtracts the decoded values.  After a non-zero status
 * (overflow, abort), d_e is unspecified. */
QSGD_API int qsgd_encode_ef(const float* d_g, float* d_e, uint64_t n, uint32_t d, uint32_t s, uint64_t seed,
                            uint32_t norm_kind, uint32_t* d_words, uint64_t words_capacity,
                            uint64_t* d_offsets, void* d_ws, size_t ws_bytes, uint32_t* d_status,
                            cudaStream_t stream);

/* Decoder: writes Q_s(v) as dense fp32 d_out[0..n) (definition paragraph:
 * ||v||_2 * sgn(v_i) * k_i / s, evaluated as fl(fl(norm/s) * k), sign last; +0.0 off
 * the support).  Buckets are decoded in parallel from d_offsets.
 *   d_words, num_words  the stream and its length in words (bounds every read)
 *   d_offsets           uint64[nb+1] as written by qsgd_encode
 * Sets QSGD_ST_BAD_STREAM for a bucket whose bits overrun offsets[b+1], whose header
 * range is shorter than 32 bits or passes 32*num_words, or that holds an index
 * >= bucket length, a level k > s or 0, or a negative / non-finite norm, or a zero
 * norm with records.  A malformed bucket's outputs are unspecified; nothing outside
 * that bucket's range of d_out is written. */
QSGD_API int qsgd_decode(const uint32_t* d_words, uint64_t num_words, const uint64_t* d_offsets,
                uint64_t n, uint32_t d, uint32_t s, float* d_out, uint32_t* d_status,
                cudaStream_t stream);

/* Receiver aggregation: d_out[i] <- (((d_out[i] + q^0_i) + q^1_i) + ... + q^{K-1}_i),
 * fp32 adds in stream order j = 0..K-1, q^j the decoded stream j (+0.0 off its
 * support).  All K streams were encoded with the same (n, d, s).
 *   h_words, h_num_words, h_offsets  host arrays of K entries holding device
 *                                    pointers / word counts (copied at the call)
 *   1 <= K <= 1024
 * Status bits as for qsgd_decode.  Up to 16 streams go to one launch (launches in
 * stream order).  With a 16-byte aligned d_out and d % 4 == 0: for d <= 1024 and
 * s <= 127 the streams are parsed side by side (a warp per stream) into byte codes
 * and added segment by segment, d_out read and written once per eight streams; for
 * d <= 4096 and s < 1024 otherwise they are decoded side by side onto fp32 tiles; for
 * d <= 1024 and larger s they are added onto fp32 tiles one after another; for
 * d > 1024 the launch adds +0 to the buckets' outputs and then each stream's records
 * in order.  One stream on d <= 1024 takes the one-stream row decoder.  The result is
 * the same on every path. */
QSGD_API int qsgd_decode_accumulate(const uint32_t* const* h_words, const uint64_t* h_num_words,
                           const uint64_t* const* h_offsets, int K, uint64_t n, uint32_t d,
                           uint32_t s, float* d_out, uint32_t* d_status, cudaStream_t stream);

/* The mean of K received streams, the update of a node in data-parallel training (the
 * definition paragraph places QSGD in distributed data-parallel optimisation).
 *   d_out[i] = (q^0[i] + q^1[i] + ... + q^{K-1}[i]) / K
 * The sum runs left to right from +0, in fp32, as in qsgd_decode_accumulate; then one
 * IEEE division by K per coordinate.  d_out is overwritten, not accumulated.  The
 * arguments and the status are those of qsgd_decode_accumulate (1 <= K <= 1024, host
 * arrays of device pointers).  Every stream is checked before the first launch.  Two
 * or more streams on the shapes qsgd_decode_accumulate decodes side by side divide in
 * the same pass.  One stream, or another shape, is decoded, accumulated and then
 * divided in a separate pass. */
QSGD_API int qsgd_decode_mean(const uint32_t* const* h_words, const uint64_t* h_num_words,
                              const uint64_t* const* h_offsets, int K, uint64_t n, uint32_t d,
                              uint32_t s, float* d_out, uint32_t* d_status, cudaStream_t stream);

/* Encoder for callers that cannot allocate device memory.  (The paper has no
 * counterpart: this is a deployment variant of qsgd_encode.)
 *
 * Who needs it: code that compresses a gradient at a point where it may not call
 * cudaMalloc -- inside a caching allocator's own callbacks, in a communication
 * library's progress thread that must not take the allocator's lock, or in an
 * embedding that only passes the codec its input and output buffers.  The output
 * buffers are still the caller's; only the encoder's scan state (the workspace of
 * qsgd_encode) moves into a fixed array of device memory owned by the library.
 *
 * Same arguments and results as qsgd_encode without d_ws / ws_bytes; the stream
 * is bit-identical to qsgd_encode's for the same (d_in, n, d, s, seed).
 *   - The array is qsgd_static_workspace_limit() bytes (4 MiB).  Every GPU that
 *     loads the library holds it until the process exits.  A problem whose
 *     one-pass scan state does not fit is rejected with QSGD_ERR_STATIC_LIMIT
 *     before anything is enqueued (about 1.4 million buckets at d = 512).  A
 *     problem whose staging slots also fit takes the two-launch encoder; the
 *     others take the one-pass encoder.  The stream is the same either way.
 *   - The first call on a device looks up the array's device address (once per
 *     device, with that device current).  Make that first call before any stream
 *     capture.
 *   - Every call shares the one array.  Its state is tagged with a call counter
 *     and reset by the end of each call, so no call needs to clear it, but calls
 *     that may overlap on the GPU (different streams, or different host threads)
 *     race and must be serialised by the caller.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library routine. */
QSGD_API int qsgd_encode_static_ws(const float* d_in, uint64_t n, uint32_t d, uint32_t s, uint64_t seed,
                                   uint32_t* d_words, uint64_t words_capacity, uint64_t* d_offsets,
                                   uint32_t* d_status, cudaStream_t stream);

/* Bytes of the fixed device workspace behind qsgd_encode_static_ws. */
QSGD_API size_t qsgd_static_workspace_limit(void);

/* ---- Fixed-width b-bit QSGD (b = 2, 4, 8) ---------------------------------------
 * The "4-bit and 2-bit QSGD" of the claim "QSVRG, non-convex and multi-GPU bucketed
 * training" (and the 4/8-bit of the curated limitations): s = 2^(b-1) - 1 levels with
 * the quantiser, random words and bucket norms of qsgd_encode; no Elias coding.  The
 * page gives no layout; this library's (its "Fixed-width b-bit variant" section):
 *   d_norms  float32[nb], the sent norm of every bucket (0 for a zero, non-finite or
 *            out-of-range bucket, which also sets NONFINITE / RANGE);
 *   d_codes  uint32[qsgd_bbit_code_words(n, b)]: coordinate i has the code
 *            (sign << (b-1)) | k at bits [i*b, i*b + b), MSB-first in each word (bit j
 *            is bit 31 - j%32 of word j/32); the sign bit is 1 only for k >= 1 and a
 *            negative v_i; bits past n*b are 0.
 * Every code sits at a fixed place, so both directions are data-parallel passes. */

/* Words of the code array: ceil(n * b / 32). */
QSGD_API uint64_t qsgd_bbit_code_words(uint64_t n, uint32_t b);

/* b-bit encoder.  b in {2, 4, 8}, else QSGD_ERR_ARG; d_norms 4-byte aligned, d_codes
 * 4-byte aligned with qsgd_bbit_code_words(n, b) words.  Allocates nothing; one or two
 * kernel launches on `stream`.  Codes are a deterministic function of
 * (d_in, n, d, b, seed); norms within 1e-6 relative of the exactly rounded norm. */
QSGD_API int qsgd_bbit_encode(const float* d_in, uint64_t n, uint32_t d, uint32_t b, uint64_t seed,
                              float* d_norms, uint32_t* d_codes, uint32_t* d_status, cudaStream_t stream);

/* qsgd_bbit_encode with the bucket scale chosen by norm_kind (QSGD_NORM_L2 or
 * QSGD_NORM_MAX, else QSGD_ERR_ARG). */
QSGD_API int qsgd_bbit_encode_ex(const float* d_in, uint64_t n, uint32_t d, uint32_t b, uint64_t seed,
                                 uint32_t norm_kind, float* d_norms, uint32_t* d_codes, uint32_t* d_status,
                                 cudaStream_t stream);

/* Error feedback around the b-bit codec: p = fl(e + g) is coded as qsgd_bbit_encode_ex
 * would code it, and e becomes fl(p - q) (q as qsgd_bbit_decode gives it), or p where
 * the code's level is 0.  The argument rules are those of qsgd_encode_ef: d_g is read,
 * d_e is overwritten, and the two must not overlap.  The encode is one kernel for
 * d in {128, 256, 512, 1024} with d_g and d_e 16-byte aligned, else three. */
QSGD_API int qsgd_bbit_encode_ef(const float* d_g, float* d_e, uint64_t n, uint32_t d, uint32_t b,
                                 uint64_t seed, uint32_t norm_kind, float* d_norms, uint32_t* d_codes,
                                 uint32_t* d_status, cudaStream_t stream);

/* b-bit decoder: d_out[0..n) = fl(fl(norm/s) * k), negated for sign 1, +0.0 for k = 0.
 * Sets QSGD_ST_BAD_STREAM for a negative or non-finite norm, a non-zero code under a
 * zero norm or a zero scale, or a code with sign 1 and k = 0 (that bucket's output is
 * then unspecified; nothing outside d_out[0..n) is written). */
QSGD_API int qsgd_bbit_decode(const float* d_norms, const uint32_t* d_codes, uint64_t n, uint32_t d,
                              uint32_t b, float* d_out, uint32_t* d_status, cudaStream_t stream);

/* b-bit receiver aggregation: d_out[i] <- ((d_out[i] + q^0_i) + ...) + q^{K-1}_i, fp32
 * adds in stream order.  h_norms, h_codes: host arrays of K device pointers; 1 <= K. */
QSGD_API int qsgd_bbit_decode_accumulate(const float* const* h_norms, const uint32_t* const* h_codes, int K,
                                         uint64_t n, uint32_t d, uint32_t b, float* d_out, uint32_t* d_status,
                                         cudaStream_t stream);

/* The mean of K b-bit streams: d_out[i] = (q^0[i] + ... + q^{K-1}[i]) / K, with the
 * order, rounding and arguments of qsgd_decode_mean. */
QSGD_API int qsgd_bbit_decode_mean(const float* const* h_norms, const uint32_t* const* h_codes, int K,
                                   uint64_t n, uint32_t d, uint32_t b, float* d_out, uint32_t* d_status,
                                   cudaStream_t stream);

/* Static description of a host return code. */
QSGD_API const char* qsgd_error_string(int code);

/* Library version string. */
QSGD_API const char* qsgd_version(void);

#ifdef __cplusplus
}
#endif
#endif
