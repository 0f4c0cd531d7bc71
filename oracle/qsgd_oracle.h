/*
 * CPU oracle for the QSGD codec.  TEST INFRASTRUCTURE ONLY.
 *
 * Plain, slow, single-threaded C that follows the method step by step so that a
 * reader can check it against the source page by eye.  Only the test suite, the
 * smoke check and the CPU-baseline leg of the benchmark may load it.  It shares
 * no code, header, table or constant with the CUDA library.
 *
 * Source of the method: "QSGD (Quantized Stochastic Gradient Descent) with Elias
 * Coding" (AIMech curated entry) -- its definition paragraph (quantiser, coded
 * tuple), claim "Elias coding communication complexity tradeoff" (fields that are
 * coded, F = 32-bit norm) and claim "QSVRG, non-convex and multi-GPU bucketed
 * training" (d-block bucketing).  Random source: Philox4x32-10 from Salmon et al.,
 * "Parallel Random Numbers: As Easy as 1, 2, 3" (SC'11).  Elias omega code:
 * P. Elias, "Universal codeword sets and representations of the integers" (1975).
 *
 * Pins (tests/test_oracle_*.py): Philox known-answer vectors; omega code brute
 * force over 1..2^20 and textbook codewords; hand-derived golden bitstreams;
 * unbiasedness, the closed-form variance, the sparsity bound and the 2.818n+32
 * bit bound from the page's claims; the size bound by brute force.  Error feedback
 * ("Sparsified SGD with Memory", abstract): exact steps, closed-form outcomes and the
 * telescoping sum of sent values plus memory (tests/test_oracle_ef.py).  The mean of
 * K received streams: hand values, K = 1 and 2, the rounding bound, unbiasedness
 * (tests/test_oracle_mean.py).
 */
#ifndef QSGD_ORACLE_H
#define QSGD_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* status bits, OR-ed into *status */
#define QO_ST_NONFINITE 1u
#define QO_ST_BAD_STREAM 2u
#define QO_ST_OVERFLOW 8u
#define QO_ST_RANGE 16u

/* Philox4x32-10 block function: out = philox(ctr, key). */
void qo_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]);

/* The 32-bit random word r_i drawn for global coordinate i. */
uint32_t qo_random_word(uint64_t seed, uint64_t i);

/* Number of bits of the Elias omega codeword of N (N >= 1). */
int qo_omega_len(uint64_t N);

/* Writes the omega codeword of N (MSB first) into bits[0..len-1] as 0/1 bytes;
 * returns len. */
int qo_omega_bits(uint64_t N, uint8_t* bits);

/* Encodes N at bit position *pos of words[cap_words] (MSB-first words, the
 * caller zeroes the words); returns 0, or -1 if it would pass the end. */
int qo_omega_put(uint32_t* words, uint64_t cap_words, uint64_t* pos, uint64_t N);

/* Decodes one omega codeword starting at *pos, reading no bit at or past
 * end_bit; returns 0 and sets *N, or -1 on overrun / value above 2^62. */
int qo_omega_get(const uint32_t* words, uint64_t* pos, uint64_t end_bit, uint64_t* N);

/* fp32 L2 norm of one bucket: exact-ish sum of squares in double, rounded once. */
float qo_bucket_norm(const float* v, uint64_t m);

/* max_i |v_i| of m values (NaN if any value is NaN): the QSGDinf scale.  Passed to
 * the encoders as norms_in, it gives the max-norm variant of either format. */
float qo_bucket_maxnorm(const float* v, uint64_t m);

/* Quantises one bucket v[0..m) that starts at global index base.  Writes the
 * signed levels (+k or -k; 0 off the support) to levels[0..m) and returns the
 * norm that is sent (0 for a degenerate bucket).  norm_in: if non-NULL, this
 * norm is used instead of qo_bucket_norm (re-quantisation with another
 * implementation's norm). */
float qo_quantize_bucket(const float* v, uint64_t m, uint64_t base, uint32_t s,
                         uint64_t seed, const float* norm_in, int32_t* levels,
                         uint32_t* status);

/* Size bound in bits of one bucket of m coordinates. */
uint64_t qo_bucket_bit_bound(uint64_t m, uint32_t s);

/* Capacity in 32-bit words for the whole stream. */
uint64_t qo_capacity_words(uint64_t n, uint64_t d, uint32_t s);

/* Encoder.  words[cap_words] (zeroed here), offsets[nb+1].  norms_in: NULL or
 * nb norms to use instead of the oracle's own.  norms_out: NULL or nb floats
 * (the norm each bucket sends).  Returns 0, or -1 on a bad argument. */
int qo_encode(const float* v, uint64_t n, uint64_t d, uint32_t s, uint64_t seed,
              const float* norms_in, uint32_t* words, uint64_t cap_words,
              uint64_t* offsets, float* norms_out, uint32_t* status);

/* Encoder of the buckets [b0, b1) of the vector v[0..n) as a standalone stream:
 * the same bits as bits [offsets[b0], offsets[b1]) of qo_encode's stream (every
 * coordinate keeps its global index, so its Philox word), shifted to start at bit 0.
 * words[cap_words] (zeroed here), offsets[b1 - b0 + 1] relative to the slice start;
 * norms_in / norms_out: NULL or b1 - b0 norms of these buckets.  Returns 0 or -1. */
int qo_encode_range(const float* v, uint64_t n, uint64_t d, uint32_t s, uint64_t seed, uint64_t b0,
                    uint64_t b1, const float* norms_in, uint32_t* words, uint64_t cap_words,
                    uint64_t* offsets, float* norms_out, uint32_t* status);

/* Encodes one bucket v[0..m) whose first coordinate has global index base at bit
 * *pos (advanced); levels[m] is scratch.  Returns 0 or -1 on overflow. */
int qo_encode_bucket(const float* v, uint64_t m, uint64_t base, uint32_t s, uint64_t seed,
                     const float* norm_in, uint32_t* words, uint64_t cap_words, uint64_t* pos,
                     float* norm_out, int32_t* levels, uint32_t* status);

/* Decodes the bucket stored in bits [begin, end) (m coordinates) into out[m]. */
int qo_decode_bucket(const uint32_t* words, uint64_t begin, uint64_t end, uint64_t m,
                     uint32_t s, float* out, uint32_t* status);

/* Decoder: out[n]. */
int qo_decode(const uint32_t* words, const uint64_t* offsets, uint64_t n, uint64_t d,
              uint32_t s, float* out, uint32_t* status);

/* Decoded signed levels instead of values (levels[n], 0 off the support). */
int qo_decode_levels(const uint32_t* words, const uint64_t* offsets, uint64_t n,
                     uint64_t d, uint32_t s, int32_t* levels, float* norms,
                     uint32_t* status);

/* out[i] <- out[i] + q^0[i] + ... + q^{K-1}[i], left to right. */
int qo_decode_accumulate(const uint32_t* const* words, const uint64_t* const* offsets,
                         int K, uint64_t n, uint64_t d, uint32_t s, float* out,
                         uint32_t* status);

/* ---- Fixed-width b-bit variant (b = 2, 4, 8) ----------------------------------
 * The "4-bit and 2-bit QSGD" of the claim "QSVRG, non-convex and multi-GPU bucketed
 * training" (and the 4/8-bit of the curated limitations): s = 2^(b-1) - 1 levels, the
 * same quantiser and random words as above, and per coordinate a b-bit code
 * (sign << (b-1)) | k packed densely at bits [i*b, i*b + b) of the code words,
 * MSB-first; one fp32 norm per bucket in its own array. */

/* s = 2^(b-1) - 1 for b in {2, 4, 8}; 0 otherwise. */
uint32_t qo_bbit_levels(uint32_t b);

/* Words of the code array for n coordinates: ceil(n*b / 32). */
uint64_t qo_bbit_code_words(uint64_t n, uint32_t b);

/* codes must hold qo_bbit_code_words(n, b) words (cleared here); norms_out[nb]
 * receives the sent norms.  norms_in (nullable) replaces the computed norms. */
int qo_bbit_encode(const float* v, uint64_t n, uint64_t d, uint32_t b, uint64_t seed,
                   const float* norms_in, float* norms_out, uint32_t* codes, uint32_t* status);

/* Dense decode; BAD_STREAM for a negative or non-finite norm, a non-zero code under
 * a zero norm or a zero scale fl(norm/s), or a code with sign 1 and k = 0. */
int qo_bbit_decode(const float* norms, const uint32_t* codes, uint64_t n, uint64_t d, uint32_t b,
                   float* out, uint32_t* status);

/* out[i] <- out[i] + q^0[i] + ... + q^{K-1}[i], left to right. */
int qo_bbit_decode_accumulate(const float* const* norms, const uint32_t* const* codes, int K,
                              uint64_t n, uint64_t d, uint32_t b, float* out, uint32_t* status);

/* ---- Error feedback ("Sparsified SGD with Memory", abstract) -------------------
 * p = e + g; the stream (or codes) carries Q(p); e <- p - Q(p), Q(p) as decoded, and
 * e <- p where a coordinate has no record.  max_norm: scale by the max-norms of p
 * (QSGDinf) when norms_in is NULL.  e[n] is read and overwritten. */
int qo_encode_ef(const float* g, float* e, uint64_t n, uint64_t d, uint32_t s, uint64_t seed,
                 int max_norm, const float* norms_in, uint32_t* words, uint64_t cap_words,
                 uint64_t* offsets, float* norms_out, uint32_t* status);
int qo_bbit_encode_ef(const float* g, float* e, uint64_t n, uint64_t d, uint32_t b, uint64_t seed,
                      int max_norm, const float* norms_in, float* norms_out, uint32_t* codes,
                      uint32_t* status);
/* ---- Data-parallel exchange ("for distributed data-parallel optimization") -------
 * out[i] = (q^0[i] + ... + q^{K-1}[i]) / K: the sum left to right from +0, then one
 * fp32 division by K. */
int qo_decode_mean(const uint32_t* const* words, const uint64_t* const* offsets, int K, uint64_t n,
                   uint64_t d, uint32_t s, float* out, uint32_t* status);
int qo_bbit_decode_mean(const float* const* norms, const uint32_t* const* codes, int K, uint64_t n,
                        uint64_t d, uint32_t b, float* out, uint32_t* status);
#ifdef __cplusplus
}
#endif
#endif
