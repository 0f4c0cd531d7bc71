/*
 * CPU oracle for the QSGD codec.  TEST INFRASTRUCTURE ONLY (see qsgd_oracle.h).
 *
 * Build: gcc -O2 -std=c99 -ffp-contract=off -fno-fast-math -shared -fPIC.
 * Every float operation below is a single IEEE binary32 operation rounded to
 * nearest-even (x86-64 SSE; no contraction into FMA).
 */
#include "qsgd_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------- */
/* Philox4x32-10 (Salmon, Moraes, Dror, Shaw, SC'11, section 4: the Philox    */
/* S-box is a 32x32->64 multiply; the bijection is                            */
/*   (x0,x1,x2,x3) -> (hi(M1*x2)^x1^k0, lo(M1*x2), hi(M0*x0)^x3^k1, lo(M0*x0)) */
/* and the key is bumped by the Weyl constants between rounds).               */
/* ------------------------------------------------------------------------- */

void qo_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]) {
    const uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u;
    const uint32_t W0 = 0x9E3779B9u, W1 = 0xBB67AE85u;
    uint32_t x0 = ctr[0], x1 = ctr[1], x2 = ctr[2], x3 = ctr[3];
    uint32_t k0 = key[0], k1 = key[1];
    for (int round = 0; round < 10; ++round) {
        if (round > 0) {
            k0 += W0;
            k1 += W1;
        }
        uint64_t prod0 = (uint64_t)M0 * (uint64_t)x0;
        uint64_t prod1 = (uint64_t)M1 * (uint64_t)x2;
        uint32_t hi0 = (uint32_t)(prod0 >> 32), lo0 = (uint32_t)prod0;
        uint32_t hi1 = (uint32_t)(prod1 >> 32), lo1 = (uint32_t)prod1;
        uint32_t y0 = hi1 ^ x1 ^ k0;
        uint32_t y1 = lo1;
        uint32_t y2 = hi0 ^ x3 ^ k1;
        uint32_t y3 = lo0;
        x0 = y0;
        x1 = y1;
        x2 = y2;
        x3 = y3;
    }
    out[0] = x0;
    out[1] = x1;
    out[2] = x2;
    out[3] = x3;
}

/* Counter (i div 4) in the first two counter words, seed as the key, word i mod 4. */
uint32_t qo_random_word(uint64_t seed, uint64_t i) {
    uint64_t j = i / 4;
    uint32_t ctr[4] = {(uint32_t)(j & 0xFFFFFFFFu), (uint32_t)(j >> 32), 0u, 0u};
    uint32_t key[2] = {(uint32_t)(seed & 0xFFFFFFFFu), (uint32_t)(seed >> 32)};
    uint32_t out[4];
    qo_philox4x32_10(ctr, key, out);
    return out[i % 4];
}

/* ------------------------------------------------------------------------- */
/* Elias omega code (Elias 1975, "recursive" code): start with "0"; while     */
/* N > 1, prepend binary(N) and replace N by (number of bits of N) - 1.       */
/* The page names "Elias recursive gamma/omega integer coding" in its         */
/* definition paragraph and "Elias recursive prefix codes" in the claim       */
/* "Elias coding communication complexity tradeoff".                          */
/* ------------------------------------------------------------------------- */

static int bit_length(uint64_t x) {
    int b = 0;
    while (x != 0) {
        b += 1;
        x >>= 1;
    }
    return b;
}

int qo_omega_len(uint64_t N) {
    int len = 1; /* the final "0" */
    while (N > 1) {
        int b = bit_length(N);
        len += b;
        N = (uint64_t)(b - 1);
    }
    return len;
}

int qo_omega_bits(uint64_t N, uint8_t* bits) {
    /* Collect the groups from the last prepended to the first, then emit them
     * in stream order. */
    uint64_t groups[8];
    int ngroups = 0;
    while (N > 1) {
        groups[ngroups++] = N;
        N = (uint64_t)(bit_length(N) - 1);
    }
    int len = 0;
    for (int g = ngroups - 1; g >= 0; --g) {
        int b = bit_length(groups[g]);
        for (int t = b - 1; t >= 0; --t) bits[len++] = (uint8_t)((groups[g] >> t) & 1u);
    }
    bits[len++] = 0;
    return len;
}

static int put_bit(uint32_t* words, uint64_t cap_words, uint64_t* pos, int bit) {
    uint64_t w = *pos / 32;
    if (w >= cap_words) return -1;
    if (bit) words[w] |= (uint32_t)1u << (31 - (unsigned)(*pos % 32));
    *pos += 1;
    return 0;
}

static int get_bit(const uint32_t* words, uint64_t* pos, uint64_t end_bit, int* bit) {
    if (*pos >= end_bit) return -1;
    *bit = (int)((words[*pos / 32] >> (31 - (unsigned)(*pos % 32))) & 1u);
    *pos += 1;
    return 0;
}

int qo_omega_put(uint32_t* words, uint64_t cap_words, uint64_t* pos, uint64_t N) {
    uint8_t bits[160];
    int len = qo_omega_bits(N, bits);
    for (int t = 0; t < len; ++t)
        if (put_bit(words, cap_words, pos, bits[t]) != 0) return -1;
    return 0;
}

int qo_omega_get(const uint32_t* words, uint64_t* pos, uint64_t end_bit, uint64_t* N) {
    uint64_t value = 1;
    for (;;) {
        int bit;
        if (get_bit(words, pos, end_bit, &bit) != 0) return -1;
        if (bit == 0) break;
        /* a 1 starts the next group: it is the leading bit of a (value+1)-bit number */
        if (value > 62) return -1;
        uint64_t next = 1;
        for (uint64_t t = 0; t < value; ++t) {
            if (get_bit(words, pos, end_bit, &bit) != 0) return -1;
            next = (next << 1) | (uint64_t)bit;
        }
        value = next;
    }
    *N = value;
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Quantiser: definition paragraph of "QSGD ... with Elias Coding":           */
/*   Q_s(v)_i = ||v||_2 * sgn(v_i) * xi_i(v, s),                              */
/*   l_i = floor(s |v_i| / ||v||_2), p_i = s |v_i| / ||v||_2 - l_i,            */
/*   xi_i = (l_i + 1)/s with probability p_i, else l_i / s,                   */
/*   levels k_i = s * xi_i.                                                   */
/* Buckets (claim "QSVRG, non-convex and multi-GPU bucketed training",       */
/* section 3.3): each d-block is quantised with its own norm.                 */
/* ------------------------------------------------------------------------- */

float qo_bucket_norm(const float* v, uint64_t m) {
    double sum = 0.0;
    for (uint64_t i = 0; i < m; ++i) sum += (double)v[i] * (double)v[i];
    return (float)sqrt(sum);
}

/* The max-norm ||v||_inf of a bucket: the scale of the QSGDinf heuristic (named
   in the NUQSGD abstract; the name gives the norm).  NaN when any value is NaN, so
   that such a bucket is non-finite like under the L2 norm. */
float qo_bucket_maxnorm(const float* v, uint64_t m) {
    float mx = 0.0f;
    for (uint64_t i = 0; i < m; ++i) {
        if (isnan(v[i])) return NAN;
        if (fabsf(v[i]) > mx) mx = fabsf(v[i]);
    }
    return mx;
}

float qo_quantize_bucket(const float* v, uint64_t m, uint64_t base, uint32_t s,
                         uint64_t seed, const float* norm_in, int32_t* levels,
                         uint32_t* status) {
    for (uint64_t i = 0; i < m; ++i) levels[i] = 0;
    float norm = norm_in ? *norm_in : qo_bucket_norm(v, m);
    if (!isfinite(norm)) {
        *status |= QO_ST_NONFINITE;
        return 0.0f;
    }
    if (norm == 0.0f) return 0.0f;
    float sinv = (float)s / norm; /* s / ||v||_2, one division per bucket */
    if (!isfinite(sinv)) {
        *status |= QO_ST_RANGE;
        return 0.0f;
    }
    for (uint64_t i = 0; i < m; ++i) {
        float t = fabsf(v[i]) * sinv; /* s |v_i| / ||v||_2 */
        float l = floorf(t);          /* l_i */
        float p = t - l;              /* p_i, exact */
        uint32_t r = qo_random_word(seed, base + i);
        float u = (float)(r >> 9) * 0x1p-23f; /* uniform on the 2^-23 grid, exact */
        uint32_t k = (uint32_t)l;
        if (u < p) k += 1; /* round up with probability p_i */
        if (k > s) k = s;
        levels[i] = signbit(v[i]) ? -(int32_t)k : (int32_t)k;
    }
    return norm;
}

/* ------------------------------------------------------------------------- */
/* Coding: the tuple (||v||_2, signs, run-length gaps, levels k_i) of the     */
/* definition paragraph; F = 32 bits for the norm (claim "Elias coding        */
/* communication complexity tradeoff").  Records are omega(gap) sign omega(k) */
/* per non-zero in ascending index, the first gap counted from index -1.      */
/* ------------------------------------------------------------------------- */

uint64_t qo_bucket_bit_bound(uint64_t m, uint32_t s) {
    return 32u + m * (uint64_t)(2 + qo_omega_len(s));
}

uint64_t qo_capacity_words(uint64_t n, uint64_t d, uint32_t s) {
    if (n == 0) return 0;
    uint64_t nb = (n + d - 1) / d;
    uint64_t bits = 0;
    for (uint64_t b = 0; b < nb; ++b) {
        uint64_t m = (b + 1 == nb) ? n - b * d : d;
        bits += qo_bucket_bit_bound(m, s);
    }
    return (bits + 31) / 32;
}

static int put_bits_msb_first(uint32_t* words, uint64_t cap, uint64_t* pos, uint32_t value,
                              int nbits) {
    for (int t = nbits - 1; t >= 0; --t)
        if (put_bit(words, cap, pos, (int)((value >> t) & 1u)) != 0) return -1;
    return 0;
}

int qo_encode_bucket(const float* v, uint64_t m, uint64_t base, uint32_t s, uint64_t seed,
                     const float* norm_in, uint32_t* words, uint64_t cap_words, uint64_t* pos,
                     float* norm_out, int32_t* levels, uint32_t* status) {
    float norm = qo_quantize_bucket(v, m, base, s, seed, norm_in, levels, status);
    if (norm_out) *norm_out = norm;
    uint32_t norm_bits;
    memcpy(&norm_bits, &norm, sizeof norm_bits);
    int err = put_bits_msb_first(words, cap_words, pos, norm_bits, 32);
    int64_t prev = -1;
    for (uint64_t i = 0; i < m && err == 0; ++i) {
        if (levels[i] == 0) continue;
        uint64_t gap = (uint64_t)((int64_t)i - prev);
        prev = (int64_t)i;
        uint32_t k = (uint32_t)(levels[i] < 0 ? -levels[i] : levels[i]);
        err |= qo_omega_put(words, cap_words, pos, gap);
        err |= put_bit(words, cap_words, pos, levels[i] < 0);
        err |= qo_omega_put(words, cap_words, pos, k);
    }
    if (err) *status |= QO_ST_OVERFLOW;
    return err ? -1 : 0;
}

int qo_encode(const float* v, uint64_t n, uint64_t d, uint32_t s, uint64_t seed,
              const float* norms_in, uint32_t* words, uint64_t cap_words,
              uint64_t* offsets, float* norms_out, uint32_t* status) {
    if (d < 1 || s < 1) return -1;
    uint64_t nb = (n + d - 1) / d;
    memset(words, 0, cap_words * sizeof(uint32_t));
    int32_t* levels = (int32_t*)malloc((size_t)(d < n ? d : (n ? n : 1)) * sizeof(int32_t));
    if (!levels) return -1;
    uint64_t pos = 0;
    for (uint64_t b = 0; b < nb; ++b) {
        uint64_t base = b * d;
        uint64_t m = (b + 1 == nb) ? n - base : d;
        offsets[b] = pos;
        if (qo_encode_bucket(v + base, m, base, s, seed, norms_in ? norms_in + b : NULL, words,
                             cap_words, &pos, norms_out ? norms_out + b : NULL, levels,
                             status) != 0) {
            free(levels);
            return -1;
        }
    }
    offsets[nb] = pos;
    free(levels);
    return 0;
}

int qo_encode_range(const float* v, uint64_t n, uint64_t d, uint32_t s, uint64_t seed, uint64_t b0,
                    uint64_t b1, const float* norms_in, uint32_t* words, uint64_t cap_words,
                    uint64_t* offsets, float* norms_out, uint32_t* status) {
    if (d < 1 || s < 1) return -1;
    uint64_t nb = (n + d - 1) / d;
    if (b0 > b1 || b1 > nb) return -1;
    memset(words, 0, cap_words * sizeof(uint32_t));
    int32_t* levels = (int32_t*)malloc((size_t)(d < n ? d : (n ? n : 1)) * sizeof(int32_t));
    if (!levels) return -1;
    uint64_t pos = 0;
    for (uint64_t b = b0; b < b1; ++b) {
        uint64_t base = b * d;
        uint64_t m = (b + 1 == nb) ? n - base : d;
        offsets[b - b0] = pos;
        if (qo_encode_bucket(v + base, m, base, s, seed, norms_in ? norms_in + (b - b0) : NULL, words,
                             cap_words, &pos, norms_out ? norms_out + (b - b0) : NULL, levels,
                             status) != 0) {
            free(levels);
            return -1;
        }
    }
    offsets[b1 - b0] = pos;
    free(levels);
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Decoder: Q_s(v)_i = ||v||_2 * sgn(v_i) * k_i / s, evaluated as             */
/* fl(fl(norm / s) * k) with the sign applied last; zeros off the support.   */
/* ------------------------------------------------------------------------- */

/* Parses bucket b into levels[0..m); returns 0 or -1 on a malformed bucket. */
static int parse_bucket(const uint32_t* words, uint64_t begin, uint64_t end, uint64_t m,
                        uint32_t s, int32_t* levels, float* norm_out) {
    for (uint64_t i = 0; i < m; ++i) levels[i] = 0;
    *norm_out = 0.0f;
    if (end < begin || end - begin < 32) return -1;
    uint64_t pos = begin;
    uint32_t norm_bits = 0;
    for (int t = 0; t < 32; ++t) {
        int bit;
        get_bit(words, &pos, end, &bit);
        norm_bits = (norm_bits << 1) | (uint32_t)bit;
    }
    float norm;
    memcpy(&norm, &norm_bits, sizeof norm);
    *norm_out = norm;
    if (!isfinite(norm) || signbit(norm)) return -1;
    if (norm == 0.0f) return pos == end ? 0 : -1;
    /* a norm whose scale norm/s rounds to zero: no conforming encoder sends records
       under it (s/norm overflows, so the bucket goes out as a zero bucket) */
    if (norm / (float)s == 0.0f && pos < end) return -1;
    int64_t idx = -1;
    while (pos < end) {
        uint64_t gap, k;
        int sign;
        if (qo_omega_get(words, &pos, end, &gap) != 0) return -1;
        if (gap > m || (uint64_t)(idx + (int64_t)gap) >= m) return -1;
        idx += (int64_t)gap;
        if (get_bit(words, &pos, end, &sign) != 0) return -1;
        if (qo_omega_get(words, &pos, end, &k) != 0) return -1;
        if (k > s) return -1;
        levels[idx] = sign ? -(int32_t)k : (int32_t)k;
    }
    return 0;
}

int qo_decode_bucket(const uint32_t* words, uint64_t begin, uint64_t end, uint64_t m,
                     uint32_t s, float* out, uint32_t* status) {
    int32_t* levels = (int32_t*)malloc((size_t)(m ? m : 1) * sizeof(int32_t));
    if (!levels) return -1;
    float norm;
    if (parse_bucket(words, begin, end, m, s, levels, &norm) != 0) *status |= QO_ST_BAD_STREAM;
    float scale = norm / (float)s;
    for (uint64_t i = 0; i < m; ++i) {
        int32_t q = levels[i];
        float value = 0.0f;
        if (q != 0) {
            value = scale * (float)(q < 0 ? -q : q);
            if (q < 0) value = -value;
        }
        out[i] = value;
    }
    free(levels);
    return 0;
}

int qo_decode_levels(const uint32_t* words, const uint64_t* offsets, uint64_t n,
                     uint64_t d, uint32_t s, int32_t* levels, float* norms,
                     uint32_t* status) {
    if (d < 1 || s < 1) return -1;
    uint64_t nb = (n + d - 1) / d;
    for (uint64_t b = 0; b < nb; ++b) {
        uint64_t base = b * d;
        uint64_t m = (b + 1 == nb) ? n - base : d;
        float norm;
        if (parse_bucket(words, offsets[b], offsets[b + 1], m, s, levels + base, &norm) != 0)
            *status |= QO_ST_BAD_STREAM;
        if (norms) norms[b] = norm;
    }
    return 0;
}

int qo_decode(const uint32_t* words, const uint64_t* offsets, uint64_t n, uint64_t d,
              uint32_t s, float* out, uint32_t* status) {
    if (d < 1 || s < 1) return -1;
    uint64_t nb = (n + d - 1) / d;
    for (uint64_t b = 0; b < nb; ++b) {
        uint64_t base = b * d;
        uint64_t m = (b + 1 == nb) ? n - base : d;
        if (qo_decode_bucket(words, offsets[b], offsets[b + 1], m, s, out + base, status) != 0)
            return -1;
    }
    return 0;
}

int qo_decode_accumulate(const uint32_t* const* words, const uint64_t* const* offsets,
                         int K, uint64_t n, uint64_t d, uint32_t s, float* out,
                         uint32_t* status) {
    if (K < 1) return -1;
    float* q = (float*)malloc((size_t)(n ? n : 1) * sizeof(float));
    if (!q) return -1;
    for (int j = 0; j < K; ++j) {
        if (qo_decode(words[j], offsets[j], n, d, s, q, status) != 0) {
            free(q);
            return -1;
        }
        for (uint64_t i = 0; i < n; ++i) out[i] = out[i] + q[i];
    }
    free(q);
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Fixed-width b-bit variant: the quantiser above with s = 2^(b-1) - 1, each  */
/* coordinate's level and sign in b bits at a fixed place; no gaps, no omega. */
/* ------------------------------------------------------------------------- */

uint32_t qo_bbit_levels(uint32_t b) {
    return (b == 2 || b == 4 || b == 8) ? (1u << (b - 1)) - 1u : 0u;
}

uint64_t qo_bbit_code_words(uint64_t n, uint32_t b) {
    return (n * (uint64_t)b + 31u) / 32u;
}

int qo_bbit_encode(const float* v, uint64_t n, uint64_t d, uint32_t b, uint64_t seed,
                   const float* norms_in, float* norms_out, uint32_t* codes, uint32_t* status) {
    uint32_t s = qo_bbit_levels(b);
    if (s == 0 || d < 1) return -1;
    uint64_t nw = qo_bbit_code_words(n, b);
    for (uint64_t w = 0; w < nw; ++w) codes[w] = 0;
    uint64_t nb = (n + d - 1) / d;
    int32_t* levels = (int32_t*)malloc((size_t)(d ? d : 1) * sizeof(int32_t));
    if (!levels) return -1;
    for (uint64_t bk = 0; bk < nb; ++bk) {
        uint64_t base = bk * d;
        uint64_t m = (bk + 1 == nb) ? n - base : d;
        float norm = qo_quantize_bucket(v + base, m, base, s, seed, norms_in ? norms_in + bk : 0, levels, status);
        norms_out[bk] = norm;
        for (uint64_t i = 0; i < m; ++i) {
            uint32_t k = (uint32_t)(levels[i] < 0 ? -levels[i] : levels[i]);
            uint32_t code = ((levels[i] < 0 ? 1u : 0u) << (b - 1)) | k;
            uint64_t pos = (base + i) * b;
            put_bits_msb_first(codes, nw, &pos, code, (int)b);
        }
    }
    free(levels);
    return 0;
}

int qo_bbit_decode(const float* norms, const uint32_t* codes, uint64_t n, uint64_t d, uint32_t b,
                   float* out, uint32_t* status) {
    uint32_t s = qo_bbit_levels(b);
    if (s == 0 || d < 1) return -1;
    uint64_t nw = qo_bbit_code_words(n, b);
    uint64_t nb = (n + d - 1) / d;
    for (uint64_t bk = 0; bk < nb; ++bk) {
        uint64_t base = bk * d;
        uint64_t m = (bk + 1 == nb) ? n - base : d;
        float norm = norms[bk];
        float bscale = norm / (float)s; /* fl(norm / s) */
        int bad = !isfinite(norm) || signbit(norm);
        for (uint64_t i = 0; i < m; ++i) {
            uint64_t pos = (base + i) * b;
            uint32_t code = 0;
            for (uint32_t t = 0; t < b; ++t) {
                int bit = 0;
                get_bit(codes, &pos, nw * 32u, &bit);
                code = (code << 1) | (uint32_t)bit;
            }
            uint32_t sign = code >> (b - 1);
            uint32_t k = code & s;
            float value = 0.0f;
            if (k == 0) {
                if (sign) bad = 1; /* a sign on a zero level: no encoder writes it */
            } else if (norm == 0.0f || bscale == 0.0f) {
                bad = 1; /* levels under a norm that carries none */
            } else {
                value = bscale * (float)k;
                if (sign) value = -value;
            }
            out[base + i] = value;
        }
        if (bad) {
            *status |= QO_ST_BAD_STREAM;
            for (uint64_t i = 0; i < m; ++i) out[base + i] = 0.0f;
        }
    }
    return 0;
}

int qo_bbit_decode_accumulate(const float* const* norms, const uint32_t* const* codes, int K,
                              uint64_t n, uint64_t d, uint32_t b, float* out, uint32_t* status) {
    if (K < 1) return -1;
    float* q = (float*)malloc((size_t)(n ? n : 1) * sizeof(float));
    if (!q) return -1;
    for (int j = 0; j < K; ++j) {
        if (qo_bbit_decode(norms[j], codes[j], n, d, b, q, status) != 0) {
            free(q);
            return -1;
        }
        for (uint64_t i = 0; i < n; ++i) out[i] += q[i]; /* one fp32 add, as above */
    }
    free(q);
    return 0;
}

/* ---- Error feedback ------------------------------------------------------------
 * "Sparsified SGD with Memory" (abstract): the compressor keeps what it did not send
 * in a memory and adds it to the next gradient.  Step by step: p = e + g, the stream
 * carries Q(p), and the memory becomes p minus Q(p) as a receiver decodes it.  A
 * coordinate with no record decodes to 0 and keeps p in the memory unchanged. */

/* p[i] = e[i] + g[i] (one fp32 add); the caller frees p. */
static float* ef_sum(const float* g, const float* e, uint64_t n) {
    float* p = (float*)malloc((size_t)(n ? n : 1) * sizeof(float));
    if (!p) return NULL;
    for (uint64_t i = 0; i < n; ++i) p[i] = e[i] + g[i];
    return p;
}

/* max_i |p_i| of every bucket (the QSGDinf scale of p); the caller frees it. */
static float* ef_max_norms(const float* p, uint64_t n, uint64_t d) {
    const uint64_t nb = (n + d - 1) / d;
    float* mx = (float*)malloc((size_t)(nb ? nb : 1) * sizeof(float));
    if (!mx) return NULL;
    for (uint64_t b = 0; b < nb; ++b) {
        const uint64_t m = (b + 1) * d <= n ? d : n - b * d;
        mx[b] = qo_bucket_maxnorm(p + b * d, m);
    }
    return mx;
}

/* e[i] <- p[i] - q[i] where a record was sent (q[i] != 0), else p[i]. */
static void ef_update(float* e, const float* p, const float* q, uint64_t n) {
    for (uint64_t i = 0; i < n; ++i) e[i] = q[i] != 0.0f ? p[i] - q[i] : p[i];
}

int qo_encode_ef(const float* g, float* e, uint64_t n, uint64_t d, uint32_t s, uint64_t seed,
                 int max_norm, const float* norms_in, uint32_t* words, uint64_t cap_words,
                 uint64_t* offsets, float* norms_out, uint32_t* status) {
    if (d == 0) return -1;
    int rc = -1;
    float* p = ef_sum(g, e, n);
    float* q = (float*)malloc((size_t)(n ? n : 1) * sizeof(float));
    float* mx = (p && max_norm && !norms_in) ? ef_max_norms(p, n, d) : NULL;
    const float* nin = norms_in ? norms_in : mx;
    if (!p || !q || (max_norm && !nin)) goto done;
    if (qo_encode(p, n, d, s, seed, nin, words, cap_words, offsets, norms_out, status) != 0) goto done;
    if (qo_decode(words, offsets, n, d, s, q, status) != 0) goto done;
    ef_update(e, p, q, n);
    rc = 0;
done:
    free(mx);
    free(q);
    free(p);
    return rc;
}

int qo_bbit_encode_ef(const float* g, float* e, uint64_t n, uint64_t d, uint32_t b, uint64_t seed,
                      int max_norm, const float* norms_in, float* norms_out, uint32_t* codes,
                      uint32_t* status) {
    if (d == 0) return -1;
    int rc = -1;
    float* p = ef_sum(g, e, n);
    float* q = (float*)malloc((size_t)(n ? n : 1) * sizeof(float));
    float* mx = (p && max_norm && !norms_in) ? ef_max_norms(p, n, d) : NULL;
    const float* nin = norms_in ? norms_in : mx;
    if (!p || !q || (max_norm && !nin)) goto done;
    if (qo_bbit_encode(p, n, d, b, seed, nin, norms_out, codes, status) != 0) goto done;
    if (qo_bbit_decode(norms_out, codes, n, d, b, q, status) != 0) goto done;
    ef_update(e, p, q, n);
    rc = 0;
done:
    free(mx);
    free(q);
    free(p);
    return rc;
}

/* ---- Data-parallel exchange: the mean of K received streams ---------------------
 * "for distributed data-parallel optimization" (definition paragraph): every node
 * quantises its gradient and the nodes exchange the encodings; a node's update is
 * the mean of the K decoded gradients.  The sum runs left to right from +0 as in
 * decode-accumulate, then one fp32 division by K per coordinate. */
int qo_decode_mean(const uint32_t* const* words, const uint64_t* const* offsets, int K, uint64_t n,
                   uint64_t d, uint32_t s, float* out, uint32_t* status) {
    if (K < 1) return -1;
    for (uint64_t i = 0; i < n; ++i) out[i] = 0.0f;
    if (qo_decode_accumulate(words, offsets, K, n, d, s, out, status) != 0) return -1;
    for (uint64_t i = 0; i < n; ++i) out[i] = out[i] / (float)K;
    return 0;
}

int qo_bbit_decode_mean(const float* const* norms, const uint32_t* const* codes, int K, uint64_t n,
                        uint64_t d, uint32_t b, float* out, uint32_t* status) {
    if (K < 1) return -1;
    for (uint64_t i = 0; i < n; ++i) out[i] = 0.0f;
    if (qo_bbit_decode_accumulate(norms, codes, K, n, d, b, out, status) != 0) return -1;
    for (uint64_t i = 0; i < n; ++i) out[i] = out[i] / (float)K;
    return 0;
}
