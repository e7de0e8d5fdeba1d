/*
 * tlc_oracle.c -- plain, single-threaded CPU oracle for the 3LC state-change
 * compression pipeline.  TEST INFRASTRUCTURE ONLY: the tests, the smoke check
 * and the benchmark's CPU-baseline leg may call it; the library's product path
 * never does.  It shares no code with the CUDA path.
 *
 * Source: the review page "3LC: Lightweight and Effective Traffic Compression
 * for Distributed Machine Learning" (Lim, Andersen et al., 2018).  Its section
 * "Proposed method" (提出的方法) names the three steps:
 *   bullet 1  3-value quantization with sparsity multiplication and an
 *             error-accumulation buffer,
 *   bullet 2  quartic encoding (five ternary values in one byte),
 *   bullet 3  zero-run encoding (a run-length variant for zero byte groups),
 *   bullet 4  one pipeline for gradients and model deltas.
 * The page prints no formula or byte layout.  This library fixes them as:
 *   x' = x + err;  M = max|x'|;  q = round(x' / (M*s)) in {-1,0,1}, s in [1,2);
 *   err = x' - q*M*s;  byte = sum_d (q_d + 1) * 3^(4-d) over five consecutive
 *   values (first value most significant), so an all-zero group is 121;
 *   a run of 2..14 consecutive 121-bytes becomes one escape byte 243..255.
 * Every step below is written in that order and notation, one element or one
 * byte at a time, in index order, with no blocking or fusion.
 *
 * Floating point: IEEE binary32, round-to-nearest-even, no contraction into
 * FMA and no flush-to-zero (built with -ffp-contract=off -fno-fast-math on
 * SSE).  round() is C's round-half-away-from-zero.
 */
#include "tlc_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* Step 1: error feedback and magnitude.                                      */
/* "Proposed method" bullet 1: the error-accumulation buffer corrects the     */
/* quantization error, so the value quantized this step is x' = x + err.      */
/* ------------------------------------------------------------------------ */
int orc_error_feedback(const float *x, const float *err, size_t n, float *xp)
{
    for (size_t i = 0; i < n; ++i)
        xp[i] = x[i] + err[i];
    return ORC_OK;
}

/* M = max_i |x'_i|.  A NaN or an infinity anywhere makes the step
 * non-finite: the page says nothing about such values, and this library
 * refuses to quantize them (the error buffer is then left as it was). */
int orc_magnitude(const float *xp, size_t n, float *m_out)
{
    float m = 0.0f;
    for (size_t i = 0; i < n; ++i) {
        if (!isfinite(xp[i]))
            return ORC_NONFINITE;
        float a = fabsf(xp[i]);
        if (a > m)
            m = a;
    }
    *m_out = m;
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Step 2: 3-value quantization with sparsity multiplication.                 */
/* "Proposed method" bullet 1 and the abstract: values map to {-1, 0, 1};     */
/* the tunable parameter s (sparsity multiplication) widens the zero band.    */
/*   q_i = round(x'_i / (M * s)),   err_i = x'_i - q_i * M * s.               */
/* M = 0 means every x' is zero: all q are 0 and no division is made.         */
/* A product M*s that overflows to infinity makes the step non-finite, like   */
/* a NaN in x': the scale written to the stream is always finite.             */
/* ------------------------------------------------------------------------ */
int orc_quantize(const float *xp, size_t n, float M, float s,
                 int8_t *q, float *err_out, float *scale_out)
{
    float scale = M * s;
    *scale_out = scale;
    if (!isfinite(scale))
        return ORC_NONFINITE;
    for (size_t i = 0; i < n; ++i) {
        int qi = 0;
        if (M != 0.0f) {
            float r = xp[i] / scale;
            qi = (int)roundf(r);
        }
        q[i] = (int8_t)qi;
        err_out[i] = xp[i] - (float)qi * scale;
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Step 3: quartic encoding.                                                  */
/* "Proposed method" bullet 2: five ternary values share one byte.  Group j   */
/* holds q[5j..5j+4]; digit d = q + 1 in {0,1,2}; the first value of the      */
/* group is the most significant base-3 digit.  Values past n are padded      */
/* with q = 0.  All-zero group: 1*81 + 1*27 + 1*9 + 1*3 + 1*1 = 121.          */
/* ------------------------------------------------------------------------ */
static const int POW3[5] = {81, 27, 9, 3, 1};

size_t orc_groups(size_t n) { return (n + 4) / 5; }

void orc_quartic_pack(const int8_t *q, size_t n, uint8_t *bytes)
{
    size_t g = orc_groups(n);
    for (size_t j = 0; j < g; ++j) {
        int v = 0;
        for (int d = 0; d < 5; ++d) {
            size_t i = 5 * j + (size_t)d;
            int qi = (i < n) ? q[i] : 0;
            v += (qi + 1) * POW3[d];
        }
        bytes[j] = (uint8_t)v;
    }
}

/* Inverse of the packing.  Bytes above 242 are not quartic codes. */
int orc_quartic_unpack(const uint8_t *bytes, size_t n, int8_t *q)
{
    size_t g = orc_groups(n);
    for (size_t j = 0; j < g; ++j) {
        int v = bytes[j];
        if (v > 242)
            return ORC_CORRUPT;
        for (int d = 0; d < 5; ++d) {
            int digit = v / POW3[d];
            v -= digit * POW3[d];
            size_t i = 5 * j + (size_t)d;
            if (i < n)
                q[i] = (int8_t)(digit - 1);
        }
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Step 4: zero-run encoding.                                                 */
/* "Proposed method" bullet 3: a run-length variant for consecutive all-zero  */
/* byte groups (121).  A maximal run of L such bytes is cut into chunks of    */
/* 14 from its start, the remainder last; a chunk of c >= 2 bytes becomes     */
/* the single escape byte 241 + c (243..255), a chunk of 1 stays 121.         */
/* Every other byte is copied.  Output length never exceeds the input's.      */
/* ------------------------------------------------------------------------ */
size_t orc_zre_encode(const uint8_t *bytes, size_t g, uint8_t *out)
{
    size_t m = 0;
    size_t j = 0;
    while (j < g) {
        if (bytes[j] != 121) {
            out[m++] = bytes[j++];
            continue;
        }
        size_t L = 0;
        while (j < g && bytes[j] == 121) {
            ++L;
            ++j;
        }
        while (L >= 14) {
            out[m++] = (uint8_t)(241 + 14);
            L -= 14;
        }
        if (L == 1)
            out[m++] = 121;
        else if (L >= 2)
            out[m++] = (uint8_t)(241 + L);
    }
    return m;
}

/* Inverse: an escape byte b in 243..255 stands for b - 241 bytes of 121;
 * any other byte is itself.  The expansion must give exactly g bytes. */
int orc_zre_decode(const uint8_t *in, size_t m, uint8_t *bytes, size_t g)
{
    size_t j = 0;
    for (size_t k = 0; k < m; ++k) {
        size_t e = (in[k] >= 243) ? (size_t)(in[k] - 241) : 1;
        if (j + e > g)
            return ORC_CORRUPT;
        for (size_t t = 0; t < e; ++t)
            bytes[j++] = (in[k] >= 243) ? 121 : in[k];
    }
    return (j == g) ? ORC_OK : ORC_CORRUPT;
}

/* ------------------------------------------------------------------------ */
/* Stream: 4-byte little-endian fp32 scale = M*s, then the zero-run payload.  */
/* The element count n is not stored; both sides know it.                     */
/* ------------------------------------------------------------------------ */
size_t orc_compress_bound(size_t n) { return 4 + orc_groups(n); }

static void put_f32le(uint8_t *p, float v)
{
    uint32_t u;
    memcpy(&u, &v, 4);
    p[0] = (uint8_t)(u & 0xFF);
    p[1] = (uint8_t)((u >> 8) & 0xFF);
    p[2] = (uint8_t)((u >> 16) & 0xFF);
    p[3] = (uint8_t)((u >> 24) & 0xFF);
}

static float get_f32le(const uint8_t *p)
{
    uint32_t u = (uint32_t)p[0] | ((uint32_t)p[1] << 8) |
                 ((uint32_t)p[2] << 16) | ((uint32_t)p[3] << 24);
    float v;
    memcpy(&v, &u, 4);
    return v;
}

static int valid_s(float s) { return s >= 1.0f && s < 2.0f; }

/* Full compression: steps 1..4 in order.  err is updated only on success. */
int orc_compress(const float *x, size_t n, float s, float *err,
                 uint8_t *out, size_t out_cap, size_t *out_len)
{
    *out_len = 0;
    if (n == 0 || !valid_s(s) || out_cap < orc_compress_bound(n))
        return ORC_INVALID;
    size_t g = orc_groups(n);
    float *xp = (float *)malloc(n * sizeof(float));
    float *e2 = (float *)malloc(n * sizeof(float));
    int8_t *q = (int8_t *)malloc(n);
    uint8_t *b = (uint8_t *)malloc(g);
    int rc = ORC_NOMEM;
    if (!xp || !e2 || !q || !b)
        goto done;

    float M, scale;
    orc_error_feedback(x, err, n, xp);
    rc = orc_magnitude(xp, n, &M);
    if (rc != ORC_OK)
        goto done;
    rc = orc_quantize(xp, n, M, s, q, e2, &scale);
    if (rc != ORC_OK)
        goto done;
    orc_quartic_pack(q, n, b);
    put_f32le(out, scale);
    size_t m = orc_zre_encode(b, g, out + 4);
    memcpy(err, e2, n * sizeof(float));
    *out_len = 4 + m;
    rc = ORC_OK;
done:
    free(xp);
    free(e2);
    free(q);
    free(b);
    return rc;
}

/* Dequantization: q * M * s, i.e. +scale, -scale, or +0 for q = 0. */
static float dequant(int qi, float scale)
{
    if (qi == 0)
        return 0.0f;
    return (float)qi * scale;
}

/* Decode one stream into q and its scale.  The encoder only writes a
 * finite, non-negative scale (M >= 0, s >= 1, overflow is refused), so a
 * header with the sign bit set or an all-ones exponent marks the stream as
 * corrupt. */
static int decode_stream(const uint8_t *in, size_t in_len, size_t n,
                         int8_t *q, float *scale_out)
{
    if (in_len < 4)
        return ORC_INVALID;
    float sc = get_f32le(in);
    if (!(isfinite(sc) && !signbit(sc)))
        return ORC_CORRUPT;
    size_t g = orc_groups(n);
    uint8_t *b = (uint8_t *)malloc(g);
    if (!b)
        return ORC_NOMEM;
    int rc = orc_zre_decode(in + 4, in_len - 4, b, g);
    if (rc == ORC_OK)
        rc = orc_quartic_unpack(b, n, q);
    free(b);
    *scale_out = get_f32le(in);
    return rc;
}

int orc_decompress(const uint8_t *in, size_t in_len, size_t n, float *y)
{
    if (n == 0)
        return ORC_INVALID;
    int8_t *q = (int8_t *)malloc(n);
    if (!q)
        return ORC_NOMEM;
    float scale;
    int rc = decode_stream(in, in_len, n, q, &scale);
    if (rc == ORC_OK)
        for (size_t i = 0; i < n; ++i)
            y[i] = dequant(q[i], scale);
    free(q);
    return rc;
}

/* Receive side of aggregation: acc += sum over k of the k-th worker's
 * decoded values, streams in order k = 0..K-1, adding only where q != 0 so
 * that acc keeps its exact bits where a worker sent a zero. */
int orc_decompress_accumulate(const uint8_t *const *ins, const size_t *in_lens,
                              int k, size_t n, float *acc)
{
    if (n == 0 || k < 1)
        return ORC_INVALID;
    int8_t *q = (int8_t *)malloc(n);
    if (!q)
        return ORC_NOMEM;
    int rc = ORC_OK;
    for (int w = 0; w < k && rc == ORC_OK; ++w) {
        float scale;
        rc = decode_stream(ins[w], in_lens[w], n, q, &scale);
        if (rc != ORC_OK)
            break;
        for (size_t i = 0; i < n; ++i)
            if (q[i] != 0)
                acc[i] = acc[i] + dequant(q[i], scale);
    }
    free(q);
    return rc;
}
