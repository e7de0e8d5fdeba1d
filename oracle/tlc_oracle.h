/*
 * tlc_oracle.h -- the CPU oracle's interface.  TEST INFRASTRUCTURE ONLY:
 * used by the tests, the smoke check and the benchmark's CPU-baseline leg,
 * never by the library.  Independent of the CUDA path (no shared headers).
 *
 * All arrays are plain host memory, caller-owned.  n is the element count,
 * g = ceil(n/5) the number of quartic bytes.
 */
#ifndef TLC_ORACLE_H
#define TLC_ORACLE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
    ORC_OK = 0,
    ORC_INVALID = 1,   /* n = 0, s outside [1,2), capacity too small, K < 1 */
    ORC_NONFINITE = 2, /* a NaN or infinity in x + err; err left unchanged */
    ORC_CORRUPT = 3,   /* stream does not expand to exactly g quartic bytes */
    ORC_NOMEM = 6
};

int orc_error_feedback(const float *x, const float *err, size_t n, float *xp);
int orc_magnitude(const float *xp, size_t n, float *m_out);
int orc_quantize(const float *xp, size_t n, float M, float s,
                 int8_t *q, float *err_out, float *scale_out);
size_t orc_groups(size_t n);
void orc_quartic_pack(const int8_t *q, size_t n, uint8_t *bytes);
int orc_quartic_unpack(const uint8_t *bytes, size_t n, int8_t *q);
size_t orc_zre_encode(const uint8_t *bytes, size_t g, uint8_t *out);
int orc_zre_decode(const uint8_t *in, size_t m, uint8_t *bytes, size_t g);
size_t orc_compress_bound(size_t n);
int orc_compress(const float *x, size_t n, float s, float *err,
                 uint8_t *out, size_t out_cap, size_t *out_len);
int orc_decompress(const uint8_t *in, size_t in_len, size_t n, float *y);
int orc_decompress_accumulate(const uint8_t *const *ins, const size_t *in_lens,
                              int k, size_t n, float *acc);

#ifdef __cplusplus
}
#endif
#endif
