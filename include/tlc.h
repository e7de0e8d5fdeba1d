/*
 * tlc.h -- C ABI of the 3LC state-change compression library for NVIDIA B200
 * (sm_100a).  libtlc.so implements it with hand-written CUDA kernels.
 *
 * Source: the review page "3LC: Lightweight and Effective Traffic Compression
 * for Distributed Machine Learning" (Lim, Andersen et al., 2018).  Section
 * "Proposed method" names the pipeline:
 *   bullet 1  3-value quantization with sparsity multiplication, with an
 *             error-accumulation buffer that carries the quantization error,
 *   bullet 2  quartic encoding: five ternary values in one byte,
 *   bullet 3  zero-run encoding of consecutive all-zero byte groups,
 *   bullet 4  the same pipeline for gradients and model deltas.
 * The Abstract adds that nodes exchange these compressed state changes; the
 * receive side is the decompress-and-accumulate call below.
 *
 * The page gives no formula or byte layout.  This library fixes them:
 *   x' = x + err                      (fp32, round to nearest)
 *   M  = max_i |x'_i|
 *   scale = M * s,  s in [1, 2)       (sparsity multiplication)
 *   q_i = round(x'_i / scale)  in {-1, 0, 1}, ties away from zero
 *                                     (q = 0 for every i when M = 0)
 *   err_i = x'_i - q_i * scale        (written back to the caller's buffer)
 *   byte_j = sum_{d=0..4} (q_{5j+d} + 1) * 3^(4-d)   in 0..242,
 *            values past n count as q = 0; an all-zero group is 121
 *   zero-run encoding: a maximal run of L bytes equal to 121 is cut into
 *            chunks of 14 from its start, the remainder last; a chunk of
 *            c >= 2 bytes becomes the escape byte 241 + c (243..255), a chunk
 *            of 1 stays 121; all other bytes are copied.
 *   stream = 4-byte little-endian fp32 scale, then the zero-run payload.
 * All arithmetic is IEEE binary32 with round-to-nearest-even, without FMA
 * contraction and without flushing subnormals; results are bit-identical to
 * a plain sequential implementation of the rules above.
 *
 * Conventions for every call
 * - Buffers named x, err, out, in, y, acc are DEVICE memory; the caller owns
 *   them.  They must not overlap one another.  Any 4-byte alignment works;
 *   16-byte alignment of the fp32 buffers takes the vectorised path.
 * - out_len, in_len(s) and dev_status must be readable/writable by the
 *   device (device memory, or pinned host memory mapped into the device).
 * - stream is a cudaStream_t (NULL = the legacy default stream).  Every call
 *   only enqueues work: it never synchronises the host, and returns as soon
 *   as the work is queued.  Results are valid once the stream reaches them.
 * - The library allocates its scratch stream-ordered from its own memory
 *   pool (one per device, kept until exit) and frees it on the same stream.
 *   Calls on different streams may run concurrently.
 * - The return value reports what the host can check before launching:
 *   TLC_ERR_INVALID_ARG for bad arguments (nothing is enqueued), and
 *   TLC_ERR_CUDA when an allocation or launch fails.
 * - Errors that depend on the data are found on the device and written to
 *   *dev_status (if dev_status is not NULL): the library writes a non-zero
 *   tlc_status there when the call fails and never writes zero, so the
 *   caller sets it to 0 first; the first error of a sequence of calls that
 *   share one status word is kept.
 */
#ifndef TLC_H
#define TLC_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t (a pointer to the runtime's opaque stream). */
typedef struct CUstream_st *tlc_stream_t;

typedef enum {
    TLC_OK = 0,
    TLC_ERR_INVALID_ARG = 1, /* host-detected: bad size, s, pointer, capacity */
    TLC_ERR_NONFINITE = 2,   /* x + err holds NaN/Inf, or M*s overflows      */
    TLC_ERR_CORRUPT = 3,     /* stream does not decode to exactly ceil(n/5)  */
    TLC_ERR_TIMEOUT = 4,     /* a cross-block wait gave up (see below)       */
    TLC_ERR_CUDA = 5         /* CUDA allocation or launch failure            */
} tlc_status;

/* Largest stream tlc_compress can write for n values: 4 + ceil(n/5) bytes
 * (zero-run encoding never lengthens the quartic bytes).  Returns 0 for
 * n = 0 or n >= 2^32. */
size_t tlc_compress_bound(size_t n);

/* Compress one fp32 tensor ("Proposed method" bullets 1-3).
 *
 *   x        [in]     device fp32[n], the new state change (gradient/delta)
 *   n        [in]     1 <= n < 2^32
 *   s        [in]     sparsity multiplier, 1 <= s < 2
 *   err      [in,out] device fp32[n], the error-accumulation buffer; on
 *                     success it becomes x + err - q*scale
 *   out      [out]    device bytes, capacity out_cap >= tlc_compress_bound(n)
 *   out_len  [out]    device-writable uint64: the stream length 4 + m
 *   dev_status [out]  device-writable int32 or NULL
 *
 * Non-finite step: if any x + err is NaN or +-Inf, or M*s is not finite,
 * *dev_status gets TLC_ERR_NONFINITE, *out_len gets 0, err is left
 * unchanged and out holds no stream.
 * Host errors: TLC_ERR_INVALID_ARG if a pointer is NULL, n is out of range,
 * s is outside [1, 2) or NaN, out_cap is too small, or x/err/out overlap.
 * Scratch: about 8 bytes per 10240 values; from 768 * 10240 values on, also
 * a staging area of about n/5 bytes (the placement of the zero-run encoded
 * bytes then runs as a separate kernel). */
tlc_status tlc_compress(const float *x, size_t n, float s, float *err,
                        uint8_t *out, size_t out_cap, uint64_t *out_len,
                        int32_t *dev_status, tlc_stream_t stream);

/* What one compression did, written by the device ("Findings" bullet 1
 * quotes the method's effect as bits per value and compression ratio):
 *   m_bits    IEEE-754 bits of M = max_i |x_i + err_i| (0x7f800000 or more:
 *             the step was non-finite)
 *   scale     M * s, the value in the stream header (0 when non-finite)
 *   nonzeros  number of values with q != 0
 *   length    stream length 4 + m in bytes (0 when non-finite), the same
 *             value as *out_len; bits per value = 8 * length / n. */
typedef struct {
    uint32_t m_bits;
    float scale;
    uint64_t nonzeros;
    uint64_t length;
} tlc_compress_record;

/* tlc_compress that also fills *record (device-writable memory: device or
 * mapped pinned host memory), in the same stream order as the stream
 * itself.  Arguments, results and errors otherwise those of tlc_compress;
 * record == NULL is TLC_ERR_INVALID_ARG.  The stream and error buffer are
 * bit-identical to tlc_compress's. */
tlc_status tlc_compress_recorded(const float *x, size_t n, float s, float *err,
                                 uint8_t *out, size_t out_cap, uint64_t *out_len,
                                 int32_t *dev_status, tlc_compress_record *record,
                                 tlc_stream_t stream);

/* Decompress one stream into a dense fp32 tensor (inverse of bullets 1-3):
 * y_i = +scale, -scale or +0.0 for q_i = 1, -1, 0.
 *
 *   in       [in]   device bytes: header + payload
 *   in_len   [in]   device-readable uint64 holding the stream length, or
 *                   NULL when in_cap is the exact length
 *   in_cap   [in]   bytes of `in` that may be read, 4 <= in_cap; with
 *                   in_len == NULL also in_cap - 4 <= ceil(n/5)
 *   n        [in]   element count the stream was made from, 1 <= n < 2^32
 *   y        [out]  device fp32[n]
 *
 * TLC_ERR_CORRUPT in *dev_status when the length read from in_len is below
 * 4 or above in_cap, the header is negative or not finite, or the payload
 * does not expand to exactly ceil(n/5) groups.  Then y holds unspecified
 * values, but nothing outside y is written.
 * When min(in_cap - 4, ceil(n/5)) spans 16384 or more 512-byte units
 * (about 8 MiB), an index (a count kernel and a scan kernel) runs before the
 * decode kernel; the result is the same. */
tlc_status tlc_decompress(const uint8_t *in, const uint64_t *in_len,
                          size_t in_cap, size_t n, float *y,
                          int32_t *dev_status, tlc_stream_t stream);

/* Receive side of aggregation: add K workers' decompressed streams into one
 * dense fp32 buffer, acc_i += y_{k,i} for k = 0..K-1 in that order, adding
 * only where q_{k,i} != 0 (acc keeps its exact bits where every worker sent
 * a zero).  Bit-identical to K sequential single-stream additions.
 *
 *   ins      [in]     HOST array of k device pointers to streams
 *   in_lens  [in]     device-readable uint64[k] of stream lengths, or NULL
 *                     when in_caps holds the exact lengths
 *   in_caps  [in]     HOST size_t[k], readable bytes of each stream (same
 *                     rules as tlc_decompress's in_cap)
 *   k        [in]     1 <= k
 *   n        [in]     element count, 1 <= n < 2^32
 *   acc      [in,out] device fp32[n]
 *
 * TLC_ERR_CORRUPT as for tlc_decompress; acc is then unspecified. */
tlc_status tlc_decompress_accumulate(const uint8_t *const *ins,
                                     const uint64_t *in_lens,
                                     const size_t *in_caps, int k, size_t n,
                                     float *acc, int32_t *dev_status,
                                     tlc_stream_t stream);

/* ---- Tensor lists ------------------------------------------------------
 * A training step compresses many tensors (one per layer).  A plan binds a
 * fixed list of tensors once; each step then compresses (or decompresses)
 * the whole list with one launch set, each tensor with its own M, scale and
 * error buffer, exactly as tlc_compress / tlc_decompress would one by one.
 * The streams live in one caller-owned arena: tensor i's stream starts at
 * tlc_plan_stream_offset(plan, i) and has room for 4 + ceil(n_i/5) bytes.
 *
 * A plan holds device memory for its descriptor tables and scratch (allocated
 * once, at creation) and belongs to the device current at creation; calls
 * must be made with that device current.  Calls with the same plan share its
 * scratch, so their work must not overlap on the GPU (keep them on one
 * stream or order the streams).  Different plans are independent. */
typedef struct tlc_plan_s *tlc_plan;

/* Create a plan for count tensors of ns[i] values.  xs/errs (arrays of
 * count device pointers; both or neither) are the inputs and error buffers
 * of tlc_compress_batch; ys (count device pointers, or NULL) are the outputs
 * of tlc_decompress_batch.  Synchronous (copies the tables to the device).
 * TLC_ERR_INVALID_ARG for count < 1, a bad n, a NULL entry, or x/err
 * overlap; TLC_ERR_CUDA if the device allocation fails. */
tlc_status tlc_plan_create(int count, const size_t *ns, const float *const *xs,
                           float *const *errs, float *const *ys, tlc_plan *plan);

/* Free a plan (synchronous; no call using it may still be running). */
void tlc_plan_destroy(tlc_plan plan);

/* Arena size for one set of streams, and tensor i's stream offset in it
 * (16-byte aligned); (size_t)-1 for a bad i. */
size_t tlc_plan_arena_bytes(tlc_plan plan);
size_t tlc_plan_stream_offset(tlc_plan plan, int i);

/* Compress every tensor of the plan ("Proposed method" bullets 1-3), each
 * as tlc_compress would: err_i is updated in place, stream i is written at
 * its arena offset and its length to out_lens[i] (device uint64[count]).  A
 * non-finite tensor gets out_lens[i] = 0 and its err_i unchanged;
 * TLC_ERR_NONFINITE goes to *dev_status while the other tensors are still
 * compressed.  Launches: one memset, a magnitude pass, one quantize+encode
 * pass over all tensors. */
tlc_status tlc_compress_batch(tlc_plan plan, float s, uint8_t *arena, uint64_t *out_lens,
                              int32_t *dev_status, tlc_stream_t stream);

/* Decompress every tensor's stream from the arena (lengths in in_lens,
 * device uint64[count]) into the plan's ys: overwrite (accumulate = 0, as
 * tlc_decompress) or add where q != 0 (accumulate = 1, as one stream of
 * tlc_decompress_accumulate).  A corrupt stream sets TLC_ERR_CORRUPT and
 * leaves its y unspecified; the others are still decoded. */
tlc_status tlc_decompress_batch(tlc_plan plan, const uint8_t *arena, const uint64_t *in_lens,
                                int accumulate, int32_t *dev_status, tlc_stream_t stream);

/* Largest n accepted by tlc_compress_noalloc. */
#define TLC_NOALLOC_MAX_N ((size_t)1 << 29)

/* tlc_compress without any device memory allocation.
 *
 * This has no counterpart on the page; it exists for callers that cannot
 * allocate device memory while they run: a process whose device memory is
 * all handed to a framework's caching allocator up front, code that must not
 * allocate on its hot path (real-time or certified loops), or a runtime
 * without stream-ordered memory pools.  tlc_compress takes its scratch from
 * a pool; this call takes it from a fixed 256 KiB array inside the library's
 * own device memory, which every device that loads the library holds until
 * the process exits.  It calls no allocation or free routine.
 *
 * Arguments, results and errors are those of tlc_compress, and the output is
 * bit-identical to it, with one more limit: n <= TLC_NOALLOC_MAX_N (2^29),
 * else TLC_ERR_INVALID_ARG and nothing is enqueued.
 * - The first call on a device resolves the array's device address (with
 *   that device current); make that first call before any stream capture.
 *   If resolving fails, that call returns TLC_ERR_CUDA without enqueuing
 *   anything, and the next call on the device tries again.
 * - Every call on a device shares the one array.  Calls whose work overlaps
 *   on the GPU (different streams, or different host threads without
 *   ordering between their streams) race on it and give wrong results;
 *   order them, e.g. keep them on one stream.  The kernels clear what they
 *   need at the start of each call, so a call never sees an earlier call's
 *   leftovers. */
tlc_status tlc_compress_noalloc(const float *x, size_t n, float s, float *err,
                                uint8_t *out, size_t out_cap, uint64_t *out_len,
                                int32_t *dev_status, tlc_stream_t stream);

/* Debug build.  libtlc_debug.so (the same sources compiled with
 * -DTLC_DEBUG) checks every index of its shared-memory staging, stream
 * placement and entry lists before the access, and puts 256-byte canaries of
 * 0xA5 on both sides of every scratch allocation, checked by a small kernel
 * when the scratch is freed.  A failing check never faults: it records its
 * location (source line | file id << 16; file ids 1 compress, 2 decode,
 * 3 API) and skips the access.
 * tlc_debug_build() is 1 in that library and 0 in libtlc.so.
 * tlc_debug_fault(reset) returns the first recorded location, or 0 (always
 * 0 in libtlc.so), and clears it when reset is non-zero.  It reads device
 * memory, so it waits for the device's queued work. */
int tlc_debug_build(void);
uint32_t tlc_debug_fault(int reset);

/* Human-readable name of a status code (static string). */
const char *tlc_status_string(tlc_status status);

/* Library version, "major.minor.patch" (static string). */
const char *tlc_version(void);

/* Cross-block waits.  The single-pass scans in the compress and decode
 * kernels wait for earlier tiles' results.  Each wait polls at most
 * `max_polls` times (with a short sleep between polls) before it gives up,
 * writes TLC_ERR_TIMEOUT to *dev_status and lets the kernel finish with
 * unspecified (but in-bounds) output.  The default, 0, means the library's
 * built-in limit (about 2^22 polls, on the order of seconds).  Applies to
 * calls enqueued after it returns, process-wide. */
void tlc_set_wait_limit(uint32_t max_polls);

/* Testing hook for the bounded waits: runs the decode kernel's cross-block
 * wait for one tile whose predecessor never publishes, with the given poll
 * limit, and writes TLC_ERR_TIMEOUT to *dev_status when the wait gives up.
 * Makes no other change.  Returns TLC_ERR_INVALID_ARG for max_polls = 0 or a
 * NULL dev_status. */
tlc_status tlc_test_wait_timeout(uint32_t max_polls, int32_t *dev_status,
                                 tlc_stream_t stream);

/* The same check for the compress kernel's cross-block wait (the look-back
 * that places a tile's zero-run encoded bytes): one tile waits for a
 * predecessor that never publishes.  Same arguments and results. */
tlc_status tlc_test_compress_wait_timeout(uint32_t max_polls, int32_t *dev_status,
                                          tlc_stream_t stream);

/* Per-kernel timing, for benchmarks.  While enabled, the library counts
 * every kernel it launches, by kind, and records a CUDA event pair on the
 * caller's stream around each launch of the selected kinds.
 * tlc_kernel_timing(1) clears the totals and starts; (0) stops.
 * tlc_kernel_timing_kinds(mask) selects the kinds that get event pairs (bit
 * k = kind k; all kinds at load time); an event pair costs a few
 * microseconds of device time, so a benchmark may time one kind only.
 * tlc_kernel_timing_read waits for the recorded events and, for each kernel
 * kind k < max_kinds, stores the number of launches in launches[k] and the
 * summed device time of its timed launches in total_ms[k] (0 for a kind
 * that was not selected); it returns the number of kinds.
 * tlc_kernel_name(k) names kind k (NULL past the last one). */
void tlc_kernel_timing(int enable);
void tlc_kernel_timing_kinds(uint32_t mask);
int tlc_kernel_timing_read(uint64_t *launches, double *total_ms, int max_kinds);
const char *tlc_kernel_name(int kind);

#ifdef __cplusplus
}
#endif
#endif /* TLC_H */
