/*
 * qga.h -- C ABI of libqga.so: quantized gradient aggregation on B200 (sm_100a).
 *
 * Sources (cited by page title and section):
 *   [MX] MXNet pull request #8342 "[WIP] 2bit gradient compression":
 *        "Approach", "Two bit quantization", "Format of compressed gradient",
 *        "Operators", "Local kvstore".
 *   [GC] gradient-compression README (vineeths96), "About The Project",
 *        "Results": names QSGDMaxNorm quantization (all-reduce compatible),
 *        its two-scale and GlobalRandK variants, without formulas; their
 *        definitions here are this library's own.
 *   [SC11] Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As Easy as
 *        1, 2, 3", SC'11 (Philox4x32-10).
 *
 * Conventions shared by every entry point
 *   - Every pointer named grad/residual/compr/out/max is DEVICE memory of the
 *     current CUDA device, owned by the caller.  Pointer ARRAYS (`const T*
 *     const* compr`) and descriptor tables are HOST memory read during the
 *     call only.  The library allocates nothing and keeps no pointer after
 *     the call returns.
 *   - Work is enqueued on `stream` (0 = legacy default stream) and is
 *     asynchronous: no call synchronizes the host with the device.
 *   - Arguments are validated on the host before anything is enqueued; an
 *     invalid call returns a negative status and enqueues nothing.  Device
 *     pointers must be aligned to their element size (4 bytes for float and
 *     uint32_t, 2 bytes for bfloat16); 16-byte-aligned buffers take the
 *     vectorised path, others a scalar path with identical results.
 *   - Outputs are overwritten, never accumulated into.  Buffers of one call
 *     must not overlap unless stated (the residual is updated in place).
 *   - The element count n of a record is the caller's; the header's float
 *     copy of n is informational (binary32 is not exact above 2^24).
 *   - Calls on different streams that touch the same buffers race; order
 *     them with events as for any kernel.
 */
#ifndef QGA_H
#define QGA_H

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h> /* cudaStream_t */

#ifdef __cplusplus
extern "C" {
#endif

/* ---------------------------------------------------------------- status */
#define QGA_OK 0
#define QGA_ERR_INVALID_ARG (-1) /* null/misaligned pointer, bad size, bad threshold, ... */
#define QGA_ERR_UNSUPPORTED (-2) /* valid request outside what is built (e.g. bits) */
#define QGA_ERR_CUDA (-3)        /* a CUDA runtime call or launch failed; see qga_last_cuda_error */

#define QGA_MAX_WORKERS 64       /* W per merge / max call */
#define QGA_DTYPE_F32 0
#define QGA_DTYPE_BF16 1

/* Text for a status code (static storage, never NULL). */
const char *qga_strerror(int status);

/* cudaError_t value behind the most recent QGA_ERR_CUDA returned on the
 * calling host thread (0 if none). */
int qga_last_cuda_error(void);

/* Library ABI version: major * 10000 + minor * 100 + patch. */
int qga_version(void);

/* ======================================================= 2-bit threshold ==
 *
 * Record layout ([MX] "Format of compressed gradient"): uint32 words
 *   word 0 = binary32 bits of neg_threshold
 *   word 1 = binary32 bits of pos_threshold
 *   word 2 = binary32 bits of (float)n (round to nearest even)
 *   word 3 + k = codes of elements 16k .. 16k+15, element 16k in bits 31..30,
 *                element 16k+15 in bits 1..0; codes of elements >= n are 00.
 * Codes ([MX] "Two bit quantization"): 01 if x >= pos_threshold, else 10 if
 * x <= neg_threshold, else 00 (the positive test first).  A code stands for
 * pos_threshold (01), neg_threshold (10) or +0 (00; also the unused 11).
 */

/* create_2bit of [MX] "Operators" as a size query: the number of uint32
 * words of a record for n elements, 3 + ceil(n / 16).  Returns
 * QGA_ERR_INVALID_ARG for n < 0. */
int64_t qga_2bit_words(int64_t n);

/* quantize_2bit(grad, residual, compr, neg_threshold, pos_threshold) of
 * [MX] "Operators", with the error feedback of [MX] "Approach": for every
 * element e < n, in binary32 round-to-nearest with no contraction,
 *   x = grad[e] + residual[e];  code = code(x);  residual[e] = x - value(code)
 * and the record (header + packed codes) is written to compr.
 *   grad      float[n], read only
 *   residual  float[n], read and updated in place (must not alias grad/compr)
 *   compr     uint32[qga_2bit_words(n)], overwritten (the tail is zeroed)
 *   n >= 0    (n == 0 writes the header only; grad/residual may be NULL)
 *   thresholds finite.  */
int qga_quantize_2bit(const float *grad, float *residual, uint32_t *compr, int64_t n,
                      float neg_threshold, float pos_threshold, cudaStream_t stream);

/* The same for a bfloat16 gradient (uint16 bit patterns, widened exactly to
 * binary32 before the add); residual and record as above. */
int qga_quantize_2bit_bf16(const uint16_t *grad, float *residual, uint32_t *compr, int64_t n,
                           float neg_threshold, float pos_threshold, cudaStream_t stream);

/* dequantize_2bit(compr, decompr) of [MX] "Operators": out[e] = value of
 * element e's code, thresholds read from the record's header on the device.
 *   compr  uint32[qga_2bit_words(n)] record written by a quantize call
 *   out    float[n], overwritten.  n == 0 enqueues nothing. */
int qga_dequantize_2bit(const uint32_t *compr, float *out, int64_t n, cudaStream_t stream);

/* The receiver's merge of [MX] "Local kvstore": each of the W workers'
 * records is dequantized with its own header's thresholds and the values are
 * summed, starting from +0 and adding workers 0, 1, ..., W-1 in that order
 * (binary32, round to nearest):
 *   out[e] = (((+0 + v_0[e]) + v_1[e]) + ...) + v_{W-1}[e]
 *   compr        HOST array of W device pointers, each a record of n elements
 *   num_workers  1 .. QGA_MAX_WORKERS
 *   out          float[n], overwritten; must not overlap any record. */
int qga_dequant_accumulate_2bit(const uint32_t *const *compr, int num_workers, float *out,
                                int64_t n, cudaStream_t stream);

/* The reducing worker's step of [MX] "Local kvstore" in one launch: the
 * device that merges the workers' gradients also quantizes its own ([MX]
 * "Questions", 1).  Worker `own`'s gradient is quantized exactly as by
 * qga_quantize_2bit (residual updated in place, record written to
 * compr[own]), and the W records are merged exactly as by
 * qga_dequant_accumulate_2bit (worker order 0..W-1, own included).  The
 * results are bit for bit those of the two calls in sequence.
 *   grad, residual  float[n] of worker `own`
 *   compr           HOST array of W device pointers to records of n
 *                   elements; compr[own] is overwritten, the others are read
 *   own             0 .. W-1;  num_workers 1 .. QGA_MAX_WORKERS
 *   out             float[n], overwritten; no buffer may overlap another.
 * 32-byte-aligned grad and residual with a 16-byte-aligned out take the
 * vector path, other element-aligned pointers a scalar path with identical
 * results. */
int qga_quantize_merge_2bit(const float *grad, float *residual, int64_t n, float neg_threshold,
                            float pos_threshold, uint32_t *const *compr, int num_workers, int own,
                            float *out, cudaStream_t stream);

/* ---------------------------------------------------------- 2-bit bucket --
 * A bucket is T tensors quantized in ONE launch.  Its compressed form is the
 * T standalone records one after the other (tensor t's record starts at word
 * sum_{u<t} qga_2bit_words(n_u)), each padded to whole words like any
 * record, so every tensor keeps its own thresholds and header. */
typedef struct qga_bucket_tensor {
    const void *grad;    /* device float[n] or bfloat16[n] (bucket-wide dtype) */
    float *residual;     /* device float[n], updated in place */
    int64_t n;           /* elements, >= 0 */
    float neg_threshold; /* finite */
    float pos_threshold; /* finite */
} qga_bucket_tensor;

/* Words of the compressed bucket: sum of qga_2bit_words(n[t]).  n is a HOST
 * array of num_tensors sizes.  Negative on invalid input. */
int64_t qga_2bit_bucket_words(const int64_t *n, int num_tensors);

/* qga_quantize_2bit for every tensor of the bucket.
 *   tensors     HOST array of num_tensors descriptors (read during the call)
 *   grad_dtype  QGA_DTYPE_F32 or QGA_DTYPE_BF16
 *   compr       device uint32[qga_2bit_bucket_words(...)], overwritten
 * Tables of more than 256 tensors are split into several launches. */
int qga_quantize_2bit_bucket(const qga_bucket_tensor *tensors, int num_tensors, int grad_dtype,
                             uint32_t *compr, cudaStream_t stream);

/* Merge of W compressed buckets of the same layout: for every tensor t,
 * out_t = qga_dequant_accumulate_2bit of the W workers' records of t, with
 * the T results one after the other in out (tensor t at element offset
 * sum_{u<t} n[u]).
 *   compr  HOST array of W device pointers to compressed buckets
 *   n      HOST array of num_tensors sizes (the layout of every bucket)
 *   out    device float[sum n], overwritten. */
int qga_dequant_accumulate_2bit_bucket(const uint32_t *const *compr, int num_workers,
                                       const int64_t *n, int num_tensors, float *out,
                                       cudaStream_t stream);

/* ===================================================== dense ternary 2-bit ==
 * [MX] "Two bit quantization" observes that three code values waste a bit
 * and defers the fix.  Dense record (this library's format): the same codes
 * 00 / 01 / 10 as trits 0 / 1 / 2, five elements per byte as the base-3
 * numeral t0 t1 t2 t3 t4 (element 0 most significant; a byte is <= 242),
 * payload byte j = elements 5j..5j+4 at byte 12 + j of the record, after the
 * same header [neg, pos, (float)n]; padded to whole words with zero bytes,
 * trits past n zero.  0.2 bytes per element instead of 0.25.
 *
 * Words of a dense record: 3 + ceil(n / 20).  QGA_ERR_INVALID_ARG for n < 0. */
int64_t qga_ternary_words(int64_t n);

/* qga_quantize_2bit's error feedback (same codes, same residual, bit for bit)
 * written as a dense record.
 *   grad float[n], residual float[n] (in place), compr uint32[qga_ternary_words(n)] */
int qga_quantize_ternary(const float *grad, float *residual, uint32_t *compr, int64_t n,
                         float neg_threshold, float pos_threshold, cudaStream_t stream);

/* Dense-record dequantize: out[e] = value of element e's code. */
int qga_dequantize_ternary(const uint32_t *compr, float *out, int64_t n, cudaStream_t stream);

/* Dense-record merge: out[e] = sum over w of the values, from +0 in worker
 * order 0..W-1 (the same sums as qga_dequant_accumulate_2bit). */
int qga_dequant_accumulate_ternary(const uint32_t *const *compr, int num_workers, float *out,
                                   int64_t n, cudaStream_t stream);

/* ==================================================== QSGD-MaxNorm, b bits ==
 * QSGDMaxNorm is named in [GC]; this library defines it as follows.
 *   s = 2^(b-1) - 1,  M = max over all workers and elements of |g|.
 *   u(e) = (Philox4x32-10 [SC11], key (lo32 seed, hi32 seed), counter
 *          (lo32(e/4), hi32(e/4), 0, 0), output word e mod 4) >> 8, times 2^-24
 *   t = ((|g| / M) * s) + u   (three binary32 operations, in this order)
 *   q = sign(g) * min(floor(t), s);  q = 0 when t is not finite or g == 0.
 * Record: word 0 = M, word 1 = (float)b, word 2 = (float)n (binary32 bits),
 * then 32/b two's-complement b-bit codes per word, first element in the most
 * significant bits, unused tail codes zero. */

/* Words of a record: 3 + ceil(n * bits / 32).  Negative on invalid input. */
int64_t qga_qsgd_words(int64_t n, int bits);

/* M = max |grad_w[e]| over w < num_workers and e < n, written to *max_out
 * (device float).  NaN elements are skipped.  max_out is first cleared with
 * cudaMemsetAsync on the same stream, then reduced into by one kernel. */
int qga_qsgd_mn_max(const float *const *grad, int num_workers, int64_t n, float *max_out,
                    cudaStream_t stream);

/* One worker's record from its gradient, the seed and the global M, which is
 * read from device memory (*max_in, e.g. written by qga_qsgd_mn_max) so no
 * host round trip is needed.
 *   grad   float[n];  compr uint32[qga_qsgd_words(n, bits)], overwritten
 *   bits   2, 4 or 8 (others: QGA_ERR_UNSUPPORTED) */
int qga_qsgd_mn_quantize(const float *grad, uint32_t *compr, int64_t n, int bits, uint64_t seed,
                         const float *max_in, cudaStream_t stream);

/* Merge: out[e] = (float)(sum_w q_w[e]) * (M / s), the level sum exact in
 * integers (so independent of worker order), M read from worker 0's header,
 * M / s one binary32 division.  This is the sum-then-scale form that makes
 * the scheme all-reduce compatible ([GC] "About The Project"). */
int qga_qsgd_mn_dequant_accumulate(const uint32_t *const *compr, int num_workers, float *out,
                                   int64_t n, int bits, cudaStream_t stream);

/* ============================= QSGD-MaxNorm with two scales (QSGD-MN-TS) ==
 * [GC] "Results" names QSGDMaxNormMultiScale quantization run with two
 * scales, each run labelled with the bit widths of its two scales, and
 * [GC] "About The Project" counts it among the all-reduce compatible
 * schemes; no formula is given.  This library's definition:
 *   coarse scale M1 = M (the global max |g|, e.g. from qga_qsgd_mn_max) with
 *     bits_coarse bits, s1 = 2^(bits_coarse-1) - 1 levels;
 *   fine scale M2 = M1 / s1 (one binary32 division: the coarse grid's first
 *     step) with bits_fine bits, s2 = 2^(bits_fine-1) - 1 levels;
 *   an element with |g| <= M2 gets its QSGD-MaxNorm level on the fine scale
 *     (M2, s2) and level 0 on the coarse one; any other element its level on
 *     the coarse scale (M1, s1) and 0 on the fine one; both use the element's
 *     QSGD-MaxNorm draw u(e) of the worker's seed.
 * Record: the coarse levels as a QSGD-MaxNorm record of bits_coarse bits
 * (header [M1, bits_coarse, n]) immediately followed by the fine levels as a
 * QSGD-MaxNorm record of bits_fine bits (header [M2, bits_fine, n]).
 * With bits_coarse = 2 the scales coincide and the fine part is the
 * QSGD-MaxNorm record of bits_fine bits. */

/* Words of a two-scale record: qga_qsgd_words(n, bits_coarse) +
 * qga_qsgd_words(n, bits_fine).  Negative on invalid input. */
int64_t qga_qsgd_mnts_words(int64_t n, int bits_coarse, int bits_fine);

/* One worker's two-scale record; M1 read from *max_in (device).
 *   grad   float[n];  compr uint32[qga_qsgd_mnts_words(n, ...)], overwritten
 *   bits_coarse, bits_fine  2, 4 or 8 each (others: QGA_ERR_UNSUPPORTED) */
int qga_qsgd_mnts_quantize(const float *grad, uint32_t *compr, int64_t n, int bits_coarse,
                           int bits_fine, uint64_t seed, const float *max_in, cudaStream_t stream);

/* Merge of W two-scale records: out[e] = A + B (binary32), where
 *   A = (float)(sum_w coarse level) * (M1 / s1),  B = (float)(sum_w fine
 *   level) * (M2 / s2), M1 and M2 read from worker 0's two headers.
 * Both level sums are exact integers (all-reduce compatible).
 *   out  float[n], overwritten. */
int qga_qsgd_mnts_dequant_accumulate(const uint32_t *const *compr, int num_workers, float *out,
                                     int64_t n, int bits_coarse, int bits_fine, cudaStream_t stream);

/* ============================================ GRandK-MaxNorm, b bits ==
 * GlobalRandKMaxNorm compression is named in [GC] "Results" (K = 10000) as
 * the sparsified variant of QSGDMaxNorm, without a formula; this library
 * defines it as follows.  All workers keep the same K coordinates index[k]
 * (int64, drawn by the caller from a seed the workers share, distinct); the
 * kept values x[k] = grad[index[k]] are quantized exactly as QSGD-MaxNorm
 * quantizes a K-element gradient: M = max |x| over all workers, the draw u of
 * position k (not of the coordinate), the record of qga_qsgd_words(K, bits)
 * words with header [M, b, K].  The merge scatters the scaled level sums to
 * their coordinates; every other coordinate of the result is +0.
 * A coordinate outside [0, n) is skipped everywhere: it does not enter M, its
 * level is 0 and nothing is stored for it.  With repeated coordinates the
 * merge stores one of their values (which one is unspecified).
 *   index  device int64[K], 8-byte aligned, owned by the caller; K >= 0. */

/* M = max |grad_w[index[k]]| over w < num_workers and k < K, written to
 * *max_out (device float, cleared first with cudaMemsetAsync); NaN skipped. */
int qga_grandk_mn_max(const float *const *grad, int num_workers, int64_t n, const int64_t *index,
                      int64_t k, float *max_out, cudaStream_t stream);

/* One worker's record of its kept values; M read from *max_in (device).
 *   grad   float[n];  compr uint32[qga_qsgd_words(k, bits)], overwritten
 *   bits   2, 4 or 8 (others: QGA_ERR_UNSUPPORTED) */
int qga_grandk_mn_quantize(const float *grad, int64_t n, const int64_t *index, int64_t k,
                           uint32_t *compr, int bits, uint64_t seed, const float *max_in,
                           cudaStream_t stream);

/* Merge of W records over the same index: out (float[n]) is cleared to +0
 * with cudaMemsetAsync, then out[index[k]] = (float)(sum_w q_w[k]) * (M / s),
 * M from worker 0's header, M / s one binary32 division. */
int qga_grandk_mn_dequant_accumulate(const uint32_t *const *compr, int num_workers,
                                     const int64_t *index, int64_t k, float *out, int64_t n,
                                     int bits, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* QGA_H */
