/*
 * qga_oracle.c -- the CPU oracle for quantized gradient aggregation.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, obviously-correct
 * statement of what the GPU library computes.  Only the test suite, the
 * smoke check of the package entry point and the CPU-baseline leg of the
 * benchmark may load it.  The CUDA library never links, includes or calls it,
 * and it shares no header, helper, table or constant with the CUDA sources.
 *
 * Build: gcc -std=c11 -O2 -ffp-contract=off -fno-fast-math -fPIC -shared.
 * On x86-64 every `float` expression below is one IEEE-754 binary32 operation
 * rounded to nearest-even (SSE arithmetic, FLT_EVAL_METHOD == 0); with
 * contraction off, no fused multiply-add is ever formed.
 *
 * Sources, cited by page title and section:
 *   [MX]  MXNet pull request #8342 "[WIP] 2bit gradient compression":
 *         sections "Approach", "Two bit quantization", "Format of compressed
 *         gradient", "Operators", "Local kvstore".
 *   [GC]  gradient-compression README (vineeths96), "About The Project" and
 *         "Results": names QSGDMaxNorm quantization and calls it all-reduce
 *         compatible; it prints no formula.  The QSGD-MaxNorm steps below are
 *         this library's definition of the method (global max-norm scale,
 *         s = 2^(b-1)-1 levels, stochastic rounding, signed b-bit codes).
 *         "Results" also names GlobalRandKMaxNorm compression (K = 10000) as
 *         its sparsified variant, again without a formula; the GRandK-MN
 *         functions state this library's reading of it.  It names the
 *         two-scale QSGDMaxNormMultiScale variant (QSGD-MN-TS) the same way;
 *         the QSGD-MN-TS functions state this library's reading of that.
 *   [SC11] J. Salmon, M. Moraes, R. Dror, D. Shaw, "Parallel Random Numbers:
 *         As Easy as 1, 2, 3", SC'11 -- the Philox4x32-10 generator.
 *
 * Pinning (what checks this file against something other than itself) is
 * done by the CPU tests: the worked example printed in [MX] "Format of
 * compressed gradient", exhaustive round trips, IEEE rounding bounds checked
 * in exact rational arithmetic, error-feedback telescoping, closed-form
 * aggregates, published Philox known-answer vectors and statistical
 * properties of the stochastic rounding.  Every function here has at least
 * one such pin; none is "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

/* ------------------------------------------------------------------ */
/* bit views of binary32                                               */
/* ------------------------------------------------------------------ */
static uint32_t bits_of(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return u;
}

static float float_of(uint32_t u)
{
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* ------------------------------------------------------------------ */
/* 2-bit threshold quantization with error feedback  [MX]              */
/* ------------------------------------------------------------------ */

/* [MX] "Format of compressed gradient": two thresholds, the original size,
 * then one 32-bit word per (up to) 16 original elements. */
int64_t oracle_2bit_words(int64_t n)
{
    return 3 + (n + 15) / 16;
}

/* [MX] "Two bit quantization": a value at or above the positive threshold
 * gets code 01, a value at or below the negative threshold gets code 10,
 * anything else gets code 00.  The positive test is taken first. */
static uint32_t two_bit_code(float value, float neg_thr, float pos_thr)
{
    if (value >= pos_thr)
        return 1u;
    if (value <= neg_thr)
        return 2u;
    return 0u;
}

/* Value a code stands for: the threshold that produced it, or zero.  The
 * header keeps the thresholds because decoding needs them ([MX] "Format of
 * compressed gradient").  Code 11 is never produced; it decodes to zero. */
static float two_bit_value(uint32_t code, float neg_thr, float pos_thr)
{
    if (code == 1u)
        return pos_thr;
    if (code == 2u)
        return neg_thr;
    return 0.0f;
}

/* Shift that puts the code of the element at position p (0..15) of its word
 * into place: the first element of a word sits in the two most significant
 * bits (the worked example's bit string 00 01 00 10 01 00 00 10 0...0). */
static int two_bit_shift(int64_t e)
{
    return 30 - 2 * (int)(e % 16);
}

static void write_2bit_header(uint32_t *compr, int64_t n, float neg_thr, float pos_thr)
{
    compr[0] = bits_of(neg_thr);
    compr[1] = bits_of(pos_thr);
    compr[2] = bits_of((float)n); /* the example prints n as the float 8 */
}

/* One element of the error-feedback step ([MX] "Approach", "Two bit
 * quantization"): the stored residual is added to the gradient, the sum is
 * coded, and what the code does not carry stays in the residual. */
static uint32_t quantize_one(float grad, float *residual, float neg_thr, float pos_thr)
{
    float with_residual = grad + *residual;
    uint32_t code = two_bit_code(with_residual, neg_thr, pos_thr);
    *residual = with_residual - two_bit_value(code, neg_thr, pos_thr);
    return code;
}

/* quantize_2bit(grad, residual, compr, neg_threshold, pos_threshold) of
 * [MX] "Operators", fp32 gradient.  compr holds oracle_2bit_words(n) words. */
void oracle_quantize_2bit(const float *grad, float *residual, uint32_t *compr,
                          int64_t n, float neg_thr, float pos_thr)
{
    write_2bit_header(compr, n, neg_thr, pos_thr);
    for (int64_t w = 0; w < (n + 15) / 16; ++w)
        compr[3 + w] = 0u;
    for (int64_t e = 0; e < n; ++e) {
        uint32_t code = quantize_one(grad[e], &residual[e], neg_thr, pos_thr);
        compr[3 + e / 16] |= code << two_bit_shift(e);
    }
}

/* bfloat16 is the upper half of a binary32 bit pattern, so widening it is
 * exact: append sixteen zero bits. */
static float widen_bf16(uint16_t h)
{
    return float_of((uint32_t)h << 16);
}

/* The same operator for a bfloat16 gradient and an fp32 residual. */
void oracle_quantize_2bit_bf16(const uint16_t *grad, float *residual, uint32_t *compr,
                               int64_t n, float neg_thr, float pos_thr)
{
    write_2bit_header(compr, n, neg_thr, pos_thr);
    for (int64_t w = 0; w < (n + 15) / 16; ++w)
        compr[3 + w] = 0u;
    for (int64_t e = 0; e < n; ++e) {
        uint32_t code = quantize_one(widen_bf16(grad[e]), &residual[e], neg_thr, pos_thr);
        compr[3 + e / 16] |= code << two_bit_shift(e);
    }
}

static uint32_t two_bit_code_at(const uint32_t *compr, int64_t e)
{
    return (compr[3 + e / 16] >> two_bit_shift(e)) & 3u;
}

/* dequantize_2bit(compr, decompr) of [MX] "Operators": every element becomes
 * the value of its code, with the thresholds read from the record's header.
 * n is the caller's element count (the header's float copy of n is not exact
 * above 2^24). */
void oracle_dequantize_2bit(const uint32_t *compr, float *out, int64_t n)
{
    float neg_thr = float_of(compr[0]);
    float pos_thr = float_of(compr[1]);
    for (int64_t e = 0; e < n; ++e)
        out[e] = two_bit_value(two_bit_code_at(compr, e), neg_thr, pos_thr);
}

/* The receiver's merge of [MX] "Local kvstore": every worker's record is
 * dequantized with its own header and the results are summed.  The sum
 * starts from +0 and adds the workers in the order 0, 1, ..., W-1. */
void oracle_dequant_accumulate_2bit(const uint32_t *const *compr, int W, float *out, int64_t n)
{
    for (int64_t e = 0; e < n; ++e) {
        float sum = 0.0f;
        for (int w = 0; w < W; ++w) {
            float neg_thr = float_of(compr[w][0]);
            float pos_thr = float_of(compr[w][1]);
            sum = sum + two_bit_value(two_bit_code_at(compr[w], e), neg_thr, pos_thr);
        }
        out[e] = sum;
    }
}

/* Bucket of T tensors: the compressed bucket is the T standalone records one
 * after the other, each padded to whole words as every record is. */
int64_t oracle_2bit_bucket_words(const int64_t *n, int T)
{
    int64_t words = 0;
    for (int t = 0; t < T; ++t)
        words += oracle_2bit_words(n[t]);
    return words;
}

/* grads[t] points at an fp32 array when grad_is_bf16 == 0, else at bf16. */
void oracle_quantize_2bit_bucket(const void *const *grads, float *const *residuals,
                                 const int64_t *n, const float *neg_thr, const float *pos_thr,
                                 int T, int grad_is_bf16, uint32_t *compr)
{
    int64_t offset = 0;
    for (int t = 0; t < T; ++t) {
        if (grad_is_bf16)
            oracle_quantize_2bit_bf16((const uint16_t *)grads[t], residuals[t], compr + offset,
                                      n[t], neg_thr[t], pos_thr[t]);
        else
            oracle_quantize_2bit((const float *)grads[t], residuals[t], compr + offset,
                                 n[t], neg_thr[t], pos_thr[t]);
        offset += oracle_2bit_words(n[t]);
    }
}

/* Merge of W compressed buckets into one fp32 buffer holding the T tensors
 * one after the other. */
void oracle_dequant_accumulate_2bit_bucket(const uint32_t *const *compr, int W,
                                           const int64_t *n, int T, float *out)
{
    const uint32_t *records[64];
    int64_t word_offset = 0, elem_offset = 0;
    for (int t = 0; t < T; ++t) {
        for (int w = 0; w < W; ++w)
            records[w] = compr[w] + word_offset;
        oracle_dequant_accumulate_2bit(records, W, out + elem_offset, n[t]);
        word_offset += oracle_2bit_words(n[t]);
        elem_offset += n[t];
    }
}

/* ------------------------------------------------------------------ */
/* Philox4x32-10  [SC11]                                               */
/* ------------------------------------------------------------------ */

/* One round: two 32x32->64 products of the even counter words with the
 * round multipliers; the high halves are mixed with the odd words and the
 * key, the low halves move into the odd slots. */
static void philox_round(uint32_t ctr[4], const uint32_t key[2])
{
    uint64_t p0 = (uint64_t)0xD2511F53u * ctr[0];
    uint64_t p1 = (uint64_t)0xCD9E8D57u * ctr[2];
    uint32_t next[4];
    next[0] = (uint32_t)(p1 >> 32) ^ ctr[1] ^ key[0];
    next[1] = (uint32_t)p1;
    next[2] = (uint32_t)(p0 >> 32) ^ ctr[3] ^ key[1];
    next[3] = (uint32_t)p0;
    memcpy(ctr, next, sizeof next);
}

/* Ten rounds; the key is advanced by the Weyl increments (golden ratio and
 * sqrt(3)-1 in 0.32 fixed point) before every round after the first. */
void oracle_philox4x32_10(const uint32_t counter[4], const uint32_t key_in[2], uint32_t out[4])
{
    uint32_t ctr[4] = {counter[0], counter[1], counter[2], counter[3]};
    uint32_t key[2] = {key_in[0], key_in[1]};
    for (int round = 0; round < 10; ++round) {
        if (round > 0) {
            key[0] += 0x9E3779B9u;
            key[1] += 0xBB67AE85u;
        }
        philox_round(ctr, key);
    }
    memcpy(out, ctr, sizeof ctr);
}

/* ------------------------------------------------------------------ */
/* QSGD-MaxNorm, b bits  ([GC] names it; steps as defined above)       */
/* ------------------------------------------------------------------ */

/* The global scale M: the largest |g| over every worker's buffer.  A NaN
 * element never compares greater, so it is skipped. */
float oracle_qsgd_mn_max(const float *const *grad, int W, int64_t n)
{
    float m = 0.0f;
    for (int w = 0; w < W; ++w)
        for (int64_t e = 0; e < n; ++e) {
            float a = fabsf(grad[w][e]);
            if (a > m)
                m = a;
        }
    return m;
}

/* The uniform draw of element e: Philox4x32-10 keyed by the 64-bit seed
 * (low word first), counter (e/4 low word, e/4 high word, 0, 0); element e
 * takes output word e mod 4, keeps its top 24 bits and scales by 2^-24, so
 * u is a multiple of 2^-24 in [0, 1 - 2^-24], exact in binary32. */
float oracle_qsgd_uniform(uint64_t seed, int64_t e)
{
    uint64_t block = (uint64_t)e / 4;
    uint32_t ctr[4] = {(uint32_t)block, (uint32_t)(block >> 32), 0u, 0u};
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    uint32_t out[4];
    oracle_philox4x32_10(ctr, key, out);
    return (float)(out[e % 4] >> 8) * 0x1p-24f;
}

static int qsgd_levels(int b)
{
    return (1 << (b - 1)) - 1;
}

/* The signed level of one element: scale |g| by the global max, stretch to
 * s levels, add the uniform draw and round down, cap at s, restore the sign.
 * Each arithmetic step is one binary32 operation in this order:
 *   t = ((|g| / M) * s) + u,   q = sign(g) * min(floor(t), s).
 * A non-finite t (M == 0, or non-finite input) gives level 0. */
int32_t oracle_qsgd_level(float grad, float M, int b, uint64_t seed, int64_t e)
{
    int s = qsgd_levels(b);
    float u = oracle_qsgd_uniform(seed, e);
    float scaled = fabsf(grad) / M;
    float stretched = scaled * (float)s;
    float t = stretched + u;
    if (!isfinite(t))
        return 0;
    float level = floorf(t);
    if (level > (float)s)
        level = (float)s;
    int32_t q = (int32_t)level;
    return grad < 0.0f ? -q : q;
}

int64_t oracle_qsgd_words(int64_t n, int b)
{
    return 3 + (n * b + 31) / 32;
}

/* Record: header [M, b, n] as binary32, then 32/b two's-complement codes of
 * b bits per word, the first element of a word in its most significant bits
 * (the same order as the 2-bit format), unused tail codes zero. */
void oracle_qsgd_mn_quantize(const float *grad, uint32_t *compr, int64_t n, int b,
                             uint64_t seed, float M)
{
    int per_word = 32 / b;
    uint32_t mask = (1u << b) - 1u;
    compr[0] = bits_of(M);
    compr[1] = bits_of((float)b);
    compr[2] = bits_of((float)n);
    for (int64_t w = 0; w < (n * b + 31) / 32; ++w)
        compr[3 + w] = 0u;
    for (int64_t e = 0; e < n; ++e) {
        int32_t q = oracle_qsgd_level(grad[e], M, b, seed, e);
        uint32_t code = (uint32_t)q & mask;
        int shift = 32 - b * (int)(e % per_word + 1);
        compr[3 + e / per_word] |= code << shift;
    }
}

/* Level of element e read back from a record: the b-bit field, sign-extended. */
static int32_t qsgd_level_at(const uint32_t *compr, int64_t e, int b)
{
    int per_word = 32 / b;
    int shift = 32 - b * (int)(e % per_word + 1);
    uint32_t code = (compr[3 + e / per_word] >> shift) & ((1u << b) - 1u);
    int32_t q = (int32_t)code;
    if (code >= (1u << (b - 1)))
        q -= (int32_t)(1u << b);
    return q;
}

/* Aggregate of W records: the integer levels are summed (exact), then scaled
 * once by M / s, with M read from worker 0's header (every worker quantized
 * with the same global M).  This is the sum-then-scale form that makes the
 * scheme all-reduce compatible ([GC] "About The Project"). */
void oracle_qsgd_mn_dequant_accumulate(const uint32_t *const *compr, int W, float *out,
                                       int64_t n, int b)
{
    float M = float_of(compr[0][0]);
    float step = M / (float)qsgd_levels(b);
    for (int64_t e = 0; e < n; ++e) {
        int32_t sum = 0;
        for (int w = 0; w < W; ++w)
            sum += qsgd_level_at(compr[w], e, b);
        out[e] = (float)sum * step;
    }
}

/* ------------------------------------------------------------------ */
/* QSGD-MaxNorm with two scales (QSGD-MN-TS)                           */
/* ------------------------------------------------------------------ */
/* [GC] "Results" names QSGDMaxNormMultiScale quantization run with two
 * scales (TS) of compression, each run labelled with the bit widths of its
 * two scales, and gives no formula; [GC] "About The Project" counts it among
 * the all-reduce compatible schemes.  This library's reading:
 *   - the coarse scale is the QSGD-MaxNorm scale M1 = M (the global max |g|)
 *     with b1 bits, s1 = 2^(b1-1) - 1 levels;
 *   - the fine scale is the coarse grid's first step, M2 = M1 / s1 (one
 *     binary32 division), with b2 bits, s2 = 2^(b2-1) - 1 levels;
 *   - an element with |g| <= M2 takes the fine scale, any other element the
 *     coarse one: its level is the QSGD-MaxNorm level with that scale's M and
 *     s and the element's own draw; its level on the other scale is 0;
 *   - the record is the coarse levels as a QSGD-MaxNorm record of b1 bits
 *     (header [M1, b1, n]) followed by the fine levels as a QSGD-MaxNorm
 *     record of b2 bits (header [M2, b2, n]);
 *   - the merge sums each scale's levels over the workers in integers, scales
 *     each sum once (the QSGD-MaxNorm merge of that scale's records) and adds
 *     the two: out = A + B.  Both integer sums can be formed by an
 *     all-reduce, as in the one-scale scheme.
 * With b1 = 2 (s1 = 1) the two scales coincide, every element with |g| <= M
 * is fine, and the fine record is the QSGD-MaxNorm record of b2 bits. */

int64_t oracle_qsgd_mnts_words(int64_t n, int b1, int b2)
{
    return oracle_qsgd_words(n, b1) + oracle_qsgd_words(n, b2);
}

/* The fine scale: the coarse scale's quantization step. */
float oracle_qsgd_mnts_fine_scale(float M, int b1)
{
    return M / (float)qsgd_levels(b1);
}

/* The two levels of element e: q[0] on the coarse scale, q[1] on the fine
 * one (one of them is 0). */
void oracle_qsgd_mnts_levels(float grad, float M, int b1, int b2, uint64_t seed, int64_t e,
                             int32_t q[2])
{
    float M2 = oracle_qsgd_mnts_fine_scale(M, b1);
    int is_fine = fabsf(grad) <= M2;
    q[0] = is_fine ? 0 : oracle_qsgd_level(grad, M, b1, seed, e);
    q[1] = is_fine ? oracle_qsgd_level(grad, M2, b2, seed, e) : 0;
}

void oracle_qsgd_mnts_quantize(const float *grad, uint32_t *compr, int64_t n, int b1, int b2,
                               uint64_t seed, float M)
{
    float M2 = oracle_qsgd_mnts_fine_scale(M, b1);
    uint32_t *coarse = compr;
    uint32_t *fine = compr + oracle_qsgd_words(n, b1);
    coarse[0] = bits_of(M);
    coarse[1] = bits_of((float)b1);
    coarse[2] = bits_of((float)n);
    fine[0] = bits_of(M2);
    fine[1] = bits_of((float)b2);
    fine[2] = bits_of((float)n);
    for (int64_t w = 0; w < (n * b1 + 31) / 32; ++w)
        coarse[3 + w] = 0u;
    for (int64_t w = 0; w < (n * b2 + 31) / 32; ++w)
        fine[3 + w] = 0u;
    for (int64_t e = 0; e < n; ++e) {
        int32_t q[2];
        oracle_qsgd_mnts_levels(grad[e], M, b1, b2, seed, e, q);
        int per1 = 32 / b1, per2 = 32 / b2;
        coarse[3 + e / per1] |= ((uint32_t)q[0] & ((1u << b1) - 1u)) << (32 - b1 * (int)(e % per1 + 1));
        fine[3 + e / per2] |= ((uint32_t)q[1] & ((1u << b2) - 1u)) << (32 - b2 * (int)(e % per2 + 1));
    }
}

void oracle_qsgd_mnts_dequant_accumulate(const uint32_t *const *compr, int W, float *out,
                                         int64_t n, int b1, int b2)
{
    int64_t fine_off = oracle_qsgd_words(n, b1);
    float step1 = float_of(compr[0][0]) / (float)qsgd_levels(b1);
    float step2 = float_of(compr[0][fine_off]) / (float)qsgd_levels(b2);
    for (int64_t e = 0; e < n; ++e) {
        int32_t sum1 = 0, sum2 = 0;
        for (int w = 0; w < W; ++w) {
            sum1 += qsgd_level_at(compr[w], e, b1);
            sum2 += qsgd_level_at(compr[w] + fine_off, e, b2);
        }
        float coarse_part = (float)sum1 * step1;
        float fine_part = (float)sum2 * step2;
        out[e] = coarse_part + fine_part;
    }
}

/* ------------------------------------------------------------------ */
/* GlobalRandKMaxNorm (GRandK-MN): QSGD-MaxNorm of K shared coordinates */
/* ------------------------------------------------------------------ */
/* [GC] "Results" names GlobalRandKMaxNorm compression, with K = 10000, as the
 * sparsified variant of QSGDMaxNorm and gives no formula.  This library's
 * reading: every worker keeps the same K coordinates index[0..K-1] (drawn by
 * the caller, shared by all workers, so the sparse vectors still add up in
 * an all-reduce); the kept values x[k] = g[index[k]] form a K-vector that is
 * quantized exactly as QSGD-MaxNorm quantizes a gradient (M = max |x| over
 * all workers, draw k for position k, header [M, b, K]); the merge sums the
 * levels, scales them once and scatters them back to their coordinates, every
 * other coordinate of the n-element result being +0.  A coordinate outside
 * [0, n) is skipped: it does not enter M, gets level 0 and is not stored. */

static int index_in_range(int64_t i, int64_t n)
{
    return i >= 0 && i < n;
}

float oracle_grandk_mn_max(const float *const *grad, int W, int64_t n, const int64_t *index,
                           int64_t K)
{
    float m = 0.0f;
    for (int w = 0; w < W; ++w)
        for (int64_t k = 0; k < K; ++k) {
            if (!index_in_range(index[k], n))
                continue;
            float a = fabsf(grad[w][index[k]]);
            if (a > m)
                m = a;
        }
    return m;
}

void oracle_grandk_mn_quantize(const float *grad, int64_t n, const int64_t *index, int64_t K,
                               uint32_t *compr, int b, uint64_t seed, float M)
{
    int per_word = 32 / b;
    uint32_t mask = (1u << b) - 1u;
    compr[0] = bits_of(M);
    compr[1] = bits_of((float)b);
    compr[2] = bits_of((float)K);
    for (int64_t w = 0; w < (K * b + 31) / 32; ++w)
        compr[3 + w] = 0u;
    for (int64_t k = 0; k < K; ++k) {
        int32_t q = 0;
        if (index_in_range(index[k], n))
            q = oracle_qsgd_level(grad[index[k]], M, b, seed, k);
        uint32_t code = (uint32_t)q & mask;
        compr[3 + k / per_word] |= code << (32 - b * (int)(k % per_word + 1));
    }
}

void oracle_grandk_mn_dequant_accumulate(const uint32_t *const *compr, int W,
                                         const int64_t *index, int64_t K, float *out, int64_t n,
                                         int b)
{
    float M = float_of(compr[0][0]);
    float step = M / (float)qsgd_levels(b);
    for (int64_t e = 0; e < n; ++e)
        out[e] = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
        if (!index_in_range(index[k], n))
            continue;
        int32_t sum = 0;
        for (int w = 0; w < W; ++w)
            sum += qsgd_level_at(compr[w], k, b);
        out[index[k]] = (float)sum * step;
    }
}

/* ------------------------------------------------------------------ */
/* Dense ternary packing of the 2-bit threshold codes                  */
/* ------------------------------------------------------------------ */
/* [MX] "Two bit quantization" notes that three values need only log2(3)
 * bits and leaves the wasted code for later.  This library's dense format:
 * the three codes 00, 01, 10 become the trits 0, 1, 2; five consecutive
 * elements form one byte as the base-3 numeral t0 t1 t2 t3 t4 (element 0 the
 * most significant trit, so a byte is at most 242); payload byte j holds
 * elements 5j..5j+4 and sits at byte 12 + j of the record (memory order)
 * after the same three-word header [neg, pos, n]; the record is padded to
 * whole 32-bit words, and trits past n and padding bytes are zero.  The
 * error feedback is exactly that of the 2-bit operator. */

int64_t oracle_ternary_words(int64_t n)
{
    return 3 + (n + 19) / 20;
}

void oracle_quantize_ternary(const float *grad, float *residual, uint32_t *compr, int64_t n,
                             float neg_thr, float pos_thr)
{
    unsigned char *payload = (unsigned char *)(compr + 3);
    write_2bit_header(compr, n, neg_thr, pos_thr);
    for (int64_t w = 0; w < (n + 19) / 20; ++w)
        compr[3 + w] = 0u;
    for (int64_t j = 0; 5 * j < n; ++j) {
        unsigned value = 0;
        for (int64_t e = 5 * j; e < 5 * j + 5; ++e) {
            unsigned trit = 0;
            if (e < n)
                trit = quantize_one(grad[e], &residual[e], neg_thr, pos_thr);
            value = value * 3 + trit;
        }
        payload[j] = (unsigned char)value;
    }
}

/* Trit of element e: digit e mod 5 (most significant first) of byte e / 5. */
static uint32_t ternary_code_at(const uint32_t *compr, int64_t e)
{
    const unsigned char *payload = (const unsigned char *)(compr + 3);
    unsigned value = payload[e / 5];
    for (int64_t k = e % 5; k < 4; ++k)
        value /= 3;
    return value % 3;
}

void oracle_dequantize_ternary(const uint32_t *compr, float *out, int64_t n)
{
    float neg_thr = float_of(compr[0]);
    float pos_thr = float_of(compr[1]);
    for (int64_t e = 0; e < n; ++e)
        out[e] = two_bit_value(ternary_code_at(compr, e), neg_thr, pos_thr);
}

void oracle_dequant_accumulate_ternary(const uint32_t *const *compr, int W, float *out, int64_t n)
{
    for (int64_t e = 0; e < n; ++e) {
        float sum = 0.0f;
        for (int w = 0; w < W; ++w) {
            float neg_thr = float_of(compr[w][0]);
            float pos_thr = float_of(compr[w][1]);
            sum = sum + two_bit_value(ternary_code_at(compr[w], e), neg_thr, pos_thr);
        }
        out[e] = sum;
    }
}
