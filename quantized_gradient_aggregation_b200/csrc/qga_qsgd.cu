// qga_qsgd.cu -- QSGD-MaxNorm with b-bit signed codes: the global max|g|,
// the per-worker stochastic quantizer and the integer-sum merge.
//
// The gradient-compression README (vineeths96), "About The Project" and
// "Results", names QSGDMaxNorm quantization and calls it all-reduce
// compatible; it prints no formula.  This library's definition:
//   s = 2^(b-1) - 1,  M = max |g| over every worker's gradient,
//   u = Philox4x32-10 draw of the element (Salmon et al., "Parallel Random
//       Numbers: As Easy as 1, 2, 3", SC'11), top 24 bits times 2^-24,
//   t = ((|g| / M) * s) + u  (three binary32 operations in this order),
//   q = sign(g) * min(floor(t), s), 0 when t is not finite,
// packed as b-bit two's complement, 32/b per word, first element in the most
// significant bits, after a header [M, b, n].  The merge adds the integer
// levels of all workers and scales once by M / s, which is what lets the
// codes be summed by an all-reduce.
//
// Tile geometry as in the 2-bit path: a warp owns 128 groups of 4 elements;
// lane l handles groups l, l+32, l+64, l+96 (coalesced 128-bit loads).  One
// Philox block (one counter) yields the 4 draws of one group.

#include <float.h>

#include "qga_common.cuh"
#include "qga_qsgd_level.cuh"

namespace qga {
namespace {

constexpr int kThreads = 256;
constexpr int kWarpsPerBlock = kThreads / kWarp;
constexpr int kGroupsPerLane = 4;
constexpr int kTileGroups = kWarp * kGroupsPerLane;

struct GradSet {
    const float *g[QGA_MAX_WORKERS];
};

struct RecordSet {
    const uint32_t *rec[QGA_MAX_WORKERS];
};

// ------------------------------------------------------------------- max ----
__global__ void __launch_bounds__(kThreads)
    qsgd_max_kernel(const __grid_constant__ GradSet set, int W, int64_t n, float *__restrict__ M)
{
    __shared__ float s_part[kWarpsPerBlock];
    const int64_t tid = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    const int64_t nthreads = (int64_t)gridDim.x * kThreads;
    const int64_t groups = n >> 2;
    float m = 0.0f;
    for (int w = 0; w < W; ++w) {
        const float *g = set.g[w];
        if (((uintptr_t)g & 15u) == 0) {
            int64_t i = tid;
            for (; i + 3 * nthreads < groups; i += 4 * nthreads) {
                const float4 a = ld_stream_f4(g + 4 * i);
                const float4 b = ld_stream_f4(g + 4 * (i + nthreads));
                const float4 c = ld_stream_f4(g + 4 * (i + 2 * nthreads));
                const float4 d = ld_stream_f4(g + 4 * (i + 3 * nthreads));
                m = fmaxf(m, fmaxf(fmaxf(fabsf(a.x), fabsf(a.y)), fmaxf(fabsf(a.z), fabsf(a.w))));
                m = fmaxf(m, fmaxf(fmaxf(fabsf(b.x), fabsf(b.y)), fmaxf(fabsf(b.z), fabsf(b.w))));
                m = fmaxf(m, fmaxf(fmaxf(fabsf(c.x), fabsf(c.y)), fmaxf(fabsf(c.z), fabsf(c.w))));
                m = fmaxf(m, fmaxf(fmaxf(fabsf(d.x), fabsf(d.y)), fmaxf(fabsf(d.z), fabsf(d.w))));
            }
            for (; i < groups; i += nthreads) {
                const float4 a = ld_stream_f4(g + 4 * i);
                m = fmaxf(m, fmaxf(fmaxf(fabsf(a.x), fabsf(a.y)), fmaxf(fabsf(a.z), fabsf(a.w))));
            }
            for (int64_t e = 4 * groups + tid; e < n; e += nthreads)
                m = fmaxf(m, fabsf(ld_stream_f1(g + e)));
        } else {
            for (int64_t e = tid; e < n; e += nthreads)
                m = fmaxf(m, fabsf(ld_stream_f1(g + e)));
        }
    }
    // fmaxf drops a NaN operand, so m is never NaN
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
        m = fmaxf(m, __shfl_xor_sync(kFullMask, m, off));
    if ((threadIdx.x & 31) == 0)
        s_part[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        float b = s_part[0];
#pragma unroll
        for (int i = 1; i < kWarpsPerBlock; ++i)
            b = fmaxf(b, s_part[i]);
        // non-negative binary32 values order like their bit patterns
        if (b > 0.0f)
            atomicMax(reinterpret_cast<unsigned int *>(M), __float_as_uint(b));
    }
}

// -------------------------------------------------------------- quantize ----
template <int B, bool kVec>
__global__ void __launch_bounds__(kThreads)
    qsgd_quantize_kernel(const float *__restrict__ grad, uint32_t *__restrict__ compr, int64_t n,
                         uint32_t key0, uint32_t key1, const float *__restrict__ max_in)
{
    using L = Levels<B>;
    const float M = *max_in;
    const bool fast = M > 0.0f && M <= FLT_MAX;          // uniform over the grid
    const float k = __fdiv_rn((float)L::s, M);
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        compr[0] = bits_from_f32(M);
        compr[1] = bits_from_f32((float)B);
        compr[2] = bits_from_f32(__ll2float_rn(n));
    }
    uint32_t *payload = compr + 3;
    const int lane = threadIdx.x & (kWarp - 1);
    const int64_t full_groups = n >> 2;
    const int64_t groups = (n + 3) >> 2;
    const int64_t nwords = (n * B + 31) >> 5;
    const int64_t tiles = (groups + kTileGroups - 1) / kTileGroups;
    const int64_t stride = (int64_t)gridDim.x * kWarpsPerBlock;
    for (int64_t tile = (int64_t)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5); tile < tiles;
         tile += stride) {
        const int64_t g0 = tile * kTileGroups;
        float4 gv[kGroupsPerLane];
#pragma unroll
        for (int j = 0; j < kGroupsPerLane; ++j) {
            const int64_t gi = g0 + j * kWarp + lane;
            if (kVec && gi < full_groups) {
                gv[j] = ld_stream_f4(grad + 4 * gi);
            } else {
                float t[4];
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    t[k] = (4 * gi + k < n) ? ld_stream_f1(grad + 4 * gi + k) : 0.0f;
                gv[j] = make_float4(t[0], t[1], t[2], t[3]);
            }
        }
        // the lane's four Philox chains side by side (independent, so their
        // fixed-latency round dependencies overlap), then the levels
        uint4 draws[kGroupsPerLane];
#pragma unroll
        for (int j = 0; j < kGroupsPerLane; ++j) {
            const int64_t gi = g0 + j * kWarp + lane;
            draws[j] = philox4x32_10(
                make_uint4((uint32_t)gi, (uint32_t)((uint64_t)gi >> 32), 0u, 0u), key0, key1);
        }
#pragma unroll
        for (int j = 0; j < kGroupsPerLane; ++j) {
            const int64_t gi = g0 + j * kWarp + lane;
            const uint4 r = draws[j];
            uint32_t c0, c1, c2, c3;
            if (fast) {
                c0 = (uint32_t)qsgd_level<B>(gv[j].x, M, k, r.x) & L::mask;
                c1 = (uint32_t)qsgd_level<B>(gv[j].y, M, k, r.y) & L::mask;
                c2 = (uint32_t)qsgd_level<B>(gv[j].z, M, k, r.z) & L::mask;
                c3 = (uint32_t)qsgd_level<B>(gv[j].w, M, k, r.w) & L::mask;
            } else {
                c0 = (uint32_t)qsgd_level_exact<B>(gv[j].x, M, unit_draw(r.x)) & L::mask;
                c1 = (uint32_t)qsgd_level_exact<B>(gv[j].y, M, unit_draw(r.y)) & L::mask;
                c2 = (uint32_t)qsgd_level_exact<B>(gv[j].z, M, unit_draw(r.z)) & L::mask;
                c3 = (uint32_t)qsgd_level_exact<B>(gv[j].w, M, unit_draw(r.w)) & L::mask;
            }
            uint32_t piece = (c0 << (3 * B)) | (c1 << (2 * B)) | (c2 << B) | c3;
            // codes of elements >= n are zero
            const int64_t valid = n - 4 * gi;
            if (valid < 4)
                piece = valid <= 0 ? 0u : (piece & ~((1u << (B * (4 - (int)valid))) - 1u));
            constexpr int LW = L::lanes_per_word;
            uint32_t word = piece << (32 - 4 * B * (1 + (lane % LW)));
            if (LW >= 2)
                word |= __shfl_xor_sync(kFullMask, word, 1);
            if (LW >= 4)
                word |= __shfl_xor_sync(kFullMask, word, 2);
            const int64_t wi = gi / LW;
            if ((lane % LW) == 0 && wi < nwords)
                st_stream_u32(payload + wi, word);
        }
    }
}

// The quantize in lane-owned words, for a 32-byte-aligned gradient: lane l
// of warp t owns the 16 consecutive elements 16 (32 t + l) .. + 15 (two
// 256-bit loads, the 4 Philox blocks of its 4 groups), forms their levels
// with the fixed-point level (qsgd_level_lean) and packs its b / 2 record
// words in registers: no shuffles and one check per lane.  A lane whose
// check flags any element recomputes all 16 by the definition's operations.
template <int B>
__global__ void __launch_bounds__(kThreads)
    qsgd_quantize_words_kernel(const float *__restrict__ grad, uint32_t *__restrict__ compr, int64_t n,
                               uint32_t key0, uint32_t key1, const float *__restrict__ max_in)
{
    using L = Levels<B>;
    constexpr int E = B - 1;
    constexpr int kWords = B / 2; // record words per 16 elements
    constexpr int kPer = 32 / B;  // elements per word
    const float M = *max_in;
    const bool fast = M > 0.0f && M <= FLT_MAX; // uniform over the grid
    const float k = __fdiv_rn((float)L::s, M);
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        compr[0] = bits_from_f32(M);
        compr[1] = bits_from_f32((float)B);
        compr[2] = bits_from_f32(__ll2float_rn(n));
    }
    uint32_t *payload = compr + 3;
    const int lane = threadIdx.x & (kWarp - 1);
    const int64_t nwords = (n * B + 31) >> 5;
    const int64_t runs = (n + 16 * kWarp - 1) / (16 * kWarp);
    for (int64_t t = (int64_t)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5); t < runs;
         t += (int64_t)gridDim.x * kWarpsPerBlock) {
        const int64_t r = t * kWarp + lane; // this lane's run of 16 elements
        const int64_t e0 = 16 * r;
        float g[16];
        if (e0 + 16 <= n) {
            ld_stream_f8(grad + e0, g);
            ld_stream_f8(grad + e0 + 8, g + 8);
        } else {
#pragma unroll
            for (int p = 0; p < 16; ++p)
                g[p] = e0 + p < n ? ld_stream_f1(grad + e0 + p) : 0.0f;
        }
        uint4 d[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int64_t gi = 4 * r + j;
            d[j] = philox4x32_10(make_uint4((uint32_t)gi, (uint32_t)((uint64_t)gi >> 32), 0u, 0u), key0, key1);
        }
        const uint32_t x[16] = {d[0].x, d[0].y, d[0].z, d[0].w, d[1].x, d[1].y, d[1].z, d[1].w,
                                d[2].x, d[2].y, d[2].z, d[2].w, d[3].x, d[3].y, d[3].z, d[3].w};
        uint32_t w[kWords] = {};
        uint32_t fmin = 0xFFFFFFFFu, tmax = 0u;
#pragma unroll
        for (int p = 0; p < 16; ++p) {
            const uint32_t c = signed_code<B>(qsgd_level_lean<E>(g[p], k, x[p], fmin, tmax), g[p]);
            w[p / kPer] |= c << (32 - B * (p % kPer + 1));
        }
        if (!fast || LeanLevel<E>::needs_exact(fmin, tmax, (uint32_t)L::s)) {
#pragma unroll
            for (int i = 0; i < kWords; ++i)
                w[i] = 0u;
#pragma unroll
            for (int p = 0; p < 16; ++p) {
                const uint32_t c = (uint32_t)qsgd_level_exact<B>(g[p], M, unit_draw(x[p])) & L::mask;
                w[p / kPer] |= c << (32 - B * (p % kPer + 1));
            }
        }
        // elements past n loaded as 0 have level 0, so their codes are 0
#pragma unroll
        for (int i = 0; i < kWords; ++i)
            if (r * kWords + i < nwords)
                st_stream_u32(payload + r * kWords + i, w[i]);
    }
}

// ----------------------------------------------------------------- merge ----
// Integer sum of the W workers' levels a whole record word at a time
// (LevelSum in qga_qsgd_level.cuh).  A thread owns whole words: word l of
// each 32-word block of its warp (for b = 2, also word 32 + l, loaded
// together for more bytes in flight), and stores its 32/b outputs as 128-bit
// (b = 8) or 256-bit rows.
template <int B> constexpr int kMergeSlotsFor = B == 2 ? 2 : 1; // words per thread (measured best)

// Outputs of one record word from its lane sums: element e sits in field
// kFields - 1 - e (counted from the least significant).
template <int B, bool kVec>
__device__ __forceinline__ void merge_store_word(LevelSum<B> &acc, int64_t kw, float offset, float step,
                                                 float *__restrict__ out, int64_t n)
{
    using S = LevelSum<B>;
    acc.finish();
    float v[S::kFields];
#pragma unroll
    for (int e = 0; e < S::kFields; ++e)
        v[e] = __fmul_rn(__fsub_rn(__uint_as_float(0x4B000000u | acc.field_sum(e)), offset), step);
    const int64_t e0 = kw * S::kFields;
    if (kVec && e0 + S::kFields <= n) {
        if (S::kFields == 4)
            st_stream_f4(out + e0, make_float4(v[0], v[1], v[2], v[3]));
        else
#pragma unroll
            for (int c = 0; c < S::kFields; c += 8)
                st_stream_f8(out + e0 + c, v + c);
    } else {
#pragma unroll
        for (int e = 0; e < S::kFields; ++e)
            if (e0 + e < n)
                st_stream_f1(out + e0 + e, v[e]);
    }
}

// Any worker count (used for W > 16): batches of 8 workers, the payload
// pointers read from the kernel's parameter space.  Measured at n = 2^27,
// b = 4, W = 9 / 16 / 32: 212 / 279 / 467 us, against 230 / 312 / 533 us
// with the pointers read back from shared memory in every iteration (b = 2
// and 8 unchanged).  Two slots per lane for every b, 4 blocks per SM and a
// separate full-batch path measured far slower (b = 8, W = 32: 1448 us).
template <int B, bool kVec>
__global__ void __launch_bounds__(kThreads)
    qsgd_merge_kernel(const __grid_constant__ RecordSet set, int W, float *__restrict__ out,
                      int64_t n)
{
    constexpr int kBatch = 8;
    static_assert(kBatch <= LevelSum<B>::kBatchMax, "a batch fits the narrow lanes");
    const float step = __fdiv_rn(f32_from_bits(set.rec[0][0]), (float)Levels<B>::s);
    // 2^23 + W 2^(b-1): the magic-number conversion's offset and the bias
    const float offset = 8388608.0f + (float)(W << (B - 1));
    const int64_t nwords = (n * B + 31) >> 5;
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    if constexpr (kMergeSlotsFor<B> == 1) {
        for (int64_t kw = (int64_t)blockIdx.x * kThreads + threadIdx.x; kw < nwords; kw += stride) {
            LevelSum<B> acc;
            for (int wb = 0; wb < W; wb += kBatch) {
                uint32_t words[kBatch];
#pragma unroll
                for (int i = 0; i < kBatch; ++i)
                    words[i] = wb + i < W ? ld_stream_u32(set.rec[wb + i] + 3 + kw) : 0u;
#pragma unroll
                for (int i = 0; i < kBatch; ++i) {
                    if (wb + i >= W) // warp-uniform
                        break;
                    acc.add(words[i]);
                }
                acc.end_batch();
            }
            merge_store_word<B, kVec>(acc, kw, offset, step, out, n);
        }
    } else {
        // a warp takes 2 x 32 consecutive words: lane l the words l and 32 + l,
        // loaded together for more bytes in flight
        const int lane = threadIdx.x & (kWarp - 1);
        const int64_t nslices = (nwords + 2 * kWarp - 1) / (2 * kWarp);
        for (int64_t sl = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5; sl < nslices;
             sl += stride >> 5) {
            const int64_t k0 = sl * (2 * kWarp) + lane, k1 = k0 + kWarp;
            LevelSum<B> acc0, acc1;
            for (int wb = 0; wb < W; wb += kBatch) {
                uint32_t w0[kBatch], w1[kBatch];
#pragma unroll
                for (int i = 0; i < kBatch; ++i) {
                    w0[i] = (wb + i < W && k0 < nwords) ? ld_stream_u32(set.rec[wb + i] + 3 + k0) : 0u;
                    w1[i] = (wb + i < W && k1 < nwords) ? ld_stream_u32(set.rec[wb + i] + 3 + k1) : 0u;
                }
#pragma unroll
                for (int i = 0; i < kBatch; ++i) {
                    if (wb + i >= W) // warp-uniform
                        break;
                    acc0.add(w0[i]);
                    acc1.add(w1[i]);
                }
                acc0.end_batch();
                acc1.end_batch();
            }
            if (k0 < nwords)
                merge_store_word<B, kVec>(acc0, k0, offset, step, out, n);
            if (k1 < nwords)
                merge_store_word<B, kVec>(acc1, k1, offset, step, out, n);
        }
    }
}

// The merge for a worker count known at compile time (W <= 8, one batch of
// the level sums): the W payload pointers come from the kernel's parameter
// space, and the W words of each of the lane's slots are all loaded before
// any is summed.  A warp takes kMergeWSlots x 32 consecutive words: slot s of
// lane l is word 32 s + l.  Four resident blocks of 256 threads per SM (at
// most 64 registers).  Measured at n = 2^27, W = 8, b = 2 / 4 / 8: 125.4 /
// 169.9 / 252.3 us, against 148.8 / 199 / 285 us for the runtime-W kernel
// above when it read the payload pointers back from shared memory in every
// iteration; one slot per lane took 124.6 / 210.8 / 255.3 us, and 6 or 8
// blocks per SM 140 / 171-217 / 256-263 us.
#ifndef QGA_QSGD_MERGE_W_SLOTS
#define QGA_QSGD_MERGE_W_SLOTS 2
#endif
#ifndef QGA_QSGD_MERGE_W_MIN_BLOCKS
#define QGA_QSGD_MERGE_W_MIN_BLOCKS 4
#endif
constexpr int kMergeWSlots = QGA_QSGD_MERGE_W_SLOTS;

// kPad: any W up to kW; the words of workers W .. kW - 1 are taken as 0, a
// word of levels 0, which adds nothing to the sums (the bias it adds is the
// one the offset removes for kW words).  Measured at n = 2^27, W = 16, b = 2
// / 4 / 8: 180 / 262 / 423 us, against 222 / 277 / 470 us for the runtime-W
// kernel.
template <int B, bool kVec, int kW, bool kPad>
__global__ void __launch_bounds__(kThreads, QGA_QSGD_MERGE_W_MIN_BLOCKS)
    qsgd_merge_w_kernel(const __grid_constant__ RecordSet set, int W, float *__restrict__ out, int64_t n)
{
    constexpr int kSlots = kMergeWSlots;
    static_assert(kW >= 1 && kW <= LevelSum<B>::kBatchMax, "one batch fits the narrow lanes");
    const float step = __fdiv_rn(f32_from_bits(set.rec[0][0]), (float)Levels<B>::s);
    const float offset = 8388608.0f + (float)(kW << (B - 1));
    const int64_t nwords = (n * B + 31) >> 5;
    const int lane = threadIdx.x & (kWarp - 1);
    const int64_t nslices = (nwords + kSlots * kWarp - 1) / (kSlots * kWarp);
    for (int64_t sl = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5; sl < nslices;
         sl += ((int64_t)gridDim.x * kThreads) >> 5) {
        uint32_t wd[kSlots][kW];
#pragma unroll
        for (int s = 0; s < kSlots; ++s) {
            const int64_t k = (sl * kSlots + s) * kWarp + lane;
#pragma unroll
            for (int i = 0; i < kW; ++i)
                wd[s][i] = ((!kPad || i < W) && k < nwords) ? ld_stream_u32(set.rec[i] + 3 + k) : 0u;
        }
#pragma unroll
        for (int s = 0; s < kSlots; ++s) {
            const int64_t k = (sl * kSlots + s) * kWarp + lane;
            LevelSum<B> acc;
#pragma unroll
            for (int i = 0; i < kW; ++i)
                acc.add(wd[s][i]);
            acc.end_batch();
            if (k < nwords)
                merge_store_word<B, kVec>(acc, k, offset, step, out, n);
        }
    }
}

std::atomic<int> occ_max[64];
std::atomic<int> occ_q[3][2][64];
std::atomic<int> occ_qw[3][64];
#ifndef QGA_QSGD_LANE_WORDS
#define QGA_QSGD_LANE_WORDS 1
#endif
std::atomic<int> occ_m[3][2][64];
std::atomic<int> occ_mw[3][2][17][64]; // [bits][vec][W][device]

int bits_slot(int bits) { return bits == 2 ? 0 : (bits == 4 ? 1 : (bits == 8 ? 2 : -1)); }

// Grid waves (see grid_for), measured at n = 2^27: quantize b = 2 / 4 / 8
// 220 / 218 / 197 us at 1 wave, 205 / 203 / 185 at 8, 205 / 203 / 187 at 16;
// merge (W = 8) b = 2 150 / 148 / 148, b = 4 231 / 206 / 201, b = 8 263 / 268 /
// 266 us at 1 / 8 / 16 waves.  The max stays persistent (one atomic per block;
// 606 / 602 / 606 / 696 us at 1 / 8 / 16 / 32).
#ifndef QGA_QSGD_QUANTIZE_WAVES
#define QGA_QSGD_QUANTIZE_WAVES 8
#endif
constexpr int kQsgdQuantizeWaves = QGA_QSGD_QUANTIZE_WAVES;
template <int B> constexpr int kQsgdMergeWaves = B == 8 ? 1 : 16;
// W <= 8 kernel: 4 / 16 / 32 waves at b = 2, W = 8: 136 / 124 / 123 us; at
// b = 4, W = 1 .. 8 and b = 8 the 32-wave grid is 1-4 us faster than 16.
#ifndef QGA_QSGD_MERGE_W_WAVES
#define QGA_QSGD_MERGE_W_WAVES 32
#endif
constexpr int kQsgdMergeWWaves = QGA_QSGD_MERGE_W_WAVES;

template <int B>
unsigned merge_grid(int64_t n, int resident)
{
    const int64_t nwords = (n * B + 31) >> 5;
    const int64_t per_block = (int64_t)kThreads * kMergeSlotsFor<B>;
    return grid_for((nwords + per_block - 1) / per_block, resident, kQsgdMergeWaves<B>);
}

unsigned group_grid(int64_t n, int resident)
{
    const int64_t groups = (n + 3) >> 2;
    const int64_t tiles = (groups + kTileGroups - 1) / kTileGroups;
    return grid_for((tiles + kWarpsPerBlock - 1) / kWarpsPerBlock, resident, kQsgdQuantizeWaves);
}

template <int B>
void launch_quantize(const float *grad, uint32_t *compr, int64_t n, uint64_t seed, const float *M,
                     cudaStream_t stream)
{
    const uint32_t k0 = (uint32_t)seed, k1 = (uint32_t)(seed >> 32);
    const int s = bits_slot(B);
    if (QGA_QSGD_LANE_WORDS && aligned(grad, 32)) {
        auto k = qsgd_quantize_words_kernel<B>;
        const int64_t runs = (n + 16 * kWarp - 1) / (16 * kWarp);
        k<<<grid_for((runs + kWarpsPerBlock - 1) / kWarpsPerBlock, resident_blocks(k, kThreads, occ_qw[s]),
                     kQsgdQuantizeWaves),
            kThreads, 0, stream>>>(grad, compr, n, k0, k1, M);
    } else if (aligned(grad, 16)) {
        auto k = qsgd_quantize_kernel<B, true>;
        k<<<group_grid(n, resident_blocks(k, kThreads, occ_q[s][0])), kThreads, 0, stream>>>(
            grad, compr, n, k0, k1, M);
    } else {
        auto k = qsgd_quantize_kernel<B, false>;
        k<<<group_grid(n, resident_blocks(k, kThreads, occ_q[s][1])), kThreads, 0, stream>>>(
            grad, compr, n, k0, k1, M);
    }
}

template <int B, bool kVec, int kW, bool kPad = false>
void launch_merge_w(const RecordSet &set, int W, float *out, int64_t n, cudaStream_t stream)
{
    auto k = qsgd_merge_w_kernel<B, kVec, kW, kPad>;
    const int64_t nwords = (n * B + 31) >> 5;
    const int64_t per_block = (int64_t)kThreads * kMergeWSlots;
    k<<<grid_for((nwords + per_block - 1) / per_block, resident_blocks(k, kThreads, occ_mw[bits_slot(B)][kVec][kW]),
                 kQsgdMergeWWaves),
        kThreads, 0, stream>>>(set, W, out, n);
}

template <int B, bool kVec>
void launch_merge_w(const RecordSet &set, int W, float *out, int64_t n, cudaStream_t stream)
{
    switch (W) {
    case 1: launch_merge_w<B, kVec, 1>(set, W, out, n, stream); break;
    case 2: launch_merge_w<B, kVec, 2>(set, W, out, n, stream); break;
    case 3: launch_merge_w<B, kVec, 3>(set, W, out, n, stream); break;
    case 4: launch_merge_w<B, kVec, 4>(set, W, out, n, stream); break;
    case 5: launch_merge_w<B, kVec, 5>(set, W, out, n, stream); break;
    case 6: launch_merge_w<B, kVec, 6>(set, W, out, n, stream); break;
    case 7: launch_merge_w<B, kVec, 7>(set, W, out, n, stream); break;
    case 8: launch_merge_w<B, kVec, 8>(set, W, out, n, stream); break;
    default: launch_merge_w<B, kVec, 16, true>(set, W, out, n, stream); break; // 9 .. 16
    }
}

template <int B>
void launch_merge(const RecordSet &set, int W, float *out, int64_t n, cudaStream_t stream)
{
    const int s = bits_slot(B);
    if (W <= 16) {
        if (aligned(out, 32))
            launch_merge_w<B, true>(set, W, out, n, stream);
        else
            launch_merge_w<B, false>(set, W, out, n, stream);
        return;
    }
    if (aligned(out, 32)) {
        auto k = qsgd_merge_kernel<B, true>;
        k<<<merge_grid<B>(n, resident_blocks(k, kThreads, occ_m[s][0])), kThreads, 0, stream>>>(
            set, W, out, n);
    } else {
        auto k = qsgd_merge_kernel<B, false>;
        k<<<merge_grid<B>(n, resident_blocks(k, kThreads, occ_m[s][1])), kThreads, 0, stream>>>(
            set, W, out, n);
    }
}

} // namespace
} // namespace qga

using namespace qga;

extern "C" int64_t qga_qsgd_words(int64_t n, int bits)
{
    if (n < 0 || bits_slot(bits) < 0)
        return n < 0 ? QGA_ERR_INVALID_ARG : QGA_ERR_UNSUPPORTED;
    return 3 + (n * bits + 31) / 32;
}

extern "C" int qga_qsgd_mn_max(const float *const *grad, int num_workers, int64_t n,
                               float *max_out, cudaStream_t stream)
{
    if (grad == nullptr || num_workers < 1 || num_workers > QGA_MAX_WORKERS || n < 0 ||
        max_out == nullptr || !aligned(max_out, 4))
        return QGA_ERR_INVALID_ARG;
    GradSet set{};
    for (int w = 0; w < num_workers; ++w) {
        if (n > 0 && (grad[w] == nullptr || !aligned(grad[w], 4)))
            return QGA_ERR_INVALID_ARG;
        set.g[w] = grad[w];
    }
    int st = cuda_status(cudaMemsetAsync(max_out, 0, sizeof(float), stream));
    if (st != QGA_OK || n == 0)
        return st;
    const int64_t groups = (n + 3) >> 2;
    const int resident = resident_blocks(qsgd_max_kernel, kThreads, occ_max);
    qsgd_max_kernel<<<grid_for((groups + kThreads - 1) / kThreads, resident), kThreads, 0, stream>>>(
        set, num_workers, n, max_out);
    return launch_status();
}

extern "C" int qga_qsgd_mn_quantize(const float *grad, uint32_t *compr, int64_t n, int bits,
                                    uint64_t seed, const float *max_in, cudaStream_t stream)
{
    if (n < 0 || compr == nullptr || !aligned(compr, 4) || max_in == nullptr || !aligned(max_in, 4))
        return QGA_ERR_INVALID_ARG;
    if (n > 0 && (grad == nullptr || !aligned(grad, 4)))
        return QGA_ERR_INVALID_ARG;
    switch (bits) {
    case 2: launch_quantize<2>(grad, compr, n, seed, max_in, stream); break;
    case 4: launch_quantize<4>(grad, compr, n, seed, max_in, stream); break;
    case 8: launch_quantize<8>(grad, compr, n, seed, max_in, stream); break;
    default: return QGA_ERR_UNSUPPORTED;
    }
    return launch_status();
}

extern "C" int qga_qsgd_mn_dequant_accumulate(const uint32_t *const *compr, int num_workers,
                                              float *out, int64_t n, int bits, cudaStream_t stream)
{
    if (compr == nullptr || num_workers < 1 || num_workers > QGA_MAX_WORKERS || n < 0)
        return QGA_ERR_INVALID_ARG;
    if (bits_slot(bits) < 0)
        return QGA_ERR_UNSUPPORTED;
    RecordSet set{};
    for (int w = 0; w < num_workers; ++w) {
        if (compr[w] == nullptr || !aligned(compr[w], 4))
            return QGA_ERR_INVALID_ARG;
        set.rec[w] = compr[w];
    }
    if (n == 0)
        return QGA_OK;
    if (out == nullptr || !aligned(out, 4))
        return QGA_ERR_INVALID_ARG;
    switch (bits) {
    case 2: launch_merge<2>(set, num_workers, out, n, stream); break;
    case 4: launch_merge<4>(set, num_workers, out, n, stream); break;
    default: launch_merge<8>(set, num_workers, out, n, stream); break;
    }
    return launch_status();
}
