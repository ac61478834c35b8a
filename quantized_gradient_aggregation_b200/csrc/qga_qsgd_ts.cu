// qga_qsgd_ts.cu -- QSGD-MaxNorm with two scales (QSGD-MN-TS): quantize and
// merge.  The global max is the one-scale max (qga_qsgd_mn_max).
//
// The gradient-compression README (vineeths96), "Results", names
// QSGDMaxNormMultiScale quantization run with two scales, each run labelled
// with the bit widths of its two scales, and "About The Project" counts it
// among the all-reduce compatible schemes; no formula is printed.  This
// library's definition:
//   coarse scale M1 = M (global max |g|), b1 bits, s1 = 2^(b1-1) - 1 levels;
//   fine scale   M2 = fl(M1 / s1) (the coarse grid's first step), b2 bits,
//                s2 = 2^(b2-1) - 1 levels;
//   an element with |g| <= M2 is quantized on the fine scale, any other on
//   the coarse one, each by the QSGD-MaxNorm level of that scale (the draw of
//   the element, Philox4x32-10 as in qga_qsgd.cu); its level on the other
//   scale is 0;
//   record = the coarse levels as a QSGD-MaxNorm record of b1 bits (header
//   [M1, b1, n]) followed by the fine levels as one of b2 bits (header [M2,
//   b2, n]);
//   merge: out = fl(fl((sum_w q1) fl(M1 / s1)) + fl((sum_w q2) fl(M2 / s2))),
//   both level sums exact in integers, so an all-reduce could form them.
//
// Quantize: the one-scale kernel's tile geometry (a warp owns 128 groups of
// 4 elements, lane l groups l, l+32, l+64, l+96; one Philox block per group),
// the fixed-point level of qga_qsgd_level.cuh with E = max(b1, b2) - 1 and
// the scale picked per element, and two packed outputs.  Merge: each scale's
// levels summed over the workers in SIMD lanes of registers (LevelSum)
// in that sub-record's own coalesced layout, converted and scaled once, and
// the two parts added in shared memory (see qsgd_ts_merge_kernel).

#include <float.h>

#include "qga_common.cuh"
#include "qga_qsgd_level.cuh"

namespace qga {
namespace {

constexpr int kThreads = 256;
constexpr int kWarpsPerBlock = kThreads / kWarp;
constexpr int kGroupsPerLane = 4;
constexpr int kTileGroups = kWarp * kGroupsPerLane;

struct RecordSet {
    const uint32_t *rec[QGA_MAX_WORKERS];
};

__host__ __device__ constexpr int64_t sub_words(int64_t n, int b) { return 3 + (n * b + 31) / 32; }

// Packs the 4 codes of group gi (piece: first element in the top b bits of
// its 4b bits) into word gi / (8 / b) of a payload; lanes sharing a word
// combine with xor-shuffles.  All 32 lanes call this together.
template <int B>
__device__ __forceinline__ void store_piece(uint32_t *__restrict__ payload, uint32_t piece, int64_t gi,
                                            int64_t n, int64_t nwords, int lane)
{
    const int64_t valid = n - 4 * gi; // codes of elements >= n are zero
    if (valid < 4)
        piece = valid <= 0 ? 0u : (piece & ~((1u << (B * (4 - (int)valid))) - 1u));
    constexpr int LW = Levels<B>::lanes_per_word;
    uint32_t word = piece << (32 - 4 * B * (1 + (lane % LW)));
    if (LW >= 2)
        word |= __shfl_xor_sync(kFullMask, word, 1);
    if (LW >= 4)
        word |= __shfl_xor_sync(kFullMask, word, 2);
    const int64_t wi = gi / LW;
    if ((lane % LW) == 0 && wi < nwords)
        st_stream_u32(payload + wi, word);
}

template <int B1, int B2, bool kVec>
__global__ void __launch_bounds__(kThreads)
    qsgd_ts_quantize_kernel(const float *__restrict__ grad, uint32_t *__restrict__ compr, int64_t n,
                            uint32_t key0, uint32_t key1, const float *__restrict__ max_in)
{
    using L1 = Levels<B1>;
    using L2 = Levels<B2>;
    constexpr int E = (B1 > B2 ? B1 : B2) - 1;
    using Fx = FixLevel<E>;
    const float M1 = *max_in;
    const float M2 = __fdiv_rn(M1, (float)L1::s);
    // fast path for a finite positive M1 whose fine scale is positive too
    const bool fast = M2 > 0.0f && M1 <= FLT_MAX; // uniform over the grid
    const float k1 = __fdiv_rn((float)L1::s, M1);
    const float k2 = __fdiv_rn((float)L2::s, M2);
    uint32_t *coarse = compr;
    uint32_t *fine = compr + sub_words(n, B1);
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        coarse[0] = bits_from_f32(M1);
        coarse[1] = bits_from_f32((float)B1);
        coarse[2] = bits_from_f32(__ll2float_rn(n));
        fine[0] = bits_from_f32(M2);
        fine[1] = bits_from_f32((float)B2);
        fine[2] = bits_from_f32(__ll2float_rn(n));
    }
    const int lane = threadIdx.x & (kWarp - 1);
    const int64_t full_groups = n >> 2;
    const int64_t groups = (n + 3) >> 2;
    const int64_t nwords1 = (n * B1 + 31) >> 5, nwords2 = (n * B2 + 31) >> 5;
    const int64_t tiles = (groups + kTileGroups - 1) / kTileGroups;
    const int64_t stride = (int64_t)gridDim.x * kWarpsPerBlock;
    for (int64_t tile = (int64_t)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5); tile < tiles;
         tile += stride) {
        const int64_t g0 = tile * kTileGroups;
        float gv[kGroupsPerLane][4];
#pragma unroll
        for (int j = 0; j < kGroupsPerLane; ++j) {
            const int64_t gi = g0 + j * kWarp + lane;
            if (kVec && gi < full_groups) {
                const float4 v = ld_stream_f4(grad + 4 * gi);
                gv[j][0] = v.x, gv[j][1] = v.y, gv[j][2] = v.z, gv[j][3] = v.w;
            } else {
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    gv[j][q] = (4 * gi + q < n) ? ld_stream_f1(grad + 4 * gi + q) : 0.0f;
            }
        }
        uint4 draws[kGroupsPerLane];
#pragma unroll
        for (int j = 0; j < kGroupsPerLane; ++j) {
            const int64_t gi = g0 + j * kWarp + lane;
            draws[j] = philox4x32_10(make_uint4((uint32_t)gi, (uint32_t)((uint64_t)gi >> 32), 0u, 0u),
                                     key0, key1);
        }
        uint32_t p1[kGroupsPerLane], p2[kGroupsPerLane];
        uint32_t fmin, xmax;
        Fx::reset(fmin, xmax);
#pragma unroll
        for (int j = 0; j < kGroupsPerLane; ++j) {
            const uint32_t x[4] = {draws[j].x, draws[j].y, draws[j].z, draws[j].w};
            p1[j] = p2[j] = 0u;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const bool is_fine = fabsf(gv[j][q]) <= M2;
                const int32_t lv = qsgd_level_fixed<E>(gv[j][q], is_fine ? k2 : k1,
                                                       is_fine ? (uint32_t)L2::s : (uint32_t)L1::s, x[q],
                                                       fmin, xmax);
                p1[j] |= (is_fine ? 0u : ((uint32_t)lv & L1::mask)) << (B1 * (3 - q));
                p2[j] |= (is_fine ? ((uint32_t)lv & L2::mask) : 0u) << (B2 * (3 - q));
            }
        }
        if (!fast || Fx::needs_exact(fmin, xmax)) {
            // rare: this lane's elements by the definition's operations
#pragma unroll
            for (int j = 0; j < kGroupsPerLane; ++j) {
                const uint32_t x[4] = {draws[j].x, draws[j].y, draws[j].z, draws[j].w};
                p1[j] = p2[j] = 0u;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float u = unit_draw(x[q]);
                    if (fabsf(gv[j][q]) <= M2)
                        p2[j] |= ((uint32_t)qsgd_level_exact<B2>(gv[j][q], M2, u) & L2::mask) << (B2 * (3 - q));
                    else
                        p1[j] |= ((uint32_t)qsgd_level_exact<B1>(gv[j][q], M1, u) & L1::mask) << (B1 * (3 - q));
                }
            }
        }
#pragma unroll
        for (int j = 0; j < kGroupsPerLane; ++j) {
            const int64_t gi = g0 + j * kWarp + lane;
            store_piece<B1>(coarse + 3, p1[j], gi, n, nwords1, lane);
            store_piece<B2>(fine + 3, p2[j], gi, n, nwords2, lane);
        }
    }
}

// The quantize in lane-owned words, for a 32-byte-aligned gradient: lane l
// of warp t owns the 16 consecutive elements 16 (32 t + l) .. + 15 (two
// 256-bit loads, the 4 Philox blocks of its 4 groups) and packs their codes
// into its b1 / 2 coarse and b2 / 2 fine record words in registers (no
// shuffles, one check per lane).  The level: X = fl(|g| k + 2^E) in one
// fused multiply-add with the element's scale, then as in
// qsgd_level_fixed (cap at the scale's s; fall back when any fraction of
// T + 8 is below 16 units or X >= 2^(E+1)).
template <int B1, int B2>
__global__ void __launch_bounds__(kThreads)
    qsgd_ts_quantize_words_kernel(const float *__restrict__ grad, uint32_t *__restrict__ compr, int64_t n,
                                  uint32_t key0, uint32_t key1, const float *__restrict__ max_in)
{
    using L1 = Levels<B1>;
    using L2 = Levels<B2>;
    constexpr int E = (B1 > B2 ? B1 : B2) - 1;
    constexpr int F = 23 - E;
    constexpr uint32_t kOne = (127u + E) << 23, kTwo = (128u + E) << 23;
    constexpr int kWords1 = B1 / 2, kWords2 = B2 / 2, kPer1 = 32 / B1, kPer2 = 32 / B2;
    const float M1 = *max_in;
    const float M2 = __fdiv_rn(M1, (float)L1::s);
    const bool fast = M2 > 0.0f && M1 <= FLT_MAX; // uniform over the grid
    const float k1 = __fdiv_rn((float)L1::s, M1);
    const float k2 = __fdiv_rn((float)L2::s, M2);
    uint32_t *coarse = compr;
    uint32_t *fine = compr + sub_words(n, B1);
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        coarse[0] = bits_from_f32(M1);
        coarse[1] = bits_from_f32((float)B1);
        coarse[2] = bits_from_f32(__ll2float_rn(n));
        fine[0] = bits_from_f32(M2);
        fine[1] = bits_from_f32((float)B2);
        fine[2] = bits_from_f32(__ll2float_rn(n));
    }
    const int lane = threadIdx.x & (kWarp - 1);
    const int64_t nwords1 = (n * B1 + 31) >> 5, nwords2 = (n * B2 + 31) >> 5;
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
        uint32_t w1[kWords1] = {}, w2[kWords2] = {};
        uint32_t fmin = 0xFFFFFFFFu, xmax = 0u;
#pragma unroll
        for (int p = 0; p < 16; ++p) {
            const bool is_fine = fabsf(g[p]) <= M2;
            const uint32_t xb = __float_as_uint(__fmaf_rn(fabsf(g[p]), is_fine ? k2 : k1, (float)(1 << E)));
            const uint32_t t8 = xb + (x[p] >> (32 - F)) + (8u - kOne);
            fmin = min(fmin, t8 << (32 - F));
            xmax = max(xmax, xb);
            const uint32_t lv = min(t8 >> F, is_fine ? (uint32_t)L2::s : (uint32_t)L1::s);
            const int32_t q = (int32_t)lv * (((int32_t)__float_as_uint(g[p]) >> 31) * 2 + 1);
            w1[p / kPer1] |= (is_fine ? 0u : ((uint32_t)q & L1::mask)) << (32 - B1 * (p % kPer1 + 1));
            w2[p / kPer2] |= (is_fine ? ((uint32_t)q & L2::mask) : 0u) << (32 - B2 * (p % kPer2 + 1));
        }
        if (!fast || fmin < (16u << (32 - F)) || xmax >= kTwo) {
#pragma unroll
            for (int i = 0; i < kWords1; ++i)
                w1[i] = 0u;
#pragma unroll
            for (int i = 0; i < kWords2; ++i)
                w2[i] = 0u;
#pragma unroll
            for (int p = 0; p < 16; ++p) {
                const float u = unit_draw(x[p]);
                if (fabsf(g[p]) <= M2)
                    w2[p / kPer2] |= ((uint32_t)qsgd_level_exact<B2>(g[p], M2, u) & L2::mask)
                                     << (32 - B2 * (p % kPer2 + 1));
                else
                    w1[p / kPer1] |= ((uint32_t)qsgd_level_exact<B1>(g[p], M1, u) & L1::mask)
                                     << (32 - B1 * (p % kPer1 + 1));
            }
        }
        // elements past n loaded as 0 have level 0 on the fine scale and code 0
#pragma unroll
        for (int i = 0; i < kWords1; ++i)
            if (r * kWords1 + i < nwords1)
                st_stream_u32(coarse + 3 + r * kWords1 + i, w1[i]);
#pragma unroll
        for (int i = 0; i < kWords2; ++i)
            if (r * kWords2 + i < nwords2)
                st_stream_u32(fine + 3 + r * kWords2 + i, w2[i]);
    }
}

// ----------------------------------------------------------------- merge ----
// A warp owns chunks of 512 elements.  Each sub-record is summed in its own
// coalesced layout: the chunk's 16 b words, lane l owning words l, 32 + l,
// ... (b / 2 of them), the levels of all workers added in SIMD lanes of
// registers (LevelSum); each element's sum is converted exactly,
// scaled once by that scale's step and written to the warp's 2 KB of shared
// memory (the coarse part), or added there to the coarse part (the fine
// part).  The 512 results then leave as coalesced 128-bit rows.
constexpr int kChunk = 512;

// One scale's part of a chunk: this lane's words c * 32 + lane (c < b / 2)
// of the chunk's 16 b words, summed over the workers in SIMD lanes of
// registers, converted exactly, scaled once by the scale's step and stored
// to sv (the coarse part) or added to the value there (kAdd, the fine part).
// Word c * 32 + lane holds the elements (c * 32 + lane) * 32 / b ...
#ifndef QGA_TS_MERGE_BATCH
#define QGA_TS_MERGE_BATCH 4
#endif

// Shared-memory slot of group g (4 elements) of a chunk.  A lane writes the
// kFields / 4 consecutive groups of its word, so at b = 2 (b = 4) the lanes
// of a quarter-warp are 4 (2) groups apart and meet in the same banks.  With
// kSwizzle the XOR with bits 3..5 of g spreads them over all 8 slots of a
// 128-byte row for b = 2, 4 and 8 alike, and keeps the 8 consecutive groups
// of a coalesced output row in one row of 8 slots.  Measured at 2^27
// (plain / swizzled, us): (2, 4) W = 1 172 / 123, W = 2 184 / 142, W = 4
// 181 / 172, W = 6 204 / 211, W = 8 226 / 234; (4, 8) W = 1 128 / 142, W = 4
// 231 / 222, W = 8 354 / 356.  So the swizzle is used where a part has b = 2
// and the worker count is at most 4.
template <bool kSwizzle>
__device__ __forceinline__ int group_slot(int g) { return kSwizzle ? g ^ ((g >> 3) & 7) : g; }

template <int B, bool kAdd, int kW, bool kSwizzle>
__device__ __forceinline__ void chunk_part(const RecordSet &set, int W, int64_t payload_off, int64_t chunk,
                                           int64_t nwords, int lane, float step, float bias,
                                           float *__restrict__ sv)
{
    using S = LevelSum<B>;
    constexpr int kWords = B / 2;
    constexpr int kBatch = kW > 0 ? kW : QGA_TS_MERGE_BATCH;
    static_assert(kBatch <= LevelSum<B>::kBatchMax, "a batch fits the narrow lanes");
    if (kW > 0)
        W = kW;
    LevelSum<B> acc[kWords];
    for (int wb = 0; wb < W; wb += kBatch) {
        uint32_t words[kBatch][kWords];
#pragma unroll
        for (int i = 0; i < kBatch; ++i)
#pragma unroll
            for (int c = 0; c < kWords; ++c) {
                const int64_t k = chunk * (16 * B) + c * kWarp + lane;
                words[i][c] = (wb + i < W && k < nwords) ? ld_stream_u32(set.rec[wb + i] + payload_off + k)
                                                         : S::kSign; // the biased 0 of an absent level
            }
#pragma unroll
        for (int i = 0; i < kBatch; ++i) {
            if (wb + i >= W) // warp-uniform
                break;
#pragma unroll
            for (int c = 0; c < kWords; ++c)
                acc[c].add(words[i][c]);
        }
#pragma unroll
        for (int c = 0; c < kWords; ++c)
            acc[c].end_batch();
    }
#pragma unroll
    for (int c = 0; c < kWords; ++c) {
        acc[c].finish();
        float v[S::kFields];
#pragma unroll
        for (int e = 0; e < S::kFields; ++e)
            v[e] = __fmul_rn(__fsub_rn(__uint_as_float(0x4B000000u | acc[c].field_sum(e)), bias), step);
        float4 *sv4 = reinterpret_cast<float4 *>(sv);
#pragma unroll
        for (int q = 0; q < S::kFields / 4; ++q) {
            const int slot = group_slot<kSwizzle>((c * kWarp + lane) * (S::kFields / 4) + q);
            float4 x = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
            if (kAdd) {
                const float4 a = sv4[slot];
                x = make_float4(__fadd_rn(a.x, x.x), __fadd_rn(a.y, x.y), __fadd_rn(a.z, x.z), __fadd_rn(a.w, x.w));
            }
            sv4[slot] = x;
        }
    }
}

template <int B1, int B2, bool kVec, int kW>
__global__ void __launch_bounds__(kThreads)
    qsgd_ts_merge_kernel(const __grid_constant__ RecordSet set, int W, float *__restrict__ out, int64_t n)
{
    if (kW > 0)
        W = kW;
    constexpr bool kSwizzle = (B1 == 2 || B2 == 2) && kW >= 1 && kW <= 4;
    __shared__ __align__(16) float s_vals[kWarpsPerBlock][kChunk];
    const int64_t off2 = sub_words(n, B1) + 3; // payload of the fine sub-record
    const float step1 = __fdiv_rn(f32_from_bits(set.rec[0][0]), (float)Levels<B1>::s);
    const float step2 = __fdiv_rn(f32_from_bits(set.rec[0][off2 - 3]), (float)Levels<B2>::s);
    // 2^23 + W 2^(b-1): the exact conversion's offset and the bias
    const float bias1 = 8388608.0f + (float)(W << (B1 - 1));
    const float bias2 = 8388608.0f + (float)(W << (B2 - 1));
    const int64_t nwords1 = (n * B1 + 31) >> 5, nwords2 = (n * B2 + 31) >> 5;
    const int lane = threadIdx.x & (kWarp - 1);
    float *sv = s_vals[threadIdx.x >> 5];
    const float4 *sv4 = reinterpret_cast<const float4 *>(sv);
    const int64_t chunks = (n + kChunk - 1) / kChunk;
    for (int64_t ch = (int64_t)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5); ch < chunks;
         ch += (int64_t)gridDim.x * kWarpsPerBlock) {
        chunk_part<B1, false, kW, kSwizzle>(set, W, 3, ch, nwords1, lane, step1, bias1, sv);
        __syncwarp();
        chunk_part<B2, true, kW, kSwizzle>(set, W, off2, ch, nwords2, lane, step2, bias2, sv);
        __syncwarp();
#pragma unroll
        for (int j = 0; j < kChunk / 4 / kWarp; ++j) {
            const int q = j * kWarp + lane; // group of 4 within the chunk
            const int64_t gi = ch * (kChunk / 4) + q;
            const float4 x = sv4[group_slot<kSwizzle>(q)];
            if (kVec && gi < (n >> 2)) {
                st_stream_f4(out + 4 * gi, x);
            } else {
                const float xx[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    if (4 * gi + e < n)
                        st_stream_f1(out + 4 * gi + e, xx[e]);
            }
        }
        __syncwarp();
    }
}

int bits_slot(int bits) { return bits == 2 ? 0 : (bits == 4 ? 1 : (bits == 8 ? 2 : -1)); }

std::atomic<int> occ_tq[3][3][2][64];
std::atomic<int> occ_tw[3][3][64];
#ifndef QGA_TS_LANE_WORDS
#define QGA_TS_LANE_WORDS 1
#endif
std::atomic<int> occ_tm[3][3][2][64];

#ifndef QGA_TS_MERGE_WAVES
#define QGA_TS_MERGE_WAVES 8
#endif
#ifndef QGA_TS_QUANTIZE_WAVES
#define QGA_TS_QUANTIZE_WAVES 8
#endif
constexpr int kTsQuantizeWaves = QGA_TS_QUANTIZE_WAVES, kTsMergeWaves = QGA_TS_MERGE_WAVES;

template <int B1, int B2>
void launch_quantize(const float *grad, uint32_t *compr, int64_t n, uint64_t seed, const float *M,
                     cudaStream_t stream)
{
    const uint32_t k0 = (uint32_t)seed, k1 = (uint32_t)(seed >> 32);
    const int64_t groups = (n + 3) >> 2;
    const int64_t tiles = (groups + kTileGroups - 1) / kTileGroups;
    const int64_t blocks = (tiles + kWarpsPerBlock - 1) / kWarpsPerBlock;
    auto &occ = occ_tq[bits_slot(B1)][bits_slot(B2)];
    if (QGA_TS_LANE_WORDS && aligned(grad, 32)) {
        auto k = qsgd_ts_quantize_words_kernel<B1, B2>;
        const int64_t runs = (n + 16 * kWarp - 1) / (16 * kWarp);
        k<<<grid_for((runs + kWarpsPerBlock - 1) / kWarpsPerBlock, resident_blocks(k, kThreads, occ_tw[bits_slot(B1)][bits_slot(B2)]),
                     kTsQuantizeWaves),
            kThreads, 0, stream>>>(grad, compr, n, k0, k1, M);
    } else if (aligned(grad, 16)) {
        auto k = qsgd_ts_quantize_kernel<B1, B2, true>;
        k<<<grid_for(blocks, resident_blocks(k, kThreads, occ[0]), kTsQuantizeWaves), kThreads, 0,
            stream>>>(grad, compr, n, k0, k1, M);
    } else {
        auto k = qsgd_ts_quantize_kernel<B1, B2, false>;
        k<<<grid_for(blocks, resident_blocks(k, kThreads, occ[1]), kTsQuantizeWaves), kThreads, 0,
            stream>>>(grad, compr, n, k0, k1, M);
    }
}

// W <= 8 with an aligned output: the worker count as a template argument
// (all W workers' words of a part loaded at once, payload pointers from the
// parameter space).  Measured at n = 2^27, W = 8: (4, 8) 354 us, (2, 4) 226
// us, (8, 2) 324 us, against 433 / 258 / 439 us with the runtime count.
std::atomic<int> occ_tmw[3][3][9][64]; // [b1][b2][W][device]

template <int B1, int B2, int kW>
void launch_merge_w(const RecordSet &set, float *out, int64_t n, int64_t blocks, cudaStream_t stream)
{
    auto k = qsgd_ts_merge_kernel<B1, B2, true, kW>;
    k<<<grid_for(blocks, resident_blocks(k, kThreads, occ_tmw[bits_slot(B1)][bits_slot(B2)][kW]), kTsMergeWaves),
        kThreads, 0, stream>>>(set, kW, out, n);
}

template <int B1, int B2>
void launch_merge(const RecordSet &set, int W, float *out, int64_t n, cudaStream_t stream)
{
    const int64_t chunks = (n + kChunk - 1) / kChunk;
    const int64_t blocks = (chunks + kWarpsPerBlock - 1) / kWarpsPerBlock;
    auto &occ = occ_tm[bits_slot(B1)][bits_slot(B2)];
    if (W <= 8 && aligned(out, 16)) {
        switch (W) {
        case 1: launch_merge_w<B1, B2, 1>(set, out, n, blocks, stream); break;
        case 2: launch_merge_w<B1, B2, 2>(set, out, n, blocks, stream); break;
        case 3: launch_merge_w<B1, B2, 3>(set, out, n, blocks, stream); break;
        case 4: launch_merge_w<B1, B2, 4>(set, out, n, blocks, stream); break;
        case 5: launch_merge_w<B1, B2, 5>(set, out, n, blocks, stream); break;
        case 6: launch_merge_w<B1, B2, 6>(set, out, n, blocks, stream); break;
        case 7: launch_merge_w<B1, B2, 7>(set, out, n, blocks, stream); break;
        default: launch_merge_w<B1, B2, 8>(set, out, n, blocks, stream); break;
        }
        return;
    }
    if (aligned(out, 16)) {
        auto k = qsgd_ts_merge_kernel<B1, B2, true, 0>;
        k<<<grid_for(blocks, resident_blocks(k, kThreads, occ[0]), kTsMergeWaves), kThreads, 0,
            stream>>>(set, W, out, n);
    } else {
        auto k = qsgd_ts_merge_kernel<B1, B2, false, 0>;
        k<<<grid_for(blocks, resident_blocks(k, kThreads, occ[1]), kTsMergeWaves), kThreads, 0,
            stream>>>(set, W, out, n);
    }
}

// The (b1, b2) pair as template arguments (every width 2, 4 or 8; checked
// by the caller).
#define QGA_TS_DISPATCH(b1, b2, CALL)                                                      \
    do {                                                                                   \
        const int p_ = (b1) * 16 + (b2);                                                   \
        if (p_ == 0x22) { constexpr int B1 = 2, B2 = 2; CALL; }                            \
        else if (p_ == 0x24) { constexpr int B1 = 2, B2 = 4; CALL; }                       \
        else if (p_ == 0x28) { constexpr int B1 = 2, B2 = 8; CALL; }                       \
        else if (p_ == 0x42) { constexpr int B1 = 4, B2 = 2; CALL; }                       \
        else if (p_ == 0x44) { constexpr int B1 = 4, B2 = 4; CALL; }                       \
        else if (p_ == 0x48) { constexpr int B1 = 4, B2 = 8; CALL; }                       \
        else if (p_ == 0x82) { constexpr int B1 = 8, B2 = 2; CALL; }                       \
        else if (p_ == 0x84) { constexpr int B1 = 8, B2 = 4; CALL; }                       \
        else { constexpr int B1 = 8, B2 = 8; CALL; }                                       \
    } while (0)

} // namespace
} // namespace qga

using namespace qga;

extern "C" int64_t qga_qsgd_mnts_words(int64_t n, int bits_coarse, int bits_fine)
{
    if (n < 0)
        return QGA_ERR_INVALID_ARG;
    if (bits_slot(bits_coarse) < 0 || bits_slot(bits_fine) < 0)
        return QGA_ERR_UNSUPPORTED;
    return sub_words(n, bits_coarse) + sub_words(n, bits_fine);
}

extern "C" int qga_qsgd_mnts_quantize(const float *grad, uint32_t *compr, int64_t n, int bits_coarse,
                                      int bits_fine, uint64_t seed, const float *max_in,
                                      cudaStream_t stream)
{
    if (n < 0 || compr == nullptr || !aligned(compr, 4) || max_in == nullptr || !aligned(max_in, 4))
        return QGA_ERR_INVALID_ARG;
    if (n > 0 && (grad == nullptr || !aligned(grad, 4)))
        return QGA_ERR_INVALID_ARG;
    if (bits_slot(bits_coarse) < 0 || bits_slot(bits_fine) < 0)
        return QGA_ERR_UNSUPPORTED;
    QGA_TS_DISPATCH(bits_coarse, bits_fine, (launch_quantize<B1, B2>(grad, compr, n, seed, max_in, stream)));
    return launch_status();
}

extern "C" int qga_qsgd_mnts_dequant_accumulate(const uint32_t *const *compr, int num_workers, float *out,
                                                int64_t n, int bits_coarse, int bits_fine,
                                                cudaStream_t stream)
{
    if (compr == nullptr || num_workers < 1 || num_workers > QGA_MAX_WORKERS || n < 0)
        return QGA_ERR_INVALID_ARG;
    if (bits_slot(bits_coarse) < 0 || bits_slot(bits_fine) < 0)
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
    QGA_TS_DISPATCH(bits_coarse, bits_fine, (launch_merge<B1, B2>(set, num_workers, out, n, stream)));
    return launch_status();
}
