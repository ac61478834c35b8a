// qga_ternary.cu -- dense ternary records of the 2-bit threshold codes:
// quantize (fp32 gradient), dequantize and the W-worker merge.
//
// MXNet pull request #8342 "[WIP] 2bit gradient compression", "Two bit
// quantization", notes that the three code values need fewer than two bits
// and leaves the wasted code for later.  This library's dense record keeps
// the same codes (00, 01, 10 -> trits 0, 1, 2) and the same error feedback,
// and packs five elements per byte as the base-3 numeral t0 t1 t2 t3 t4
// (element 0 most significant): payload byte j holds elements 5j..5j+4 and
// sits at byte 12 + j of the record, after the header [neg, pos, n]; four
// bytes (20 elements) fill one 32-bit word, and unused trits and padding
// bytes are zero.  Record: 3 + ceil(n / 20) words (0.2 bytes per element
// instead of 0.25).
//
// Quantize geometry: a warp owns a tile of 640 elements (160 groups of 4,
// five per lane, every load a coalesced 512-byte row) = 32 payload words.
// Each lane writes its groups' codes as bytes to a per-warp shared buffer;
// lane l then reads the 20 codes of word l (five conflict-free 32-bit
// loads: the stride of 5 words is odd) and forms each payload byte with one
// byte-wise dot product against the weights 81, 27, 9, 3 (plus the fifth
// code).  Decode geometry: a lane owns one payload word (20 elements); a
// 256-entry shared table turns each byte into its five 2-bit codes or into
// the bit masks of its codes 01 and 10, and the outputs leave through a
// shared stage (again stride 5, conflict-free) as coalesced 128-bit rows.

#include "qga_2bit_tiles.cuh"

namespace qga {
namespace {

constexpr int kThreads = 256;
constexpr int kWarpsPerBlock = kThreads / kWarp;
constexpr int kTGroups = 5;                             // groups of 4 per lane per tile
constexpr int kTTileElems = kWarp * kTGroups * 4;        // 640 elements = 32 words
constexpr uint32_t kWeights = 0x03091B51u;               // bytes 81, 27, 9, 3 (little endian)

__device__ __forceinline__ int64_t warp_id() { return (int64_t)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5); }
__device__ __forceinline__ int64_t warp_stride() { return (int64_t)gridDim.x * kWarpsPerBlock; }

// Payload word from 20 codes held one per byte in five 32-bit words (code of
// element 4i + k in byte k of c[i]).
__device__ __forceinline__ uint32_t pack_ternary_word(const uint32_t (&c)[5])
{
    uint32_t word = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        // codes 5k .. 5k+3 start at byte 5k: word 5k / 4, byte offset (5k) % 4 = k
        const int i = (5 * k) >> 2, o = k;
        const uint32_t four = o == 0 ? c[i] : __funnelshift_r(c[i], c[i + 1], 8 * o);
        const uint32_t fifth = (c[(5 * k + 4) >> 2] >> (8 * ((5 * k + 4) & 3))) & 0xFFu;
        word |= (uint32_t)__dp4a(four, kWeights, fifth) << (8 * k);
    }
    return word;
}

template <bool kVec>
__global__ void __launch_bounds__(kThreads)
    quantize_ternary_kernel(const float *__restrict__ grad, float *__restrict__ residual,
                            uint32_t *__restrict__ compr, int64_t n, float neg, float pos)
{
    __shared__ uint32_t s_codes[kWarpsPerBlock][kTTileElems / 4];
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        compr[0] = bits_from_f32(neg);
        compr[1] = bits_from_f32(pos);
        compr[2] = bits_from_f32(__ll2float_rn(n));
    }
    uint32_t *payload = compr + 3;
    uint32_t *codes = s_codes[threadIdx.x >> 5];
    const int lane = threadIdx.x & (kWarp - 1);
    const int64_t full_groups = n >> 2;
    const int64_t nwords = (n + 19) / 20;
    const int64_t tiles = (n + kTTileElems - 1) / kTTileElems;
    for (int64_t t = warp_id(); t < tiles; t += warp_stride()) {
        const int64_t g0 = t * (kWarp * kTGroups);
        float4 gv[kTGroups], rv[kTGroups];
#pragma unroll
        for (int j = 0; j < kTGroups; ++j) {
            const int64_t gi = g0 + j * kWarp + lane;
            if (kVec && gi < full_groups) {
                gv[j] = ld_stream_f4(grad + 4 * gi);
                rv[j] = ld_stream_f4(residual + 4 * gi);
            } else {
                float tg[4], tr[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int64_t e = 4 * gi + k;
                    tg[k] = e < n ? ld_stream_f1(grad + e) : 0.0f;
                    tr[k] = e < n ? ld_stream_f1(residual + e) : 0.0f;
                }
                gv[j] = make_float4(tg[0], tg[1], tg[2], tg[3]);
                rv[j] = make_float4(tr[0], tr[1], tr[2], tr[3]);
            }
        }
#pragma unroll
        for (int j = 0; j < kTGroups; ++j) {
            const int64_t gi = g0 + j * kWarp + lane;
            float4 r = rv[j];
            uint32_t c0 = tb_step(gv[j].x, r.x, neg, pos);
            uint32_t c1 = tb_step(gv[j].y, r.y, neg, pos);
            uint32_t c2 = tb_step(gv[j].z, r.z, neg, pos);
            uint32_t c3 = tb_step(gv[j].w, r.w, neg, pos);
            if (kVec && gi < full_groups) {
                st_stream_f4(residual + 4 * gi, r);
            } else {
                const int64_t valid = n - 4 * gi;
                const float rr[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    if (k < valid)
                        st_stream_f1(residual + 4 * gi + k, rr[k]);
                c0 = valid > 0 ? c0 : 0u;
                c1 = valid > 1 ? c1 : 0u;
                c2 = valid > 2 ? c2 : 0u;
                c3 = valid > 3 ? c3 : 0u;
            }
            codes[j * kWarp + lane] = c0 | (c1 << 8) | (c2 << 16) | (c3 << 24);
        }
        __syncwarp();
        uint32_t c[5];
#pragma unroll
        for (int i = 0; i < 5; ++i)
            c[i] = codes[5 * lane + i];
        const int64_t w = t * kWarp + lane;
        if (w < nwords)
            st_stream_u32(payload + w, pack_ternary_word(c));
        __syncwarp();
    }
}

// Byte -> (mask of its codes 01 in bits 4..0, mask of its codes 10 in bits
// 9..5), element 5j + i of the byte at bit 4 - i; and byte -> its five 2-bit
// codes, element 5j + i in bits 9 - 2i .. 8 - 2i.  Digits are taken mod 3
// (bytes above 242 never occur in a record).
__device__ __forceinline__ void build_byte_tables(uint16_t *masks, uint16_t *codes)
{
    for (int b = threadIdx.x; b < 256; b += blockDim.x) {
        uint32_t v = (uint32_t)b, m01 = 0, m10 = 0, c = 0;
#pragma unroll
        for (int i = 4; i >= 0; --i) {
            const uint32_t d = v % 3u;
            v /= 3u;
            m01 |= (d == 1u ? 1u : 0u) << (4 - i);
            m10 |= (d == 2u ? 1u : 0u) << (4 - i);
            c |= (d & 3u) << (2 * (4 - i));
        }
        masks[b] = (uint16_t)(m01 | (m10 << 5));
        codes[b] = (uint16_t)c;
    }
}

// The 01 / 10 masks of a payload word's 20 elements, element p at bit 19 - p.
__device__ __forceinline__ void word_masks(const uint16_t *table, uint32_t word, uint32_t &is01,
                                           uint32_t &is10)
{
    is01 = 0;
    is10 = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const uint32_t m = table[(word >> (8 * k)) & 0xFFu];
        is01 |= (m & 0x1Fu) << (15 - 5 * k);
        is10 |= ((m >> 5) & 0x1Fu) << (15 - 5 * k);
    }
}

struct RecordSet {
    const uint32_t *rec[QGA_MAX_WORKERS];
};

// Of every QGA_TERNARY_TABLE_PERIOD consecutive workers, the first
// QGA_TERNARY_TABLE_SHARE go through the pair table, the others through the
// code masks.
#ifndef QGA_TERNARY_TABLE_PERIOD
#define QGA_TERNARY_TABLE_PERIOD 2
#endif
#ifndef QGA_TERNARY_TABLE_SHARE
#define QGA_TERNARY_TABLE_SHARE 1
#endif

// The dequantize of one dense record: a lane owns one word (20 elements),
// turns its 4 bytes into 01 / 10 code masks through a 256-entry shared
// table and writes each element's value; outputs leave through a stride-5
// stage as coalesced 128-bit rows.
template <bool kVec>
__global__ void __launch_bounds__(kThreads)
    dequantize_ternary_kernel(const uint32_t *__restrict__ compr, float *__restrict__ out, int64_t n)
{
    __shared__ uint16_t s_masks[256], s_codes[256];
    __shared__ float4 s_stage[kWarpsPerBlock][kWarp * 5];
    build_byte_tables(s_masks, s_codes);
    __syncthreads();
    const float neg = f32_from_bits(compr[0]), pos = f32_from_bits(compr[1]);
    const uint32_t *payload = compr + 3;
    float4 *stage = s_stage[threadIdx.x >> 5];
    const int lane = threadIdx.x & (kWarp - 1);
    const int64_t nwords = (n + 19) / 20;
    const int64_t tiles = (nwords + kWarp - 1) / kWarp;
    for (int64_t t = warp_id(); t < tiles; t += warp_stride()) {
        const int64_t w = t * kWarp + lane;
        const uint32_t word = w < nwords ? ld_stream_u32(payload + w) : 0u;
        uint32_t is01, is10;
        word_masks(s_masks, word, is01, is10);
        float v[20];
#pragma unroll
        for (int p = 0; p < 20; ++p) {
            const uint32_t bit = 1u << (19 - p);
            v[p] = (is01 & bit) ? pos : ((is10 & bit) ? neg : 0.0f);
        }
#pragma unroll
        for (int c = 0; c < 5; ++c)
            stage[5 * lane + c] = make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
        __syncwarp();
#pragma unroll
        for (int j = 0; j < 5; ++j) {
            const int q = j * kWarp + lane; // group of 4 within the tile
            store_group<kVec>(out, n, t * (kWarp * 5) + q, stage[q]);
        }
        __syncwarp();
    }
}

// ------------------------------------------------------ merge by sum table --
// W <= 8: the merge through the table of all 3^W sums (build_sum_table in
// qga_2bit_tiles.cuh: entry sum_k d_k 3^k holds the definition's sum of the
// workers' code values, d_k the trit of worker k).  A lane owns one payload
// word (20 elements) and turns every worker's 4 bytes into trits without
// a lookup table: two bytes at a time in 16-bit lanes, floor(v / 3) =
// (171 v) >> 9 (exact for v < 256), trit = v - 3 floor(v / 3), four times;
// the leading trit is taken mod 3 like every other (a byte above 242 never
// occurs in a record).  The trits of worker k, times 4 3^k, accumulate into
// the byte offsets of the table entries (at most 4 * 6560 < 2^16).
__device__ __forceinline__ uint32_t div3_16(uint32_t v) // two 16-bit lanes, each below 256
{
    return ((v * 171u) >> 9) & 0x007F007Fu;
}

// acc[i]: table offsets of trit i (0 = most significant) of the two bytes in
// the lanes of v, plus 4 3^k times worker k's trits.
__device__ __forceinline__ void add_trits(uint32_t v, uint32_t weight, uint32_t (&acc)[5])
{
    const uint32_t q1 = div3_16(v), q2 = div3_16(q1), q3 = div3_16(q2), q4 = div3_16(q3);
    acc[4] += (v - 3u * q1) * weight;
    acc[3] += (q1 - 3u * q2) * weight;
    acc[2] += (q2 - 3u * q3) * weight;
    acc[1] += (q3 - 3u * q4) * weight;
    acc[0] += (q4 - 3u * ((q4 >> 1) & q4 & 0x00010001u)) * weight; // 3 -> 0
}

// Words per lane of a table-merge tile (build-time setting; the default is
// the measured best): lane l owns words l, 32 + l, ... and loads all of them,
// of every worker, before using any.  With QGA_TERNARY_TABLE_PREFETCH the
// words of the warp's next tile are loaded before the current tile is
// decoded and stored, so that they are in flight meanwhile.  Measured at
// n = 138M, W = 8: 2 slots with the next tile in flight 142.0 us; 2 slots
// loaded just before use 148.9 us; 1 slot 158.7 us, with the next tile in
// flight and 4 blocks per SM 145.7 us.
#ifndef QGA_TERNARY_TABLE_SLOTS
#define QGA_TERNARY_TABLE_SLOTS 2
#endif
#ifndef QGA_TERNARY_TABLE_PREFETCH
#define QGA_TERNARY_TABLE_PREFETCH 1
#endif
#ifdef QGA_TERNARY_TABLE_MIN_BLOCKS
#define QGA_TERNARY_TABLE_BOUNDS __launch_bounds__(kThreads, QGA_TERNARY_TABLE_MIN_BLOCKS)
#else
#define QGA_TERNARY_TABLE_BOUNDS __launch_bounds__(kThreads)
#endif
constexpr int kTernarySlots = QGA_TERNARY_TABLE_SLOTS;
constexpr bool kTernaryPrefetch = QGA_TERNARY_TABLE_PREFETCH != 0;

template <int kW>
__device__ __forceinline__ void load_ternary_tile(const RecordSet &set, int64_t t, int64_t nwords, int lane,
                                                  uint32_t (&words)[kTernarySlots][kW])
{
#pragma unroll
    for (int sl = 0; sl < kTernarySlots; ++sl) {
        const int64_t w = (t * kTernarySlots + sl) * kWarp + lane;
#pragma unroll
        for (int k = 0; k < kW; ++k)
            words[sl][k] = w < nwords ? ld_stream_u32(set.rec[k] + 3 + w) : 0u;
    }
}

template <bool kVec, int kW>
__global__ void QGA_TERNARY_TABLE_BOUNDS
    merge_ternary_table_kernel(const __grid_constant__ RecordSet set, float *__restrict__ out, int64_t n)
{
    __shared__ float s_neg[kW], s_pos[kW];
    __shared__ float s_sum[Pow3<kW>::value];
    __shared__ float4 s_stage[kWarpsPerBlock][kWarp * 5];
    if (threadIdx.x < kW) {
        const uint32_t *r = set.rec[threadIdx.x];
        s_neg[threadIdx.x] = f32_from_bits(r[0]);
        s_pos[threadIdx.x] = f32_from_bits(r[1]);
    }
    const char *tb = reinterpret_cast<const char *>(s_sum);
    float4 *stage = s_stage[threadIdx.x >> 5];
    const int lane = threadIdx.x & (kWarp - 1);
    const int64_t nwords = (n + 19) / 20;
    const int64_t tiles = (nwords + kWarp * kTernarySlots - 1) / (kWarp * kTernarySlots);
    int64_t t = warp_id();
    uint32_t words[kTernarySlots][kW];
    if (t < tiles) // the first tile's words are in flight while the table is built
        load_ternary_tile<kW>(set, t, nwords, lane, words);
    __syncthreads();
    build_sum_table<kW>(s_sum, [&](int w) { return s_neg[w]; }, [&](int w) { return s_pos[w]; });
    for (; t < tiles; t += warp_stride()) {
        const int64_t tn = t + warp_stride();
        uint32_t next[kTernarySlots][kW];
        if (kTernaryPrefetch) {
            if (tn < tiles)
                load_ternary_tile<kW>(set, tn, nwords, lane, next);
            else
#pragma unroll
                for (int sl = 0; sl < kTernarySlots; ++sl)
#pragma unroll
                    for (int k = 0; k < kW; ++k)
                        next[sl][k] = 0u;
        }
#pragma unroll
        for (int sl = 0; sl < kTernarySlots; ++sl) {
            // lanes: ev = bytes 0 and 2 of the word, od = bytes 1 and 3
            uint32_t ev[5] = {}, od[5] = {};
            uint32_t weight = 4u;
#pragma unroll
            for (int k = 0; k < kW; ++k) {
                add_trits(words[sl][k] & 0x00FF00FFu, weight, ev);
                add_trits((words[sl][k] >> 8) & 0x00FF00FFu, weight, od);
                weight *= 3u;
            }
            // byte b of the word holds elements 5b .. 5b + 4 (trit i = element 5b + i)
            float v[20];
#pragma unroll
            for (int i = 0; i < 5; ++i) {
                v[i] = *reinterpret_cast<const float *>(tb + (ev[i] & 0xFFFFu));   // byte 0
                v[10 + i] = *reinterpret_cast<const float *>(tb + (ev[i] >> 16)); // byte 2
                v[5 + i] = *reinterpret_cast<const float *>(tb + (od[i] & 0xFFFFu)); // byte 1
                v[15 + i] = *reinterpret_cast<const float *>(tb + (od[i] >> 16));   // byte 3
            }
#pragma unroll
            for (int c = 0; c < 5; ++c)
                stage[5 * lane + c] = make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
            __syncwarp();
            const int64_t g0 = (t * kTernarySlots + sl) * (kWarp * 5); // first group of this word slot
#pragma unroll
            for (int j = 0; j < 5; ++j) {
                const int q = j * kWarp + lane; // group of 4 within the slot's 32 words
                store_group<kVec>(out, n, g0 + q, stage[q]);
            }
            __syncwarp();
        }
        if (kTernaryPrefetch) {
#pragma unroll
            for (int sl = 0; sl < kTernarySlots; ++sl)
#pragma unroll
                for (int k = 0; k < kW; ++k)
                    words[sl][k] = next[sl][k];
        } else if (tn < tiles) {
            load_ternary_tile<kW>(set, tn, nwords, lane, words);
        }
    }
}

// W > 8: the first 8 workers' sum of each element from the 3^8 table (as in
// merge_ternary_table_kernel), which is exactly the definition's running sum
// after worker 7, then workers 8 .. W-1 added in order by the per-worker
// decode (pair tables for even workers, code masks for odd ones).  The 3^8
// table (26,244 B) sits in dynamic
// shared memory.
constexpr int kTernaryPrefix = 8;
constexpr int kTernaryPrefixBytes = Pow3<kTernaryPrefix>::value * 4;

template <bool kVec>
__global__ void __launch_bounds__(kThreads)
    merge_ternary_prefix_kernel(const __grid_constant__ RecordSet set, int W, float *__restrict__ out,
                                int64_t n)
{
    extern __shared__ __align__(16) unsigned char s_dyn[];
    float *s_sum = reinterpret_cast<float *>(s_dyn);
    __shared__ uint16_t s_masks[256], s_codes[256];
    __shared__ float s_neg[QGA_MAX_WORKERS], s_pos[QGA_MAX_WORKERS];
    __shared__ float2 s_pair[QGA_MAX_WORKERS][16];
    __shared__ float4 s_stage[kWarpsPerBlock][kWarp * 5];
    build_byte_tables(s_masks, s_codes);
    for (int w = threadIdx.x; w < W; w += kThreads) {
        const uint32_t *r = set.rec[w];
        s_neg[w] = f32_from_bits(r[0]);
        s_pos[w] = f32_from_bits(r[1]);
    }
    __syncthreads();
    for (int i = kTernaryPrefix * 16 + threadIdx.x; i < W * 16; i += kThreads)
        s_pair[i >> 4][i & 15] = pair_entry(i & 15, s_neg[i >> 4], s_pos[i >> 4]);
    build_sum_table<kTernaryPrefix>(s_sum, [&](int w) { return s_neg[w]; }, [&](int w) { return s_pos[w]; });
    __syncthreads();
    const char *tb = reinterpret_cast<const char *>(s_sum);
    float4 *stage = s_stage[threadIdx.x >> 5];
    const int lane = threadIdx.x & (kWarp - 1);
    const int64_t nwords = (n + 19) / 20;
    const int64_t tiles = (nwords + kWarp - 1) / kWarp;
    for (int64_t t = warp_id(); t < tiles; t += warp_stride()) {
        const int64_t w = t * kWarp + lane;
        const bool ok = w < nwords;
        float2 acc[10];
        {
            uint32_t ev[5] = {}, od[5] = {};
            uint32_t weight = 4u;
#pragma unroll
            for (int k = 0; k < kTernaryPrefix; ++k) {
                const uint32_t word = ok ? ld_stream_u32(set.rec[k] + 3 + w) : 0u;
                add_trits(word & 0x00FF00FFu, weight, ev);
                add_trits((word >> 8) & 0x00FF00FFu, weight, od);
                weight *= 3u;
            }
            // byte b of the word holds elements 5b .. 5b + 4 (trit i = element 5b + i)
            float v[20];
#pragma unroll
            for (int i = 0; i < 5; ++i) {
                v[i] = *reinterpret_cast<const float *>(tb + (ev[i] & 0xFFFFu));
                v[10 + i] = *reinterpret_cast<const float *>(tb + (ev[i] >> 16));
                v[5 + i] = *reinterpret_cast<const float *>(tb + (od[i] & 0xFFFFu));
                v[15 + i] = *reinterpret_cast<const float *>(tb + (od[i] >> 16));
            }
#pragma unroll
            for (int q = 0; q < 10; ++q)
                acc[q] = make_float2(v[2 * q], v[2 * q + 1]);
        }
        constexpr int kBatch = 8;
        for (int wb = kTernaryPrefix; wb < W; wb += kBatch) {
            uint32_t words[kBatch];
#pragma unroll
            for (int i = 0; i < kBatch; ++i)
                words[i] = (ok && wb + i < W) ? ld_stream_u32(set.rec[wb + i] + 3 + w) : 0u;
#pragma unroll
            for (int i = 0; i < kBatch; ++i) {
                if (wb + i >= W) // warp-uniform
                    break;
                const uint32_t word = words[i];
                if ((i % QGA_TERNARY_TABLE_PERIOD) < QGA_TERNARY_TABLE_SHARE) {
                    // the 20 codes as a 40-bit string, element 0 in bits 39..38
                    const uint32_t c0 = s_codes[word & 0xFFu], c1 = s_codes[(word >> 8) & 0xFFu];
                    const uint32_t c2 = s_codes[(word >> 16) & 0xFFu], c3 = s_codes[word >> 24];
                    const uint32_t hi = c0 >> 2;
                    const uint32_t lo = (c0 << 30) | (c1 << 20) | (c2 << 10) | c3;
                    const char *pt = reinterpret_cast<const char *>(s_pair[wb + i]);
#pragma unroll
                    for (int q = 0; q < 10; ++q) {
                        const int sh = 36 - 4 * q;
                        const uint32_t nib = sh >= 32 ? (hi >> (sh - 32)) : (lo >> sh);
                        acc[q] = __fadd2_rn(acc[q], *reinterpret_cast<const float2 *>(pt + ((nib & 0xFu) << 3)));
                    }
                } else {
                    const float neg = s_neg[wb + i], pos = s_pos[wb + i];
                    uint32_t is01, is10;
                    word_masks(s_masks, word, is01, is10);
#pragma unroll
                    for (int p = 0; p < 20; ++p) {
                        const uint32_t bit = 1u << (19 - p);
                        float &a = (p & 1) ? acc[p >> 1].y : acc[p >> 1].x;
                        if (is01 & bit)
                            a = __fadd_rn(a, pos);
                        if (is10 & bit)
                            a = __fadd_rn(a, neg);
                    }
                }
            }
        }
#pragma unroll
        for (int c = 0; c < 5; ++c)
            stage[5 * lane + c] = make_float4(acc[2 * c].x, acc[2 * c].y, acc[2 * c + 1].x, acc[2 * c + 1].y);
        __syncwarp();
#pragma unroll
        for (int j = 0; j < 5; ++j) {
            const int q = j * kWarp + lane; // group of 4 within the tile
            store_group<kVec>(out, n, t * (kWarp * 5) + q, stage[q]);
        }
        __syncwarp();
    }
}

std::atomic<int> occ_tq[2][64], occ_td[2][2][9][64]; // td: [vec][merge][kW]
std::atomic<bool> prefix_attr_set[2][64];

// Grid waves (see grid_for), measured at n = 138M: quantize 287 / 253 / 247 /
// 243 / 240 us at 1 / 8 / 16 / 32 / 128 waves; merge (W = 8) 206 / 199 / 206
// / 224 us at 1 / 8 / 16 / 32.
constexpr int kTernaryQuantizeWaves = 32, kTernaryDecodeWaves = 8;
// The table merge by worker count (the table is rebuilt by every block):
// measured at n = 138M (us at 1 / 4 / 8 / 16 waves): W = 1 106 / 95 / 93 /
// 91, W = 2 112 / 100 / 97 / 96, W = 3 117 / 105 / 101 / 99, W = 4 123 / 110
// / 107 / 111, W = 5 128 / 114 / 110 / 115, W = 6 134 / 119 / 119 / 134,
// W = 7 139 / 125 / 131 / 152, W = 8 142 / 147 / 158 / 187.
#ifdef QGA_TERNARY_TABLE_WAVES
constexpr int ternary_table_waves(int) { return QGA_TERNARY_TABLE_WAVES; }
#else
constexpr int ternary_table_waves(int w) { return w <= 3 ? 16 : (w <= 5 ? 8 : (w <= 7 ? 4 : 1)); }
#endif

unsigned warps_grid(int64_t warp_items, int resident, int waves)
{
    return grid_for((warp_items + kWarpsPerBlock - 1) / kWarpsPerBlock, resident, waves);
}

template <bool kVec, bool kMerge, int kW>
void launch_decode_k(const RecordSet &set, int W, float *out, int64_t n, cudaStream_t stream)
{
    const int64_t tiles = ((n + 19) / 20 + kWarp - 1) / kWarp;
    if constexpr (kMerge && kW > 0) {
        auto k = merge_ternary_table_kernel<kVec, kW>;
        const int64_t table_tiles = ((n + 19) / 20 + kWarp * kTernarySlots - 1) / (kWarp * kTernarySlots);
        k<<<warps_grid(table_tiles, resident_blocks(k, kThreads, occ_td[kVec][kMerge][kW]),
                       ternary_table_waves(kW)),
            kThreads, 0, stream>>>(set, out, n);
    } else if constexpr (kMerge) {
        // W > 8: the prefix table takes more than the default 48 KB of shared memory
        auto k = merge_ternary_prefix_kernel<kVec>;
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
            dev = 0;
        if (!prefix_attr_set[kVec][dev].load(std::memory_order_relaxed)) {
            cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kTernaryPrefixBytes);
            prefix_attr_set[kVec][dev].store(true, std::memory_order_relaxed);
        }
        k<<<warps_grid(tiles, resident_blocks(k, kThreads, occ_td[kVec][kMerge][0], kTernaryPrefixBytes),
                       kTernaryDecodeWaves),
            kThreads, kTernaryPrefixBytes, stream>>>(set, W, out, n);
    } else {
        auto k = dequantize_ternary_kernel<kVec>;
        k<<<warps_grid(tiles, resident_blocks(k, kThreads, occ_td[kVec][0][0]), kTernaryDecodeWaves),
            kThreads, 0, stream>>>(set.rec[0], out, n);
    }
}

template <bool kVec>
void launch_merge_v(const RecordSet &set, int W, float *out, int64_t n, cudaStream_t stream)
{
    switch (W) {
    case 1: launch_decode_k<kVec, true, 1>(set, W, out, n, stream); break;
    case 2: launch_decode_k<kVec, true, 2>(set, W, out, n, stream); break;
    case 3: launch_decode_k<kVec, true, 3>(set, W, out, n, stream); break;
    case 4: launch_decode_k<kVec, true, 4>(set, W, out, n, stream); break;
    case 5: launch_decode_k<kVec, true, 5>(set, W, out, n, stream); break;
    case 6: launch_decode_k<kVec, true, 6>(set, W, out, n, stream); break;
    case 7: launch_decode_k<kVec, true, 7>(set, W, out, n, stream); break;
    case 8: launch_decode_k<kVec, true, 8>(set, W, out, n, stream); break;
    default: launch_decode_k<kVec, true, 0>(set, W, out, n, stream); break;
    }
}

int launch_decode(const RecordSet &set, int W, float *out, int64_t n, cudaStream_t stream,
                  bool merge)
{
    const bool vec = aligned(out, 16);
    if (merge) {
        if (vec)
            launch_merge_v<true>(set, W, out, n, stream);
        else
            launch_merge_v<false>(set, W, out, n, stream);
    } else {
        if (vec)
            launch_decode_k<true, false, 1>(set, 1, out, n, stream);
        else
            launch_decode_k<false, false, 1>(set, 1, out, n, stream);
    }
    return launch_status();
}

} // namespace
} // namespace qga

using namespace qga;

extern "C" int64_t qga_ternary_words(int64_t n)
{
    if (n < 0)
        return QGA_ERR_INVALID_ARG;
    return 3 + (n + 19) / 20;
}

extern "C" int qga_quantize_ternary(const float *grad, float *residual, uint32_t *compr, int64_t n,
                                    float neg_threshold, float pos_threshold, cudaStream_t stream)
{
    if (n < 0 || compr == nullptr || !aligned(compr, 4) || !finite_f32(neg_threshold) ||
        !finite_f32(pos_threshold))
        return QGA_ERR_INVALID_ARG;
    if (n > 0 && (grad == nullptr || residual == nullptr || !aligned(grad, 4) || !aligned(residual, 4)))
        return QGA_ERR_INVALID_ARG;
    const int64_t tiles = (n + kTTileElems - 1) / kTTileElems;
    if (aligned(grad, 16) && aligned(residual, 16)) {
        auto k = quantize_ternary_kernel<true>;
        k<<<warps_grid(tiles, resident_blocks(k, kThreads, occ_tq[1]), kTernaryQuantizeWaves), kThreads,
            0, stream>>>(
            grad, residual, compr, n, neg_threshold, pos_threshold);
    } else {
        auto k = quantize_ternary_kernel<false>;
        k<<<warps_grid(tiles, resident_blocks(k, kThreads, occ_tq[0]), kTernaryQuantizeWaves), kThreads,
            0, stream>>>(
            grad, residual, compr, n, neg_threshold, pos_threshold);
    }
    return launch_status();
}

extern "C" int qga_dequantize_ternary(const uint32_t *compr, float *out, int64_t n,
                                      cudaStream_t stream)
{
    if (n < 0 || compr == nullptr || !aligned(compr, 4))
        return QGA_ERR_INVALID_ARG;
    if (n == 0)
        return QGA_OK;
    if (out == nullptr || !aligned(out, 4))
        return QGA_ERR_INVALID_ARG;
    RecordSet set{};
    set.rec[0] = compr;
    return launch_decode(set, 1, out, n, stream, false);
}

extern "C" int qga_dequant_accumulate_ternary(const uint32_t *const *compr, int num_workers,
                                              float *out, int64_t n, cudaStream_t stream)
{
    if (n < 0 || compr == nullptr || num_workers < 1 || num_workers > QGA_MAX_WORKERS)
        return QGA_ERR_INVALID_ARG;
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
    return launch_decode(set, num_workers, out, n, stream, true);
}
