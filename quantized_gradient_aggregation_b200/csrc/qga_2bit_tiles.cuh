// qga_2bit_tiles.cuh -- the per-warp tiles of the 2-bit threshold path,
// shared by the single-tensor kernels (qga_2bit.cu) and the bucket kernels
// (qga_bucket.cu).
//
// Method: MXNet pull request #8342 "[WIP] 2bit gradient compression",
// "Approach" (the residual carries the quantization error into the next
// step), "Two bit quantization" (codes 01 / 10 / 00 against the two
// thresholds) and "Format of compressed gradient" (16 codes per 32-bit word,
// the first element in the two most significant bits).
//
// Tile geometry.  One warp owns a tile of consecutive elements in groups of
// 4: 128 groups (512 elements, 32 packed words) for an fp32 gradient, 256
// groups (1024 elements) for a bfloat16 one, whose narrower gradient loads
// need more groups per lane to keep as many bytes in flight.  Lane l handles
// groups l, l+32, l+64, ..., so every load or store instruction of the warp
// touches contiguous bytes (fully coalesced vector accesses).  A group's 4
// codes form one byte of its word; the 4 lanes sharing a word combine their
// bytes with two xor-shuffles (no shared memory, so no bank conflicts), and
// the first of them stores the word.
#pragma once

#include "qga_common.cuh"

namespace qga {

constexpr int kGroupsPerLane = 4;                   // fp32 tiles; see GradLoad::kGroups
constexpr int kTileGroups = kWarp * kGroupsPerLane; // 128 groups of 4 elements
constexpr int kTileElems = kTileGroups * 4;         // 512 elements
constexpr int kTileWords = kTileElems / 16;         // 32 words

// "Two bit quantization": at or above the positive threshold -> 01, else at
// or below the negative threshold -> 10, else 00.
__device__ __forceinline__ uint32_t tb_code(float x, float neg, float pos)
{
    return (x >= pos) ? 1u : ((x <= neg) ? 2u : 0u);
}

// The value a code stands for (11 is never written and reads as 0).
__device__ __forceinline__ float tb_value(uint32_t c, float neg, float pos)
{
    return (c == 1u) ? pos : ((c == 2u) ? neg : 0.0f);
}

// Error feedback for one element: x = g + r; code; r = x - value(code).
// Two separately rounded binary32 operations, never fused.
__device__ __forceinline__ uint32_t tb_step(float g, float &r, float neg, float pos)
{
    const float x = __fadd_rn(g, r);
    const uint32_t c = tb_code(x, neg, pos);
    r = __fsub_rn(x, tb_value(c, neg, pos));
    return c;
}

// Gradient access by element type: fp32, or bfloat16 bit patterns.  A
// group is loaded raw (one vector load) and widened to fp32 when it is used.
template <typename G> struct GradLoad;

template <> struct GradLoad<float> {
    static constexpr uintptr_t kVecAlign = 16;
    static constexpr int kGroups = 4; // groups per lane per tile
    using Raw = float4;
    static __device__ __forceinline__ Raw raw(const float *g, int64_t gi) { return ld_stream_f4(g + 4 * gi); }
    static __device__ __forceinline__ float4 widen(Raw v) { return v; }
    static __device__ __forceinline__ Raw pack(const float t[4]) { return make_float4(t[0], t[1], t[2], t[3]); }
    static __device__ __forceinline__ float one(const float *g, int64_t e) { return ld_stream_f1(g + e); }
};

template <> struct GradLoad<uint16_t> {
    static constexpr uintptr_t kVecAlign = 8;
    static constexpr int kGroups = 8;
    using Raw = uint2; // 4 bfloat16, element 0 in the low half of .x (little endian)
    static __device__ __forceinline__ Raw raw(const uint16_t *g, int64_t gi) { return ld_stream_u2(g + 4 * gi); }
    static __device__ __forceinline__ float4 widen(Raw v)
    {
        return make_float4(widen_bf16(v.x & 0xffffu), widen_bf16(v.x >> 16),
                           widen_bf16(v.y & 0xffffu), widen_bf16(v.y >> 16));
    }
    static __device__ __forceinline__ Raw pack(const float t[4])
    {
        // t holds widened bfloat16 values: their high halves are the originals
        return make_uint2((__float_as_uint(t[0]) >> 16) | (__float_as_uint(t[1]) & 0xffff0000u),
                          (__float_as_uint(t[2]) >> 16) | (__float_as_uint(t[3]) & 0xffff0000u));
    }
    static __device__ __forceinline__ float one(const uint16_t *g, int64_t e)
    {
        return widen_bf16(ld_stream_u16(g + e));
    }
};

// Elements of one quantize tile for gradient type G.
template <typename G> __host__ __device__ constexpr int64_t quantize_tile_elems() { return (int64_t)kWarp * GradLoad<G>::kGroups * 4; }

// Codes of elements at or beyond n are forced to 00: keep the top 2*valid
// bits of a group's byte.
__device__ __forceinline__ uint32_t keep_valid_codes(uint32_t byte, int64_t valid)
{
    const int v = valid <= 0 ? 0 : (valid >= 4 ? 4 : (int)valid);
    return byte & ((0xFF00u >> (2 * v)) & 0xFFu);
}

// Quantize + residual update + pack of tile `tile` of one tensor.
//   kVec: grad and residual are aligned for vector access (16 B fp32 / 8 B bf16).
// All 32 lanes must call this together (warp-uniform `tile`).
template <typename G, bool kVec>
__device__ __forceinline__ void quantize_2bit_tile(const G *__restrict__ grad,
                                                   float *__restrict__ residual,
                                                   uint32_t *__restrict__ payload, int64_t n,
                                                   int64_t tile, float neg, float pos, int lane)
{
    using GL = GradLoad<G>;
    constexpr int kG = GL::kGroups;
    const int64_t full_groups = n >> 2;
    const int64_t nwords = (n + 15) >> 4;
    const int64_t g0 = tile * (kWarp * kG);

    typename GL::Raw gv[kG];
    float4 rv[kG];
#pragma unroll
    for (int j = 0; j < kG; ++j) {
        const int64_t gi = g0 + j * kWarp + lane;
        if (kVec && gi < full_groups) {
            gv[j] = GL::raw(grad, gi);
            rv[j] = ld_stream_f4(residual + 4 * gi);
        } else {
            float tg[4], tr[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int64_t e = 4 * gi + k;
                tg[k] = e < n ? GL::one(grad, e) : 0.0f;
                tr[k] = e < n ? ld_stream_f1(residual + e) : 0.0f;
            }
            gv[j] = GL::pack(tg);
            rv[j] = make_float4(tr[0], tr[1], tr[2], tr[3]);
        }
    }

#pragma unroll
    for (int j = 0; j < kG; ++j) {
        const int64_t gi = g0 + j * kWarp + lane;
        const float4 g = GL::widen(gv[j]);
        float4 r = rv[j];
        const uint32_t c0 = tb_step(g.x, r.x, neg, pos);
        const uint32_t c1 = tb_step(g.y, r.y, neg, pos);
        const uint32_t c2 = tb_step(g.z, r.z, neg, pos);
        const uint32_t c3 = tb_step(g.w, r.w, neg, pos);
        uint32_t byte = (c0 << 6) | (c1 << 4) | (c2 << 2) | c3;
        if (kVec && gi < full_groups) {
            st_stream_f4(residual + 4 * gi, r);
        } else {
            const int64_t valid = n - 4 * gi;
            const float rr[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
            for (int k = 0; k < 4; ++k)
                if (k < valid)
                    st_stream_f1(residual + 4 * gi + k, rr[k]);
            byte = keep_valid_codes(byte, valid);
        }
        // lanes 4q..4q+3 hold the 4 bytes of word q of this slice, the lowest
        // lane the most significant byte
        uint32_t word = byte << (24 - 8 * (lane & 3));
        word |= __shfl_xor_sync(kFullMask, word, 1);
        word |= __shfl_xor_sync(kFullMask, word, 2);
        const int64_t wi = (g0 >> 2) + j * (kWarp / 4) + (lane >> 2);
        if ((lane & 3) == 0 && wi < nwords)
            st_stream_u32(payload + wi, word);
    }
}

// ---------------------------------------------------- lane-owned words --
// The other geometry for an fp32 gradient whose gradient and residual are
// 32-byte aligned: a lane owns whole words (16 consecutive elements), loads
// them with two 256-bit loads each of g and r, packs its 16 codes in
// registers (no shuffle) and stores r with two 256-bit stores.  Each warp
// access still uses whole 32-byte sectors, with a quarter of the memory
// instructions of the group tiles.  load_word and quantize_word are its two
// halves (the loads of several words can be issued before any is used).
// Codes of elements >= n are 00.
template <bool kVec>
__device__ __forceinline__ void load_word(const float *__restrict__ grad,
                                          const float *__restrict__ residual, int64_t n,
                                          int64_t k, float (&g)[16], float (&r)[16])
{
    const int64_t e0 = 16 * k;
    if (kVec && e0 + 16 <= n) {
        ld_stream_f8(grad + e0, g);
        ld_stream_f8(grad + e0 + 8, g + 8);
        ld_stream_f8(residual + e0, r);
        ld_stream_f8(residual + e0 + 8, r + 8);
    } else {
#pragma unroll
        for (int p = 0; p < 16; ++p) {
            g[p] = e0 + p < n ? ld_stream_f1(grad + e0 + p) : 0.0f;
            r[p] = e0 + p < n ? ld_stream_f1(residual + e0 + p) : 0.0f;
        }
    }
}

// Codes and residual update of word k from its loaded elements; writes the
// residual and the word, and returns the word.
template <bool kVec>
__device__ __forceinline__ uint32_t quantize_word(float *__restrict__ residual,
                                                  uint32_t *__restrict__ payload, int64_t n,
                                                  int64_t k, float neg, float pos,
                                                  const float (&g)[16], float (&r)[16])
{
    const int64_t e0 = 16 * k;
    const bool full = kVec && e0 + 16 <= n;
    uint32_t word = 0u;
#pragma unroll
    for (int p = 0; p < 16; ++p) {
        const uint32_t c = tb_step(g[p], r[p], neg, pos);
        if (full || e0 + p < n)
            word |= c << (30 - 2 * p);
    }
    if (full) {
        st_stream_f8(residual + e0, r);
        st_stream_f8(residual + e0 + 8, r + 8);
    } else {
#pragma unroll
        for (int p = 0; p < 16; ++p)
            if (e0 + p < n)
                st_stream_f1(residual + e0 + p, r[p]);
    }
    st_stream_u32(payload + k, word);
    return word;
}

// Store the 4 values of group gi of an fp32 output of n elements.
template <bool kVec>
__device__ __forceinline__ void store_group(float *__restrict__ out, int64_t n, int64_t gi, float4 v)
{
    if (kVec && gi < (n >> 2)) {
        st_stream_f4(out + 4 * gi, v);
    } else {
        const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int k = 0; k < 4; ++k)
            if (4 * gi + k < n)
                st_stream_f1(out + 4 * gi + k, vv[k]);
    }
}

// ------------------------------------------------------------------ merge --
// Decoding the way the quantizer packs (one byte per lane, a shuffle per
// worker) leaves the merge bound by instruction issue, far from HBM.  So
// the merge has its own geometry: a warp owns a slice of 64 consecutive
// words (1024 elements), lane l owns words l and 32 + l of the slice and
// decodes all 16 codes of each itself -- one coalesced 32-bit load per lane
// per worker, no shuffle -- keeping both words in flight together.
//
// Two decoders share the work so that neither execution pipe saturates:
//   even workers: a 16-entry table per worker in shared memory maps 4 code
//     bits (two elements) to the two values they stand for; one 64-bit
//     shared load and one paired add (__fadd2_rn) per two elements (load
//     / store pipe + FMA pipe);
//   odd workers: each word becomes two bit masks (elements coded 01, coded
//     10; 11 is in neither) and every element takes a predicated add of the
//     threshold its code stands for (integer pipe + FMA pipe).
// Both add exactly the oracle's value in the oracle's order: the table holds
// the thresholds themselves, paired adds are two independent round-to-
// nearest adds, and skipping the add of +0 for code 00 changes nothing (the
// sum starts at +0, can never become -0 in round-to-nearest, and x + (+0) ==
// x for every other x).
// The 16 sums of a word are consecutive floats owned by one lane; they leave
// through a per-warp shared-memory stage (xor-swizzled so that both the
// 128-bit writes and the 128-bit reads are free of bank conflicts) as fully
// coalesced 128-bit rows.
#ifndef QGA_MERGE_SLOTS
#define QGA_MERGE_SLOTS 2
#endif
constexpr int kMergeSlots = QGA_MERGE_SLOTS;           // words per lane per slice
constexpr int kSliceWords = kWarp * kMergeSlots;       // 64
constexpr int64_t kSliceElems = kSliceWords * 16;      // 1024
constexpr int kStagePerWarp = kSliceWords * 4;         // float4 per warp (4 KB)
constexpr int kMergeBatch = 8;                         // workers loaded before decoding

// Stage position of chunk c (elements 4c..4c+3) of lane L's word.
__device__ __forceinline__ int stage_slot(int L, int c) { return L * 4 + (c ^ ((L >> 1) & 3)); }

// Pair table of one worker: entry e = (value of code e >> 2, value of code
// e & 3), the first element of the pair in the high bits.
__device__ __forceinline__ float2 pair_entry(int e, float neg, float pos)
{
    return make_float2(tb_value((uint32_t)e >> 2, neg, pos), tb_value((uint32_t)e & 3u, neg, pos));
}

// Merge slice `slice` of W records into out (n elements), values summed
// from +0 in worker order 0..W-1.
//   payload_of(w) -> worker w's payload (word 3 of its record)
//   neg_of(w), pos_of(w) -> its thresholds
//   table -> QGA_MAX_WORKERS x 16 pair entries (built by the caller for w < W)
//   stage -> this warp's kStagePerWarp float4 of shared memory
//   kW > 0: the worker count is the compile-time constant kW (W is ignored)
// All 32 lanes must call this together (warp-uniform `slice`).
template <bool kVec, int kW, typename PayloadOf, typename NegOf, typename PosOf>
__device__ __forceinline__ void dequant_accumulate_2bit_slice(int W_runtime, PayloadOf payload_of,
                                                              NegOf neg_of, PosOf pos_of,
                                                              const float2 (*table)[16],
                                                              float *__restrict__ out, int64_t n,
                                                              int64_t slice, int lane,
                                                              float4 *__restrict__ stage)
{
    const int W = kW > 0 ? kW : W_runtime;
    const int64_t nwords = (n + 15) >> 4;
    int64_t k[kMergeSlots];
    bool ok[kMergeSlots];
#pragma unroll
    for (int s = 0; s < kMergeSlots; ++s) {
        k[s] = slice * kSliceWords + s * kWarp + lane;
        ok[s] = k[s] < nwords;
    }
    float2 acc[kMergeSlots][8];
#pragma unroll
    for (int s = 0; s < kMergeSlots; ++s)
#pragma unroll
        for (int p = 0; p < 8; ++p)
            acc[s][p] = make_float2(0.0f, 0.0f);

    for (int wb = 0; wb < W; wb += kMergeBatch) {
        uint32_t words[kMergeSlots][kMergeBatch];
#pragma unroll
        for (int i = 0; i < kMergeBatch; ++i)
#pragma unroll
            for (int s = 0; s < kMergeSlots; ++s)
                words[s][i] = (ok[s] && wb + i < W) ? ld_stream_u32(payload_of(wb + i) + k[s]) : 0u;
#pragma unroll
        for (int i = 0; i < kMergeBatch; ++i) {
            if (wb + i >= W) // warp-uniform
                break;
            if ((i & 1) == 0) {
                const char *tb = reinterpret_cast<const char *>(table[wb + i]);
#pragma unroll
                for (int s = 0; s < kMergeSlots; ++s)
#pragma unroll
                    for (int p = 0; p < 8; ++p) {
                        // 4 code bits of elements 2p, 2p+1, times the 8-byte entry size
                        const int sh = 25 - 4 * p;
                        const uint32_t off =
                            (sh >= 0 ? (words[s][i] >> sh) : (words[s][i] << (-sh))) & 0x78u;
                        acc[s][p] = __fadd2_rn(acc[s][p], *reinterpret_cast<const float2 *>(tb + off));
                    }
            } else {
                const float neg = neg_of(wb + i), pos = pos_of(wb + i);
#pragma unroll
                for (int s = 0; s < kMergeSlots; ++s) {
                    const uint32_t lo = words[s][i] & 0x55555555u;
                    const uint32_t hi = (words[s][i] >> 1) & 0x55555555u;
                    const uint32_t is01 = lo & ~hi, is10 = hi & ~lo;
#pragma unroll
                    for (int p = 0; p < 16; ++p) {
                        const uint32_t bit = 1u << (30 - 2 * p);
                        float &a = (p & 1) ? acc[s][p >> 1].y : acc[s][p >> 1].x;
                        if (is01 & bit)
                            a = __fadd_rn(a, pos);
                        if (is10 & bit)
                            a = __fadd_rn(a, neg);
                    }
                }
            }
        }
    }

    const int f = (lane >> 1) & 3;
#pragma unroll
    for (int s = 0; s < kMergeSlots; ++s)
#pragma unroll
        for (int c = 0; c < 4; ++c)
            stage[s * (kWarp * 4) + lane * 4 + (c ^ f)] =
                make_float4(acc[s][2 * c].x, acc[s][2 * c].y, acc[s][2 * c + 1].x, acc[s][2 * c + 1].y);
    __syncwarp();
#pragma unroll
    for (int s = 0; s < kMergeSlots; ++s) {
        const int64_t g0 = (slice * kSliceWords + s * kWarp) * 4; // first group of this slot
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int q = j * kWarp + lane;
            store_group<kVec>(out, n, g0 + q, stage[s * (kWarp * 4) + stage_slot(q >> 2, q & 3)]);
        }
    }
    __syncwarp();
}

// ------------------------------------------------------ merge by sum table --
// With at most 8 workers the merged value of an element depends on nothing
// but its W codes, and a code reads as one of three values (11 reads as 00).
// So every sum the merge can produce is an entry of a table of 3^W floats
// (6561 at W = 8, 26 KB of shared memory): entry i = sum_k d_k 3^k, digit
// d_k = 0 / 1 / 2 for codes 00 / 01 / 10 of worker k, holds the sum of those
// codes' values.  The table is filled with the same binary32 adds in worker
// order as the definition:
//   T[0] = +0;  for k = 0 .. W-1, i < 3^k:  T[i + 3^k] = T[i] + pos_k,
//                                            T[i + 2 3^k] = T[i] + neg_k
// (T[i] for i < 3^k already holds the sum of workers 0 .. k-1 with the later
// workers' codes 00, and adding their +0 changes nothing: the running sum
// starts at +0 and is never -0 in round-to-nearest).  Each entry is thus the
// definition's sum bit for bit, per-worker thresholds included.
//
// Per element the merge computes its table index from the W codes and loads
// one float: the W sequential adds and decodes per element leave the loop.
// The index is formed for the 16 elements of a word position at once, in
// fields of wider and wider registers (SIMD within a register):
//   - every code 11 is cleared to 00;
//   - even and odd 2-bit fields go to the low half of 4-bit nibbles;
//   - two workers combine in a nibble as d_k + 3 d_{k+1} (at most 8);
//   - two such pairs combine in a byte (at most 80: workers 0-3, and 4-7);
//   - the two groups combine in 16-bit halves as 4 (A + 81 B), the table
//     offset in bytes (at most 26240).
// Integer adds of fields never carry into the neighbouring field: every field
// is wide enough for its largest value.
template <int W> struct Pow3 {
    static constexpr int value = 3 * Pow3<W - 1>::value;
};
template <> struct Pow3<0> {
    static constexpr int value = 1;
};
constexpr int kTableMaxWorkers = 8;

// Fill T (3^kW floats of shared memory) from the workers' thresholds.  All
// threads of the block take part; ends with a barrier.
template <int kW, typename NegOf, typename PosOf>
__device__ __forceinline__ void build_sum_table(float *T, NegOf neg_of, PosOf pos_of)
{
    if (threadIdx.x == 0)
        T[0] = 0.0f;
    __syncthreads();
    int P = 1;
#pragma unroll
    for (int k = 0; k < kW; ++k) {
        const float pos = pos_of(k), neg = neg_of(k);
        for (int i = threadIdx.x; i < 2 * P; i += blockDim.x) {
            const bool one = i < P;
            const int j = one ? i : i - P;
            T[j + (one ? P : 2 * P)] = __fadd_rn(T[j], one ? pos : neg);
        }
        __syncthreads();
        P *= 3;
    }
}

// A record word with every code 11 turned into 00.
__device__ __forceinline__ uint32_t clear_code_11(uint32_t w)
{
    const uint32_t t = w & (w >> 1) & 0x55555555u; // low bit of each 11
    return w ^ (t * 3u);
}

// Byte offsets into the sum table of the 16 elements of one word position:
// wd[k] is worker k's word (k < kW), off[p] the offset of element p (element
// p's code sits in bits 31-2p .. 30-2p).
template <int kW>
__device__ __forceinline__ void sum_table_offsets(const uint32_t (&wd)[kTableMaxWorkers],
                                                  uint32_t (&off)[16])
{
    static_assert(kW >= 1 && kW <= kTableMaxWorkers, "table merge: 1..8 workers");
    // nibble i of e[k] / o[k] = field 2i / 2i+1 of worker k (field q = bits 2q..2q+1)
    uint32_t e[kTableMaxWorkers], o[kTableMaxWorkers];
#pragma unroll
    for (int k = 0; k < kW; ++k) {
        const uint32_t c = clear_code_11(wd[k]);
        e[k] = c & 0x33333333u;
        o[k] = (c >> 2) & 0x33333333u;
    }
    // pairs of workers: d_2j + 3 d_2j+1 per nibble
    constexpr int kPairs = (kW + 1) / 2;
    uint32_t pe[4], po[4];
#pragma unroll
    for (int j = 0; j < kPairs; ++j) {
        pe[j] = e[2 * j];
        po[j] = o[2 * j];
        if (2 * j + 1 < kW) {
            pe[j] += 3u * e[2 * j + 1];
            po[j] += 3u * o[2 * j + 1];
        }
    }
    // groups of two pairs, in byte lanes; X = 0..3 holds the fields
    // 4b + {0, 2, 1, 3}[X] in byte b
    constexpr int kGroups = (kPairs + 1) / 2;
    uint32_t g[2][4];
#pragma unroll
    for (int h = 0; h < kGroups; ++h) {
        const uint32_t lo_e = pe[2 * h] & 0x0F0F0F0Fu, hi_e = (pe[2 * h] >> 4) & 0x0F0F0F0Fu;
        const uint32_t lo_o = po[2 * h] & 0x0F0F0F0Fu, hi_o = (po[2 * h] >> 4) & 0x0F0F0F0Fu;
        g[h][0] = lo_e;
        g[h][1] = hi_e;
        g[h][2] = lo_o;
        g[h][3] = hi_o;
        if (2 * h + 1 < kPairs) {
            g[h][0] += 9u * (pe[2 * h + 1] & 0x0F0F0F0Fu);
            g[h][1] += 9u * ((pe[2 * h + 1] >> 4) & 0x0F0F0F0Fu);
            g[h][2] += 9u * (po[2 * h + 1] & 0x0F0F0F0Fu);
            g[h][3] += 9u * ((po[2 * h + 1] >> 4) & 0x0F0F0F0Fu);
        }
    }
    constexpr int kBase[4] = {0, 2, 1, 3};
#pragma unroll
    for (int X = 0; X < 4; ++X) {
        // 16-bit halves: `ev` holds bytes 0 and 2 of the groups, `od` bytes 1 and 3
        uint32_t ev = 4u * (g[0][X] & 0x00FF00FFu);
        uint32_t od = 4u * ((g[0][X] >> 8) & 0x00FF00FFu);
        if (kGroups > 1) {
            ev += 324u * (g[1][X] & 0x00FF00FFu);
            od += 324u * ((g[1][X] >> 8) & 0x00FF00FFu);
        }
        const int q = kBase[X]; // field of byte 0; element p = 15 - field
        off[15 - q] = ev & 0xFFFFu;
        off[15 - (q + 8)] = ev >> 16;
        off[15 - (q + 4)] = od & 0xFFFFu;
        off[15 - (q + 12)] = od >> 16;
    }
}

// Words per lane of a table-merge slice (build-time setting; the default is
// the measured best).
#ifndef QGA_TABLE_MERGE_SLOTS
#define QGA_TABLE_MERGE_SLOTS 2
#endif
constexpr int kTableSlots = QGA_TABLE_MERGE_SLOTS;
constexpr int64_t kTableSliceElems = (int64_t)kWarp * kTableSlots * 16;

// Merge slice `slice` of kW <= 8 records through the sum table T (built by
// build_sum_table for the same records).  A warp's slice is 32 kS consecutive
// words; lane l owns words l, 32 + l, ..., loads all of its words of every
// worker before using any (merge_2bit_table_load), and computes the 16 sums
// of each (merge_2bit_table_store).  The sums leave through `stage` (this
// warp's 2 KB, 128 float4) one word slot at a time, as fully coalesced
// 128-bit rows (xor-swizzled: both sides free of bank conflicts).  All 32
// lanes must call these together (warp-uniform `slice`).
// skip: a worker whose words the caller fills in itself (-1: none).
template <int kW, int kS, typename PayloadOf>
__device__ __forceinline__ void merge_2bit_table_load(PayloadOf payload_of, int64_t nwords, int64_t slice,
                                                      int lane, int skip,
                                                      uint32_t (&wd)[kS][kTableMaxWorkers])
{
#pragma unroll
    for (int s = 0; s < kS; ++s) {
        const int64_t k = (slice * kS + s) * kWarp + lane;
#pragma unroll
        for (int w = 0; w < kTableMaxWorkers; ++w)
            wd[s][w] = (w < kW && w != skip && k < nwords) ? ld_stream_u32(payload_of(w) + k) : 0u;
    }
}

template <bool kVec, int kW, int kS>
__device__ __forceinline__ void merge_2bit_table_store(const uint32_t (&wd)[kS][kTableMaxWorkers],
                                                       const float *T, float *__restrict__ out, int64_t n,
                                                       int64_t slice, int lane, float4 *__restrict__ stage)
{
    const char *tb = reinterpret_cast<const char *>(T);
    const int f = (lane >> 1) & 3;
#pragma unroll
    for (int s = 0; s < kS; ++s) {
        uint32_t off[16];
        sum_table_offsets<kW>(wd[s], off);
        float v[16];
#pragma unroll
        for (int p = 0; p < 16; ++p)
            v[p] = *reinterpret_cast<const float *>(tb + off[p]);
#pragma unroll
        for (int c = 0; c < 4; ++c)
            stage[lane * 4 + (c ^ f)] = make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
        __syncwarp();
        const int64_t g0 = (slice * kS + s) * kWarp * 4; // first group of this word slot
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int q = j * kWarp + lane;
            store_group<kVec>(out, n, g0 + q, stage[stage_slot(q >> 2, q & 3)]);
        }
        __syncwarp();
    }
}

template <bool kVec, int kW, int kS, typename PayloadOf>
__device__ __forceinline__ void merge_2bit_table_slice(PayloadOf payload_of, const float *T,
                                                       float *__restrict__ out, int64_t n,
                                                       int64_t slice, int lane,
                                                       float4 *__restrict__ stage)
{
    uint32_t wd[kS][kTableMaxWorkers];
    merge_2bit_table_load<kW, kS>(payload_of, (n + 15) >> 4, slice, lane, -1, wd);
    merge_2bit_table_store<kVec, kW, kS>(wd, T, out, n, slice, lane, stage);
}

} // namespace qga
