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
// Tile geometry.  One warp owns a tile of 512 consecutive elements = 128
// groups of 4 = 32 packed words.  Lane l handles groups l, l+32, l+64, l+96,
// so every load or store instruction of the warp touches 512 contiguous
// bytes of fp32 (fully coalesced 128-bit accesses).  A group's 4 codes form
// one byte of its word; the 4 lanes sharing a word combine their bytes with
// two xor-shuffles (no shared memory, so no bank conflicts), and the first
// of them stores the word.
#pragma once

#include "qga_common.cuh"

namespace qga {

constexpr int kGroupsPerLane = 4;
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

// Gradient access by element type: fp32, or bfloat16 bit patterns.
template <typename G> struct GradLoad;

template <> struct GradLoad<float> {
    static constexpr uintptr_t kVecAlign = 16;
    static __device__ __forceinline__ float4 group(const float *g, int64_t gi)
    {
        return ld_stream_f4(g + 4 * gi);
    }
    static __device__ __forceinline__ float one(const float *g, int64_t e)
    {
        return ld_stream_f1(g + e);
    }
};

template <> struct GradLoad<uint16_t> {
    static constexpr uintptr_t kVecAlign = 8;
    static __device__ __forceinline__ float4 group(const uint16_t *g, int64_t gi)
    {
        const uint2 v = ld_stream_u2(g + 4 * gi); // little endian: element 0 in v.x low half
        return make_float4(widen_bf16(v.x & 0xffffu), widen_bf16(v.x >> 16),
                           widen_bf16(v.y & 0xffffu), widen_bf16(v.y >> 16));
    }
    static __device__ __forceinline__ float one(const uint16_t *g, int64_t e)
    {
        return widen_bf16(ld_stream_u16(g + e));
    }
};

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
    const int64_t full_groups = n >> 2;
    const int64_t nwords = (n + 15) >> 4;
    const int64_t g0 = tile * kTileGroups;

    float4 gv[kGroupsPerLane], rv[kGroupsPerLane];
#pragma unroll
    for (int j = 0; j < kGroupsPerLane; ++j) {
        const int64_t gi = g0 + j * kWarp + lane;
        if (kVec && gi < full_groups) {
            gv[j] = GradLoad<G>::group(grad, gi);
            rv[j] = ld_stream_f4(residual + 4 * gi);
        } else {
            float tg[4], tr[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int64_t e = 4 * gi + k;
                tg[k] = e < n ? GradLoad<G>::one(grad, e) : 0.0f;
                tr[k] = e < n ? ld_stream_f1(residual + e) : 0.0f;
            }
            gv[j] = make_float4(tg[0], tg[1], tg[2], tg[3]);
            rv[j] = make_float4(tr[0], tr[1], tr[2], tr[3]);
        }
    }

#pragma unroll
    for (int j = 0; j < kGroupsPerLane; ++j) {
        const int64_t gi = g0 + j * kWarp + lane;
        float4 r = rv[j];
        const uint32_t c0 = tb_step(gv[j].x, r.x, neg, pos);
        const uint32_t c1 = tb_step(gv[j].y, r.y, neg, pos);
        const uint32_t c2 = tb_step(gv[j].z, r.z, neg, pos);
        const uint32_t c3 = tb_step(gv[j].w, r.w, neg, pos);
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

// Values of the 4 codes in a byte (first element in bits 7..6).
__device__ __forceinline__ float4 tb_decode4(uint32_t byte, float neg, float pos)
{
    return make_float4(tb_value((byte >> 6) & 3u, neg, pos), tb_value((byte >> 4) & 3u, neg, pos),
                       tb_value((byte >> 2) & 3u, neg, pos), tb_value(byte & 3u, neg, pos));
}

// The byte of group slot j of this lane, given the lane's own word of the
// tile (word `lane` of the tile's 32 words).
__device__ __forceinline__ uint32_t tb_group_byte(uint32_t my_word, int j, int lane)
{
    const uint32_t w = __shfl_sync(kFullMask, my_word, j * (kWarp / 4) + (lane >> 2));
    return (w >> (24 - 8 * (lane & 3))) & 0xFFu;
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

// Dequantize tile `tile` of one record.
template <bool kVec>
__device__ __forceinline__ void dequantize_2bit_tile(const uint32_t *__restrict__ payload,
                                                     float *__restrict__ out, int64_t n,
                                                     int64_t tile, float neg, float pos, int lane)
{
    const int64_t nwords = (n + 15) >> 4;
    const int64_t w = tile * kTileWords + lane;
    const uint32_t my_word = w < nwords ? ld_stream_u32(payload + w) : 0u;
#pragma unroll
    for (int j = 0; j < kGroupsPerLane; ++j) {
        const uint32_t byte = tb_group_byte(my_word, j, lane);
        store_group<kVec>(out, n, tile * kTileGroups + j * kWarp + lane, tb_decode4(byte, neg, pos));
    }
}

// Merge of W records for tile `tile`: values summed from +0 in worker order.
//   payload_of(w) -> pointer to worker w's payload (word 3 of its record)
//   neg_of(w), pos_of(w) -> its thresholds
// Words of 8 workers are loaded before any is decoded, so each lane keeps 8
// independent loads in flight.
template <bool kVec, typename PayloadOf, typename NegOf, typename PosOf>
__device__ __forceinline__ void dequant_accumulate_2bit_tile(int W, PayloadOf payload_of,
                                                             NegOf neg_of, PosOf pos_of,
                                                             float *__restrict__ out, int64_t n,
                                                             int64_t tile, int lane)
{
    constexpr int kBatch = 8;
    const int64_t nwords = (n + 15) >> 4;
    const int64_t w_idx = tile * kTileWords + lane;
    const bool in_range = w_idx < nwords;
    float4 acc[kGroupsPerLane];
#pragma unroll
    for (int j = 0; j < kGroupsPerLane; ++j)
        acc[j] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);

    for (int wb = 0; wb < W; wb += kBatch) {
        uint32_t words[kBatch];
#pragma unroll
        for (int k = 0; k < kBatch; ++k)
            words[k] = (wb + k < W && in_range) ? ld_stream_u32(payload_of(wb + k) + w_idx) : 0u;
#pragma unroll
        for (int k = 0; k < kBatch; ++k) {
            if (wb + k < W) { // warp-uniform
                const float neg = neg_of(wb + k), pos = pos_of(wb + k);
#pragma unroll
                for (int j = 0; j < kGroupsPerLane; ++j) {
                    const float4 v = tb_decode4(tb_group_byte(words[k], j, lane), neg, pos);
                    acc[j].x = __fadd_rn(acc[j].x, v.x);
                    acc[j].y = __fadd_rn(acc[j].y, v.y);
                    acc[j].z = __fadd_rn(acc[j].z, v.z);
                    acc[j].w = __fadd_rn(acc[j].w, v.w);
                }
            }
        }
    }
#pragma unroll
    for (int j = 0; j < kGroupsPerLane; ++j)
        store_group<kVec>(out, n, tile * kTileGroups + j * kWarp + lane, acc[j]);
}

} // namespace qga
