// qga_2bit.cu -- single-tensor 2-bit threshold kernels and their C ABI:
// quantize (fp32 / bf16 gradient), dequantize, and the W-worker merge.
//
// MXNet pull request #8342 "[WIP] 2bit gradient compression": "Operators"
// (create_2bit / quantize_2bit / dequantize_2bit), "Format of compressed
// gradient" (header [neg, pos, n] then 16 codes per word) and "Local kvstore"
// (the receiver dequantizes every worker's gradient and sums them).
//
// Each kernel is one pass over HBM: warps stride over tiles (512 elements
// for an fp32 quantize or a dequantize, 1024 for a bf16 quantize or a merge
// slice) on a grid of a few waves of resident blocks, the count measured
// best for each kernel (see grid_for).  Nothing is filled
// or cleared by a separate launch: the quantize kernel writes every payload
// word (including the zero tail codes) and its block 0 writes the header.
// The merge's occupancy and words per lane are build-time settings
// (QGA_MERGE_MIN_BLOCKS, QGA_MERGE_SLOTS); the defaults are the measured best.

#include "qga_2bit_tiles.cuh"

namespace qga {
namespace {

constexpr int kThreads = 256;
constexpr int kWarpsPerBlock = kThreads / kWarp;

__device__ __forceinline__ int64_t first_tile() { return (int64_t)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5); }
__device__ __forceinline__ int64_t tile_stride() { return (int64_t)gridDim.x * kWarpsPerBlock; }

template <typename G, bool kVec>
__global__ void __launch_bounds__(kThreads)
    quantize_2bit_kernel(const G *__restrict__ grad, float *__restrict__ residual,
                         uint32_t *__restrict__ compr, int64_t n, float neg, float pos)
{
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        compr[0] = bits_from_f32(neg);
        compr[1] = bits_from_f32(pos);
        compr[2] = bits_from_f32(__ll2float_rn(n));
    }
    const int lane = threadIdx.x & (kWarp - 1);
    constexpr int64_t kElems = quantize_tile_elems<G>();
    const int64_t tiles = (n + kElems - 1) / kElems;
    for (int64_t t = first_tile(); t < tiles; t += tile_stride())
        quantize_2bit_tile<G, kVec>(grad, residual, compr + 3, n, t, neg, pos, lane);
}

// fp32 quantize in lane-owned words (gradient and residual 32-byte aligned):
// warp t of the grid owns words 32 t .. 32 t + 31, one per lane.
__global__ void __launch_bounds__(kThreads)
    quantize_2bit_words_kernel(const float *__restrict__ grad, float *__restrict__ residual,
                               uint32_t *__restrict__ compr, int64_t n, float neg, float pos)
{
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        compr[0] = bits_from_f32(neg);
        compr[1] = bits_from_f32(pos);
        compr[2] = bits_from_f32(__ll2float_rn(n));
    }
    const int lane = threadIdx.x & (kWarp - 1);
    const int64_t nwords = (n + 15) >> 4;
    const int64_t runs = (nwords + kWarp - 1) / kWarp;
    for (int64_t t = first_tile(); t < runs; t += tile_stride()) {
        const int64_t k = t * kWarp + lane;
        if (k < nwords) {
            float g[16], r[16];
            load_word<true>(grad, residual, n, k, g, r);
            quantize_word<true>(residual, compr + 3, n, k, neg, pos, g, r);
        }
    }
}

template <bool kVec>
__global__ void __launch_bounds__(kThreads)
    dequantize_2bit_kernel(const uint32_t *__restrict__ compr, float *__restrict__ out, int64_t n)
{
    const float neg = f32_from_bits(compr[0]);
    const float pos = f32_from_bits(compr[1]);
    const int lane = threadIdx.x & (kWarp - 1);
    const int64_t tiles = (n + kTileElems - 1) / kTileElems;
    for (int64_t t = first_tile(); t < tiles; t += tile_stride())
        dequantize_2bit_tile<kVec>(compr + 3, out, n, t, neg, pos, lane);
}

struct RecordSet {
    const uint32_t *rec[QGA_MAX_WORKERS];
};

// kW > 0: compiled for exactly kW workers (record pointers and loop bounds
// are constants); kW == 0: any W up to QGA_MAX_WORKERS.
#ifndef QGA_MERGE_MIN_BLOCKS
#define QGA_MERGE_MIN_BLOCKS 4
#endif

template <bool kVec, int kW>
__global__ void __launch_bounds__(kThreads, QGA_MERGE_MIN_BLOCKS)
    dequant_accumulate_2bit_kernel(const __grid_constant__ RecordSet set, int W,
                                   float *__restrict__ out, int64_t n)
{
    __shared__ const uint32_t *s_payload[QGA_MAX_WORKERS];
    __shared__ float s_neg[QGA_MAX_WORKERS], s_pos[QGA_MAX_WORKERS];
    __shared__ float2 s_table[QGA_MAX_WORKERS][16];
    __shared__ float4 s_stage[kWarpsPerBlock][kStagePerWarp];
    if (threadIdx.x < W) {
        const uint32_t *r = set.rec[threadIdx.x];
        s_payload[threadIdx.x] = r + 3;
        s_neg[threadIdx.x] = f32_from_bits(r[0]);
        s_pos[threadIdx.x] = f32_from_bits(r[1]);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < W * 16; i += kThreads)
        s_table[i >> 4][i & 15] = pair_entry(i & 15, s_neg[i >> 4], s_pos[i >> 4]);
    __syncthreads();
    const int lane = threadIdx.x & (kWarp - 1);
    const int64_t slices = (n + kSliceElems - 1) / kSliceElems;
    for (int64_t sl = first_tile(); sl < slices; sl += tile_stride()) {
        if (kW > 0)
            dequant_accumulate_2bit_slice<kVec, kW>(
                W, [&](int w) { return set.rec[w] + 3; }, [&](int w) { return s_neg[w]; },
                [&](int w) { return s_pos[w]; }, s_table, out, n, sl, lane, s_stage[threadIdx.x >> 5]);
        else
            dequant_accumulate_2bit_slice<kVec, 0>(
                W, [&](int w) { return s_payload[w]; }, [&](int w) { return s_neg[w]; },
                [&](int w) { return s_pos[w]; }, s_table, out, n, sl, lane, s_stage[threadIdx.x >> 5]);
    }
}

// W <= 8: the merge through the table of all 3^W sums (build_sum_table,
// merge_2bit_table_store): one table index and one shared-memory load per
// element instead of W decodes and adds.  A lane owns one word of each of
// its warp's slices (32 words, 512 elements), and the W words of the next
// slice are already in flight while the current one is summed and stored;
// the first slice's words are loaded before the table is built.  The table
// (26 KB at W = 8) and the per-warp 2 KB output stage fit 4 blocks per SM,
// which leaves the SM's L1 room for the loads in flight (5 blocks left too
// little: 182 us).  Measured at n = 138M, W = 8: 139.2 us, against 145.5 us
// for two words per lane loaded just before use.
constexpr int64_t kMergeSliceElems = (int64_t)kWarp * 16;

template <bool kVec, int kW>
__global__ void __launch_bounds__(kThreads, 4)
    merge_2bit_table_kernel(const __grid_constant__ RecordSet set, float *__restrict__ out, int64_t n)
{
    __shared__ float s_neg[kW], s_pos[kW];
    __shared__ float s_sum[Pow3<kW>::value];
    __shared__ float4 s_stage[kWarpsPerBlock][kWarp * 4];
    if (threadIdx.x < kW) {
        const uint32_t *r = set.rec[threadIdx.x];
        s_neg[threadIdx.x] = f32_from_bits(r[0]);
        s_pos[threadIdx.x] = f32_from_bits(r[1]);
    }
    const int lane = threadIdx.x & (kWarp - 1);
    const int64_t nwords = (n + 15) >> 4;
    const int64_t slices = (n + kMergeSliceElems - 1) / kMergeSliceElems;
    auto payload_of = [&](int w) { return set.rec[w] + 3; };
    int64_t sl = first_tile();
    uint32_t wd[1][kTableMaxWorkers];
    if (sl < slices)
        merge_2bit_table_load<kW, 1>(payload_of, nwords, sl, lane, -1, wd);
    __syncthreads();
    build_sum_table<kW>(s_sum, [&](int w) { return s_neg[w]; }, [&](int w) { return s_pos[w]; });
    for (; sl < slices; sl += tile_stride()) {
        uint32_t next[1][kTableMaxWorkers];
        if (sl + tile_stride() < slices)
            merge_2bit_table_load<kW, 1>(payload_of, nwords, sl + tile_stride(), lane, -1, next);
        else
#pragma unroll
            for (int w = 0; w < kTableMaxWorkers; ++w)
                next[0][w] = 0u;
        merge_2bit_table_store<kVec, kW, 1>(wd, s_sum, out, n, sl, lane, s_stage[threadIdx.x >> 5]);
#pragma unroll
        for (int w = 0; w < kTableMaxWorkers; ++w)
            wd[0][w] = next[0][w];
    }
}

std::atomic<int> occ_q_f32_w[64], occ_q_f32_v[64], occ_q_f32_s[64], occ_q_bf16_v[64], occ_q_bf16_s[64];
std::atomic<int> occ_dq_v[64], occ_dq_s[64];
std::atomic<int> occ_acc[2][64];    // [vec][device]: W > 8
std::atomic<int> occ_tab[2][9][64]; // [vec][kW][device]: W <= 8

// Grid waves (see grid_for), measured at n = 138M: quantize in group tiles
// 270-286 / 263 / 259 / 256 / 258 us at 1 / 8 / 16 / 32 / 128 waves, in
// lane-owned words 252 / 243 us at 8 / 32 waves (2 words per lane: 253 /
// 256); dequantize 109 / 97 / 96 / 101 us at 1 / 8 / 16 / 32; merge (W = 8)
// 180 / 174 / 176 / 181 us at 1 / 8 / 16 / 32.
constexpr int kQuantizeWaves = 32, kDequantizeWaves = 16, kMergeWaves = 8;
// The table merge by worker count: every block builds the 3^W-entry table
// once, so small tables take many waves and large ones one persistent wave.
// Measured at n = 138M (us at 1 / 2 / 4 / 8 / 16 waves): W = 1 108 / 103 /
// 97 / 95 / 93, W = 2 115 / 112 / 104 / 99 / 98, W = 3 121 / 118 / 110 / 105
// / 103, W = 4 127 / 123 / 115 / 111 / 112, W = 5 120 / 119 / 119 / 119 /
// 121, W = 6 126 / 127 / 127 / 132 / 138, W = 7 131 / 132 / 133 / 136 / 144,
// W = 8 142 / 142 / 144 / 152 / 169.
#ifdef QGA_TABLE_MERGE_WAVES
constexpr int table_merge_waves(int) { return QGA_TABLE_MERGE_WAVES; }
#else
constexpr int table_merge_waves(int w) { return w <= 3 ? 16 : (w == 4 ? 8 : (w == 5 ? 2 : 1)); }
#endif

unsigned tiles_grid(int64_t n, int resident, int64_t elems_per_warp, int waves)
{
    const int64_t tiles = (n + elems_per_warp - 1) / elems_per_warp;
    return grid_for((tiles + kWarpsPerBlock - 1) / kWarpsPerBlock, resident, waves);
}

template <bool kVec, int kW>
void launch_merge_k(const RecordSet &set, int W, float *out, int64_t n, cudaStream_t stream)
{
    if constexpr (kW > 0) {
        auto k = merge_2bit_table_kernel<kVec, kW>;
        k<<<tiles_grid(n, resident_blocks(k, kThreads, occ_tab[kVec][kW]), kMergeSliceElems,
                       table_merge_waves(kW)),
            kThreads, 0, stream>>>(set, out, n);
    } else {
        auto k = dequant_accumulate_2bit_kernel<kVec, 0>;
        k<<<tiles_grid(n, resident_blocks(k, kThreads, occ_acc[kVec]), kSliceElems, kMergeWaves),
            kThreads, 0, stream>>>(set, W, out, n);
    }
}

template <bool kVec>
void launch_merge_v(const RecordSet &set, int W, float *out, int64_t n, cudaStream_t stream)
{
    switch (W) {
    case 1: launch_merge_k<kVec, 1>(set, W, out, n, stream); break;
    case 2: launch_merge_k<kVec, 2>(set, W, out, n, stream); break;
    case 3: launch_merge_k<kVec, 3>(set, W, out, n, stream); break;
    case 4: launch_merge_k<kVec, 4>(set, W, out, n, stream); break;
    case 5: launch_merge_k<kVec, 5>(set, W, out, n, stream); break;
    case 6: launch_merge_k<kVec, 6>(set, W, out, n, stream); break;
    case 7: launch_merge_k<kVec, 7>(set, W, out, n, stream); break;
    case 8: launch_merge_k<kVec, 8>(set, W, out, n, stream); break;
    default: launch_merge_k<kVec, 0>(set, W, out, n, stream); break;
    }
}

void launch_merge(const RecordSet &set, int W, float *out, int64_t n, cudaStream_t stream, bool vec)
{
    if (vec)
        launch_merge_v<true>(set, W, out, n, stream);
    else
        launch_merge_v<false>(set, W, out, n, stream);
}

template <typename G>
int launch_quantize(const G *grad, float *residual, uint32_t *compr, int64_t n, float neg, float pos,
                    cudaStream_t stream, std::atomic<int> *occ_v, std::atomic<int> *occ_s,
                    std::atomic<int> *occ_w = nullptr)
{
    if (n < 0 || compr == nullptr || !aligned(compr, 4) || !finite_f32(neg) || !finite_f32(pos))
        return QGA_ERR_INVALID_ARG;
    if (n > 0 && (grad == nullptr || residual == nullptr || !aligned(grad, sizeof(G)) ||
                  !aligned(residual, 4)))
        return QGA_ERR_INVALID_ARG;
    const bool vec = aligned(grad, GradLoad<G>::kVecAlign) && aligned(residual, 16);
    constexpr int64_t kElems = quantize_tile_elems<G>();
    if constexpr (sizeof(G) == sizeof(float)) {
        if (aligned(grad, 32) && aligned(residual, 32)) {
            auto k = quantize_2bit_words_kernel;
            k<<<tiles_grid(n, resident_blocks(k, kThreads, occ_w), 16 * kWarp, kQuantizeWaves),
                kThreads, 0, stream>>>(grad, residual, compr, n, neg, pos);
            return launch_status();
        }
    }
    if (vec) {
        auto k = quantize_2bit_kernel<G, true>;
        k<<<tiles_grid(n, resident_blocks(k, kThreads, occ_v), kElems, kQuantizeWaves), kThreads, 0,
            stream>>>(
            grad, residual, compr, n, neg, pos);
    } else {
        auto k = quantize_2bit_kernel<G, false>;
        k<<<tiles_grid(n, resident_blocks(k, kThreads, occ_s), kElems, kQuantizeWaves), kThreads, 0,
            stream>>>(
            grad, residual, compr, n, neg, pos);
    }
    return launch_status();
}

} // namespace
} // namespace qga

using namespace qga;

extern "C" int64_t qga_2bit_words(int64_t n)
{
    if (n < 0)
        return QGA_ERR_INVALID_ARG;
    return 3 + (n + 15) / 16;
}

extern "C" int qga_quantize_2bit(const float *grad, float *residual, uint32_t *compr, int64_t n,
                                 float neg_threshold, float pos_threshold, cudaStream_t stream)
{
    return launch_quantize<float>(grad, residual, compr, n, neg_threshold, pos_threshold, stream,
                                  occ_q_f32_v, occ_q_f32_s, occ_q_f32_w);
}

extern "C" int qga_quantize_2bit_bf16(const uint16_t *grad, float *residual, uint32_t *compr,
                                      int64_t n, float neg_threshold, float pos_threshold,
                                      cudaStream_t stream)
{
    return launch_quantize<uint16_t>(grad, residual, compr, n, neg_threshold, pos_threshold,
                                     stream, occ_q_bf16_v, occ_q_bf16_s);
}

extern "C" int qga_dequantize_2bit(const uint32_t *compr, float *out, int64_t n,
                                   cudaStream_t stream)
{
    if (n < 0 || compr == nullptr || !aligned(compr, 4))
        return QGA_ERR_INVALID_ARG;
    if (n == 0)
        return QGA_OK;
    if (out == nullptr || !aligned(out, 4))
        return QGA_ERR_INVALID_ARG;
    if (aligned(out, 16)) {
        auto k = dequantize_2bit_kernel<true>;
        k<<<tiles_grid(n, resident_blocks(k, kThreads, occ_dq_v), kTileElems, kDequantizeWaves),
            kThreads, 0, stream>>>(compr, out, n);
    } else {
        auto k = dequantize_2bit_kernel<false>;
        k<<<tiles_grid(n, resident_blocks(k, kThreads, occ_dq_s), kTileElems, kDequantizeWaves),
            kThreads, 0, stream>>>(compr, out, n);
    }
    return launch_status();
}

extern "C" int qga_dequant_accumulate_2bit(const uint32_t *const *compr, int num_workers,
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
    launch_merge(set, num_workers, out, n, stream, aligned(out, 16));
    return launch_status();
}
