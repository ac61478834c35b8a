// qga_local_reduce.cu -- the reducing worker's step of the local kvstore as
// one kernel: quantize its own gradient and merge all W records.
//
// MXNet pull request #8342 "[WIP] 2bit gradient compression", "Local
// kvstore": the device that sums the gradients dequantizes every worker's
// compressed gradient and merges them, and it also quantizes (and so
// error-feeds) its own gradient, so that its own samples are treated like
// every other worker's (the page's reason, and its "Questions", 1).
// Done as two calls, that device's own quantize writes its record and the
// merge reads it straight back.  Here one kernel does both: a warp quantizes
// the words of its slice of the own gradient (residual updated, record words
// written), then merges the slice of all W records in worker order exactly as
// the merge kernel does, so the results are bit for bit those of
// qga_quantize_2bit followed by qga_dequant_accumulate_2bit.  One pass over
// HBM instead of two: 18 bytes per element at W = 8 (read g and r, write r,
// write the own codes, read the other 7 records, write the aggregate)
// against 12.25 + 6.
//
// Geometry: the merge's (a warp owns a slice of 64 words, lane l words l and
// 32 + l).  For the quantize half a lane therefore owns 16 consecutive
// elements per word: two 256-bit loads each of g and r, the 16 codes packed
// in the lane (no shuffle), two 256-bit stores of r.  Each such warp access
// uses every byte of the 32-byte sectors it touches.  The merge half reads
// the own word back from the address this same thread has just written
// (program order makes the value visible to it; the line is still in L2).

#include "qga_2bit_tiles.cuh"

namespace qga {
namespace {

constexpr int kThreads = 256;
constexpr int kWarpsPerBlock = kThreads / kWarp;

// Blocks per SM the register budget is fitted to (64 registers a thread at 4).
// Measured at n = 138M, W = 8: 4 blocks 426 us, 3 blocks 428 us, 2 blocks
// 496 us.  Issuing both words' loads before either is quantized (470-618 us)
// and prefetching the next slice into L2 (570-602 us) were slower; issuing
// the received records' loads before the own quantize changed nothing
// (426 us, at 3 blocks to avoid spills).  More grid waves: 426 / 440 us at 8
// / 32; with one word per lane in the merge slice 432 / 411 / 424 us at 1 /
// 8 / 32 waves (that slice width is shared with the plain and bucket merges).
#ifndef QGA_LOCAL_REDUCE_MIN_BLOCKS
#define QGA_LOCAL_REDUCE_MIN_BLOCKS 4
#endif

struct RecordSet {
    const uint32_t *rec[QGA_MAX_WORKERS];
};

// kW > 0: compiled for exactly kW workers; kW == 0: any W up to QGA_MAX_WORKERS.
template <bool kVec, int kW>
__global__ void __launch_bounds__(kThreads, QGA_LOCAL_REDUCE_MIN_BLOCKS)
    quantize_merge_2bit_kernel(const float *__restrict__ grad, float *__restrict__ residual,
                               int64_t n, float neg, float pos,
                               const __grid_constant__ RecordSet set, int W, int own,
                               float *__restrict__ out)
{
    __shared__ float s_neg[QGA_MAX_WORKERS], s_pos[QGA_MAX_WORKERS];
    __shared__ float2 s_table[QGA_MAX_WORKERS][16];
    __shared__ float4 s_stage[kWarpsPerBlock][kStagePerWarp];
    uint32_t *own_rec = const_cast<uint32_t *>(set.rec[own]);
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        own_rec[0] = bits_from_f32(neg);
        own_rec[1] = bits_from_f32(pos);
        own_rec[2] = bits_from_f32(__ll2float_rn(n));
    }
    // the own thresholds come from the arguments: its header is being
    // written by this same launch
    if (threadIdx.x < W) {
        const uint32_t *r = set.rec[threadIdx.x];
        s_neg[threadIdx.x] = threadIdx.x == own ? neg : f32_from_bits(r[0]);
        s_pos[threadIdx.x] = threadIdx.x == own ? pos : f32_from_bits(r[1]);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < W * 16; i += kThreads)
        s_table[i >> 4][i & 15] = pair_entry(i & 15, s_neg[i >> 4], s_pos[i >> 4]);
    __syncthreads();
    uint32_t *own_payload = own_rec + 3;
    const int lane = threadIdx.x & (kWarp - 1);
    const int64_t nwords = (n + 15) >> 4;
    const int64_t slices = (n + kSliceElems - 1) / kSliceElems;
    const int64_t stride = (int64_t)gridDim.x * kWarpsPerBlock;
    for (int64_t sl = (int64_t)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5); sl < slices;
         sl += stride) {
#pragma unroll
        for (int s = 0; s < kMergeSlots; ++s) {
            const int64_t k = sl * kSliceWords + s * kWarp + lane;
            if (k < nwords) {
                float g[16], r[16];
                load_word<kVec>(grad, residual, n, k, g, r);
                quantize_word<kVec>(residual, own_payload, n, k, neg, pos, g, r);
            }
        }
        dequant_accumulate_2bit_slice<kVec, kW>(
            W, [&](int w) { return set.rec[w] + 3; }, [&](int w) { return s_neg[w]; },
            [&](int w) { return s_pos[w]; }, s_table, out, n, sl, lane, s_stage[threadIdx.x >> 5]);
    }
}

// W <= 8: the same step with the merge through the table of all 3^W sums
// (build_sum_table, merge_2bit_table_*).  The received records' words of a
// slice are loaded first, so they are in flight while the lane quantizes
// its own words; the own word goes from the register straight into the
// table index (it is stored too, and never read back).
// Blocks per SM the table kernel's registers are fitted to: 3 spill (435 us
// against 404 us at 2, n = 138M, W = 8).
#ifndef QGA_LOCAL_REDUCE_TABLE_MIN_BLOCKS
#define QGA_LOCAL_REDUCE_TABLE_MIN_BLOCKS 1
#endif

template <bool kVec, int kW>
__global__ void __launch_bounds__(kThreads, QGA_LOCAL_REDUCE_TABLE_MIN_BLOCKS)
    quantize_merge_2bit_table_kernel(const float *__restrict__ grad, float *__restrict__ residual,
                                     int64_t n, float neg, float pos,
                                     const __grid_constant__ RecordSet set, int own,
                                     uint32_t *__restrict__ own_rec, float *__restrict__ out)
{
    __shared__ float s_neg[kW], s_pos[kW];
    __shared__ float s_sum[Pow3<kW>::value];
    __shared__ float4 s_stage[kWarpsPerBlock][kWarp * 4];
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        own_rec[0] = bits_from_f32(neg);
        own_rec[1] = bits_from_f32(pos);
        own_rec[2] = bits_from_f32(__ll2float_rn(n));
    }
    if (threadIdx.x < kW) {
        const uint32_t *r = set.rec[threadIdx.x];
        s_neg[threadIdx.x] = (int)threadIdx.x == own ? neg : f32_from_bits(r[0]);
        s_pos[threadIdx.x] = (int)threadIdx.x == own ? pos : f32_from_bits(r[1]);
    }
    __syncthreads();
    build_sum_table<kW>(s_sum, [&](int w) { return s_neg[w]; }, [&](int w) { return s_pos[w]; });
    uint32_t *own_payload = own_rec + 3;
    const int lane = threadIdx.x & (kWarp - 1);
    const int64_t nwords = (n + 15) >> 4;
    const int64_t slices = (n + kTableSliceElems - 1) / kTableSliceElems;
    const int64_t stride = (int64_t)gridDim.x * kWarpsPerBlock;
    for (int64_t sl = (int64_t)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5); sl < slices;
         sl += stride) {
        uint32_t wd[kTableSlots][kTableMaxWorkers];
        merge_2bit_table_load<kW, kTableSlots>([&](int w) { return set.rec[w] + 3; }, nwords, sl, lane,
                                               own, wd);
#pragma unroll
        for (int s = 0; s < kTableSlots; ++s) {
            const int64_t k = (sl * kTableSlots + s) * kWarp + lane;
            uint32_t word = 0u;
            if (k < nwords) {
                float g[16], r[16];
                load_word<kVec>(grad, residual, n, k, g, r);
                word = quantize_word<kVec>(residual, own_payload, n, k, neg, pos, g, r);
            }
            // the own worker's load was skipped (its slot holds 0); a register
            // array is indexed by constants only, so the word is or-ed in by mask
#pragma unroll
            for (int w = 0; w < kW; ++w)
                wd[s][w] |= word & (0u - (uint32_t)(w == own));
        }
        merge_2bit_table_store<kVec, kW, kTableSlots>(wd, s_sum, out, n, sl, lane,
                                                      s_stage[threadIdx.x >> 5]);
    }
}

std::atomic<int> occ_lr[2][9][64]; // [vec][kW][device]

#ifndef QGA_LOCAL_REDUCE_WAVES
#define QGA_LOCAL_REDUCE_WAVES 1
#endif

template <bool kVec, int kW>
void launch_k(const float *grad, float *residual, int64_t n, float neg, float pos,
              const RecordSet &set, int W, int own, float *out, cudaStream_t stream)
{
    if constexpr (kW > 0) {
        auto k = quantize_merge_2bit_table_kernel<kVec, kW>;
        const int64_t slices = (n + kTableSliceElems - 1) / kTableSliceElems;
        const unsigned grid = grid_for((slices + kWarpsPerBlock - 1) / kWarpsPerBlock,
                                       resident_blocks(k, kThreads, occ_lr[kVec][kW]),
                                       QGA_LOCAL_REDUCE_WAVES);
        k<<<grid, kThreads, 0, stream>>>(grad, residual, n, neg, pos, set, own,
                                         const_cast<uint32_t *>(set.rec[own]), out);
    } else {
        auto k = quantize_merge_2bit_kernel<kVec, 0>;
        const int64_t slices = (n + kSliceElems - 1) / kSliceElems;
        const unsigned grid = grid_for((slices + kWarpsPerBlock - 1) / kWarpsPerBlock,
                                       resident_blocks(k, kThreads, occ_lr[kVec][0]));
        k<<<grid, kThreads, 0, stream>>>(grad, residual, n, neg, pos, set, W, own, out);
    }
}

template <bool kVec>
void launch_v(const float *grad, float *residual, int64_t n, float neg, float pos,
              const RecordSet &set, int W, int own, float *out, cudaStream_t stream)
{
    switch (W) {
    case 1: launch_k<kVec, 1>(grad, residual, n, neg, pos, set, W, own, out, stream); break;
    case 2: launch_k<kVec, 2>(grad, residual, n, neg, pos, set, W, own, out, stream); break;
    case 3: launch_k<kVec, 3>(grad, residual, n, neg, pos, set, W, own, out, stream); break;
    case 4: launch_k<kVec, 4>(grad, residual, n, neg, pos, set, W, own, out, stream); break;
    case 5: launch_k<kVec, 5>(grad, residual, n, neg, pos, set, W, own, out, stream); break;
    case 6: launch_k<kVec, 6>(grad, residual, n, neg, pos, set, W, own, out, stream); break;
    case 7: launch_k<kVec, 7>(grad, residual, n, neg, pos, set, W, own, out, stream); break;
    case 8: launch_k<kVec, 8>(grad, residual, n, neg, pos, set, W, own, out, stream); break;
    default: launch_k<kVec, 0>(grad, residual, n, neg, pos, set, W, own, out, stream); break;
    }
}

} // namespace
} // namespace qga

using namespace qga;

extern "C" int qga_quantize_merge_2bit(const float *grad, float *residual, int64_t n,
                                       float neg_threshold, float pos_threshold,
                                       uint32_t *const *compr, int num_workers, int own,
                                       float *out, cudaStream_t stream)
{
    if (n < 0 || compr == nullptr || num_workers < 1 || num_workers > QGA_MAX_WORKERS ||
        own < 0 || own >= num_workers || !finite_f32(neg_threshold) || !finite_f32(pos_threshold))
        return QGA_ERR_INVALID_ARG;
    RecordSet set{};
    for (int w = 0; w < num_workers; ++w) {
        if (compr[w] == nullptr || !aligned(compr[w], 4))
            return QGA_ERR_INVALID_ARG;
        set.rec[w] = compr[w];
    }
    if (n > 0 && (grad == nullptr || residual == nullptr || out == nullptr || !aligned(grad, 4) ||
                  !aligned(residual, 4) || !aligned(out, 4)))
        return QGA_ERR_INVALID_ARG;
    const bool vec = aligned(grad, 32) && aligned(residual, 32) && aligned(out, 16);
    if (vec)
        launch_v<true>(grad, residual, n, neg_threshold, pos_threshold, set, num_workers, own, out,
                       stream);
    else
        launch_v<false>(grad, residual, n, neg_threshold, pos_threshold, set, num_workers, own, out,
                        stream);
    return launch_status();
}
