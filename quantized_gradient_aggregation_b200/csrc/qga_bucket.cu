// qga_bucket.cu -- the ragged bucket launcher: T tensors of different sizes,
// each with its own thresholds, quantized (or merged) in ONE launch.
//
// The compressed bucket is the T standalone records of MXNet pull request
// #8342 "[WIP] 2bit gradient compression" ("Format of compressed gradient")
// one after the other, so a bucket can be split back into per-tensor records
// without copying.
//
// Work distribution.  Each tensor is cut into chunks (8192 elements for the
// quantizer, 32768 for the merge, whose blocks rebuild a per-worker table at
// every chunk; a tensor of n = 0 still owns one quantizer chunk, which writes
// its header).  The host numbers the chunks of all tensors consecutively and
// passes the descriptor table BY VALUE as a kernel parameter (no device
// table, no allocation, no copy): the grid strides over the chunk
// numbers, and each block finds its tensor by a binary search over the
// table's first-chunk column.  Tables over 256 tensors are split into
// several launches.

#include "qga_2bit_tiles.cuh"

namespace qga {
namespace {

constexpr int kThreads = 256;
constexpr int kWarpsPerBlock = kThreads / kWarp;
constexpr int64_t kChunkElems = 8192;       // quantize: a whole number of quantize tiles
constexpr int64_t kMergeChunkElems = 32768; // merge: 4 slices per warp between block barriers
constexpr int kMaxRows = 256;

struct QuantRow {
    const void *grad;
    float *residual;
    int64_t n;
    int64_t word_off;    // record start within the compressed bucket
    int64_t chunk_begin; // number of this tensor's first chunk within the launch
    float neg, pos;
    int vec;             // grad and residual aligned for vector access
};

struct QuantTable {
    int T;
    int64_t total_chunks;
    QuantRow row[kMaxRows];
};

struct MergeRow {
    int64_t n;
    int64_t word_off;
    int64_t elem_off;    // offset of the tensor within the merged output
    int64_t chunk_begin;
    int vec;
};

struct MergeTable {
    int T;
    int W;
    int64_t total_chunks;
    const uint32_t *bucket[QGA_MAX_WORKERS];
    MergeRow row[kMaxRows];
};

// Largest t with chunk_begin[t] <= chunk: the tensor owning `chunk` (a
// tensor with no chunks shares its first-chunk number with the next one and
// is never chosen).
template <typename Table>
__device__ __forceinline__ int owner_row(const Table &tab, int64_t chunk)
{
    int lo = 0, hi = tab.T - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (tab.row[mid].chunk_begin <= chunk)
            lo = mid;
        else
            hi = mid - 1;
    }
    return lo;
}

// kAllVec: every row of the table is aligned for vector access (the common
// case; only the vector path is compiled in, which keeps registers low).
template <typename G, bool kAllVec>
__global__ void __launch_bounds__(kThreads, 3)
    quantize_2bit_bucket_kernel(const __grid_constant__ QuantTable tab, uint32_t *__restrict__ compr)
{
    const int lane = threadIdx.x & (kWarp - 1);
    const int warp = threadIdx.x >> 5;
    for (int64_t chunk = blockIdx.x; chunk < tab.total_chunks; chunk += gridDim.x) {
        const QuantRow &row = tab.row[owner_row(tab, chunk)];
        const int64_t c = chunk - row.chunk_begin;
        uint32_t *rec = compr + row.word_off;
        if (c == 0 && threadIdx.x == 0) {
            rec[0] = bits_from_f32(row.neg);
            rec[1] = bits_from_f32(row.pos);
            rec[2] = bits_from_f32(__ll2float_rn(row.n));
        }
        constexpr int64_t kTile = quantize_tile_elems<G>();
        constexpr int64_t kChunkTiles = kChunkElems / kTile;
        const int64_t tiles = (row.n + kTile - 1) / kTile;
        const int64_t t_end = min((c + 1) * kChunkTiles, tiles);
        const G *grad = static_cast<const G *>(row.grad);
        if (kAllVec || row.vec) {
            for (int64_t t = c * kChunkTiles + warp; t < t_end; t += kWarpsPerBlock)
                quantize_2bit_tile<G, true>(grad, row.residual, rec + 3, row.n, t, row.neg, row.pos, lane);
        } else {
            for (int64_t t = c * kChunkTiles + warp; t < t_end; t += kWarpsPerBlock)
                quantize_2bit_tile<G, false>(grad, row.residual, rec + 3, row.n, t, row.neg, row.pos, lane);
        }
    }
}

// kW > 0: compiled for exactly kW workers; kW == 0: any W up to QGA_MAX_WORKERS.
template <int kW>
__global__ void __launch_bounds__(kThreads, 3)
    dequant_accumulate_2bit_bucket_kernel(const __grid_constant__ MergeTable tab, float *__restrict__ out)
{
    __shared__ const uint32_t *s_payload[QGA_MAX_WORKERS];
    __shared__ float s_neg[QGA_MAX_WORKERS], s_pos[QGA_MAX_WORKERS];
    __shared__ float2 s_table[QGA_MAX_WORKERS][16];
    __shared__ float4 s_stage[kWarpsPerBlock][kStagePerWarp];
    constexpr int64_t kChunkSlices = kMergeChunkElems / kSliceElems;
    const int lane = threadIdx.x & (kWarp - 1);
    const int warp = threadIdx.x >> 5;
    for (int64_t chunk = blockIdx.x; chunk < tab.total_chunks; chunk += gridDim.x) {
        const MergeRow &row = tab.row[owner_row(tab, chunk)];
        const int64_t c = chunk - row.chunk_begin;
        __syncthreads(); // the previous chunk's readers of s_* are done
        if (threadIdx.x < tab.W) {
            const uint32_t *rec = tab.bucket[threadIdx.x] + row.word_off;
            s_payload[threadIdx.x] = rec + 3;
            s_neg[threadIdx.x] = f32_from_bits(rec[0]);
            s_pos[threadIdx.x] = f32_from_bits(rec[1]);
        }
        __syncthreads();
        for (int i = threadIdx.x; i < tab.W * 16; i += kThreads)
            s_table[i >> 4][i & 15] = pair_entry(i & 15, s_neg[i >> 4], s_pos[i >> 4]);
        __syncthreads();
        const int64_t slices = (row.n + kSliceElems - 1) / kSliceElems;
        const int64_t s_end = min((c + 1) * kChunkSlices, slices);
        float *o = out + row.elem_off;
        auto payload_of = [&](int w) { return s_payload[w]; };
        auto neg_of = [&](int w) { return s_neg[w]; };
        auto pos_of = [&](int w) { return s_pos[w]; };
        float4 *stage = s_stage[warp];
        if (row.vec) {
            for (int64_t sl = c * kChunkSlices + warp; sl < s_end; sl += kWarpsPerBlock)
                dequant_accumulate_2bit_slice<true, kW>(tab.W, payload_of, neg_of, pos_of, s_table, o, row.n, sl,
                                                    lane, stage);
        } else {
            for (int64_t sl = c * kChunkSlices + warp; sl < s_end; sl += kWarpsPerBlock)
                dequant_accumulate_2bit_slice<false, kW>(tab.W, payload_of, neg_of, pos_of, s_table, o, row.n, sl,
                                                     lane, stage);
        }
    }
}

// W <= 8: each chunk's tensor merged through the table of its 3^W sums
// (build_sum_table, merge_2bit_table_load / _store); the table is rebuilt
// only when the block moves on to a chunk of another tensor.  The W payload
// pointers of the chunk's tensor are held in registers, and with
// QGA_BUCKET_MERGE_PREFETCH a warp's next slice of the chunk is loaded
// before the current one is summed and stored.  Measured on the BERT-Base
// bucket (W = 4): 2 words per lane 92.2 us, with the next slice in flight
// 92.5 us; 1 word per lane 97.7 / 96.0 us; 16 waves no change.
#ifndef QGA_BUCKET_MERGE_PREFETCH
#define QGA_BUCKET_MERGE_PREFETCH 0
#endif
#ifndef QGA_BUCKET_MERGE_SLOTS
#define QGA_BUCKET_MERGE_SLOTS 2
#endif
constexpr int kBucketSlots = QGA_BUCKET_MERGE_SLOTS;
constexpr int64_t kBucketSliceElems = (int64_t)kWarp * kBucketSlots * 16;

template <bool kVec, int kW>
__device__ __forceinline__ void merge_chunk_slices(const uint32_t *const (&pl)[kW], const float *T, float *o,
                                                   int64_t n, int64_t s_begin, int64_t s_end, int lane,
                                                   float4 *stage)
{
    const int64_t nwords = (n + 15) >> 4;
    auto payload_of = [&](int w) { return pl[w < kW ? w : 0]; };
    uint32_t wd[kBucketSlots][kTableMaxWorkers];
    int64_t sl = s_begin;
    if (QGA_BUCKET_MERGE_PREFETCH && sl < s_end)
        merge_2bit_table_load<kW, kBucketSlots>(payload_of, nwords, sl, lane, -1, wd);
    for (; sl < s_end; sl += kWarpsPerBlock) {
        if (QGA_BUCKET_MERGE_PREFETCH) {
            uint32_t next[kBucketSlots][kTableMaxWorkers];
            if (sl + kWarpsPerBlock < s_end)
                merge_2bit_table_load<kW, kBucketSlots>(payload_of, nwords, sl + kWarpsPerBlock, lane, -1, next);
            else
#pragma unroll
                for (int s = 0; s < kBucketSlots; ++s)
#pragma unroll
                    for (int w = 0; w < kTableMaxWorkers; ++w)
                        next[s][w] = 0u;
            merge_2bit_table_store<kVec, kW, kBucketSlots>(wd, T, o, n, sl, lane, stage);
#pragma unroll
            for (int s = 0; s < kBucketSlots; ++s)
#pragma unroll
                for (int w = 0; w < kTableMaxWorkers; ++w)
                    wd[s][w] = next[s][w];
        } else {
            merge_2bit_table_load<kW, kBucketSlots>(payload_of, nwords, sl, lane, -1, wd);
            merge_2bit_table_store<kVec, kW, kBucketSlots>(wd, T, o, n, sl, lane, stage);
        }
    }
}

template <int kW>
__global__ void __launch_bounds__(kThreads)
    merge_2bit_table_bucket_kernel(const __grid_constant__ MergeTable tab, float *__restrict__ out)
{
    __shared__ const uint32_t *s_payload[kW];
    __shared__ float s_neg[kW], s_pos[kW];
    __shared__ float s_sum[Pow3<kW>::value];
    __shared__ float4 s_stage[kWarpsPerBlock][kWarp * 4];
    static_assert(kMergeChunkElems % kBucketSliceElems == 0, "whole slices per chunk");
    constexpr int64_t kChunkSlices = kMergeChunkElems / kBucketSliceElems;
    const int lane = threadIdx.x & (kWarp - 1);
    const int warp = threadIdx.x >> 5;
    int loaded = -1; // the row whose table is in shared memory (block-uniform)
    const uint32_t *pl[kW];
    for (int64_t chunk = blockIdx.x; chunk < tab.total_chunks; chunk += gridDim.x) {
        const int t = owner_row(tab, chunk);
        const MergeRow &row = tab.row[t];
        if (t != loaded) {
            __syncthreads(); // the previous tensor's readers of s_* are done
            if (threadIdx.x < kW) {
                const uint32_t *rec = tab.bucket[threadIdx.x] + row.word_off;
                s_payload[threadIdx.x] = rec + 3;
                s_neg[threadIdx.x] = f32_from_bits(rec[0]);
                s_pos[threadIdx.x] = f32_from_bits(rec[1]);
            }
            __syncthreads();
            build_sum_table<kW>(s_sum, [&](int w) { return s_neg[w]; }, [&](int w) { return s_pos[w]; });
#pragma unroll
            for (int w = 0; w < kW; ++w)
                pl[w] = s_payload[w];
            loaded = t;
        }
        const int64_t c = chunk - row.chunk_begin;
        const int64_t slices = (row.n + kBucketSliceElems - 1) / kBucketSliceElems;
        const int64_t s_end = min((c + 1) * kChunkSlices, slices);
        float *o = out + row.elem_off;
        if (row.vec)
            merge_chunk_slices<true, kW>(pl, s_sum, o, row.n, c * kChunkSlices + warp, s_end, lane, s_stage[warp]);
        else
            merge_chunk_slices<false, kW>(pl, s_sum, o, row.n, c * kChunkSlices + warp, s_end, lane, s_stage[warp]);
    }
}

std::atomic<int> occ_qb_f32[2][64], occ_qb_bf16[2][64], occ_ab[9][64];

// Grid waves (see grid_for), measured on the BERT-Base bucket: bf16 quantize
// 186 / 175 / 171 / 173 us at 1 / 8 / 16 / 32 waves; 4-worker merge 113 /
// 109 / 109 us at 1 / 8 / 16.
#ifndef QGA_BUCKET_MERGE_WAVES
#define QGA_BUCKET_MERGE_WAVES 8
#endif
constexpr int kBucketQuantizeWaves = 16, kBucketMergeWaves = QGA_BUCKET_MERGE_WAVES;

template <int kW>
void launch_bucket_merge(const MergeTable &tab, float *out, cudaStream_t stream)
{
    if constexpr (kW > 0) {
        auto kernel = merge_2bit_table_bucket_kernel<kW>;
        const int resident = resident_blocks(kernel, kThreads, occ_ab[kW]);
        kernel<<<grid_for(tab.total_chunks, resident, kBucketMergeWaves), kThreads, 0, stream>>>(tab, out);
    } else {
        auto kernel = dequant_accumulate_2bit_bucket_kernel<0>;
        const int resident = resident_blocks(kernel, kThreads, occ_ab[0]);
        kernel<<<grid_for(tab.total_chunks, resident, kBucketMergeWaves), kThreads, 0, stream>>>(tab, out);
    }
}

void launch_bucket_merge_any(const MergeTable &tab, float *out, cudaStream_t stream)
{
    switch (tab.W) {
    case 1: launch_bucket_merge<1>(tab, out, stream); break;
    case 2: launch_bucket_merge<2>(tab, out, stream); break;
    case 3: launch_bucket_merge<3>(tab, out, stream); break;
    case 4: launch_bucket_merge<4>(tab, out, stream); break;
    case 5: launch_bucket_merge<5>(tab, out, stream); break;
    case 6: launch_bucket_merge<6>(tab, out, stream); break;
    case 7: launch_bucket_merge<7>(tab, out, stream); break;
    case 8: launch_bucket_merge<8>(tab, out, stream); break;
    default: launch_bucket_merge<0>(tab, out, stream); break;
    }
}

int64_t chunks_of(int64_t n, bool at_least_one, int64_t chunk_elems = kChunkElems)
{
    const int64_t c = (n + chunk_elems - 1) / chunk_elems;
    return (at_least_one && c == 0) ? 1 : c;
}

template <typename G>
int quantize_bucket(const qga_bucket_tensor *tensors, int T, uint32_t *compr, cudaStream_t stream,
                    std::atomic<int> (*occ)[64])
{
    const uintptr_t gal = GradLoad<G>::kVecAlign;
    // validate everything before the first launch
    for (int t = 0; t < T; ++t) {
        const qga_bucket_tensor &d = tensors[t];
        if (d.n < 0 || !finite_f32(d.neg_threshold) || !finite_f32(d.pos_threshold))
            return QGA_ERR_INVALID_ARG;
        if (d.n > 0 && (d.grad == nullptr || d.residual == nullptr || !aligned(d.grad, sizeof(G)) ||
                        !aligned(d.residual, 4)))
            return QGA_ERR_INVALID_ARG;
    }
    int64_t word_off = 0;
    for (int base = 0; base < T; base += kMaxRows) {
        QuantTable tab;
        tab.T = (T - base) < kMaxRows ? (T - base) : kMaxRows;
        int64_t chunk = 0;
        for (int i = 0; i < tab.T; ++i) {
            const qga_bucket_tensor &d = tensors[base + i];
            QuantRow &r = tab.row[i];
            r.grad = d.grad;
            r.residual = d.residual;
            r.n = d.n;
            r.word_off = word_off;
            r.chunk_begin = chunk;
            r.neg = d.neg_threshold;
            r.pos = d.pos_threshold;
            r.vec = aligned(d.grad, gal) && aligned(d.residual, 16);
            chunk += chunks_of(d.n, true);
            word_off += 3 + (d.n + 15) / 16;
        }
        tab.total_chunks = chunk;
        bool all_vec = true;
        for (int i = 0; i < tab.T; ++i)
            all_vec = all_vec && tab.row[i].vec;
        if (all_vec) {
            auto kernel = quantize_2bit_bucket_kernel<G, true>;
            kernel<<<grid_for(chunk, resident_blocks(kernel, kThreads, occ[1]), kBucketQuantizeWaves),
                     kThreads, 0, stream>>>(tab, compr);
        } else {
            auto kernel = quantize_2bit_bucket_kernel<G, false>;
            kernel<<<grid_for(chunk, resident_blocks(kernel, kThreads, occ[0]), kBucketQuantizeWaves),
                     kThreads, 0, stream>>>(tab, compr);
        }
        const int st = launch_status();
        if (st != QGA_OK)
            return st;
    }
    return QGA_OK;
}

} // namespace
} // namespace qga

using namespace qga;

extern "C" int64_t qga_2bit_bucket_words(const int64_t *n, int num_tensors)
{
    if (num_tensors < 0 || (num_tensors > 0 && n == nullptr))
        return QGA_ERR_INVALID_ARG;
    int64_t words = 0;
    for (int t = 0; t < num_tensors; ++t) {
        if (n[t] < 0)
            return QGA_ERR_INVALID_ARG;
        words += 3 + (n[t] + 15) / 16;
    }
    return words;
}

extern "C" int qga_quantize_2bit_bucket(const qga_bucket_tensor *tensors, int num_tensors,
                                        int grad_dtype, uint32_t *compr, cudaStream_t stream)
{
    if (num_tensors < 0 || (num_tensors > 0 && (tensors == nullptr || compr == nullptr)))
        return QGA_ERR_INVALID_ARG;
    if (compr != nullptr && !aligned(compr, 4))
        return QGA_ERR_INVALID_ARG;
    if (grad_dtype == QGA_DTYPE_F32)
        return quantize_bucket<float>(tensors, num_tensors, compr, stream, occ_qb_f32);
    if (grad_dtype == QGA_DTYPE_BF16)
        return quantize_bucket<uint16_t>(tensors, num_tensors, compr, stream, occ_qb_bf16);
    return QGA_ERR_UNSUPPORTED;
}

extern "C" int qga_dequant_accumulate_2bit_bucket(const uint32_t *const *compr, int num_workers,
                                                  const int64_t *n, int num_tensors, float *out,
                                                  cudaStream_t stream)
{
    if (compr == nullptr || num_workers < 1 || num_workers > QGA_MAX_WORKERS || num_tensors < 0 ||
        (num_tensors > 0 && n == nullptr))
        return QGA_ERR_INVALID_ARG;
    int64_t total = 0;
    for (int t = 0; t < num_tensors; ++t) {
        if (n[t] < 0)
            return QGA_ERR_INVALID_ARG;
        total += n[t];
    }
    for (int w = 0; w < num_workers; ++w)
        if (compr[w] == nullptr || !aligned(compr[w], 4))
            return QGA_ERR_INVALID_ARG;
    if (total == 0)
        return QGA_OK;
    if (out == nullptr || !aligned(out, 4))
        return QGA_ERR_INVALID_ARG;
    int64_t word_off = 0, elem_off = 0;
    for (int base = 0; base < num_tensors; base += kMaxRows) {
        MergeTable tab;
        tab.T = (num_tensors - base) < kMaxRows ? (num_tensors - base) : kMaxRows;
        tab.W = num_workers;
        for (int w = 0; w < QGA_MAX_WORKERS; ++w)
            tab.bucket[w] = w < num_workers ? compr[w] : nullptr;
        int64_t chunk = 0;
        for (int i = 0; i < tab.T; ++i) {
            MergeRow &r = tab.row[i];
            r.n = n[base + i];
            r.word_off = word_off;
            r.elem_off = elem_off;
            r.chunk_begin = chunk;
            r.vec = aligned(out + elem_off, 16);
            chunk += chunks_of(r.n, false, kMergeChunkElems);
            word_off += 3 + (r.n + 15) / 16;
            elem_off += r.n;
        }
        tab.total_chunks = chunk;
        if (chunk == 0)
            continue;
        launch_bucket_merge_any(tab, out, stream);
        const int st = launch_status();
        if (st != QGA_OK)
            return st;
    }
    return QGA_OK;
}
