// qga_2bit.cu -- single-tensor 2-bit threshold kernels and their C ABI:
// quantize (fp32 / bf16 gradient), dequantize, and the W-worker merge.
//
// MXNet pull request #8342 "[WIP] 2bit gradient compression": "Operators"
// (create_2bit / quantize_2bit / dequantize_2bit), "Format of compressed
// gradient" (header [neg, pos, n] then 16 codes per word) and "Local kvstore"
// (the receiver dequantizes every worker's gradient and sums them).
//
// Each kernel is one pass over HBM: warps stride over tiles (512 elements
// for an fp32 quantize, a dequantize or a merge slice, 1024 for a bf16
// quantize) on a grid of a few waves of resident blocks, the count measured
// best for each kernel (see grid_for).  Nothing is filled
// or cleared by a separate launch: the quantize kernel writes every payload
// word (including the zero tail codes) and its block 0 writes the header.
// The merges are built for W <= 8 from a table of all 3^W sums, and for
// W > 8 from the table of the first 8 workers' sums continued by per-worker
// adds.

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

// The dequantize in the table merge's geometry: a lane owns one word of each
// 32-word slice, and the next slice's word is in flight while the current
// one is stored; a 3-entry shared table holds the three code values (+0,
// pos, neg; code 11 reads as 00, as in the merge) and the 16 values of a
// word leave through the per-warp stage as coalesced 128-bit rows.
// Measured at n = 138M: 92.4 us at 16 waves (94.4 at 8, 96.7 at 32),
// against 96.3-96.7 us for one word per lane decoded by shuffles into
// 4-element groups.
template <bool kVec>
__global__ void __launch_bounds__(kThreads)
    dequantize_2bit_kernel(const uint32_t *__restrict__ compr, float *__restrict__ out, int64_t n)
{
    __shared__ float s_val[3];
    __shared__ float4 s_stage[kWarpsPerBlock][kWarp * 4];
    if (threadIdx.x == 0) {
        s_val[0] = 0.0f;
        s_val[1] = f32_from_bits(compr[1]);
        s_val[2] = f32_from_bits(compr[0]);
    }
    const int lane = threadIdx.x & (kWarp - 1);
    const int64_t nwords = (n + 15) >> 4;
    const int64_t slices = (nwords + kWarp - 1) / kWarp;
    auto payload_of = [&](int) { return compr + 3; };
    int64_t sl = first_tile();
    uint32_t wd[1][kTableMaxWorkers];
    if (sl < slices)
        merge_2bit_table_load<1, 1>(payload_of, nwords, sl, lane, -1, wd);
    __syncthreads();
    for (; sl < slices; sl += tile_stride()) {
        uint32_t next[1][kTableMaxWorkers];
        if (sl + tile_stride() < slices)
            merge_2bit_table_load<1, 1>(payload_of, nwords, sl + tile_stride(), lane, -1, next);
        else
            next[0][0] = 0u;
        merge_2bit_table_store<kVec, 1, 1>(wd, s_val, out, n, sl, lane, s_stage[threadIdx.x >> 5]);
        wd[0][0] = next[0][0];
    }
}

struct RecordSet {
    const uint32_t *rec[QGA_MAX_WORKERS];
};

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

// W > 8: the table of the first 8 workers' 3^8 sums gives each element's
// exact running sum after worker 7 (one table load), and workers 8 .. W-1
// are then added in order by the per-worker decode (pair tables for even
// workers, bit masks and predicated adds for odd ones), so the result is
// the definition's sum in worker order, bit for bit.  A lane owns one word
// of each 32-word slice.  The 3^8 table (26,244 B) and the W - 8 pair
// tables sit in dynamic shared memory.
// Measured at n = 138M (us, W = 9 / 16 / 32): the first 8 words loaded just
// before use 198 / 297 / 611 at 8 waves; the next slice's first 8 words in
// flight 181 / 285 / 595 at 1 wave and 199 / 293 / 566 at 8 waves, against
// 251 / 355 / 651 for the per-worker decode of all W workers.
#ifndef QGA_PREFIX_MERGE_PREFETCH
#define QGA_PREFIX_MERGE_PREFETCH 1
#endif
#ifdef QGA_PREFIX_MERGE_WAVES
inline int prefix_merge_waves(int) { return QGA_PREFIX_MERGE_WAVES; }
#else
inline int prefix_merge_waves(int w) { return w <= 16 ? 1 : 8; }
#endif
constexpr int kPrefixWorkers = 8;
constexpr int kPrefixTableBytes = Pow3<kPrefixWorkers>::value * 4;

inline int hybrid_smem_bytes(int W)
{
    return kPrefixTableBytes + 4 /* pad to 8 */ + (W - kPrefixWorkers) * 16 * 8 + 2 * W * 4;
}

template <bool kVec>
__global__ void __launch_bounds__(kThreads)
    merge_2bit_prefix_table_kernel(const __grid_constant__ RecordSet set, int W, float *__restrict__ out,
                                   int64_t n)
{
    extern __shared__ __align__(16) unsigned char s_dyn[];
    float *s_sum = reinterpret_cast<float *>(s_dyn);
    float2(*s_pair)[16] = reinterpret_cast<float2(*)[16]>(s_dyn + kPrefixTableBytes + 4);
    float *s_neg = reinterpret_cast<float *>(s_dyn + kPrefixTableBytes + 4 + (W - kPrefixWorkers) * 128);
    float *s_pos = s_neg + W;
    __shared__ float4 s_stage[kWarpsPerBlock][kWarp * 4];
    for (int w = threadIdx.x; w < W; w += kThreads) {
        const uint32_t *r = set.rec[w];
        s_neg[w] = f32_from_bits(r[0]);
        s_pos[w] = f32_from_bits(r[1]);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < (W - kPrefixWorkers) * 16; i += kThreads)
        s_pair[i >> 4][i & 15] = pair_entry(i & 15, s_neg[kPrefixWorkers + (i >> 4)], s_pos[kPrefixWorkers + (i >> 4)]);
    build_sum_table<kPrefixWorkers>(s_sum, [&](int w) { return s_neg[w]; }, [&](int w) { return s_pos[w]; });
    const char *tb = reinterpret_cast<const char *>(s_sum);
    const int lane = threadIdx.x & (kWarp - 1);
    const int f = (lane >> 1) & 3;
    float4 *stage = s_stage[threadIdx.x >> 5];
    const int64_t nwords = (n + 15) >> 4;
    const int64_t slices = (nwords + kWarp - 1) / kWarp;
#if QGA_PREFIX_MERGE_PREFETCH
    uint32_t wd[kTableMaxWorkers];
    {
        const int64_t k0 = first_tile() * kWarp + lane;
#pragma unroll
        for (int w = 0; w < kPrefixWorkers; ++w)
            wd[w] = (first_tile() < slices && k0 < nwords) ? ld_stream_u32(set.rec[w] + 3 + k0) : 0u;
    }
#endif
    for (int64_t sl = first_tile(); sl < slices; sl += tile_stride()) {
        const int64_t k = sl * kWarp + lane;
        const bool ok = k < nwords;
        float2 acc[8];
        {
#if QGA_PREFIX_MERGE_PREFETCH
            uint32_t nx[kTableMaxWorkers];
            const int64_t kn = (sl + tile_stride()) * kWarp + lane;
#pragma unroll
            for (int w = 0; w < kPrefixWorkers; ++w)
                nx[w] = (sl + tile_stride() < slices && kn < nwords) ? ld_stream_u32(set.rec[w] + 3 + kn) : 0u;
#else
            uint32_t wd[kTableMaxWorkers];
#pragma unroll
            for (int w = 0; w < kPrefixWorkers; ++w)
                wd[w] = ok ? ld_stream_u32(set.rec[w] + 3 + k) : 0u;
#endif
            uint32_t off[16];
            sum_table_offsets<kPrefixWorkers>(wd, off);
#pragma unroll
            for (int p = 0; p < 8; ++p)
                acc[p] = make_float2(*reinterpret_cast<const float *>(tb + off[2 * p]),
                                     *reinterpret_cast<const float *>(tb + off[2 * p + 1]));
#if QGA_PREFIX_MERGE_PREFETCH
#pragma unroll
            for (int w = 0; w < kPrefixWorkers; ++w)
                wd[w] = nx[w];
#endif
        }
        for (int wb = kPrefixWorkers; wb < W; wb += kMergeBatch) {
            uint32_t words[kMergeBatch];
#pragma unroll
            for (int i = 0; i < kMergeBatch; ++i)
                words[i] = (ok && wb + i < W) ? ld_stream_u32(set.rec[wb + i] + 3 + k) : 0u;
#pragma unroll
            for (int i = 0; i < kMergeBatch; ++i) {
                if (wb + i >= W) // warp-uniform
                    break;
                if ((i & 1) == 0) {
                    const char *pt = reinterpret_cast<const char *>(s_pair[wb + i - kPrefixWorkers]);
#pragma unroll
                    for (int p = 0; p < 8; ++p) {
                        // 4 code bits of elements 2p, 2p+1, times the 8-byte entry size
                        const int sh = 25 - 4 * p;
                        const uint32_t o = (sh >= 0 ? (words[i] >> sh) : (words[i] << (-sh))) & 0x78u;
                        acc[p] = __fadd2_rn(acc[p], *reinterpret_cast<const float2 *>(pt + o));
                    }
                } else {
                    const float neg = s_neg[wb + i], pos = s_pos[wb + i];
                    const uint32_t lo = words[i] & 0x55555555u;
                    const uint32_t hi = (words[i] >> 1) & 0x55555555u;
                    const uint32_t is01 = lo & ~hi, is10 = hi & ~lo;
#pragma unroll
                    for (int p = 0; p < 16; ++p) {
                        const uint32_t bit = 1u << (30 - 2 * p);
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
        for (int c = 0; c < 4; ++c)
            stage[lane * 4 + (c ^ f)] = make_float4(acc[2 * c].x, acc[2 * c].y, acc[2 * c + 1].x, acc[2 * c + 1].y);
        __syncwarp();
        const int64_t g0 = sl * kWarp * 4; // first group of this slice
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int q = j * kWarp + lane;
            store_group<kVec>(out, n, g0 + q, stage[stage_slot(q >> 2, q & 3)]);
        }
        __syncwarp();
    }
}

std::atomic<int> occ_q_f32_w[64], occ_q_f32_v[64], occ_q_f32_s[64], occ_q_bf16_v[64], occ_q_bf16_s[64];
std::atomic<int> occ_dq_v[64], occ_dq_s[64];
std::atomic<int> occ_acc[2][64];    // [vec][device]: W > 8
std::atomic<bool> smem_attr_set[2][64];
std::atomic<int> occ_tab[2][9][64]; // [vec][kW][device]: W <= 8

// Grid waves (see grid_for), measured at n = 138M: quantize in group tiles
// 270-286 / 263 / 259 / 256 / 258 us at 1 / 8 / 16 / 32 / 128 waves, in
// lane-owned words 252 / 243 us at 8 / 32 waves (2 words per lane: 253 /
// 256); dequantize 109 / 97 / 96 / 101 us at 1 / 8 / 16 / 32; merge (W = 8)
// 180 / 174 / 176 / 181 us at 1 / 8 / 16 / 32.
constexpr int kQuantizeWaves = 32, kDequantizeWaves = 16;
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
        // the prefix table needs more than the default 48 KB of shared memory:
        // the attribute is set once per device, for the largest worker count
        auto k = merge_2bit_prefix_table_kernel<kVec>;
        const int smem = hybrid_smem_bytes(W);
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
            dev = 0;
        if (!smem_attr_set[kVec][dev].load(std::memory_order_relaxed)) {
            cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 hybrid_smem_bytes(QGA_MAX_WORKERS));
            smem_attr_set[kVec][dev].store(true, std::memory_order_relaxed);
        }
        k<<<tiles_grid(n, resident_blocks(k, kThreads, occ_acc[kVec], hybrid_smem_bytes(QGA_MAX_WORKERS)),
                       16 * kWarp, prefix_merge_waves(W)),
            kThreads, smem, stream>>>(set, W, out, n);
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
        k<<<tiles_grid(n, resident_blocks(k, kThreads, occ_dq_v), 16 * kWarp, kDequantizeWaves),
            kThreads, 0, stream>>>(compr, out, n);
    } else {
        auto k = dequantize_2bit_kernel<false>;
        k<<<tiles_grid(n, resident_blocks(k, kThreads, occ_dq_s), 16 * kWarp, kDequantizeWaves),
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
