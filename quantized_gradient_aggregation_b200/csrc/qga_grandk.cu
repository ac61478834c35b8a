// qga_grandk.cu -- GlobalRandKMaxNorm (GRandK-MN): QSGD-MaxNorm of K
// coordinates that every worker keeps.
//
// The gradient-compression README (vineeths96), "Results", names
// GlobalRandKMaxNorm compression with K = 10000 as the sparsified variant of
// QSGDMaxNorm and prints no formula.  This library's reading: all workers
// keep the same K coordinates index[0..K-1] (drawn by the caller from a seed
// the workers share, so the sparse records still add up element by element
// in an all-reduce); the kept values x[k] = g[index[k]] are quantized exactly
// as the dense QSGD-MaxNorm kernels quantize a gradient of K elements (M =
// max |x| over all workers, the draw of position k, header [M, b, K]); the
// merge sums the levels, scales them once by M / s and scatters them back,
// every other coordinate of the n-element result being +0.  A coordinate
// outside [0, n) is skipped: it does not enter M, gets level 0 and is not
// stored, so no index value can make a kernel touch memory outside the
// caller's buffers.
//
// K is small (10^4) next to n (10^8): these kernels gather K scattered
// elements per worker and are bound by load latency, not by bandwidth; the
// merge's one bandwidth-heavy step is clearing the n-element result, done by
// cudaMemsetAsync before the scatter.

#include "qga_common.cuh"
#include "qga_qsgd_level.cuh"

namespace qga {
namespace {

constexpr int kThreads = 256;
constexpr int kWarpsPerBlock = kThreads / kWarp;

struct GradSet {
    const float *g[QGA_MAX_WORKERS];
};

struct RecordSet {
    const uint32_t *rec[QGA_MAX_WORKERS];
};

__device__ __forceinline__ bool in_range(int64_t i, int64_t n) { return (uint64_t)i < (uint64_t)n; }

// M = max over workers of |g_w| at the kept coordinates; one thread per
// position, its W loads issued together.
__global__ void __launch_bounds__(kThreads)
    grandk_max_kernel(const __grid_constant__ GradSet set, int W, int64_t n,
                      const int64_t *__restrict__ index, int64_t K, float *__restrict__ M)
{
    __shared__ float s_part[kWarpsPerBlock];
    constexpr int kBatch = 8;
    float m = 0.0f;
    for (int64_t k = (int64_t)blockIdx.x * kThreads + threadIdx.x; k < K;
         k += (int64_t)gridDim.x * kThreads) {
        const int64_t i = index[k];
        if (!in_range(i, n))
            continue;
        for (int wb = 0; wb < W; wb += kBatch) {
            float v[kBatch];
#pragma unroll
            for (int j = 0; j < kBatch; ++j)
                v[j] = wb + j < W ? set.g[wb + j][i] : 0.0f;
#pragma unroll
            for (int j = 0; j < kBatch; ++j)
                m = fmaxf(m, fabsf(v[j])); // fmaxf drops a NaN operand
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
        m = fmaxf(m, __shfl_xor_sync(kFullMask, m, off));
    if ((threadIdx.x & 31) == 0)
        s_part[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        float b = s_part[0];
#pragma unroll
        for (int j = 1; j < kWarpsPerBlock; ++j)
            b = fmaxf(b, s_part[j]);
        // non-negative binary32 values order like their bit patterns
        if (b > 0.0f)
            atomicMax(reinterpret_cast<unsigned int *>(M), __float_as_uint(b));
    }
}

// One worker's record of its kept values.  A warp takes 32 consecutive
// positions; the 32/b lanes of one record word OR their shifted codes
// together with shuffles, and the first of them stores the word.
template <int B>
__global__ void __launch_bounds__(kThreads)
    grandk_quantize_kernel(const float *__restrict__ grad, int64_t n,
                           const int64_t *__restrict__ index, int64_t K,
                           uint32_t *__restrict__ compr, uint32_t key0, uint32_t key1,
                           const float *__restrict__ max_in)
{
    using L = Levels<B>;
    constexpr int F = 32 / B; // codes per word
    const float M = *max_in;
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        compr[0] = bits_from_f32(M);
        compr[1] = bits_from_f32((float)B);
        compr[2] = bits_from_f32(__ll2float_rn(K));
    }
    uint32_t *payload = compr + 3;
    const int lane = threadIdx.x & (kWarp - 1);
    const int64_t nwords = (K * B + 31) >> 5;
    // base is the warp's first position, so the loop condition is warp-uniform
    // and every lane takes part in the shuffles
    for (int64_t base = (int64_t)blockIdx.x * kThreads + (threadIdx.x - lane); base < K;
         base += (int64_t)gridDim.x * kThreads) {
        const int64_t k = base + lane;
        uint32_t code = 0u;
        if (k < K) {
            const int64_t i = index[k];
            if (in_range(i, n)) {
                const uint64_t blk = (uint64_t)k >> 2;
                const uint4 r = philox4x32_10(make_uint4((uint32_t)blk, (uint32_t)(blk >> 32), 0u, 0u),
                                              key0, key1);
                const int j = (int)(k & 3);
                const uint32_t x = j == 0 ? r.x : (j == 1 ? r.y : (j == 2 ? r.z : r.w));
                code = (uint32_t)qsgd_level_exact<B>(grad[i], M, unit_draw(x)) & L::mask;
            }
        }
        uint32_t word = code << (32 - B * (lane % F + 1));
#pragma unroll
        for (int off = 1; off < F; off <<= 1)
            word |= __shfl_xor_sync(kFullMask, word, off);
        if (lane % F == 0 && k / F < nwords)
            st_stream_u32(payload + k / F, word);
    }
}

// Scatter of the merged kept values into the cleared n-element result:
// out[index[k]] = (float)(sum_w q_w[k]) * fl(M / s), M from worker 0's header.
template <int B>
__global__ void __launch_bounds__(kThreads)
    grandk_scatter_kernel(const __grid_constant__ RecordSet set, int W,
                          const int64_t *__restrict__ index, int64_t K, float *__restrict__ out,
                          int64_t n)
{
    constexpr int F = 32 / B;
    const float step = __fdiv_rn(f32_from_bits(set.rec[0][0]), (float)Levels<B>::s);
    for (int64_t k = (int64_t)blockIdx.x * kThreads + threadIdx.x; k < K;
         k += (int64_t)gridDim.x * kThreads) {
        const int64_t i = index[k];
        if (!in_range(i, n))
            continue;
        const int up = B * (int)(k % F); // field k % F moved to the top bits
        int32_t sum = 0;
        for (int w = 0; w < W; ++w)
            sum += (int32_t)(set.rec[w][3 + k / F] << up) >> (32 - B); // sign-extended level
        out[i] = __fmul_rn(__int2float_rn(sum), step);
    }
}

std::atomic<int> occ_max[64];
std::atomic<int> occ_q[3][64];
std::atomic<int> occ_s[3][64];

int bits_slot(int bits) { return bits == 2 ? 0 : (bits == 4 ? 1 : (bits == 8 ? 2 : -1)); }

unsigned position_grid(int64_t K, int resident)
{
    return grid_for((K + kThreads - 1) / kThreads, resident);
}

template <int B>
void launch_quantize(const float *grad, int64_t n, const int64_t *index, int64_t K, uint32_t *compr,
                     uint64_t seed, const float *M, cudaStream_t stream)
{
    auto k = grandk_quantize_kernel<B>;
    k<<<position_grid(K, resident_blocks(k, kThreads, occ_q[bits_slot(B)])), kThreads, 0, stream>>>(
        grad, n, index, K, compr, (uint32_t)seed, (uint32_t)(seed >> 32), M);
}

template <int B>
void launch_scatter(const RecordSet &set, int W, const int64_t *index, int64_t K, float *out,
                    int64_t n, cudaStream_t stream)
{
    auto k = grandk_scatter_kernel<B>;
    k<<<position_grid(K, resident_blocks(k, kThreads, occ_s[bits_slot(B)])), kThreads, 0, stream>>>(
        set, W, index, K, out, n);
}

} // namespace
} // namespace qga

using namespace qga;

extern "C" int qga_grandk_mn_max(const float *const *grad, int num_workers, int64_t n,
                                 const int64_t *index, int64_t k, float *max_out,
                                 cudaStream_t stream)
{
    if (grad == nullptr || num_workers < 1 || num_workers > QGA_MAX_WORKERS || n < 0 || k < 0 ||
        max_out == nullptr || !aligned(max_out, 4))
        return QGA_ERR_INVALID_ARG;
    if (k > 0 && (index == nullptr || !aligned(index, 8)))
        return QGA_ERR_INVALID_ARG;
    GradSet set{};
    for (int w = 0; w < num_workers; ++w) {
        if (n > 0 && k > 0 && (grad[w] == nullptr || !aligned(grad[w], 4)))
            return QGA_ERR_INVALID_ARG;
        set.g[w] = grad[w];
    }
    int st = cuda_status(cudaMemsetAsync(max_out, 0, sizeof(float), stream));
    if (st != QGA_OK || n == 0 || k == 0)
        return st;
    grandk_max_kernel<<<position_grid(k, resident_blocks(grandk_max_kernel, kThreads, occ_max)),
                        kThreads, 0, stream>>>(set, num_workers, n, index, k, max_out);
    return launch_status();
}

extern "C" int qga_grandk_mn_quantize(const float *grad, int64_t n, const int64_t *index,
                                      int64_t k, uint32_t *compr, int bits, uint64_t seed,
                                      const float *max_in, cudaStream_t stream)
{
    if (n < 0 || k < 0 || compr == nullptr || !aligned(compr, 4) || max_in == nullptr ||
        !aligned(max_in, 4))
        return QGA_ERR_INVALID_ARG;
    if (k > 0 && (index == nullptr || !aligned(index, 8)))
        return QGA_ERR_INVALID_ARG;
    if (n > 0 && k > 0 && (grad == nullptr || !aligned(grad, 4)))
        return QGA_ERR_INVALID_ARG;
    switch (bits) {
    case 2: launch_quantize<2>(grad, n, index, k, compr, seed, max_in, stream); break;
    case 4: launch_quantize<4>(grad, n, index, k, compr, seed, max_in, stream); break;
    case 8: launch_quantize<8>(grad, n, index, k, compr, seed, max_in, stream); break;
    default: return QGA_ERR_UNSUPPORTED;
    }
    return launch_status();
}

extern "C" int qga_grandk_mn_dequant_accumulate(const uint32_t *const *compr, int num_workers,
                                                const int64_t *index, int64_t k, float *out,
                                                int64_t n, int bits, cudaStream_t stream)
{
    if (compr == nullptr || num_workers < 1 || num_workers > QGA_MAX_WORKERS || n < 0 || k < 0)
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
    if (out == nullptr || !aligned(out, 4) || (k > 0 && (index == nullptr || !aligned(index, 8))))
        return QGA_ERR_INVALID_ARG;
    int st = cuda_status(cudaMemsetAsync(out, 0, (size_t)n * sizeof(float), stream));
    if (st != QGA_OK || k == 0)
        return st;
    switch (bits) {
    case 2: launch_scatter<2>(set, num_workers, index, k, out, n, stream); break;
    case 4: launch_scatter<4>(set, num_workers, index, k, out, n, stream); break;
    default: launch_scatter<8>(set, num_workers, index, k, out, n, stream); break;
    }
    return launch_status();
}
