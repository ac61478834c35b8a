// qga_common.cuh -- private helpers shared by the libqga.so translation units:
// cache-hinted global loads/stores, bit casts, and host-side validation,
// status and launch-geometry helpers.  Not part of the public ABI.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "qga.h"

namespace qga {

// ------------------------------------------------------------------ device --

constexpr int kWarp = 32;
constexpr unsigned kFullMask = 0xffffffffu;

__device__ __forceinline__ float f32_from_bits(uint32_t u) { return __uint_as_float(u); }
__device__ __forceinline__ uint32_t bits_from_f32(float f) { return __float_as_uint(f); }

// Streaming (evict-first) loads and stores: every byte of the hot path is
// touched once per call, so nothing is worth keeping in L1/L2 for the SAME
// call.  The 256-byte L2 prefetch hint lets one request pull the sectors the
// neighbouring lanes will ask for next.
__device__ __forceinline__ float4 ld_stream_f4(const float *p)
{
    float4 v;
    asm volatile("ld.global.cs.L2::256B.v4.f32 {%0,%1,%2,%3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ uint2 ld_stream_u2(const void *p)
{
    uint2 v;
    asm volatile("ld.global.cs.L2::256B.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
    return v;
}

__device__ __forceinline__ float ld_stream_f1(const float *p)
{
    float v;
    asm volatile("ld.global.cs.f32 %0, [%1];" : "=f"(v) : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t ld_stream_u32(const uint32_t *p)
{
    uint32_t v;
    asm volatile("ld.global.cs.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

__device__ __forceinline__ uint16_t ld_stream_u16(const uint16_t *p)
{
    unsigned short v;
    asm volatile("ld.global.cs.u16 %0, [%1];" : "=h"(v) : "l"(p));
    return v;
}

__device__ __forceinline__ void st_stream_f4(float *p, float4 v)
{
    asm volatile("st.global.cs.v4.f32 [%0], {%1,%2,%3,%4};"
                 :
                 : "l"(p), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w)
                 : "memory");
}

// 256-bit streaming load (sm_100): p must be 32-byte aligned.
__device__ __forceinline__ void ld_stream_f8(const float *p, float *v)
{
    asm volatile("ld.global.cs.L2::256B.v8.f32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]),
                   "=f"(v[6]), "=f"(v[7])
                 : "l"(p));
}

// 256-bit store (sm_100): p must be 32-byte aligned.
__device__ __forceinline__ void st_stream_f8(float *p, const float *v)
{
    asm volatile("st.global.cs.v8.f32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};"
                 :
                 : "l"(p), "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]),
                   "f"(v[6]), "f"(v[7])
                 : "memory");
}

__device__ __forceinline__ void st_stream_f1(float *p, float v)
{
    asm volatile("st.global.cs.f32 [%0], %1;" : : "l"(p), "f"(v) : "memory");
}

__device__ __forceinline__ void st_stream_u32(uint32_t *p, uint32_t v)
{
    asm volatile("st.global.cs.u32 [%0], %1;" : : "l"(p), "r"(v) : "memory");
}

// bfloat16 is the high half of a binary32 pattern: widening appends zeros.
__device__ __forceinline__ float widen_bf16(uint32_t h16) { return __uint_as_float(h16 << 16); }

// -------------------------------------------------------------------- host --

// Records the CUDA error behind a QGA_ERR_CUDA status for qga_last_cuda_error().
int cuda_status(cudaError_t err);

// Current device's SM count (cached per device).
int sm_count();

// Blocks of `threads` threads that one SM keeps resident for `kernel`
// (cached per kernel and device by the caller-provided slot).
template <typename Kernel>
int resident_blocks(Kernel kernel, int threads, std::atomic<int> *slots, size_t dynamic_smem = 0)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        dev = 0;
    int cached = slots[dev].load(std::memory_order_relaxed);
    if (cached > 0)
        return cached;
    int blocks = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks, kernel, threads, dynamic_smem) != cudaSuccess ||
        blocks < 1)
        blocks = 1;
    slots[dev].store(blocks, std::memory_order_relaxed);
    return blocks;
}

// Grid of a grid-stride kernel: `waves` times the blocks every SM holds at
// once (waves = 1 is a persistent grid), never more blocks than there are
// work items.  Each kernel passes the count measured best for it: for most of
// the streaming kernels several waves beat one persistent wave by 2-12%.
inline unsigned grid_for(int64_t work_items_per_block_rounded_up, int resident, int waves = 1)
{
    int64_t cap = (int64_t)sm_count() * resident * waves;
    int64_t g = work_items_per_block_rounded_up < cap ? work_items_per_block_rounded_up : cap;
    return (unsigned)(g < 1 ? 1 : g);
}

inline bool aligned(const void *p, uintptr_t a) { return ((uintptr_t)p % a) == 0; }

inline bool finite_f32(float x)
{
    return x == x && x <= 3.4028234663852886e38f && x >= -3.4028234663852886e38f;
}

// Launch status: the launch-configuration error of the kernel just enqueued.
inline int launch_status() { return cuda_status(cudaGetLastError()); }

} // namespace qga
