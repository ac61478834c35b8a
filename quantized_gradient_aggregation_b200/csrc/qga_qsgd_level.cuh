// qga_qsgd_level.cuh -- the QSGD-MaxNorm level of one element and the
// Philox4x32-10 draw behind it, shared by the dense QSGD-MaxNorm kernels and
// the GRandK-MaxNorm kernels of kept coordinates.  Private to libqga.so.
//
// Philox4x32-10: Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As
// Easy as 1, 2, 3", SC'11.  The level: t = ((|g| / M) * s) + u in binary32,
// q = sign(g) * min(floor(t), s), 0 when t is not finite.
#pragma once

#include <float.h>

#include "qga_common.cuh"

namespace qga {

// ----------------------------------------------------------- Philox4x32-10 --
// Ten rounds of: two 32x32 -> 64-bit products of the even counter words with
// the round multipliers; the high halves xor the odd words and the key, the
// low halves move to the odd slots.  The key is bumped by the Weyl constants
// before every round but the first.
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1)
{
#pragma unroll
    for (int round = 0; round < 10; ++round) {
        if (round > 0) {
            k0 += 0x9E3779B9u;
            k1 += 0xBB67AE85u;
        }
        const uint32_t hi0 = __umulhi(0xD2511F53u, c.x);
        const uint32_t lo0 = 0xD2511F53u * c.x;
        const uint32_t hi1 = __umulhi(0xCD9E8D57u, c.z);
        const uint32_t lo1 = 0xCD9E8D57u * c.z;
        c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
    }
    return c;
}

// Draw of an output word: its top 24 bits as a multiple of 2^-24 (exact).
__device__ __forceinline__ float unit_draw(uint32_t x)
{
    return __fmul_rn(__uint2float_rn(x >> 8), 0x1p-24f);
}

template <int B> struct Levels {
    static constexpr int s = (1 << (B - 1)) - 1;
    static constexpr uint32_t mask = (1u << B) - 1u;
    static constexpr int lanes_per_word = 8 / B; // 4 codes of B bits per lane
};

// The level by the definition's three operations, in their order.
template <int B>
__device__ __forceinline__ int32_t qsgd_level_exact(float g, float M, float u)
{
    constexpr float s = (float)Levels<B>::s;
    const float t = __fadd_rn(__fmul_rn(__fdiv_rn(fabsf(g), M), s), u);
    if (!(fabsf(t) <= FLT_MAX)) // NaN or infinite
        return 0;
    const int32_t q = (int32_t)fminf(floorf(t), s);
    return g < 0.0f ? -q : q;
}

// The same level with one multiply instead of the division, for a finite
// positive M, and k = fl(s / M).  Only floor(t) matters, so: t' = fl(fl(|g| k)
// + u) is within 2^-15 of the definition's t whenever t' < s + 1 (each of the
// two is within 1.9e-5 of the exact real |g| s / M + u: two relative
// roundings of at most 2^-24 on a value below 128, plus half an ulp below
// 128), and any t' >= s + 1 caps both to s.  So wherever t' is at least
// 2^-14 away from an integer, floor(t') == floor(t); otherwise (or if t' is
// not finite) the exact sequence decides.  Results are identical to
// qsgd_level_exact for every input.
//   x: the draw's output word; u = (x >> 8) 2^-24 enters the sum through one
//   fused multiply-add, whose product is exact, so the sum is the same single
//   rounding of |g| k + u as a separate add of u.
template <int B>
__device__ __forceinline__ int32_t qsgd_level(float g, float M, float k, uint32_t x)
{
    constexpr float s = (float)Levels<B>::s;
    constexpr float kMargin = 0x1p-14f;
    const float m = __uint2float_rn(x >> 8); // exact: below 2^24
    const float tf = __fmaf_rn(m, 0x1p-24f, __fmul_rn(fabsf(g), k));
    const float fl = floorf(tf);
    const float d = __fsub_rn(tf, fl); // exact
    // d in [2^-14, 1 - 2^-14], as one comparison (its rounding moves the
    // bound by at most 2^-25, far inside the slack of the margin)
    if (!(fabsf(__fsub_rn(d, 0.5f)) <= 0.5f - kMargin))
        return qsgd_level_exact<B>(g, M, __fmul_rn(m, 0x1p-24f));
    return (int32_t)copysignf(fminf(fl, s), g); // g = -0 gives 0
}

} // namespace qga
