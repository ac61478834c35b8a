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
// positive M, and k = fl(s / M).  Only floor(t) matters.  Each of t' =
// fl(fl(|g| k) + u) and the definition's t is within 1.9e-5 of the exact real
// |g| s / M + u whenever it is below s + 1 (two relative roundings of at most
// 2^-24 on a value below 128, 1.5e-5, plus half an ulp below 128, 3.8e-6), so
// |t - t'| <= 3.8e-5, below 2^-14 (6.1e-5); any t' >= s + 1 caps both to s.
// So wherever t' is at least 2^-14 away from an integer, floor(t') ==
// floor(t); otherwise (or if t' is not finite) the exact sequence decides.
// Results are identical to qsgd_level_exact for every input.
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

// ------------------------------------------------ fixed-point fast level --
// The level of one element without the division and without conversions
// between integers and floats, for a finite positive M and k = fl(s / M).
// 2^E must exceed every level count s the caller uses (E = b - 1 for one
// scale of b bits).  With F = 23 - E fraction bits:
//   a  = fl(|g| k)                      (one multiply)
//   X  = fl(a + 2^E)                    bits(X) - bits(2^E) = a rounded to a
//                                       multiple of 2^-F, as an integer
//   T  = that integer + (x >> (32 - F)) the draw u truncated to F fraction bits
//   level = min(floor(T / 2^F), s),  signed by g
// T / 2^F differs from the definition's t by at most 2^(E-21): a and
// fl(fl(|g| / M) s) are each within 2^(E-23) of the exact |g| s / M (two
// relative roundings of 2^-24 on a value below 2^E), a's rounding to the grid
// adds 2^-(F+1) = 2^(E-24), the truncation of u less than 2^-F = 2^(E-23),
// and the definition's last rounding 2^(E-24); the sum is below 2^(E-21),
// 4 units of 2^-F.  So wherever T is at least kFixMargin = 8 units away from
// a multiple of 2^F, floor(T / 2^F) = floor(t).  Near an integer (fraction
// of T within 8 units), and for a not below 2^E (X >= 2^(E+1), which also
// catches an infinite or NaN a), the caller recomputes the level by the
// definition's operations (qsgd_level_exact).  Levels at or above s need no
// margin: both sides cap them to s.  The checks are accumulated over a
// lane's elements (fmin, xmax) so that one test per tile decides.
//   x: the draw's Philox output word (u = (x >> 8) 2^-24).
template <int E> struct FixLevel {
    static constexpr int F = 23 - E;
    static constexpr uint32_t kOne = (127u + E) << 23;  // binary32 bits of 2^E
    static constexpr uint32_t kTwo = (128u + E) << 23;  // bits of 2^(E+1)
    static constexpr uint32_t kMargin = 8;              // units of 2^-F
    static constexpr uint32_t kFrac = (1u << F) - 1u;
    // the per-lane accumulators start here; recompute iff needs_exact()
    static __device__ __forceinline__ void reset(uint32_t &fmin, uint32_t &xmax)
    {
        fmin = 0xFFFFFFFFu;
        xmax = 0u;
    }
    static __device__ __forceinline__ bool needs_exact(uint32_t fmin, uint32_t xmax)
    {
        return fmin < 2u * kMargin || xmax >= kTwo;
    }
};

template <int E>
__device__ __forceinline__ int32_t qsgd_level_fixed(float g, float k, uint32_t s, uint32_t x,
                                                    uint32_t &fmin, uint32_t &xmax)
{
    using Fx = FixLevel<E>;
    const float a = __fmul_rn(fabsf(g), k);
    const uint32_t xb = __float_as_uint(__fadd_rn(a, (float)(1 << E)));
    // T + kMargin: its floor equals T's wherever the fraction of T + kMargin is
    // at least 2 kMargin, which is what the accumulated check demands
    const uint32_t t8 = xb + (x >> (32 - Fx::F)) + (Fx::kMargin - Fx::kOne);
    fmin = min(fmin, t8 & Fx::kFrac);
    xmax = max(xmax, xb);
    const uint32_t level = min(t8 >> Fx::F, s);
    const uint32_t sg = (uint32_t)((int32_t)__float_as_uint(g) >> 31); // all ones if g < 0
    return (int32_t)((level ^ sg) - sg);
}

// The same fixed-point level with one fused multiply-add and checks that
// cost two integer min/max per element: X = fl(|g| k + 2^E) (a single
// rounding, within half an ulp of the exact sum), T + 8 as above, and the
// level floor(T / 2^F) with no cap.  A lane falls back to
// qsgd_level_exact when, over its elements, the smallest fraction of T + 8
// (shifted to the top bits) is below 16 units, or the largest T + 8 reaches
// (s + 1) 2^F: a level above s (the cap case near |g| = M, or |g| > M),
// and an infinite or NaN X all land there.  The error bound is that of
// qsgd_level_fixed (the fused add only removes one rounding), so with the
// same margin the two floors agree everywhere else.  2^E must exceed s.
template <int E> struct LeanLevel {
    static constexpr int F = 23 - E;
    static constexpr uint32_t kOne = (127u + E) << 23;  // binary32 bits of 2^E
    static __device__ __forceinline__ bool needs_exact(uint32_t fmin, uint32_t tmax, uint32_t s)
    {
        return fmin < (16u << (32 - F)) || tmax >= ((s + 1u) << F);
    }
};

template <int E>
__device__ __forceinline__ uint32_t qsgd_level_lean(float g, float k, uint32_t x, uint32_t &fmin,
                                                    uint32_t &tmax)
{
    using Lx = LeanLevel<E>;
    const float X = __fmaf_rn(fabsf(g), k, (float)(1 << E));
    const uint32_t t8 = __float_as_uint(X) + (x >> (32 - Lx::F)) + (8u - Lx::kOne);
    fmin = min(fmin, t8 << (32 - Lx::F));
    tmax = max(tmax, t8);
    return t8 >> Lx::F;
}

// The b-bit two's-complement code of a level of magnitude L with g's sign.
template <int B>
__device__ __forceinline__ uint32_t signed_code(uint32_t L, float g)
{
    const int32_t sgn = ((int32_t)__float_as_uint(g) >> 31) * 2 + 1; // -1 or +1
    return (uint32_t)((int32_t)L * sgn) & ((1u << B) - 1u);
}

// ------------------------------------------------- integer sum of levels --
// The merges add the W workers' levels a whole record word at a time.  XOR
// with the sign bit of every b-bit field turns a two's-complement level q
// into q + 2^(b-1) in [0, 2^b), and the biased fields are added in SIMD
// lanes of registers wide enough that no add carries into the neighbouring
// lane (at most 64 workers):
//   b = 2: every fourth field in the 8-bit lanes of 4 registers (64 * 3 < 2^8);
//   b = 4: the even and odd fields in the 8-bit lanes of 2 registers, which
//          hold up to 17 words (17 * 15 < 2^8) and are widened into the
//          16-bit lanes of 4 registers after every batch of words;
//   b = 8: the even and odd fields in the 16-bit lanes of 2 registers
//          (64 * 255 < 2^16).
// A field's final sum, minus W 2^(b-1), is the exact integer level sum; it is
// below 2^23, so adding it to the bits of 2^23 and subtracting 2^23 + W
// 2^(b-1) in binary32 converts it exactly.
//   add(word) for each worker's word, end_batch() after every batch of at
//   most kBatchMax words, finish() at the end; field_sum(e) is the biased
//   sum of element e of the word (element 0 = most significant field).
template <int B> struct LevelSum;

template <> struct LevelSum<2> {
    static constexpr int kFields = 16, kBatchMax = 64;
    static constexpr uint32_t kSign = 0xAAAAAAAAu;
    uint32_t w[4] = {0u, 0u, 0u, 0u}; // register j: fields j, j + 4, j + 8, j + 12
    __device__ __forceinline__ void add(uint32_t word)
    {
        const uint32_t x = word ^ kSign;
#pragma unroll
        for (int j = 0; j < 4; ++j)
            w[j] += (x >> (2 * j)) & 0x03030303u;
    }
    __device__ __forceinline__ void end_batch() {}
    __device__ __forceinline__ void finish() {}
    __device__ __forceinline__ uint32_t field_sum(int e) const
    {
        const int f = kFields - 1 - e; // field counted from the least significant
        return (w[f & 3] >> (8 * (f >> 2))) & 0xFFu;
    }
};

template <> struct LevelSum<4> {
    static constexpr int kFields = 8, kBatchMax = 17;
    static constexpr uint32_t kSign = 0x88888888u;
    uint32_t a = 0u, b = 0u;          // 8-bit lanes: fields 2i (a), 2i + 1 (b)
    uint32_t w[4] = {0u, 0u, 0u, 0u}; // 16-bit lanes: bytes 0 / 2 and 1 / 3 of a, then of b
    __device__ __forceinline__ void add(uint32_t word)
    {
        const uint32_t x = word ^ kSign;
        a += x & 0x0F0F0F0Fu;
        b += (x >> 4) & 0x0F0F0F0Fu;
    }
    __device__ __forceinline__ void end_batch()
    {
        w[0] += a & 0x00FF00FFu;
        w[1] += (a >> 8) & 0x00FF00FFu;
        w[2] += b & 0x00FF00FFu;
        w[3] += (b >> 8) & 0x00FF00FFu;
        a = b = 0u;
    }
    __device__ __forceinline__ void finish() { end_batch(); }
    __device__ __forceinline__ uint32_t field_sum(int e) const
    {
        const int f = kFields - 1 - e;
        const int i = f >> 1; // byte of a (f even) or b (f odd)
        return (w[2 * (f & 1) + (i & 1)] >> (16 * (i >> 1))) & 0xFFFFu;
    }
};

template <> struct LevelSum<8> {
    static constexpr int kFields = 4, kBatchMax = 64;
    static constexpr uint32_t kSign = 0x80808080u;
    uint32_t w[2] = {0u, 0u}; // 16-bit lanes: bytes 0 / 2 and 1 / 3
    __device__ __forceinline__ void add(uint32_t word)
    {
        const uint32_t x = word ^ kSign;
        w[0] += x & 0x00FF00FFu;
        w[1] += (x >> 8) & 0x00FF00FFu;
    }
    __device__ __forceinline__ void end_batch() {}
    __device__ __forceinline__ void finish() {}
    __device__ __forceinline__ uint32_t field_sum(int e) const
    {
        const int f = kFields - 1 - e;
        return (w[f & 1] >> (16 * (f >> 1))) & 0xFFFFu;
    }
};

} // namespace qga
