// pa_codes.cuh -- the one-byte element formats of quantised K/V pools.
//
// "PagedAttention：大模型KV Cache分页管理优化实践" §7 names FP8 and INT8 storage of
// the cached blocks, and "vLLM用虚拟内存分页思想管理KV Cache" (工程实践与局限) names
// low-precision storage of block KV values.  A quantised pool holds one
// code per element and one scale per pool: value = decode(code) * scale.
//
//   E4m3Codes  OCP e4m3 ("e4m3fn").  Encoding rounds to nearest even and
//              saturates at +-448; NaN becomes 0x7F.
//   Int8Codes  two's complement.  Encoding rounds to nearest even and
//              saturates to [-128, 127]; NaN becomes 0.
//
// Every code of either format is an fp16 value, so the decode kernels widen
// codes to fp16 exactly and run the tensor cores in fp16.
//
//   widen4(w, lo, hi)  the four codes of w as two packed fp16 pairs:
//                      lo = (code 0, code 1), hi = (code 2, code 3), the
//                      lower-addressed code in the low half, each value
//                      plus kBias: decode(code) + kBias, exact in fp16.
//   kBias              0 for e4m3; 1152 for int8, whose widening is a byte
//                      permute that yields 1152 + c (the decode kernels
//                      remove the bias once per head instead of once per
//                      pair of codes).
//   encode2(a, b)      two fp32 values (already times 1 / scale) as two
//                      codes in the low 16 bits, a in the low byte.
//   kMax               the largest code magnitude (448 or 127): the code a
//                      row's largest element takes under a row scale.
#pragma once

#include <cuda_fp8.h>
#include <float.h>
#include <stdint.h>

#include "pa_common.cuh"

namespace pa {

struct E4m3Codes {
    static constexpr float kMax = 448.0f;
    static constexpr float kBias = 0.0f;

    static __device__ __forceinline__ void widen4(uint32_t w, uint32_t& lo, uint32_t& hi)
    {
        asm("{\n\t.reg .b16 l, h;\n\t"
            "mov.b32 {l, h}, %2;\n\t"
            "cvt.rn.f16x2.e4m3x2 %0, l;\n\t"
            "cvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
            : "=r"(lo), "=r"(hi)
            : "r"(w));
    }

    static __device__ __forceinline__ uint32_t encode2(float a, float b)
    {
        return static_cast<uint32_t>(
            __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3));
    }
};

struct Int8Codes {
    static constexpr float kMax = 127.0f;
    static constexpr float kBias = 1152.0f;

    // Exponent-field construction: with 0x64 as the high byte, an fp16 is
    // 1024 + (low byte), since its unit in [1024, 2048) is 1.  Flipping the
    // sign bit of a code c gives the byte c + 128, so the fp16 0x64:(c + 128)
    // is exactly 1152 + c.  The bias is left in (kBias).
    static __device__ __forceinline__ void widen4(uint32_t w, uint32_t& lo, uint32_t& hi)
    {
        const uint32_t u = w ^ 0x80808080u;                   // c + 128 in every byte
        lo = __byte_perm(u, 0x64646464u, 0x5140);              // [0x64 u1 0x64 u0]
        hi = __byte_perm(u, 0x64646464u, 0x5342);              // [0x64 u3 0x64 u2]
    }

    static __device__ __forceinline__ uint32_t encode1(float x)
    {
        // clamping to the integer ends before rounding equals rounding first
        const float y = x != x ? 0.f : fminf(fmaxf(x, -128.f), 127.f);
        return static_cast<uint32_t>(__float2int_rn(y)) & 0xffu;
    }

    static __device__ __forceinline__ uint32_t encode2(float a, float b)
    {
        return encode1(a) | (encode1(b) << 8);
    }
};

// Eight 16-bit elements (one 16-byte vector) as eight codes of x * inv,
// the product rounded once in fp32 before encoding.
template <typename Codes, typename T>
__device__ __forceinline__ uint2 encode8(const uint4& w, float inv)
{
    float f[8];
    unpack8<T>(w, f);
    uint32_t r[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) r[j] = Codes::encode2(f[2 * j] * inv, f[2 * j + 1] * inv);
    return make_uint2(r[0] | (r[1] << 16), r[2] | (r[3] << 16));
}

// Largest magnitude among the 8 elements of a 16-byte vector, exact.
template <typename T>
__device__ __forceinline__ float amax8(const uint4& w)
{
    float f[8];
    unpack8<T>(w, f);
    float m = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(f[i]));
    return m;
}

// One row of D elements quantised with a scale of its own, by a whole warp
// (lanes below D / 8 hold 8 elements each; every lane must call it):
//   amax = max |x|,  s = fp32(amax / kMax),  codes = encode8(x, fp32(1 / s)),
// the per-pool encoding with scale s, so the row's largest element takes the
// top code.  A row whose s is below the smallest normal fp32 (all zeros, or
// tiny values) gets s = 0 and zero codes.  `x` is the lane's 16-byte input
// vector (anything on lanes >= D / 8); returns the lane's 8 codes and sets
// `scale` on every lane.
template <typename Codes, typename T, int D>
__device__ __forceinline__ uint2 quantise_row_warp(const uint4& x, float& scale)
{
    const int lane = threadIdx.x & 31;
    float m = lane < D / 8 ? amax8<T>(x) : 0.f;
#pragma unroll
    for (int k = 16; k >= 1; k >>= 1) m = fmaxf(m, __shfl_xor_sync(kFullMask, m, k));
    const float s = m / Codes::kMax;
    if (!(s >= FLT_MIN)) {
        scale = 0.f;
        return make_uint2(0u, 0u);
    }
    scale = s;
    return encode8<Codes, T>(x, 1.0f / s);
}

}  // namespace pa
