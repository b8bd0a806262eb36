// quant_rule.cuh -- the per-token int8 code rule, shared by the activation
// kernels and the fused decode GEMV.
//
// "M8.8 - Native Binary and Ternary Transformers" 0x05C: per token
// gamma_t = max|x_t|, q = clip(rint((x*127) / (gamma_t + eps)), -128, 127)
// with one fp32 multiply and one IEEE fp32 divide, nearest-even ties
// (0x02C/0x02E); the reconstruction scale is gamma_t/127.
#pragma once

#include "lowbit_internal.cuh"

namespace lowbit {
namespace qrule {

template <typename T> struct In;
template <> struct In<float> {
    static constexpr int kPerVec = 4;
    __device__ static float get(const uint4 &v, int i) { return __uint_as_float((&v.x)[i]); }
    __device__ static float scalar(const void *p, int64_t i) { return ld_act_f32(static_cast<const float *>(p) + i); }
    // max of |x| bits over one vector (a non-finite value sorts above all finite ones)
    __device__ static uint32_t absmax_bits(const uint4 &v)
    {
        return max(max(v.x & 0x7fffffffu, v.y & 0x7fffffffu), max(v.z & 0x7fffffffu, v.w & 0x7fffffffu));
    }
};
template <> struct In<__nv_bfloat16> {
    static constexpr int kPerVec = 8;
    __device__ static float get(const uint4 &v, int i)
    {
        const uint32_t w = (&v.x)[i >> 1];
        return __uint_as_float((i & 1) ? (w & 0xffff0000u) : (w << 16));
    }
    __device__ static float scalar(const void *p, int64_t i)
    {
        const uint16_t h = ld_act_u16(static_cast<const uint16_t *>(p) + i);
        return __uint_as_float(static_cast<uint32_t>(h) << 16);
    }
    // 16-bit lane-wise max of the |x| bit patterns, then the larger half
    __device__ static uint32_t absmax_bits(const uint4 &v)
    {
        const uint32_t m = __vmaxu2(__vmaxu2(v.x & 0x7fff7fffu, v.y & 0x7fff7fffu),
                                    __vmaxu2(v.z & 0x7fff7fffu, v.w & 0x7fff7fffu));
        return max(m << 16, m & 0xffff0000u);
    }
};

__device__ __forceinline__ int8_t quant_one(float x, float d)
{
    float t = rintf(__fdiv_rn(__fmul_rn(x, 127.0f), d));
    t = fminf(fmaxf(t, -128.0f), 127.0f);
    return static_cast<int8_t>(static_cast<int>(t));
}

// Codes for four values without a divide or a conversion instruction each.
// The exact code is rint(z), z = RN(t/d), t = RN(127x).  With c = RN(127 *
// RN(1/d)) and u = RN(x*c), |u - t/d| <= (127|x|/d) * 4 * 2^-24 < 3.1e-5 and
// |z - t/d| <= 2^-18 < 3.9e-6 (|z| < 128), so |u - z| < 3.5e-5: u and z round
// to the same integer unless u lies within that distance of a midpoint
// k + 1/2.  Rounding uses the IEEE nearest-even addition v = u + 1.5*2^23,
// exact to the unit for |u| < 2^22: v - 1.5*2^23 is rint(u) and the low byte
// of v's bit pattern is the code in two's complement.  A value within 1e-4
// of a midpoint (about 2 in 10^4) sets `near`; the caller then redoes the
// four values with the IEEE divide.  |u| <= 127.0001, so no clamp is needed.
// The relative bounds need RN(1/d) and c normal and finite, i.e. d in
// [2^-121, 2^126); outside it the caller takes the divide for every value.
__device__ __forceinline__ uint32_t quant4(float x0, float x1, float x2, float x3, float c, bool &near)
{
    constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
    const float u0 = __fmul_rn(x0, c), u1 = __fmul_rn(x1, c), u2 = __fmul_rn(x2, c), u3 = __fmul_rn(x3, c);
    const float v0 = __fadd_rn(u0, kMagic), v1 = __fadd_rn(u1, kMagic);
    const float v2 = __fadd_rn(u2, kMagic), v3 = __fadd_rn(u3, kMagic);
    near |= fabsf(__fsub_rn(u0, __fsub_rn(v0, kMagic))) > 0.4999f;
    near |= fabsf(__fsub_rn(u1, __fsub_rn(v1, kMagic))) > 0.4999f;
    near |= fabsf(__fsub_rn(u2, __fsub_rn(v2, kMagic))) > 0.4999f;
    near |= fabsf(__fsub_rn(u3, __fsub_rn(v3, kMagic))) > 0.4999f;
    const uint32_t lo = __byte_perm(__float_as_uint(v0), __float_as_uint(v1), 0x0040);
    const uint32_t hi = __byte_perm(__float_as_uint(v2), __float_as_uint(v3), 0x0040);
    return __byte_perm(lo, hi, 0x5410);
}

__device__ __forceinline__ uint32_t quant4_exact(float x0, float x1, float x2, float x3, float d)
{
    return static_cast<uint32_t>(static_cast<uint8_t>(quant_one(x0, d))) |
           (static_cast<uint32_t>(static_cast<uint8_t>(quant_one(x1, d))) << 8) |
           (static_cast<uint32_t>(static_cast<uint8_t>(quant_one(x2, d))) << 16) |
           (static_cast<uint32_t>(static_cast<uint8_t>(quant_one(x3, d))) << 24);
}

}  // namespace qrule
}  // namespace lowbit
