// fo_codec.cuh - device-side formats of the FlashOptim-style compressed
// optimizer state: 16-bit downcast + ULP-normalised ECC masters, and 8-bit
// companded momentum / variance codes with one fp16 scale per 32 elements.
//
// Sources: "FlashOptim: Breaking the Memory Wall with 24-bit Weights and
// Companded States" (wispaper blog), sections "1. ULP-based Weight
// Splitting" and "2. Companded Quantization"; Davis Blalock's FlashOptim
// release thread, posts on the f32 interval that rounds to one downcast
// value, on integer-quantizing the position in it, on 8-bit states with a
// 16-bit scale per 32 elements, and on companding.
//
// Every function here is bit-exact with respect to the definitions in
// include/fo.h: only correctly rounded IEEE binary32 operations
// (__fadd_rn, __fmul_rn, __fmaf_rn, __fdiv_rn, __fsqrt_rn), documented
// conversions (round-to-nearest-even to bf16 / fp16, round-up to fp16,
// round-half-even to integer) and integer bit arithmetic are used.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace fo {

enum : int { kBF16 = 0, kFP16 = 1 };

constexpr int kGroup = 32;

template <int NB>
struct EccType;
template <>
struct EccType<8> {
    using type = int8_t;
};
template <>
struct EccType<16> {
    using type = int16_t;
};

// ---- 16-bit float <-> binary32 ------------------------------------------

template <int DT>
__device__ __forceinline__ float widen16(uint32_t h)
{
    if constexpr (DT == kBF16) {
        return __uint_as_float(h << 16);
    } else {
        return __half2float(__ushort_as_half((unsigned short)h));
    }
}

// round to nearest even (overflow -> inf); every NaN, whatever its sign and
// payload, becomes the positive quiet NaN with only the quiet bit set (bf16
// 0x7FC0, fp16 0x7E00): binary32 arithmetic gives NaNs no portable sign
template <int DT>
__device__ __forceinline__ uint32_t downcast16(float x)
{
    if (x != x) return DT == kBF16 ? 0x7FC0u : 0x7E00u;
    if constexpr (DT == kBF16) {
        return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(x));
    } else {
        return (uint32_t)__half_as_ushort(__float2half_rn(x));
    }
}

template <int DT>
__device__ __forceinline__ bool nonfinite16(uint32_t h)
{
    if constexpr (DT == kBF16) {
        return (h & 0x7F80u) == 0x7F80u;
    } else {
        return (h & 0x7C00u) == 0x7C00u;
    }
}

// ---- ULP-normalised ECC ---------------------------------------------------
//
// rho = round_half_even((x - x') * 2^N / u), clamped to +-(2^(N-1) - 1), where
// u is the spacing of the 16-bit grid at x' on the side of x' where x lies.
//
// bf16: inside the preimage of a bf16 value the binary32 grid is uniform
// with spacing u / 2^16 (also on the inward side of a power of two, where
// both spacings halve), so the code is the difference of the magnitude bit
// patterns, divided by 2^(16-N) with round-half-even.  Same sign bits cancel
// in the 32-bit subtraction.
//
// fp16: t = (|x| - |x'|) * 2^(N + 10 - E) is exact (Sterbenz for the
// difference, a power of two for the product), doubled on the inward side of
// a power of two above the smallest normal.

template <int DT, int NB>
__device__ __forceinline__ int ecc_encode(float x, uint32_t xp)
{
    constexpr int lim = (1 << (NB - 1)) - 1;
    if (nonfinite16<DT>(xp)) return 0;
    int r;
    if constexpr (DT == kBF16) {
        const int d = (int)(__float_as_uint(x) - (xp << 16));
        if constexpr (NB == 16) {
            r = d;
        } else {
            r = (d + 127 + ((d >> 8) & 1)) >> 8;
        }
    } else {
        const uint32_t ef = (xp >> 10) & 0x1Fu;
        const int E = ef ? (int)ef - 15 : -14;
        const float a = widen16<DT>(xp & 0x7FFFu);
        const float e = __fadd_rn(fabsf(x), -a);
        float t = __fmul_rn(e, __uint_as_float((uint32_t)(127 + NB + 10 - E) << 23));
        const bool pow2_above_min = ((xp & 0x3FFu) == 0) && ef > 1u;
        if (e < 0.0f && pow2_above_min) t = __fmul_rn(t, 2.0f);
        r = __float2int_rn(t);
    }
    r = r > lim ? lim : r;
    r = r < -lim ? -lim : r;
    return r;
}

template <int DT, int NB>
__device__ __forceinline__ float ecc_decode(uint32_t xp, int rho)
{
    if (rho == 0 || nonfinite16<DT>(xp)) return widen16<DT>(xp);
    if constexpr (DT == kBF16) {
        constexpr int unit = 1 << (16 - NB);
        if ((xp & 0x7FFFu) == 0u && rho < 0) {
            // inward from +-0 the value crosses zero: opposite sign, |rho| units
            return __uint_as_float(((xp ^ 0x8000u) << 16) | (uint32_t)(-rho * unit));
        }
        return __uint_as_float((xp << 16) + (uint32_t)(rho * unit));
    } else {
        const uint32_t ef = (xp >> 10) & 0x1Fu;
        const int E = ef ? (int)ef - 15 : -14;
        int k = E - 10 - NB;
        const bool pow2_above_min = ((xp & 0x3FFu) == 0) && ef > 1u;
        if (rho < 0 && pow2_above_min) k -= 1;
        float sc = __uint_as_float((uint32_t)(127 + k) << 23);
        if (xp & 0x8000u) sc = -sc;
        return __fmaf_rn((float)rho, sc, widen16<DT>(xp));
    }
}

// ---- companded 8-bit states -----------------------------------------------

// fp16 of a >= 0 rounded toward +inf, saturated at 65504 (0x7BFF)
__device__ __forceinline__ uint32_t scale_fp16_up(float a)
{
    uint32_t s = (uint32_t)__half_as_ushort(__float2half_ru(a));
    return s > 0x7BFFu ? 0x7BFFu : s;
}

// a state value that takes part in its group's scale and gets a code: inf
// and NaN do not (they are stored as code 0)
__device__ __forceinline__ bool finite32(float z) { return fabsf(z) <= 3.40282347e38f; }

// momentum: code = clamp(rint(127 * (2y / (1 + |y|))), +-127), y = z * r
__device__ __forceinline__ int m_code(float z, float r)
{
    if (!finite32(z)) return 0;
    const float y = __fmul_rn(z, r);
    const float c = __fdiv_rn(__fmul_rn(2.0f, y), __fadd_rn(1.0f, fabsf(y)));
    int q = __float2int_rn(__fmul_rn(127.0f, c));
    q = q > 127 ? 127 : q;
    q = q < -127 ? -127 : q;
    return q;
}

// variance: code = min(255, rint(sqrt(v) * k)), k = 255 / S
__device__ __forceinline__ int v_code(float sv, float k)
{
    if (!finite32(sv)) return 0;
    int q = __float2int_rn(__fmul_rn(sv, k));
    q = q > 255 ? 255 : q;
    q = q < 0 ? 0 : q;
    return q;
}

// decode tables: lut_m[b] = phi^-1((int8)b / 127), lut_v[b] = b / 255
__device__ __forceinline__ float lut_m_entry(int b)
{
    const float c = __fdiv_rn((float)(int8_t)b, 127.0f);
    return __fdiv_rn(c, __fadd_rn(2.0f, -fabsf(c)));
}

__device__ __forceinline__ float lut_v_entry(int b) { return __fdiv_rn((float)b, 255.0f); }

}  // namespace fo
