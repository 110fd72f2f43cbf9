// mx_elem.cuh -- device helpers of the MX element formats shared by the quantizer and
// the GEMM epilogue that quantizes its output: packed bf16 abs-max, the E8M0 scale of a
// block, and the hardware conversions to E2M1 / E4M3 (round to nearest even,
// saturating, sign of a zero result kept).
#pragma once

#include <stdint.h>

namespace mxq {

// Packed max of |a| and |b| over two bf16 lanes (sign of the result is the xor of the
// signs, which the caller masks off); a NaN in either input yields NaN.
__device__ __forceinline__ uint32_t absmax_bf16x2(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("max.NaN.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

__device__ __forceinline__ float lo_f(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float hi_f(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Eight fp32 -> one word of eight E2M1 codes (v[i] in nibble i).
__device__ __forceinline__ uint32_t cvt_e2m1x8(const float (&v)[8])
{
    uint32_t r;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(r)
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
    return r;
}

// Two fp32 -> two E4M3 codes in a 16-bit word (first argument in the low byte).
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi)
{
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %2, %1;" : "=h"(r) : "f"(lo), "f"(hi));
    return r;
}

// E8M0 scale code of a block from the bf16 bit pattern of its absolute maximum: bf16
// and E8M0 share the exponent bias 127, so floor(log2 amax) + 127 is the exponent
// field; code = field - emax, clamped at 0 (zero and subnormal maxima), and 255 for a
// block holding Inf or NaN (exponent field 255).
template <uint32_t kEmax>
__device__ __forceinline__ uint32_t e8m0_code(uint32_t amax_bits)
{
    const uint32_t eb = (amax_bits & 0x7FFFu) >> 7;
    return eb == 255u ? 255u : (eb > kEmax ? eb - kEmax : 0u);
}

// 2^(127 - code) as fp32, the exact reciprocal of the scale.  Finite blocks give codes
// <= 252 (bf16 exponent fields stop at 254); for 255, a non-finite block, the caller
// forces the element codes to zero, so the clamp only keeps the value finite.
__device__ __forceinline__ float e8m0_inverse(uint32_t code)
{
    return __uint_as_float((254u - min(code, 253u)) << 23);
}

}  // namespace mxq
