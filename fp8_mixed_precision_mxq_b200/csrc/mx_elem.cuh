// mx_elem.cuh -- device helpers of the MX element formats shared by the quantizer and
// the GEMM epilogue that quantizes its output: packed bf16 abs-max, the E8M0 scale of a
// block, and the hardware conversions to E2M1 / E4M3 (round to nearest even,
// saturating, sign of a zero result kept); and the exact bf16 GELU of the fused FFN
// epilogue (a shared-memory table and closed forms).
#pragma once

#include <cuda_bf16.h>
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

// ---- GELU of bf16 values ---------------------------------------------------------------
// h = bf16(GELU(x)) for a bf16 x, GELU(x) = x/2 erfc(-x / sqrt 2) (the plain erf form) rounded
// once to bf16, nearest with ties to even: what a bf16 network's GELU gives when computed
// exactly.  For 2^-10 <= |x| < 16 (14 binades of 128 significands, both signs: 3584 values)
// the result comes from a table that the kernel using it builds in shared memory from the
// fp64 erfc.  Elsewhere it has a closed form: below 2^-10 it is x/2 rounded to bf16 (the
// next term, x^2 / sqrt(2 pi), moves x/2 by less than 0.8 |x| of itself, which is under half
// a bf16 unit); from 16 up it is x (1 - Phi(16) < 2^-190); from -16 down it is -0 (below the
// smallest bf16 magnitude); +Inf gives +Inf, -Inf and NaN give NaN (0x7FC0).
constexpr uint32_t kGeluLo = 0x3A80u;                 // bf16 magnitude bits of 2^-10
constexpr uint32_t kGeluSpan = 14u * 128u;            // magnitudes 2^-10 ... 16 (exclusive)
constexpr uint32_t kGeluEntries = 2u * kGeluSpan;     // positive, then negative
constexpr uint32_t kGeluTableBytes = 2u * kGeluEntries;

// Entry i of the table: bf16 bits of GELU of the bf16 value with sign i / kGeluSpan and
// magnitude bits kGeluLo + i % kGeluSpan.  The fp64 GELU is rounded to 8 significant bits
// (to a multiple of 2^-133 below 2^-126, bf16's subnormal step) with rint, then read as
// bf16: one rounding.
__device__ __forceinline__ uint16_t gelu_table_value(uint32_t i)
{
    const uint32_t b = ((i / kGeluSpan) << 15) | (kGeluLo + i % kGeluSpan);
    const double x = static_cast<double>(__uint_as_float(b << 16));
    const double g = 0.5 * x * erfc(-x / sqrt(2.0));
    int e = 0;
    frexp(g, &e);  // |g| in [2^(e-1), 2^e)
    const double ulp = ldexp(1.0, max(e - 8, -133));
    const double r = rint(g / ulp) * ulp;
    return static_cast<uint16_t>(__float_as_uint(static_cast<float>(r)) >> 16);
}

// Threads tid, tid + nthreads, ... fill their entries of the shared-memory table.
__device__ __forceinline__ void gelu_table_fill(uint16_t* lut, uint32_t tid, uint32_t nthreads)
{
    for (uint32_t i = tid; i < kGeluEntries; i += nthreads) lut[i] = gelu_table_value(i);
}

// GELU of one bf16 value (bits b, low 16 bits) through the table.
__device__ __forceinline__ uint32_t gelu_bf16_bits(uint32_t b, const uint16_t* lut)
{
    const uint32_t m = b & 0x7FFFu;
    const uint32_t neg = b >> 15;
    const uint32_t idx = m - kGeluLo;
    const bool in = idx < kGeluSpan;
    const uint32_t t = lut[in ? neg * kGeluSpan + idx : 0u];
    const uint32_t half = __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(b << 16) * 0.5f));
    uint32_t big = neg ? 0x8000u : b;
    if (m >= 0x7F80u) big = (m == 0x7F80u && !neg) ? b : 0x7FC0u;
    return in ? t : (m < kGeluLo ? half : big);
}

}  // namespace mxq
