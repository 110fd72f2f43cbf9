// quant.cu -- MX block quantizer / dequantizer kernels (HBM-bound).
//
// The quantizer implements the MX format as the blog "Quark Mixed-Precision
// Quantization for Wan2.2 Video Generation on AMD Instinct GPUs" uses it (section
// "Quantization formats"): per block of 32 consecutive elements along K, the
// absolute maximum gives an E8M0 scale 2^(floor(log2 amax) - emax) (emax 2 for
// E2M1, 8 for E4M3; clamped at 2^-127), and each element x / scale is rounded to
// nearest-even onto the element grid with saturation (RTN).
//
// Work split: the tensor is read as a flat run of 16-byte groups of 8 bf16; four
// consecutive lanes hold one 32-element block, so the block absmax takes two
// xor-shuffles.  Each warp covers 256 consecutive elements per step; a warp step
// keeps several 16-byte loads in flight per lane.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <cmath>
#include <numeric>

#include "mx_elem.cuh"
#include "mxq_internal.h"
#include "ptx.cuh"


namespace mxq {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;  // 16-byte loads in flight per lane per step (measured best of 4, 8, 16)

// The quantizers stream their input once and write their output once: the loads carry
// an L2 evict-first policy and bypass L1, the code stores are streaming (.cs) stores, so
// neither side keeps lines in L2 that the next launch's stream would have to evict
// (measured on the 720p activations: +7 % for E2M1, +13 % for E4M3).
__device__ __forceinline__ uint4 ld_stream(const uint4* p)
{
    uint4 v;
    uint64_t pol;
    asm("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p), "l"(pol));
    return v;
}


// Byte offset of scale (r, kb) in the tiled 128x4 atom layout.
__device__ __forceinline__ uint32_t sf_offset(uint32_t r, uint32_t kb, uint32_t atoms_k)
{
    return ((r >> 7) * atoms_k + (kb >> 2)) * 512u + (r & 31u) * 16u + ((r >> 5) & 3u) * 4u + (kb & 3u);
}

// Static per-tensor E4M3 (the format template argument kFmtStatic): every element x
// becomes RNE_sat(x / s) on the E4M3 grid, x / s the exact quotient by the tensor's
// scale s; the block scales are all 127 (x1) and the GEMM applies s to its sums.
constexpr int kFmtStatic = 2;

// The scale as the static quantizer takes it: s = sn * 2^-k with sn in [1, 2), the
// reciprocal r = fl32(1/sn) in (1/2, 1], and 2^k as p1 (and p2 when two_step: k runs from
// -127 to 149, and 2^k is a binary32 normal only up to 127).
struct StaticScale {
    float sn, r, p1, p2;
    int two_step;
};

// One value's E4M3 code is RNE_sat(x / s), decided exactly in binary32:
//  * xs = x * 2^k, so that x / s = xs / sn with sn in [1, 2) (exact, except overflow, where
//    x / s is above 2^127 and saturates either way, and underflow, where x / s is below
//    2^-125 and rounds to a zero of x's sign either way); |xs| is then clamped to the
//    largest finite binary32 (sign and NaN kept: Inf saturates like any huge value), so
//    with r <= 1 every later value stays finite;
//  * q0 = fl(xs * r), then one Markstein correction q1 = fl(q0 + fl(xs - q0 sn) * r)
//    (fused multiply-adds; M. Cornea, J. Harrison, P. Tang, "Scientific Computing on
//    Itanium-based Systems", and J.-M. Muller et al., "Handbook of Floating-Point
//    Arithmetic", on division by Newton-Raphson iterations): q0 is within about 2^-23
//    relative, the correction leaves about 2^-46 before its own rounding, so q1 is within
//    half an ulp plus 2^-22 ulp of xs / sn: faithful, and the correctly rounded quotient
//    unless xs / sn lies that close to a midpoint between binary32 values;
//  * the remainder e1 = xs - q1 sn of a faithful quotient is a binary32 number whenever
//    |xs| >= 2^-102 (both terms are multiples of 2^(floor(log2 |xs|) - 47)), so the fused
//    multiply-add returns it exactly; below 2^-102 the quotient is far under E4M3's
//    smallest midpoint 2^-10 and only its sign matters;
//  * z = fl_rz(q1 + e1 r) (a fused multiply-add rounded toward zero) is the quotient
//    truncated to binary32: q1 + e1 / sn is the exact quotient, e1 r moves it by less than
//    an ulp of q1 in the same direction, and it could reach the next binary32 value only if
//    the quotient lay within 2^-24 ulp of it -- where q1 is the correctly rounded quotient
//    and |e1 / sn| is at most half an ulp;
//  * setting z's last bit when e1 != 0 gives the quotient rounded to odd (S. Boldo,
//    G. Melquiond, "Emulation of FMA and correctly rounded sums: proved algorithms using
//    rounding to odd", IEEE TC 2008), and rounding a round-to-odd value of at least two more
//    bits than the target gives the same result as rounding the exact value once: cvt's
//    round-to-nearest-even is then the exact quotient's.  The sign is copied from xs (a
//    zero quotient keeps x's sign).
__device__ __forceinline__ float clamp_finite(float v)
{
    float d;
    // sign(v) * min(|v|, largest finite), NaN kept
    asm("min.NaN.xorsign.abs.f32 %0, %1, 0f7F7FFFFF;" : "=f"(d) : "f"(v));
    return d;
}

__device__ __forceinline__ float2 static_quotient2(float2 x, const StaticScale& st)
{
    float2 xs = __fmul2_rn(x, make_float2(st.p1, st.p1));
    if (st.two_step) xs = __fmul2_rn(xs, make_float2(st.p2, st.p2));
    xs = make_float2(clamp_finite(xs.x), clamp_finite(xs.y));
    const float2 r = make_float2(st.r, st.r), ns = make_float2(-st.sn, -st.sn);
    const float2 q0 = __fmul2_rn(xs, r);
    const float2 q1 = __ffma2_rn(__ffma2_rn(q0, ns, xs), r, q0);
    const float2 e1 = __ffma2_rn(q1, ns, xs);
    const float2 z = __ffma2_rz(e1, r, q1);
    const uint32_t zx = (__float_as_uint(z.x) & 0x7FFFFFFFu) | (__float_as_uint(xs.x) & 0x80000000u);
    const uint32_t zy = (__float_as_uint(z.y) & 0x7FFFFFFFu) | (__float_as_uint(xs.y) & 0x80000000u);
    return make_float2(__uint_as_float(zx | (e1.x != 0.0f ? 1u : 0u)),
                       __uint_as_float(zy | (e1.y != 0.0f ? 1u : 0u)));
}

template <int FMT>
__global__ void __launch_bounds__(kThreads) quantize_kernel(const uint4* __restrict__ x, uint32_t n_groups,
                                                            uint32_t KB, uint64_t kb_magic, uint32_t atoms_k,
                                                            uint32_t rows, uint8_t* __restrict__ codes,
                                                            uint8_t* __restrict__ sf, StaticScale st)
{
    constexpr bool kStatic = FMT == kFmtStatic;
    constexpr int kElem = kStatic ? kFmtE4M3 : FMT;
    constexpr uint32_t kEmax = kElem == kFmtE4M3 ? 8u : 2u;
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t nwarps = gridDim.x * (kThreads / 32);
    const uint32_t warp = blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5);

    static_assert(kUnroll % 4 == 0, "the scale bytes of a step are stored kUnroll / 4 per lane");
    for (uint32_t w0 = warp; w0 * 32u < n_groups; w0 += nwarps * kUnroll) {
        uint4 v[kUnroll];
        uint32_t g[kUnroll];
        uint32_t scw[kUnroll / 4] = {};  // the scale codes of this quad's block, a byte per u
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            g[u] = (w0 + u * nwarps) * 32u + lane;
            v[u] = g[u] < n_groups ? ld_stream(x + g[u]) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            uint32_t sc;
            float inv = 1.0f;
            if constexpr (kStatic) {
                if (g[u] >= n_groups) continue;
                sc = 127u;
            } else {
                // block absmax over the quad of lanes holding the 32 elements
                uint32_t m2 = absmax_bf16x2(absmax_bf16x2(v[u].x, v[u].y), absmax_bf16x2(v[u].z, v[u].w));
                m2 = absmax_bf16x2(m2, __byte_perm(m2, 0, 0x1032));
                uint32_t amax = m2 & 0x7FFFu;
                amax = max(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
                amax = max(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 2));
                if (g[u] >= n_groups) continue;
                const uint32_t eb = amax >> 7;  // biased exponent of amax (bf16 and E8M0 share bias 127)
                sc = eb == 255u ? 255u : (eb > kEmax ? eb - kEmax : 0u);
                inv = __uint_as_float((254u - min(sc, 253u)) << 23);  // 2^(127 - sc)
            }
            const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
            float2 f[4];
            if constexpr (kStatic) {
#pragma unroll
                for (int i = 0; i < 4; ++i) f[i] = static_quotient2(make_float2(lo_f(w[i]), hi_f(w[i])), st);
            } else {
                // x * 2^-s, two lanes of binary32 a multiply (each rounded as the scalar one)
                const float2 inv2 = make_float2(inv, inv);
#pragma unroll
                for (int i = 0; i < 4; ++i) f[i] = __fmul2_rn(make_float2(lo_f(w[i]), hi_f(w[i])), inv2);
            }
            const uint32_t keep = sc == 255u ? 0u : 0xFFFFFFFFu;
            // cvt rounds to nearest even, saturates, and keeps the sign of a value that
            // rounds to zero (-0 = 0x8 / 0x80), as the format reading requires
            if (kElem == kFmtE2M1) {
                const float q[8] = {f[0].x, f[0].y, f[1].x, f[1].y, f[2].x, f[2].y, f[3].x, f[3].y};
                __stcs(reinterpret_cast<unsigned int*>(codes) + g[u], cvt_e2m1x8(q) & keep);
            } else {
                uint32_t out[2];
#pragma unroll
                for (int i = 0; i < 2; ++i)
                    out[i] = (cvt_e4m3x2(f[2 * i].x, f[2 * i].y) | (cvt_e4m3x2(f[2 * i + 1].x, f[2 * i + 1].y) << 16)) &
                             keep;
                __stcs(reinterpret_cast<uint2*>(codes) + g[u], make_uint2(out[0], out[1]));
            }
            scw[u >> 2] |= sc << (8 * (u & 3));
        }
        // The step's 8 kUnroll scale bytes (8 blocks for each u), kUnroll / 4 per lane: lane
        // 4 q + j stores those of block q for u = j, j + 4, ...
#pragma unroll
        for (int h = 0; h < kUnroll / 4; ++h) {
            const uint32_t u = (lane & 3u) + 4u * h;
            const uint32_t gq = (w0 + u * nwarps) * 32u + (lane & ~3u);  // the block's first group
            if (gq < n_groups) {
                const uint32_t blk = gq >> 2;
                // (blk * kb_magic) >> 40 without a 64-bit overflow: blk < 2^29 and
                // kb_magic <= 2^40, so the product needs up to 69 bits
                const uint32_t r = static_cast<uint32_t>(__umul64hi(static_cast<uint64_t>(blk) << 24, kb_magic));
                const uint32_t kb = blk - r * KB;
                sf[sf_offset(r, kb, atoms_k)] = static_cast<uint8_t>(scw[h] >> (8u * (lane & 3u)));
            }
        }
    }

    // zero the padding of the tiled scale buffer: k-blocks KB..4*atoms_k-1 of real
    // rows, and every k-block of rows rows..ceil128(rows)-1
    const uint32_t kbp = atoms_k * 4u;
    const uint32_t pad_k = kbp - KB;
    const uint32_t rows_p = (rows + 127u) & ~127u;
    const uint32_t n_pad_a = rows * pad_k;
    const uint32_t n_pad = n_pad_a + (rows_p - rows) * kbp;
    for (uint32_t p = blockIdx.x * kThreads + threadIdx.x; p < n_pad; p += gridDim.x * kThreads) {
        uint32_t r, kb;
        if (p < n_pad_a) {
            r = p / pad_k;
            kb = KB + (p - r * pad_k);
        } else {
            const uint32_t q = p - n_pad_a;
            r = rows + q / kbp;
            kb = q - (q / kbp) * kbp;
        }
        sf[sf_offset(r, kb, atoms_k)] = 0;
    }
}

// 2^(sc - 127) as fp32 (2^-127 is an fp32 subnormal); NaN for sc = 255.
__device__ __forceinline__ float scale_val(uint32_t sc)
{
    if (sc == 255u) return __uint_as_float(0x7FC00000u);
    return sc ? __uint_as_float(sc << 23) : __uint_as_float(0x00400000u);
}

// Two codes of one byte (E2M1 pair, first element in the low nibble) or of one 16-bit word
// (E4M3 pair, first element in the low byte) -> their values as f16x2, exactly (every E2M1
// and E4M3 value, NaN included, is an f16 value), widened to binary32.
__device__ __forceinline__ float2 e2m1x2_to_float2(uint32_t byte)
{
    uint32_t h2;
    asm("{\n\t.reg .b8 b;\n\tcvt.u8.u32 b, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, b;\n\t}" : "=r"(h2) : "r"(byte));
    return __half22float2(*reinterpret_cast<const __half2*>(&h2));
}

__device__ __forceinline__ float2 e4m3x2_to_float2(uint32_t pair)
{
    uint32_t h2;
    asm("{\n\t.reg .b16 w;\n\tcvt.u16.u32 w, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, w;\n\t}" : "=r"(h2) : "r"(pair));
    return __half22float2(*reinterpret_cast<const __half2*>(&h2));
}

// Lanes take 8-element groups in order (four lanes per MX block, like the quantizer), so the
// warp's code loads and its 16-byte bf16 stores are contiguous; kDqGroups groups per lane, one
// step per warp (the grid covers the tensor).  value = code value x 2^(scale - 127), a product
// binary32 holds exactly, rounded once to bf16 (nearest even): exact except that large scales
// overflow to Inf and E4M3 codes under scale codes 0-2 can fall below bf16's 2^-133 step.
// Measured on B200 against one lane per 32-element block: +27 to +37 %, 5.6-6.6 TB/s.
constexpr int kDqGroups = 4;
template <int FMT>
__global__ void __launch_bounds__(kThreads) dequantize_kernel(const uint8_t* __restrict__ codes,
                                                              const uint8_t* __restrict__ sf, uint32_t n_groups,
                                                              uint32_t KB, uint64_t kb_magic, uint32_t atoms_k,
                                                              uint4* __restrict__ out)
{
    constexpr int kGU = kDqGroups;
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t nwarps = gridDim.x * (kThreads / 32);
    const uint32_t warp = blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5);
    for (uint32_t w0 = warp; w0 * 32u < n_groups; w0 += nwarps * kGU) {
        uint2 c[kGU];
        uint32_t sc[kGU];
#pragma unroll
        for (int u = 0; u < kGU; ++u) {
            const uint32_t g = (w0 + u * nwarps) * 32u + lane;
            if (g >= n_groups) continue;
            if (FMT == kFmtE4M3) c[u] = __ldcs(reinterpret_cast<const uint2*>(codes) + g);
            else c[u].x = __ldcs(reinterpret_cast<const unsigned int*>(codes) + g);
            const uint32_t blk = g >> 2;
            const uint32_t r = static_cast<uint32_t>(__umul64hi(static_cast<uint64_t>(blk) << 24, kb_magic));
            sc[u] = sf[sf_offset(r, blk - r * KB, atoms_k)];
        }
#pragma unroll
        for (int u = 0; u < kGU; ++u) {
            const uint32_t g = (w0 + u * nwarps) * 32u + lane;
            if (g >= n_groups) continue;
            const float s = scale_val(sc[u]);
            const float2 s2 = make_float2(s, s);
            uint32_t o[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float2 v = FMT == kFmtE4M3 ? e4m3x2_to_float2((k < 2 ? c[u].x : c[u].y) >> (16 * (k & 1)))
                                                 : e2m1x2_to_float2(c[u].x >> (8 * k));
                const float2 y = __fmul2_rn(v, s2);
                __nv_bfloat162 h = __floats2bfloat162_rn(y.x, y.y);
                o[k] = *reinterpret_cast<uint32_t*>(&h);
            }
            __stcs(out + g, make_uint4(o[0], o[1], o[2], o[3]));
        }
    }
}

__global__ void sf_to_logical_kernel(const uint8_t* __restrict__ sf, uint32_t rows, uint32_t KB, uint32_t atoms_k,
                                     uint8_t* __restrict__ out)
{
    const uint32_t n = rows * KB;
    for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
        const uint32_t r = i / KB, kb = i - r * KB;
        out[i] = sf[sf_offset(r, kb, atoms_k)];
    }
}

int num_sms()
{
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

// ---------------------------------------------------------------------------- transform_on
// The activation (or weight) is transformed before it is quantized: t = x * mul per
// channel (SmoothQuant's 1/s for activations, s for weights; mul may be null), then each
// block of kB consecutive values along K is rotated by the Sylvester Hadamard matrix
// normalized by c = fl32(1/sqrt kB), and the result is MX-quantized from the binary32
// values.  Every step is one binary32 operation -- the multiply by mul, butterflies
// (a, b) -> (a + b, a - b) for h = 1, 2, 4, ..., kB/2, then the multiply by c -- written
// with the _rn intrinsics so the compiler cannot fuse them.  A value t thus differs from
// the exact transform by at most about (log2 kB + 4) u sum_i |x_i mul_i| / sqrt kB
// (u = 2^-24), and its code is the exact transform's wherever that lies farther than
// this from an MX rounding boundary.
// Layout for kB = 32: one lane per 32-element MX block; the 32-point transform, the
// block's abs-max and its scale byte stay in the lane.  Input: x seen as a [n_blocks, 32]
// bf16 tensor; each warp streams spans of 32 blocks (2 KB) into its own ring of
// shared-memory stages with TMA (64-byte swizzle: 16-byte chunk q of row r sits at chunk
// q ^ ((r >> 1) & 3), so the lanes' 16-byte reads of their own rows are free of bank
// conflicts).  kB = 128 has a kernel of its own below.

// threads of the transform quantizer's CTAs: 4 warps, 5 CTAs an SM
constexpr int kTThreads = 128;
constexpr int kTStages = 4;  // spans in flight per warp
constexpr uint32_t kSpanBytes = 32u * 64u;
constexpr uint64_t kTWaitNs = 1000000000ull;

__device__ uint32_t g_quant_status;

template <int FMT>
__global__ void __launch_bounds__(kTThreads, 5) quantize_transform_kernel(
    const __grid_constant__ CUtensorMap map_x, uint32_t n_blocks, uint32_t KB, uint64_t kb_magic, uint32_t atoms_k,
    uint32_t rows, const float* __restrict__ mul, float c, uint8_t* __restrict__ codes, uint8_t* __restrict__ sf,
    uint32_t debug)
{
    constexpr uint32_t kEmax = FMT == kFmtE4M3 ? 8u : 2u;
    constexpr int kWarps = kTThreads / 32;
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t wid = threadIdx.x >> 5;
    const uint32_t nwarps = gridDim.x * kWarps;
    const uint32_t warp = blockIdx.x * kWarps + wid;
    __shared__ __align__(1024) uint8_t ring[kWarps][kTStages][kSpanBytes];
    __shared__ __align__(8) uint64_t full[kWarps][kTStages];
    // The launch makes every span of a warp hold the same k-blocks in the same lanes (a
    // warp has one span, or the warp count times 32 is a multiple of KB), so each lane
    // loads the multipliers of its 32 channels once and keeps them in registers.
    float2 mreg[16];
    if (mul != nullptr) {
        const uint32_t kb0 = static_cast<uint32_t>((static_cast<uint64_t>(warp) * 32u + lane) % KB);
        const float4* m4 = reinterpret_cast<const float4*>(mul + kb0 * 32u);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const float4 v = __ldg(m4 + q);
            mreg[2 * q] = make_float2(v.x, v.y);
            mreg[2 * q + 1] = make_float2(v.z, v.w);
        }
    }
    const float2 neg1 = make_float2(-1.f, -1.f);
    const uint32_t stride = nwarps * 32u;
    const uint32_t first = warp * 32u;
    // spans of this warp: first, first + stride, ...; the one with index i sits in stage
    // i % kTStages, whose barrier completes its (i / kTStages)-th phase when it lands
    const uint32_t n_spans = first < n_blocks ? (n_blocks - first + stride - 1) / stride : 0u;
    if (lane == 0) {
        for (int st = 0; st < kTStages; ++st) mbar_init(&full[wid][st], 1);
        fence_mbar_init();
    }
    __syncwarp();
    const uint64_t policy = policy_evict_first();
    auto issue = [&](uint32_t i) {  // lane 0 only
        const int st = static_cast<int>(i % kTStages);
        fence_async_smem();  // the lanes' reads of this stage come before the copy's writes
        mbar_arrive_expect_tx(&full[wid][st], kSpanBytes);
        tma_load_2d<1>(ring[wid][st], &map_x, 0, static_cast<int32_t>(first + i * stride),
                       smem_u32(&full[wid][st]), policy);
    };
    if (lane == 0)
        for (uint32_t i = 0; i < n_spans && i < static_cast<uint32_t>(kTStages); ++i)
            if (!((debug & 2u) && warp == 0 && i == 0)) issue(i);  // debug bit 1: warp 0's first span never lands
    for (uint32_t i = 0; i < n_spans; ++i) {
        const int st = static_cast<int>(i % kTStages);
        const bool landed = mbar_wait(&full[wid][st], (i / kTStages) & 1u, kTWaitNs);
        if (!__all_sync(0xFFFFFFFFu, landed)) {
            // a copy never landed: report it, let the copies still in flight finish
            // (each wait again bounded), and leave
            if (lane == 0) {
                atomicCAS(&g_quant_status, 0u, static_cast<uint32_t>(MXQ_ERR_TIMEOUT));
                const uint32_t issued = min(n_spans, i + static_cast<uint32_t>(kTStages));
                for (uint32_t j = i; j < issued; ++j)
                    mbar_wait(&full[wid][j % kTStages], (j / kTStages) & 1u, kTWaitNs);
            }
            __syncwarp();
            return;
        }
        const uint8_t* row = ring[wid][st] + lane * 64u;
        const uint32_t sw = (lane >> 1) & 3u;
        uint4 v[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) v[q] = *reinterpret_cast<const uint4*>(row + 16u * (static_cast<uint32_t>(q) ^ sw));
        __syncwarp();  // every lane has read the stage before it is refilled
        if (lane == 0 && i + kTStages < n_spans) issue(i + kTStages);
        const uint32_t blk = first + i * stride + lane;
        const bool live = blk < n_blocks;
        float2 t[16];  // t[k] holds values 2k and 2k + 1 of the lane's block
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint32_t w[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) t[4 * q + e] = make_float2(lo_f(w[e]), hi_f(w[e]));
        }
        if (mul != nullptr)
#pragma unroll
            for (int k = 0; k < 16; ++k) t[k] = __fmul2_rn(t[k], mreg[k]);
        // Butterflies inside the lane.  h = 1 pairs the two halves of a register pair and
        // runs on scalars; h = 2, 4, 8, 16 pair whole register pairs and run as packed
        // binary32 operations (each half rounded as the scalar one), the difference a - b
        // as fma(b, -1, a): an exact product and one rounding, the IEEE difference.
#pragma unroll
        for (int k = 0; k < 16; ++k) t[k] = make_float2(__fadd_rn(t[k].x, t[k].y), __fsub_rn(t[k].x, t[k].y));
#pragma unroll
        for (int m = 1; m < 16; m <<= 1)
#pragma unroll
            for (int k = 0; k < 16; ++k)
                if ((k & m) == 0) {
                    const float2 a = t[k], b = t[k + m];
                    t[k] = __fadd2_rn(a, b);
                    t[k + m] = __ffma2_rn(b, neg1, a);
                }
        if (!live) continue;
        const uint32_t r = static_cast<uint32_t>(__umul64hi(static_cast<uint64_t>(blk) << 24, kb_magic));
        const uint32_t kb = blk - r * KB;
        // The block's scale comes from max |t c| = fl(max |t| c) (rounding is monotone and
        // c > 0; a NaN propagates through the max, and Inf or NaN gives exponent field 255,
        // so such a block gets code 255).  The element codes are cvt(fl(fl(t c) / 2^s)).
        // For 11 <= code <= 249 that equals cvt(fl(t (c 2^-s))), one multiply: c 2^-s is
        // a normal binary32, so wherever fl(t c) and the result are normal, scaling by the
        // power of two commutes with the rounding; where fl(t c) is subnormal, both
        // results lie at or below 2^-126 2^(127 - 11) = 2^-10, which E2M1 and E4M3 round
        // to a zero of the value's sign.  Other codes take the two multiplies.
        float mc[4] = {0.f, 0.f, 0.f, 0.f};  // four independent chains, then their max
#pragma unroll
        for (int k = 0; k < 16; ++k)
            asm("max.NaN.abs.f32 %0, %1, %2, %3;" : "=f"(mc[k & 3]) : "f"(mc[k & 3]), "f"(t[k].x), "f"(t[k].y));
        float m;
        asm("max.NaN.abs.f32 %0, %1, %2, %3;" : "=f"(m) : "f"(mc[0]), "f"(mc[1]), "f"(mc[2]));
        asm("max.NaN.f32 %0, %1, %2;" : "=f"(m) : "f"(m), "f"(mc[3]));
        const uint32_t eb = (__float_as_uint(__fmul_rn(m, c)) & 0x7FFFFFFFu) >> 23;
        const uint32_t sc = eb == 255u ? 255u : (eb > kEmax ? eb - kEmax : 0u);
        float mult = e8m0_inverse(sc);  // 2^-s, or c 2^-s on the one-multiply path
        const uint32_t keep = sc == 255u ? 0u : 0xFFFFFFFFu;
        if (sc - 11u <= 249u - 11u) {
            mult = __fmul_rn(c, mult);
        } else {
            const float2 c2 = make_float2(c, c);
#pragma unroll
            for (int k = 0; k < 16; ++k) t[k] = __fmul2_rn(t[k], c2);
        }
        const float2 mult2 = make_float2(mult, mult);
#pragma unroll
        for (int k = 0; k < 16; ++k) t[k] = __fmul2_rn(t[k], mult2);
        if (FMT == kFmtE2M1) {
            uint32_t w[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float q[8] = {t[4 * k].x,     t[4 * k].y,     t[4 * k + 1].x, t[4 * k + 1].y,
                                    t[4 * k + 2].x, t[4 * k + 2].y, t[4 * k + 3].x, t[4 * k + 3].y};
                w[k] = cvt_e2m1x8(q) & keep;
            }
            __stcs(reinterpret_cast<uint4*>(codes) + blk, make_uint4(w[0], w[1], w[2], w[3]));
        } else {
            uint32_t w[8];
#pragma unroll
            for (int k = 0; k < 8; ++k)
                w[k] = (cvt_e4m3x2(t[2 * k].x, t[2 * k].y) | (cvt_e4m3x2(t[2 * k + 1].x, t[2 * k + 1].y) << 16)) & keep;
            uint4* dst = reinterpret_cast<uint4*>(codes) + static_cast<size_t>(blk) * 2u;
            __stcs(dst, make_uint4(w[0], w[1], w[2], w[3]));
            __stcs(dst + 1, make_uint4(w[4], w[5], w[6], w[7]));
        }
        sf[sf_offset(r, kb, atoms_k)] = static_cast<uint8_t>(sc);
    }
    // the padding of the tiled scale buffer, as in quantize_kernel
    const uint32_t kbp = atoms_k * 4u;
    const uint32_t pad_k = kbp - KB;
    const uint32_t rows_p = (rows + 127u) & ~127u;
    const uint32_t n_pad_a = rows * pad_k;
    const uint32_t n_pad = n_pad_a + (rows_p - rows) * kbp;
    for (uint32_t p = blockIdx.x * kTThreads + threadIdx.x; p < n_pad; p += gridDim.x * kTThreads) {
        uint32_t rr, k;
        if (p < n_pad_a) {
            rr = p / pad_k;
            k = KB + (p - rr * pad_k);
        } else {
            const uint32_t q = p - n_pad_a;
            rr = rows + q / kbp;
            k = q - (q / kbp) * kbp;
        }
        sf[sf_offset(rr, k, atoms_k)] = 0;
    }
}

// kB = 128: one lane per rotation block.  The lane holds the block's 128 values (four MX
// blocks) as 64 register pairs, so all seven butterfly stages stay in the lane and no
// value crosses lanes.  A warp streams spans of 32 rows x 128 channels -- two TMA boxes
// of 32 rows x 64 channels with the 128-byte swizzle (16-byte chunk q of row r sits at
// chunk q ^ (r & 7), so the lanes' reads of their own rows are free of bank conflicts)
// -- and lane l takes row l; the 128 values take most of a thread's 164 registers, so an
// SM holds 12 warps (three CTAs of four) with two spans in flight each.  The lanes of a
// warp share the span's channels, so each multiplier is one warp-uniform load.  The
// codes of a lane's four MX blocks are 64
// (E2M1) or 128 (E4M3) contiguous bytes of its row, and its four scale bytes one 32-bit
// word of the tiled scale layout (k-blocks 4g .. 4g + 3 of a row are adjacent there).
constexpr int kT128Warps = 4;
constexpr int kT128Stages = 2;
constexpr uint32_t kBox128Bytes = 32u * 128u;          // 32 rows x 64 bf16
constexpr uint32_t kSpan128Bytes = 2u * kBox128Bytes;  // 32 rows x 128 bf16
constexpr uint32_t kT128Smem = kT128Warps * kT128Stages * kSpan128Bytes + 1024u;  // + alignment slack

template <int FMT>
__global__ void __launch_bounds__(kT128Warps * 32, 3) quantize_transform128_kernel(
    const __grid_constant__ CUtensorMap map_x, uint32_t rows, uint32_t K, uint32_t KG, uint32_t n_spans_all,
    uint32_t atoms_k, const float* __restrict__ mul, float c, uint8_t* __restrict__ codes, uint8_t* __restrict__ sf,
    uint32_t debug)
{
    constexpr uint32_t kEmax = FMT == kFmtE4M3 ? 8u : 2u;
    extern __shared__ uint8_t dsm[];
    __shared__ __align__(8) uint64_t full[kT128Warps][kT128Stages];
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t wid = threadIdx.x >> 5;
    const uint32_t warp = blockIdx.x * kT128Warps + wid;
    const uint32_t nwarps = gridDim.x * kT128Warps;
    // the 128-byte swizzle wants 1024-byte aligned boxes
    uint8_t* ring = dsm + ((1024u - (smem_u32(dsm) & 1023u)) & 1023u) + wid * (kT128Stages * kSpan128Bytes);
    // spans of this warp: warp, warp + nwarps, ...; span s covers rows 32 (s / KG) ..
    // 32 (s / KG) + 31 and channels 128 (s % KG) .. + 127; the one with index i sits in
    // stage i % kT128Stages, whose barrier completes its (i / kT128Stages)-th phase when
    // both boxes land
    const uint32_t n_spans = warp < n_spans_all ? (n_spans_all - warp + nwarps - 1) / nwarps : 0u;
    if (lane == 0) {
        for (int st = 0; st < kT128Stages; ++st) mbar_init(&full[wid][st], 1);
        fence_mbar_init();
    }
    __syncwarp();
    const uint64_t policy = policy_evict_first();
    // spans are visited in order, so their (row group, channel group) pairs are stepped by
    // nwarps = d_rg KG + d_g instead of divided out: p_ for the next span to load (lane 0),
    // c_ for the next one to quantize
    const uint32_t d_rg = nwarps / KG, d_g = nwarps - d_rg * KG;
    auto advance = [&](uint32_t& rg, uint32_t& g) {
        g += d_g;
        rg += d_rg;
        if (g >= KG) {
            g -= KG;
            ++rg;
        }
    };
    uint32_t p_rg = warp / KG, p_g = warp - (warp / KG) * KG;
    uint32_t c_rg = p_rg, c_g = p_g;
    auto issue = [&](uint32_t i, bool skip) {  // lane 0 only, spans in order
        const int st = static_cast<int>(i % kT128Stages);
        const int32_t c0 = static_cast<int32_t>(p_g * 128u);
        const int32_t c1 = static_cast<int32_t>(p_rg * 32u);
        advance(p_rg, p_g);
        if (skip) return;
        uint8_t* dst = ring + st * kSpan128Bytes;
        fence_async_smem();  // the lanes' reads of this stage come before the copy's writes
        mbar_arrive_expect_tx(&full[wid][st], kSpan128Bytes);
        tma_load_2d<1>(dst, &map_x, c0, c1, smem_u32(&full[wid][st]), policy);
        tma_load_2d<1>(dst + kBox128Bytes, &map_x, c0 + 64, c1, smem_u32(&full[wid][st]), policy);
    };
    if (lane == 0)
        for (uint32_t i = 0; i < n_spans && i < static_cast<uint32_t>(kT128Stages); ++i)
            issue(i, (debug & 2u) && warp == 0 && i == 0);  // debug bit 1: warp 0's first span never lands
    const float2 neg1 = make_float2(-1.f, -1.f);
    const uint32_t sw = lane & 7u;
    for (uint32_t i = 0; i < n_spans; ++i) {
        const int st = static_cast<int>(i % kT128Stages);
        const bool landed = mbar_wait(&full[wid][st], (i / kT128Stages) & 1u, kTWaitNs);
        if (!__all_sync(0xFFFFFFFFu, landed)) {
            // a copy never landed: report it, let the copies still in flight finish
            // (each wait again bounded), and leave
            if (lane == 0) {
                atomicCAS(&g_quant_status, 0u, static_cast<uint32_t>(MXQ_ERR_TIMEOUT));
                const uint32_t issued = min(n_spans, i + static_cast<uint32_t>(kT128Stages));
                for (uint32_t j = i; j < issued; ++j)
                    mbar_wait(&full[wid][j % kT128Stages], (j / kT128Stages) & 1u, kTWaitNs);
            }
            __syncwarp();
            return;
        }
        const uint32_t rg = c_rg, g = c_g;
        advance(c_rg, c_g);
        const uint8_t* rowp = ring + st * kSpan128Bytes + lane * 128u;
        const float4* m4 = mul != nullptr ? reinterpret_cast<const float4*>(mul + g * 128u) : nullptr;
        float2 t[64];  // t[k] holds values 2k and 2k + 1 of the lane's rotation block
#pragma unroll
        for (int q = 0; q < 16; ++q) {
            const uint4 v = *reinterpret_cast<const uint4*>(rowp + (q >> 3) * kBox128Bytes +
                                                            16u * ((static_cast<uint32_t>(q) & 7u) ^ sw));
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) t[4 * q + e] = make_float2(lo_f(w[e]), hi_f(w[e]));
            if (mul != nullptr) {
                const float4 ma = __ldg(m4 + 2 * q), mb = __ldg(m4 + 2 * q + 1);
                t[4 * q] = __fmul2_rn(t[4 * q], make_float2(ma.x, ma.y));
                t[4 * q + 1] = __fmul2_rn(t[4 * q + 1], make_float2(ma.z, ma.w));
                t[4 * q + 2] = __fmul2_rn(t[4 * q + 2], make_float2(mb.x, mb.y));
                t[4 * q + 3] = __fmul2_rn(t[4 * q + 3], make_float2(mb.z, mb.w));
            }
        }
        __syncwarp();  // every lane has read the stage before it is refilled
        if (lane == 0 && i + kT128Stages < n_spans) issue(i + kT128Stages, false);
        // butterflies: h = 1 on scalars, h = 2 ... 64 as packed binary32 operations (the
        // difference as fma(b, -1, a), one rounding, the IEEE difference)
#pragma unroll
        for (int k = 0; k < 64; ++k) t[k] = make_float2(__fadd_rn(t[k].x, t[k].y), __fsub_rn(t[k].x, t[k].y));
#pragma unroll
        for (int m = 1; m < 64; m <<= 1)
#pragma unroll
            for (int k = 0; k < 64; ++k)
                if ((k & m) == 0) {
                    const float2 a = t[k], b = t[k + m];
                    t[k] = __fadd2_rn(a, b);
                    t[k + m] = __ffma2_rn(b, neg1, a);
                }
        const uint32_t row = rg * 32u + lane;
        if (row >= rows) continue;
        // each MX block b (values 32b .. 32b + 31, pairs t[16b .. 16b + 15]): scale and
        // codes as in the 32-point kernel above
        uint32_t scw = 0;
        uint32_t cw[FMT == kFmtE2M1 ? 16 : 32];
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            float2* tb = t + 16 * b;
            float mc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int k = 0; k < 16; ++k)
                asm("max.NaN.abs.f32 %0, %1, %2, %3;" : "=f"(mc[k & 3]) : "f"(mc[k & 3]), "f"(tb[k].x), "f"(tb[k].y));
            float m;
            asm("max.NaN.abs.f32 %0, %1, %2, %3;" : "=f"(m) : "f"(mc[0]), "f"(mc[1]), "f"(mc[2]));
            asm("max.NaN.f32 %0, %1, %2;" : "=f"(m) : "f"(m), "f"(mc[3]));
            const uint32_t eb = (__float_as_uint(__fmul_rn(m, c)) & 0x7FFFFFFFu) >> 23;
            const uint32_t sc = eb == 255u ? 255u : (eb > kEmax ? eb - kEmax : 0u);
            float mult = e8m0_inverse(sc);
            const uint32_t keep = sc == 255u ? 0u : 0xFFFFFFFFu;
            if (sc - 11u <= 249u - 11u) {
                mult = __fmul_rn(c, mult);
            } else {
                const float2 c2 = make_float2(c, c);
#pragma unroll
                for (int k = 0; k < 16; ++k) tb[k] = __fmul2_rn(tb[k], c2);
            }
            const float2 mult2 = make_float2(mult, mult);
#pragma unroll
            for (int k = 0; k < 16; ++k) tb[k] = __fmul2_rn(tb[k], mult2);
            if (FMT == kFmtE2M1) {
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float q[8] = {tb[4 * k].x,     tb[4 * k].y,     tb[4 * k + 1].x, tb[4 * k + 1].y,
                                        tb[4 * k + 2].x, tb[4 * k + 2].y, tb[4 * k + 3].x, tb[4 * k + 3].y};
                    cw[4 * b + k] = cvt_e2m1x8(q) & keep;
                }
            } else {
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    cw[8 * b + k] = (cvt_e4m3x2(tb[2 * k].x, tb[2 * k].y) |
                                     (cvt_e4m3x2(tb[2 * k + 1].x, tb[2 * k + 1].y) << 16)) & keep;
            }
            scw |= sc << (8 * b);
        }
        constexpr uint32_t kCodeBytes = FMT == kFmtE2M1 ? 64u : 128u;  // per rotation block
        uint4* dst = reinterpret_cast<uint4*>(codes + static_cast<size_t>(row) * (K / (FMT == kFmtE2M1 ? 2u : 1u)) +
                                              static_cast<size_t>(g) * kCodeBytes);
#pragma unroll
        for (int k = 0; k < static_cast<int>(kCodeBytes / 16u); ++k)
            __stcs(dst + k, make_uint4(cw[4 * k], cw[4 * k + 1], cw[4 * k + 2], cw[4 * k + 3]));
        *reinterpret_cast<uint32_t*>(sf + sf_offset(row, 4u * g, atoms_k)) = scw;
    }
    // the padding of the tiled scale buffer, as in quantize_kernel
    const uint32_t KB = K / 32u;
    const uint32_t kbp = atoms_k * 4u;
    const uint32_t pad_k = kbp - KB;
    const uint32_t rows_p = (rows + 127u) & ~127u;
    const uint32_t n_pad_a = rows * pad_k;
    const uint32_t n_pad = n_pad_a + (rows_p - rows) * kbp;
    for (uint32_t p = blockIdx.x * blockDim.x + threadIdx.x; p < n_pad; p += gridDim.x * blockDim.x) {
        uint32_t rr, k;
        if (p < n_pad_a) {
            rr = p / pad_k;
            k = KB + (p - rr * pad_k);
        } else {
            const uint32_t q = p - n_pad_a;
            rr = rows + q / kbp;
            k = q - (q / kbp) * kbp;
        }
        sf[sf_offset(rr, k, atoms_k)] = 0;
    }
}

}  // namespace

// fmt: kFmtE2M1 / kFmtE4M3 (MX, scales from each block's abs-max) or kFmtStatic (E4M3
// of x / scale with block scales 127; scale positive and finite).
cudaError_t launch_quantize_any(const void* x, int64_t rows, int64_t K, int fmt, float scale, void* codes,
                                void* sf, cudaStream_t stream)
{
    StaticScale st{1.0f, 1.0f, 1.0f, 1.0f, 0};
    if (fmt == kFmtStatic) {
        int e = 0;
        const float m = std::frexp(scale, &e);  // scale = m 2^e, m in [1/2, 1)
        const int k = 1 - e;                    // sn = scale 2^k in [1, 2)
        st.sn = 2.0f * m;
        // fl32(1/sn): the double quotient is never within 2^-53 of a binary32 midpoint
        // unless it is one, so rounding it to binary32 gives the correctly rounded value
        st.r = static_cast<float>(1.0 / static_cast<double>(st.sn));
        st.two_step = k > 127 ? 1 : 0;
        st.p1 = std::ldexp(1.0f, st.two_step ? k / 2 : k);
        st.p2 = std::ldexp(1.0f, st.two_step ? k - k / 2 : 0);
    }
    const uint32_t n_groups = static_cast<uint32_t>(rows * K / 8);
    const uint32_t KB = static_cast<uint32_t>(K / 32);
    const uint32_t atoms_k = static_cast<uint32_t>(sf_atoms_k(K));
    // one step (8 groups per lane) per warp: the block scheduler streams CTAs in as others
    // finish, which measured 9-13 % faster on B200 than grids capped at 8-16 CTAs per SM
    // looping over the tensor (and faster than every cap between)
    const int64_t want = ceil_div(n_groups, kThreads * kUnroll);
    const int grid = static_cast<int>(std::max<int64_t>(1, want));
    // row = floor(block / KB) as a multiply-shift, exact for block < 2^29 and KB <= 2^11:
    // magic * KB - 2^40 < KB, so block * magic / 2^40 overshoots block / KB by less than 1 / KB
    const uint64_t kb_magic = ((uint64_t(1) << 40) + KB - 1) / KB;
    const uint4* xv = static_cast<const uint4*>(x);
    uint8_t* c = static_cast<uint8_t*>(codes);
    uint8_t* f = static_cast<uint8_t*>(sf);
    const uint32_t r = static_cast<uint32_t>(rows);
    if (fmt == kFmtStatic)
        quantize_kernel<kFmtStatic><<<grid, kThreads, 0, stream>>>(xv, n_groups, KB, kb_magic, atoms_k, r, c, f, st);
    else if (fmt == kFmtE4M3)
        quantize_kernel<kFmtE4M3><<<grid, kThreads, 0, stream>>>(xv, n_groups, KB, kb_magic, atoms_k, r, c, f, st);
    else
        quantize_kernel<kFmtE2M1><<<grid, kThreads, 0, stream>>>(xv, n_groups, KB, kb_magic, atoms_k, r, c, f, st);
    return cudaGetLastError();
}

cudaError_t launch_quantize(const void* x, int64_t rows, int64_t K, int fmt, void* codes, void* sf,
                            cudaStream_t stream)
{
    return launch_quantize_any(x, rows, K, fmt, 0.f, codes, sf, stream);
}

cudaError_t launch_quantize_static(const void* x, int64_t rows, int64_t K, float scale, void* codes, void* sf,
                                   cudaStream_t stream)
{
    return launch_quantize_any(x, rows, K, kFmtStatic, scale, codes, sf, stream);
}

cudaError_t launch_quantize_transform(const void* x, int64_t rows, int64_t K, int fmt, const float* mul, int block,
                                      float norm, void* codes, void* sf, cudaStream_t stream)
{
    const uint32_t n_blocks = static_cast<uint32_t>(rows * K / 32);
    const uint32_t KB = static_cast<uint32_t>(K / 32);
    const uint32_t atoms_k = static_cast<uint32_t>(sf_atoms_k(K));
    uint8_t* c = static_cast<uint8_t*>(codes);
    uint8_t* f = static_cast<uint8_t*>(sf);
    const uint32_t r = static_cast<uint32_t>(rows);
    const uint32_t dbg = debug_flags();
    CUtensorMap map;
    if (n_blocks == 0) return cudaSuccess;
    if (block == 128) {
        // x as [rows, K] bf16, boxes of 32 rows x 64 channels, 128-byte swizzle; rows past
        // the end read as zeros
        const uint32_t KG = static_cast<uint32_t>(K / 128);
        const uint32_t n_spans = static_cast<uint32_t>(ceil_div(rows, 32)) * KG;
        if (!make_map_2d(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, static_cast<uint64_t>(K),
                         static_cast<uint64_t>(rows), static_cast<uint64_t>(K) * 2u, 64, 32,
                         CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
        const int64_t want = ceil_div(n_spans, kT128Warps);
        const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(want, num_sms() * 3)));
        const uint32_t k32 = static_cast<uint32_t>(K);
        if (fmt == kFmtE4M3) {
            auto kern = quantize_transform128_kernel<kFmtE4M3>;
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kT128Smem);
            if (e != cudaSuccess) return e;
            kern<<<grid, kT128Warps * 32, kT128Smem, stream>>>(map, r, k32, KG, n_spans, atoms_k, mul, norm, c, f, dbg);
        } else {
            auto kern = quantize_transform128_kernel<kFmtE2M1>;
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kT128Smem);
            if (e != cudaSuccess) return e;
            kern<<<grid, kT128Warps * 32, kT128Smem, stream>>>(map, r, k32, KG, n_spans, atoms_k, mul, norm, c, f, dbg);
        }
        return cudaGetLastError();
    }
    const int64_t want = ceil_div(n_blocks, kTThreads);  // CTAs for one span per warp
    int64_t grid64 = std::max<int64_t>(1, std::min<int64_t>(want, num_sms() * 32));
    if (mul != nullptr && grid64 < want) {
        // several spans per warp: the warp count (4 per CTA) times 32 blocks must be a
        // multiple of KB, so that the multipliers a lane holds stay the ones of its channels
        const int64_t m = KB / std::gcd<int64_t>(KB, 32);  // warps
        const int64_t step = m / std::gcd<int64_t>(m, kTThreads / 32);  // CTAs
        grid64 = std::max<int64_t>(step, grid64 / step * step);
    }
    const int grid = static_cast<int>(grid64);
    // x as n_blocks rows of 32 bf16 (64 bytes), boxes of 32 rows, 64-byte swizzle; rows
    // past the end read as zeros
    if (!make_map_2d(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, 32, n_blocks, 64, 32, 32,
                     CU_TENSOR_MAP_SWIZZLE_64B))
        return cudaErrorInvalidValue;
    const uint64_t kb_magic = ((uint64_t(1) << 40) + KB - 1) / KB;
    if (fmt == kFmtE4M3)
        quantize_transform_kernel<kFmtE4M3><<<grid, kTThreads, 0, stream>>>(map, n_blocks, KB, kb_magic, atoms_k, r,
                                                                               mul, norm, c, f, dbg);
    else
        quantize_transform_kernel<kFmtE2M1><<<grid, kTThreads, 0, stream>>>(map, n_blocks, KB, kb_magic, atoms_k, r,
                                                                               mul, norm, c, f, dbg);
    return cudaGetLastError();
}

int read_and_clear_quant_status(cudaStream_t stream, uint32_t* out)
{
    uint32_t v = 0, zero = 0;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return MXQ_ERR_CUDA;
    if (cudaMemcpyFromSymbol(&v, g_quant_status, sizeof v) != cudaSuccess) return MXQ_ERR_CUDA;
    if (cudaMemcpyToSymbol(g_quant_status, &zero, sizeof zero) != cudaSuccess) return MXQ_ERR_CUDA;
    *out = v;
    return MXQ_OK;
}

cudaError_t launch_dequantize(const void* codes, const void* sf, int64_t rows, int64_t K, int fmt, void* out,
                              cudaStream_t stream)
{
    const uint32_t n_groups = static_cast<uint32_t>(rows * K / 8);
    const uint32_t KB = static_cast<uint32_t>(K / 32);
    const uint32_t atoms_k = static_cast<uint32_t>(sf_atoms_k(K));
    const uint64_t kb_magic = ((uint64_t(1) << 40) + KB - 1) / KB;
    const int grid = static_cast<int>(std::max<int64_t>(1, ceil_div(n_groups, kThreads * kDqGroups)));
    if (fmt == kFmtE4M3)
        dequantize_kernel<kFmtE4M3><<<grid, kThreads, 0, stream>>>(static_cast<const uint8_t*>(codes),
                                                                   static_cast<const uint8_t*>(sf), n_groups, KB,
                                                                   kb_magic, atoms_k, static_cast<uint4*>(out));
    else
        dequantize_kernel<kFmtE2M1><<<grid, kThreads, 0, stream>>>(static_cast<const uint8_t*>(codes),
                                                                   static_cast<const uint8_t*>(sf), n_groups, KB,
                                                                   kb_magic, atoms_k, static_cast<uint4*>(out));
    return cudaGetLastError();
}

cudaError_t launch_sf_to_logical(const void* sf, int64_t rows, int64_t K, void* out, cudaStream_t stream)
{
    const uint32_t n = static_cast<uint32_t>(rows * (K / 32));
    const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(ceil_div(n, 256), 4096)));
    sf_to_logical_kernel<<<grid, 256, 0, stream>>>(static_cast<const uint8_t*>(sf), static_cast<uint32_t>(rows),
                                                   static_cast<uint32_t>(K / 32),
                                                   static_cast<uint32_t>(sf_atoms_k(K)),
                                                   static_cast<uint8_t*>(out));
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------- calibration
namespace {

// max |x| over n bf16 values (n a multiple of 8): packed abs-max per 16-byte group, a
// warp reduction, and one atomicMax per warp on the float's bits (non-negative floats
// order like their bit patterns).  *out must hold 0 before the launch.  An Inf or NaN
// input makes the result Inf or NaN (their bit patterns lie above every finite one).
__global__ void __launch_bounds__(kThreads) absmax_kernel(const uint4* __restrict__ x, uint64_t n_groups,
                                                          uint32_t* __restrict__ out)
{
    uint32_t m = 0;
    for (uint64_t g = blockIdx.x * uint64_t(kThreads) + threadIdx.x; g < n_groups;
         g += uint64_t(gridDim.x) * kThreads) {
        const uint4 v = ld_stream(x + g);
        uint32_t m2 = absmax_bf16x2(absmax_bf16x2(v.x, v.y), absmax_bf16x2(v.z, v.w));
        m2 &= 0x7FFF7FFFu;
        m = max(m, max(m2 & 0xFFFFu, m2 >> 16));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if ((threadIdx.x & 31u) == 0) atomicMax(out, m << 16);  // bf16 bits -> fp32 bits
}

}  // namespace

namespace {

// GELU of bf16 values, elementwise, through the same table as the fused FFN epilogue: each
// CTA builds the table in shared memory, then maps its share of the elements.
__global__ void __launch_bounds__(256) gelu_bf16_kernel(const uint16_t* __restrict__ x, int64_t n,
                                                       uint16_t* __restrict__ y)
{
    __shared__ uint16_t lut[kGeluEntries];
    gelu_table_fill(lut, threadIdx.x, blockDim.x);
    __syncthreads();
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x)
        y[i] = static_cast<uint16_t>(gelu_bf16_bits(x[i], lut));
}

}  // namespace

cudaError_t launch_gelu_bf16(const void* x, int64_t n, void* y, cudaStream_t stream)
{
    const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(ceil_div(n, 256), num_sms() * 4)));
    gelu_bf16_kernel<<<grid, 256, 0, stream>>>(static_cast<const uint16_t*>(x), n, static_cast<uint16_t*>(y));
    return cudaGetLastError();
}

cudaError_t launch_absmax(const void* x, int64_t n, float* out, cudaStream_t stream)
{
    cudaError_t e = cudaMemsetAsync(out, 0, sizeof(float), stream);
    if (e != cudaSuccess) return e;
    const uint64_t n_groups = static_cast<uint64_t>(n / 8);
    const int64_t want = ceil_div(static_cast<int64_t>(n_groups), kThreads);
    const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(want, num_sms() * 8)));
    absmax_kernel<<<grid, kThreads, 0, stream>>>(static_cast<const uint4*>(x), n_groups,
                                                 reinterpret_cast<uint32_t*>(out));
    return cudaGetLastError();
}

}  // namespace mxq
