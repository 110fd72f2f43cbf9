// calib.cu -- the offline and calibration arithmetic of the mixed-precision policy, on the
// GPU: per-channel abs-max and SmoothQuant scales (the transform_on policy), the SQNR of a
// block's outputs (the block selection), and the split of a weight into the SVDQuant
// low-rank factors and residual (blog "Quark Mixed-Precision Quantization for Wan2.2 Video
// Generation on AMD Instinct GPUs", sections "Mixed-Precision selection", "Calibration-driven
// block selection" and "Results").  None of these runs on the layer's hot path; they run
// at calibration or load time.  All are HBM-bound or small.
#include <cuda_bf16.h>

#include <algorithm>
#include <cmath>

#include "mx_elem.cuh"
#include "mxq_internal.h"

namespace mxq {
namespace {

constexpr int kThreads = 256;

int num_sms_calib()
{
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

// out[k] = max over rows of |x[r, k]| as fp32 bits (non-negative floats order like their
// bit patterns; a NaN's bits lie above every finite value and Inf).  Each thread keeps the
// packed abs-max of one 16-byte group of 8 columns over the rows it visits, then one
// atomicMax per column.  out must hold zeros before the launch.
__global__ void __launch_bounds__(kThreads) channel_absmax_kernel(const uint4* __restrict__ x, uint32_t rows,
                                                                  uint32_t groups_per_row, uint32_t* __restrict__ out)
{
    const uint32_t gcol = blockIdx.x * kThreads + threadIdx.x;
    if (gcol >= groups_per_row) return;
    uint32_t m[4] = {0u, 0u, 0u, 0u};  // packed bf16x2 abs-max of columns 8 gcol ..
    for (uint32_t r = blockIdx.y; r < rows; r += gridDim.y) {
        const uint4 v = __ldg(x + static_cast<size_t>(r) * groups_per_row + gcol);
        m[0] = absmax_bf16x2(m[0], v.x);
        m[1] = absmax_bf16x2(m[1], v.y);
        m[2] = absmax_bf16x2(m[2], v.z);
        m[3] = absmax_bf16x2(m[3], v.w);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t w = m[i] & 0x7FFF7FFFu;
        atomicMax(out + 8 * gcol + 2 * i, (w & 0xFFFFu) << 16);   // bf16 bits -> fp32 bits
        atomicMax(out + 8 * gcol + 2 * i + 1, w & 0xFFFF0000u);
    }
}

// SmoothQuant's per-channel scales s_k = max|X_k|^alpha / max|W_k|^(1 - alpha), each
// maximum first raised to at least 1e-5 (an all-zero channel would otherwise divide by 0),
// and, when inv is given, their reciprocals 1 / s_k (IEEE binary32 division).
__global__ void smooth_scales_kernel(const float* __restrict__ ax, const float* __restrict__ aw, uint32_t K,
                                     float alpha, float* __restrict__ s, float* __restrict__ inv)
{
    for (uint32_t k = blockIdx.x * blockDim.x + threadIdx.x; k < K; k += gridDim.x * blockDim.x) {
        const float v = powf(fmaxf(ax[k], 1e-5f), alpha) / powf(fmaxf(aw[k], 1e-5f), 1.0f - alpha);
        s[k] = v;
        if (inv) inv[k] = 1.0f / v;
    }
}

// acc[0] += sum ref^2, acc[1] += sum (ref - test)^2 over n bf16 values (n % 8 == 0), in
// fp64 (squares and differences of bf16 values are exact there); a warp reduction and one
// atomicAdd per warp and sum.
__global__ void __launch_bounds__(kThreads) sqnr_kernel(const uint4* __restrict__ ref, const uint4* __restrict__ test,
                                                        uint64_t n_groups, double* __restrict__ acc)
{
    double s = 0.0, d = 0.0;
    for (uint64_t g = blockIdx.x * uint64_t(kThreads) + threadIdx.x; g < n_groups;
         g += uint64_t(gridDim.x) * kThreads) {
        const uint4 a = __ldg(ref + g), b = __ldg(test + g);
        const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const double r0 = lo_f(wa[i]), r1 = hi_f(wa[i]);
            const double e0 = r0 - static_cast<double>(lo_f(wb[i])), e1 = r1 - static_cast<double>(hi_f(wb[i]));
            s = fma(r0, r0, fma(r1, r1, s));
            d = fma(e0, e0, fma(e1, e1, d));
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
        d += __shfl_xor_sync(0xFFFFFFFFu, d, o);
    }
    if ((threadIdx.x & 31u) == 0) {
        atomicAdd(acc, s);
        atomicAdd(acc + 1, d);
    }
}

// acc[2] = 10 log10(acc[0] / acc[1]) (+Inf for identical tensors, NaN for 0 / 0).
__global__ void sqnr_db_kernel(double* acc) { acc[2] = 10.0 * log10(acc[0] / acc[1]); }

// The SVDQuant split of W [N, K] from its singular triplets (U [N, r] with row stride ldu,
// S [r], Vh [r, K] with row stride ldvh, fp32):
//   l2t[n, j] = bf16(U[n, j] * sqrt(S[j])),  l1t[j, k] = bf16(sqrt(S[j]) * Vh[j, k]).
__global__ void lowrank_factors_kernel(const float* __restrict__ U, int64_t ldu, const float* __restrict__ S,
                                       const float* __restrict__ Vh, int64_t ldvh, uint32_t N, uint32_t K, uint32_t r,
                                       __nv_bfloat16* __restrict__ l2t, __nv_bfloat16* __restrict__ l1t)
{
    const uint64_t n2 = uint64_t(N) * r, n1 = uint64_t(r) * K;
    for (uint64_t i = blockIdx.x * uint64_t(blockDim.x) + threadIdx.x; i < n2 + n1;
         i += uint64_t(gridDim.x) * blockDim.x) {
        if (i < n2) {
            const uint64_t n = i / r, j = i - n * r;
            l2t[i] = __float2bfloat16_rn(U[n * ldu + j] * sqrtf(S[j]));
        } else {
            const uint64_t q = i - n2, j = q / K, k = q - j * K;
            l1t[q] = __float2bfloat16_rn(sqrtf(S[j]) * Vh[j * ldvh + k]);
        }
    }
}

// resid[n, k] = bf16(W[n, k] - sum_j l2t[n, j] * l1t[j, k]), the products of bf16 values
// exact in fp32 and summed in fp32.  64 x 64 output tiles per 256-thread block, each thread
// 4 x 4 outputs; the rank is walked in chunks of 32 staged in shared memory.
constexpr int kRt = 64, kRc = 32;
__global__ void __launch_bounds__(256) lowrank_residual_kernel(const __nv_bfloat16* __restrict__ W,
                                                               const __nv_bfloat16* __restrict__ l2t,
                                                               const __nv_bfloat16* __restrict__ l1t, uint32_t N,
                                                               uint32_t K, uint32_t r, __nv_bfloat16* __restrict__ out)
{
    __shared__ float a_s[kRc][kRt + 1];  // l2t chunk, transposed: [j][n]
    __shared__ float b_s[kRc][kRt];      // l1t chunk: [j][k]
    const uint32_t n0 = blockIdx.y * kRt, k0 = blockIdx.x * kRt;
    const uint32_t tx = threadIdx.x & 15u, ty = threadIdx.x >> 4;
    float acc[4][4] = {};
    for (uint32_t j0 = 0; j0 < r; j0 += kRc) {
        for (uint32_t i = threadIdx.x; i < kRt * kRc; i += 256) {
            const uint32_t nn = i / kRc, jj = i - nn * kRc;      // l2t rows are r long
            const uint32_t n = n0 + nn, j = j0 + jj;
            a_s[jj][nn] = (n < N && j < r) ? __bfloat162float(l2t[uint64_t(n) * r + j]) : 0.0f;
            const uint32_t jb = i / kRt, kk = i - jb * kRt;       // l1t rows are K long
            const uint32_t j2 = j0 + jb, k = k0 + kk;
            b_s[jb][kk] = (j2 < r && k < K) ? __bfloat162float(l1t[uint64_t(j2) * K + k]) : 0.0f;
        }
        __syncthreads();
#pragma unroll 8
        for (int jj = 0; jj < kRc; ++jj) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                a[i] = a_s[jj][ty * 4 + i];
                b[i] = b_s[jj][tx * 4 + i];
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int c = 0; c < 4; ++c) acc[i][c] = fmaf(a[i], b[c], acc[i][c]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t n = n0 + ty * 4 + i;
        if (n >= N) continue;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const uint32_t k = k0 + tx * 4 + c;
            if (k < K) {
                const uint64_t o = uint64_t(n) * K + k;
                out[o] = __float2bfloat16_rn(__bfloat162float(W[o]) - acc[i][c]);
            }
        }
    }
}

}  // namespace

cudaError_t launch_channel_absmax(const void* x, int64_t rows, int64_t K, float* out, cudaStream_t stream)
{
    cudaError_t e = cudaMemsetAsync(out, 0, sizeof(float) * static_cast<size_t>(K), stream);
    if (e != cudaSuccess) return e;
    const uint32_t gpr = static_cast<uint32_t>(K / 8);
    const uint32_t gx = static_cast<uint32_t>(ceil_div(gpr, kThreads));
    // enough row slices to fill the SMs a few times over, each thread covering many rows
    const int64_t want_y = std::max<int64_t>(1, (int64_t(num_sms_calib()) * 8 + gx - 1) / gx);
    const uint32_t gy = static_cast<uint32_t>(std::min<int64_t>(want_y, std::min<int64_t>(rows, 65535)));
    channel_absmax_kernel<<<dim3(gx, gy), kThreads, 0, stream>>>(static_cast<const uint4*>(x),
                                                                 static_cast<uint32_t>(rows), gpr,
                                                                 reinterpret_cast<uint32_t*>(out));
    return cudaGetLastError();
}

cudaError_t launch_smooth_scales(const float* ax, const float* aw, int64_t K, float alpha, float* s, float* inv,
                                 cudaStream_t stream)
{
    const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(ceil_div(K, kThreads), 1024)));
    smooth_scales_kernel<<<grid, kThreads, 0, stream>>>(ax, aw, static_cast<uint32_t>(K), alpha, s, inv);
    return cudaGetLastError();
}

cudaError_t launch_sqnr(const void* const* ref, const void* const* test, const int64_t* n, int count, double* out,
                        cudaStream_t stream)
{
    cudaError_t e = cudaMemsetAsync(out, 0, 3 * sizeof(double), stream);
    if (e != cudaSuccess) return e;
    for (int i = 0; i < count; ++i) {
        const uint64_t groups = static_cast<uint64_t>(n[i] / 8);
        const int grid = static_cast<int>(std::max<int64_t>(
            1, std::min<int64_t>(ceil_div(static_cast<int64_t>(groups), kThreads), num_sms_calib() * 8)));
        sqnr_kernel<<<grid, kThreads, 0, stream>>>(static_cast<const uint4*>(ref[i]),
                                                   static_cast<const uint4*>(test[i]), groups, out);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    sqnr_db_kernel<<<1, 1, 0, stream>>>(out);
    return cudaGetLastError();
}

cudaError_t launch_lowrank_split(const float* U, int64_t ldu, const float* S, const float* Vh, int64_t ldvh,
                                 const void* w, int64_t N, int64_t K, int64_t r, void* l2t, void* l1t, void* resid,
                                 cudaStream_t stream)
{
    const int64_t total = N * r + r * K;
    const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(ceil_div(total, kThreads), 65535)));
    lowrank_factors_kernel<<<grid, kThreads, 0, stream>>>(U, ldu, S, Vh, ldvh, static_cast<uint32_t>(N),
                                                          static_cast<uint32_t>(K), static_cast<uint32_t>(r),
                                                          static_cast<__nv_bfloat16*>(l2t),
                                                          static_cast<__nv_bfloat16*>(l1t));
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    dim3 g2(static_cast<uint32_t>(ceil_div(K, kRt)), static_cast<uint32_t>(ceil_div(N, kRt)));
    lowrank_residual_kernel<<<g2, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(w),
                                                    static_cast<const __nv_bfloat16*>(l2t),
                                                    static_cast<const __nv_bfloat16*>(l1t), static_cast<uint32_t>(N),
                                                    static_cast<uint32_t>(K), static_cast<uint32_t>(r),
                                                    static_cast<__nv_bfloat16*>(resid));
    return cudaGetLastError();
}

}  // namespace mxq
