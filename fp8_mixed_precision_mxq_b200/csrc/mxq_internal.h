// mxq_internal.h -- declarations shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "mxq.h"

namespace mxq {

// Element formats of the activation operand.
constexpr int kFmtE2M1 = MXQ_FMT_E2M1;
constexpr int kFmtE4M3 = MXQ_FMT_E4M3;

// Tiled scale-factor layout: 512-byte atoms of 128 rows x 4 k-blocks.
inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline int64_t sf_atoms_k(int64_t K) { return ceil_div(K / 32, 4); }
inline int64_t sf_bytes(int64_t rows, int64_t K) { return ceil_div(rows, 128) * 128 * sf_atoms_k(K) * 4; }
inline int64_t codes_bytes(int64_t rows, int64_t K, int fmt) { return fmt == kFmtE4M3 ? rows * K : rows * K / 2; }

// ---- launchers (return cudaError_t of the launch) ----
cudaError_t launch_quantize(const void* x, int64_t rows, int64_t K, int fmt, void* codes, void* sf,
                            cudaStream_t stream);
// Static per-tensor E4M3: codes = RNE_sat(x / scale) (the exact quotient), block scales 127.
cudaError_t launch_quantize_static(const void* x, int64_t rows, int64_t K, float scale, void* codes, void* sf,
                                   cudaStream_t stream);
// transform_on: t = x * mul (per channel; mul may be null), each `block` (32 or 128)
// values along K rotated by the Hadamard matrix times norm, then MX-quantized in fmt.
cudaError_t launch_quantize_transform(const void* x, int64_t rows, int64_t K, int fmt, const float* mul, int block,
                                      float norm, void* codes, void* sf, cudaStream_t stream);
// *out = max |x| over n bf16 values (n % 8 == 0), as fp32.
cudaError_t launch_absmax(const void* x, int64_t n, float* out, cudaStream_t stream);
cudaError_t launch_gelu_bf16(const void* x, int64_t n, void* y, cudaStream_t stream);
cudaError_t launch_dequantize(const void* codes, const void* sf, int64_t rows, int64_t K, int fmt, void* out,
                              cudaStream_t stream);
// Calibration and load-time arithmetic of the policy (calib.cu).
cudaError_t launch_channel_absmax(const void* x, int64_t rows, int64_t K, float* out, cudaStream_t stream);
cudaError_t launch_smooth_scales(const float* ax, const float* aw, int64_t K, float alpha, float* s, float* inv,
                                 cudaStream_t stream);
cudaError_t launch_sqnr(const void* const* ref, const void* const* test, const int64_t* n, int count, double* out,
                        cudaStream_t stream);
cudaError_t launch_lowrank_split(const float* U, int64_t ldu, const float* S, const float* Vh, int64_t ldvh,
                                 const void* w, int64_t N, int64_t K, int64_t r, void* l2t, void* l1t, void* resid,
                                 cudaStream_t stream);
cudaError_t launch_sf_to_logical(const void* sf, int64_t rows, int64_t K, void* out, cudaStream_t stream);

struct GemmArgs {
    const void* a_codes;
    const void* a_sf;
    int a_fmt;  // kFmtE2M1 -> kind::mxf4, kFmtE4M3 -> kind::mxf8f6f4
    int64_t M, N, K;
    const void* w_codes;
    const void* w_sf;
    const void* bias;  // bf16 [N] or null
    void* y;           // bf16 [M, N]; with out_fmt >= 0: h in bf16, or null
    // out_fmt >= 0: the epilogue writes its output MX-quantized in that format (codes
    // [M, N/2] or [M, N], tiled scales with K = N), the next layer's input; with
    // out_gelu, GELU of it (rounded to bf16 first and after)
    int out_fmt = -1;
    bool out_gelu = true;
    void* q_codes = nullptr;
    void* q_sf = nullptr;
    // per-tensor scale of the activation (static E4M3): y = alpha * acc + bias
    float alpha = 1.0f;
    // low-rank branch (rank a multiple of 64, or 0): y += u . l2t^T, u bf16 [M, r],
    // l2t bf16 [N, r]
    int64_t lr_rank = 0;
    const void* lr_u = nullptr;
    const void* lr_l2t = nullptr;
    // plain bf16 GEMM: a_codes is A bf16 [M, K], w_codes is B bf16 [N, K] (K-major, K % 8
    // == 0), no scales; the same kernel runs only bf16 (kind::f16) stages of 64 along K
    bool bf16 = false;
    // bf16 GEMM only, N <= 128, K % 32 == 0: also MX-quantize A (format qa_fmt, or -1 for
    // no) into codes qa_codes and tiled scales qa_sf as its stages pass through the kernel,
    // the same bits as the activation quantizer writes
    int qa_fmt = -1;
    void* qa_codes = nullptr;
    void* qa_sf = nullptr;
};

// Builds the tensor maps and launches the tcgen05 GEMM.  Returns an mxq_status;
// on failure *msg points to a static description.
int launch_gemm(const GemmArgs& g, cudaStream_t stream, const char** msg, char* path, size_t path_len);

// Device status words written by kernels whose bounded waits ran out (the GEMM's and
// the quantizers'); each call synchronizes the stream, returns the word and clears it.
int read_and_clear_device_status(cudaStream_t stream, uint32_t* out);
int read_and_clear_quant_status(cudaStream_t stream, uint32_t* out);

// 2-D tiled tensor map (dims d0 inner, d1 outer; row stride in bytes; box b0 x b1);
// false if the driver entry point is missing or the encoding is refused.
bool make_map_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t d0, uint64_t d1,
                 uint64_t stride_bytes, uint32_t b0, uint32_t b1, CUtensorMapSwizzle sw);
void set_debug_flags(uint32_t flags);
uint32_t debug_flags();

}  // namespace mxq
