// qdq_gemm.cu -- the bf16 GEMM of the quantize-dequantize emulation mode.
//
// The blog "Quark Mixed-Precision Quantization for Wan2.2 Video Generation on AMD
// Instinct GPUs" measures W4A8 by QDQ emulation: both operands are dequantized to a
// high-precision type and an ordinary GEMM runs on them ("Kernel note").  Here the
// dequantization runs in this library's own kernel and the plain bf16 GEMM is a
// cuBLASLt call (fp32 accumulation, bf16 output, bias in the epilogue).
#include <cublasLt.h>

#include <mutex>
#include <unordered_map>

#include "mxq_internal.h"

namespace mxq {
namespace {

struct Handle {
    cublasLtHandle_t h = nullptr;
};

cublasLtHandle_t lt_handle(int dev)
{
    static std::mutex mu;
    static std::unordered_map<int, Handle> handles;
    std::lock_guard<std::mutex> g(mu);
    Handle& hd = handles[dev];
    if (!hd.h && cublasLtCreate(&hd.h) != CUBLAS_STATUS_SUCCESS) hd.h = nullptr;
    return hd.h;
}

}  // namespace

// Row-major Y[M, N] = Xd[M, K] . Wd[N, K]^T + bias[N]: in cuBLASLt's column-major
// view this is Y^T[N, M] = op(Wd)[N, K] . Xd^T[K, M] with op = transpose.
int qdq_bf16_gemm(const void* xd, const void* wd, const void* bias, void* y, int64_t M, int64_t N, int64_t K,
                  void* workspace, size_t ws_bytes, cudaStream_t stream, const char** msg)
{
    int dev = 0;
    cudaGetDevice(&dev);
    cublasLtHandle_t h = lt_handle(dev);
    if (!h) {
        *msg = "cublasLtCreate failed";
        return MXQ_ERR_CUDA;
    }
    cublasLtMatmulDesc_t op = nullptr;
    cublasLtMatrixLayout_t la = nullptr, lb = nullptr, lc = nullptr;
    cublasLtMatmulPreference_t pref = nullptr;
    int rc = MXQ_ERR_CUDA;
    do {
        if (cublasLtMatmulDescCreate(&op, CUBLAS_COMPUTE_32F, CUDA_R_32F) != CUBLAS_STATUS_SUCCESS) break;
        const cublasOperation_t ta = CUBLAS_OP_T, tb = CUBLAS_OP_N;
        cublasLtMatmulDescSetAttribute(op, CUBLASLT_MATMUL_DESC_TRANSA, &ta, sizeof ta);
        cublasLtMatmulDescSetAttribute(op, CUBLASLT_MATMUL_DESC_TRANSB, &tb, sizeof tb);
        if (bias) {
            const cublasLtEpilogue_t ep = CUBLASLT_EPILOGUE_BIAS;
            const cudaDataType_t bt = CUDA_R_16BF;
            cublasLtMatmulDescSetAttribute(op, CUBLASLT_MATMUL_DESC_EPILOGUE, &ep, sizeof ep);
            cublasLtMatmulDescSetAttribute(op, CUBLASLT_MATMUL_DESC_BIAS_POINTER, &bias, sizeof bias);
            cublasLtMatmulDescSetAttribute(op, CUBLASLT_MATMUL_DESC_BIAS_DATA_TYPE, &bt, sizeof bt);
        }
        if (cublasLtMatrixLayoutCreate(&la, CUDA_R_16BF, K, N, K) != CUBLAS_STATUS_SUCCESS) break;
        if (cublasLtMatrixLayoutCreate(&lb, CUDA_R_16BF, K, M, K) != CUBLAS_STATUS_SUCCESS) break;
        if (cublasLtMatrixLayoutCreate(&lc, CUDA_R_16BF, N, M, N) != CUBLAS_STATUS_SUCCESS) break;
        if (cublasLtMatmulPreferenceCreate(&pref) != CUBLAS_STATUS_SUCCESS) break;
        cublasLtMatmulPreferenceSetAttribute(pref, CUBLASLT_MATMUL_PREF_MAX_WORKSPACE_BYTES, &ws_bytes,
                                             sizeof ws_bytes);
        cublasLtMatmulHeuristicResult_t res;
        int n_res = 0;
        if (cublasLtMatmulAlgoGetHeuristic(h, op, la, lb, lc, lc, pref, 1, &res, &n_res) !=
                CUBLAS_STATUS_SUCCESS ||
            n_res == 0) {
            *msg = "cuBLASLt found no bf16 algorithm for this shape";
            break;
        }
        const float alpha = 1.f, beta = 0.f;
        if (cublasLtMatmul(h, op, &alpha, wd, la, xd, lb, &beta, y, lc, y, lc, &res.algo, workspace, ws_bytes,
                           stream) != CUBLAS_STATUS_SUCCESS) {
            *msg = "cublasLtMatmul failed";
            break;
        }
        rc = MXQ_OK;
    } while (false);
    if (rc != MXQ_OK && *msg == nullptr) *msg = "cuBLASLt setup failed";
    if (pref) cublasLtMatmulPreferenceDestroy(pref);
    if (lc) cublasLtMatrixLayoutDestroy(lc);
    if (lb) cublasLtMatrixLayoutDestroy(lb);
    if (la) cublasLtMatrixLayoutDestroy(la);
    if (op) cublasLtMatmulDescDestroy(op);
    return rc;
}

}  // namespace mxq
