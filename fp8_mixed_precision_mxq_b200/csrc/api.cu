// api.cu -- the C ABI of libmxq.so (declared in include/mxq.h): argument checks,
// workspace layout, and dispatch to the quantizer, dequantizer and GEMM kernels.
#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "mxq_internal.h"

using namespace mxq;

namespace {

thread_local char g_err[512] = "";
thread_local char g_path[256] = "";

int fail(int code, const char* fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
    return code;
}

int ok()
{
    g_err[0] = 0;
    return MXQ_OK;
}

constexpr int64_t kMaxElems = int64_t(1) << 34;  // rows*K; keeps 32-bit group / scale indices exact
constexpr int64_t kMaxK = int64_t(1) << 16;       // K/32 < 2^11 keeps the row division of the quantizer exact
constexpr int64_t kWsAlign = 256;

int64_t round_up(int64_t v, int64_t a) { return (v + a - 1) / a * a; }

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int check_ptr(const void* p, const char* name, uintptr_t align = 16)
{
    if (!p) return fail(MXQ_ERR_INVALID_ARG, "%s is NULL", name);
    if (!aligned(p, align)) return fail(MXQ_ERR_ALIGN, "%s is not %zu-byte aligned", name, (size_t)align);
    return MXQ_OK;
}

int check_fmt(int fmt)
{
    if (fmt != MXQ_FMT_E2M1 && fmt != MXQ_FMT_E4M3) return fail(MXQ_ERR_INVALID_ARG, "unknown format %d", fmt);
    return MXQ_OK;
}

int check_rows_k(int64_t rows, int64_t K, const char* what)
{
    if (rows <= 0 || K <= 0) return fail(MXQ_ERR_INVALID_ARG, "%s: sizes must be positive (rows=%lld K=%lld)", what,
                                         (long long)rows, (long long)K);
    if (K % 32 != 0) return fail(MXQ_ERR_SHAPE, "%s: K=%lld is not a multiple of 32", what, (long long)K);
    if (K > kMaxK) return fail(MXQ_ERR_SHAPE, "%s: K=%lld is above the supported maximum %lld", what, (long long)K,
                               (long long)kMaxK);
    if (rows > (int64_t(1) << 31) - 1 || rows * K > kMaxElems)
        return fail(MXQ_ERR_SHAPE, "%s: tensor too large (rows=%lld K=%lld)", what, (long long)rows, (long long)K);
    return MXQ_OK;
}

// The kernels are built for sm_100a only.
int check_device()
{
    static thread_local int checked_dev = -1;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(MXQ_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev == checked_dev) return MXQ_OK;
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (major != 10 || minor != 0)
        return fail(MXQ_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library runs on sm_100 only", dev, major, minor);
    checked_dev = dev;
    return MXQ_OK;
}

int cuda_rc(cudaError_t e, const char* what)
{
    if (e != cudaSuccess) return fail(MXQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    return ok();
}

#define RETURN_IF(x)                 \
    do {                             \
        int rc_ = (x);               \
        if (rc_ != MXQ_OK) return rc_; \
    } while (0)

int check_gemm(const void* a_codes, const void* a_sf, int a_fmt, int64_t M, int64_t K, const void* w_codes,
               const void* w_sf, int64_t N, const void* bias, const void* y)
{
    RETURN_IF(check_fmt(a_fmt));
    RETURN_IF(check_rows_k(M, K, "activation"));
    RETURN_IF(check_rows_k(N, K, "weight"));
    if (N % 8 != 0) return fail(MXQ_ERR_SHAPE, "N=%lld is not a multiple of 8", (long long)N);
    if (a_fmt == MXQ_FMT_E4M3 && K % 128 != 0)
        return fail(MXQ_ERR_SHAPE, "W4A8 native GEMM needs K %% 128 == 0 (K=%lld)", (long long)K);
    RETURN_IF(check_ptr(a_codes, "a_codes"));
    RETURN_IF(check_ptr(a_sf, "a_sf"));
    RETURN_IF(check_ptr(w_codes, "w_codes", a_fmt == MXQ_FMT_E4M3 ? 32 : 16));
    RETURN_IF(check_ptr(w_sf, "w_sf"));
    RETURN_IF(check_ptr(y, "y"));
    if (bias) RETURN_IF(check_ptr(bias, "bias"));
    return MXQ_OK;
}

int64_t linear_ws(int64_t M, int64_t N, int64_t K, int fmt, int mode)
{
    int64_t ws = round_up(codes_bytes(M, K, fmt), kWsAlign) + round_up(sf_bytes(M, K), kWsAlign);
    if (mode == MXQ_MODE_QDQ) ws += round_up(M * K * 2, kWsAlign) + round_up(N * K * 2, kWsAlign);
    return ws;
}

// y[M, N] = bf16(a[M, K] . b[N, K]^T + bias), both bf16 and K-major: the GEMM kernel with
// only bf16 (kind::f16) stages.
int run_gemm_bf16(const void* a, const void* b, const void* bias, void* y, int64_t M, int64_t N, int64_t K,
                  cudaStream_t stream)
{
    GemmArgs g{a, nullptr, MXQ_FMT_E2M1, M, N, K, b, nullptr, bias, y};
    g.bf16 = true;
    const char* msg = nullptr;
    int rc = launch_gemm(g, stream, &msg, g_path, sizeof g_path);
    if (rc != MXQ_OK) return fail(rc, "bf16 gemm: %s", msg ? msg : "launch failed");
    return ok();
}

int check_gemm_bf16(const void* a, int64_t M, int64_t K, const void* b, int64_t N, const void* bias, const void* y)
{
    if (M <= 0 || N <= 0 || K <= 0)
        return fail(MXQ_ERR_INVALID_ARG, "bf16 gemm: sizes must be positive (M=%lld N=%lld K=%lld)", (long long)M,
                    (long long)N, (long long)K);
    if (K % 8 != 0) return fail(MXQ_ERR_SHAPE, "bf16 gemm: K=%lld is not a multiple of 8", (long long)K);
    if (N % 8 != 0) return fail(MXQ_ERR_SHAPE, "N=%lld is not a multiple of 8", (long long)N);
    if (M > (int64_t(1) << 31) - 1 || N > (int64_t(1) << 31) - 1 || K > kMaxK * 4)
        return fail(MXQ_ERR_SHAPE, "bf16 gemm: sizes above the supported maximum (M=%lld N=%lld K=%lld)",
                    (long long)M, (long long)N, (long long)K);
    RETURN_IF(check_ptr(a, "a"));
    RETURN_IF(check_ptr(b, "b"));
    RETURN_IF(check_ptr(y, "y"));
    if (bias) RETURN_IF(check_ptr(bias, "bias"));
    return MXQ_OK;
}

int run_gemm(const void* a_codes, const void* a_sf, int a_fmt, int64_t M, int64_t K, const void* w_codes,
             const void* w_sf, int64_t N, const void* bias, void* y, cudaStream_t stream)
{
    GemmArgs g{a_codes, a_sf, a_fmt, M, N, K, w_codes, w_sf, bias, y};
    const char* msg = nullptr;
    int rc = launch_gemm(g, stream, &msg, g_path, sizeof g_path);
    if (rc != MXQ_OK) return fail(rc, "gemm: %s", msg ? msg : "launch failed");
    return ok();
}

// Quantize x into the workspace, then GEMM (native) or dequantize + bf16 GEMM (QDQ).
int run_linear(const void* x, int64_t M, int64_t K, const void* w_codes, const void* w_sf, int64_t N,
               const void* bias, int fmt, int mode, void* workspace, int64_t ws_bytes, void* y,
               cudaStream_t stream)
{
    const int64_t need = linear_ws(M, N, K, fmt, mode);
    if (ws_bytes < need)
        return fail(MXQ_ERR_WORKSPACE, "workspace has %lld bytes, needs %lld", (long long)ws_bytes, (long long)need);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    uint8_t* xc = ws;
    uint8_t* xs = xc + round_up(codes_bytes(M, K, fmt), kWsAlign);
    RETURN_IF(cuda_rc(launch_quantize(x, M, K, fmt, xc, xs, stream), "quantize launch"));
    if (mode == MXQ_MODE_NATIVE) return run_gemm(xc, xs, fmt, M, K, w_codes, w_sf, N, bias, y, stream);

    uint8_t* xd = xs + round_up(sf_bytes(M, K), kWsAlign);
    uint8_t* wd = xd + round_up(M * K * 2, kWsAlign);
    RETURN_IF(cuda_rc(launch_dequantize(xc, xs, M, K, fmt, xd, stream), "dequantize launch"));
    RETURN_IF(cuda_rc(launch_dequantize(w_codes, w_sf, N, K, MXQ_FMT_E2M1, wd, stream), "dequantize launch"));
    RETURN_IF(run_gemm_bf16(xd, wd, bias, y, M, N, K, stream));
    char gp[sizeof g_path];
    snprintf(gp, sizeof gp, "%s", g_path);
    snprintf(g_path, sizeof g_path, "qdq %s dequant + %.200s", fmt == MXQ_FMT_E4M3 ? "e4m3" : "e2m1", gp);
    return ok();
}

// fl32(1/sqrt B) for B = 2^j: 2^(-j/2) for even j, fl32(sqrt 2) * 2^(-(j+1)/2) for odd j
// (scaling by a power of two is exact, so both are the correctly rounded value).
float hadamard_norm(int B)
{
    int j = 0;
    while ((1 << j) < B) ++j;
    if (j % 2 == 0) return std::ldexp(1.0f, -j / 2);
    return std::ldexp(static_cast<float>(M_SQRT2), -(j + 1) / 2);
}

int check_transform(int64_t K, int block, const void* mul)
{
    if (block != 32 && block != 128) return fail(MXQ_ERR_INVALID_ARG, "rotation block must be 32 or 128 (got %d)", block);
    if (K % block != 0) return fail(MXQ_ERR_SHAPE, "K=%lld is not a multiple of the rotation block %d", (long long)K, block);
    if (mul) RETURN_IF(check_ptr(mul, "channel multiplier"));
    return MXQ_OK;
}

int check_mode(int mode)
{
    if (mode != MXQ_MODE_NATIVE && mode != MXQ_MODE_QDQ) return fail(MXQ_ERR_INVALID_ARG, "unknown mode %d", mode);
    return MXQ_OK;
}

// Checks of the quantizing-epilogue GEMM beyond those of the plain GEMM: the output is
// the next layer's activation [M, N] (K = N), so N follows the activation rules.
int check_gelu_quant(int64_t M, int64_t N, int out_fmt, const void* out_codes, const void* out_sf, const void* h)
{
    RETURN_IF(check_fmt(out_fmt));
    RETURN_IF(check_rows_k(M, N, "hidden activation"));
    RETURN_IF(check_ptr(out_codes, "out_codes"));
    RETURN_IF(check_ptr(out_sf, "out_sf"));
    if (h) RETURN_IF(check_ptr(h, "h"));
    return MXQ_OK;
}

int run_gemm_gelu_quant(const void* a_codes, const void* a_sf, int a_fmt, int64_t M, int64_t K,
                        const void* w_codes, const void* w_sf, int64_t N, const void* bias, int out_fmt,
                        void* out_codes, void* out_sf, void* h, cudaStream_t stream, bool gelu = true)
{
    GemmArgs g{a_codes, a_sf, a_fmt, M, N, K, w_codes, w_sf, bias, h};
    g.out_fmt = out_fmt;
    g.out_gelu = gelu;
    g.q_codes = out_codes;
    g.q_sf = out_sf;
    const char* msg = nullptr;
    int rc = launch_gemm(g, stream, &msg, g_path, sizeof g_path);
    if (rc != MXQ_OK) return fail(rc, "gemm: %s", msg ? msg : "launch failed");
    return ok();
}

// FFN workspace: the quantized input (up_fmt) and the quantized hidden activation
// (down_fmt), each codes then tiled scales, 256-byte aligned.
int64_t ffn_ws(int64_t M, int64_t K, int64_t H, int up_fmt, int down_fmt)
{
    return round_up(codes_bytes(M, K, up_fmt), kWsAlign) + round_up(sf_bytes(M, K), kWsAlign) +
           round_up(codes_bytes(M, H, down_fmt), kWsAlign) + round_up(sf_bytes(M, H), kWsAlign);
}

}  // namespace

extern "C" {

int mxq_version(void) { return 100; }

int64_t mxq_codes_bytes(int64_t rows, int64_t K, int fmt)
{
    if (rows <= 0 || K <= 0 || (fmt != MXQ_FMT_E2M1 && fmt != MXQ_FMT_E4M3)) return -1;
    return codes_bytes(rows, K, fmt);
}

int64_t mxq_sf_bytes(int64_t rows, int64_t K)
{
    if (rows <= 0 || K <= 0 || K % 32 != 0) return -1;
    return sf_bytes(rows, K);
}

int64_t mxq_workspace_bytes(int64_t M, int64_t N, int64_t K, int fmt, int mode)
{
    if (M <= 0 || N <= 0 || K <= 0 || K % 32 != 0) return -1;
    if ((fmt != MXQ_FMT_E2M1 && fmt != MXQ_FMT_E4M3) || (mode != MXQ_MODE_NATIVE && mode != MXQ_MODE_QDQ)) return -1;
    return linear_ws(M, N, K, fmt, mode);
}

int mxq_quantize_weight(const void* w_bf16, int64_t N, int64_t K, void* codes, void* sf, void* stream)
{
    return mxq_quantize_act(w_bf16, N, K, MXQ_FMT_E2M1, codes, sf, stream);
}

int mxq_quantize_act(const void* x_bf16, int64_t M, int64_t K, int fmt, void* codes, void* sf, void* stream)
{
    RETURN_IF(check_fmt(fmt));
    RETURN_IF(check_rows_k(M, K, "quantize"));
    RETURN_IF(check_ptr(x_bf16, "x"));
    RETURN_IF(check_ptr(codes, "codes"));
    RETURN_IF(check_ptr(sf, "sf"));
    RETURN_IF(check_device());
    snprintf(g_path, sizeof g_path, "quantize %s", fmt == MXQ_FMT_E4M3 ? "e4m3" : "e2m1");
    return cuda_rc(launch_quantize(x_bf16, M, K, fmt, codes, sf, static_cast<cudaStream_t>(stream)),
                   "quantize launch");
}

int mxq_dequantize(const void* codes, const void* sf, int64_t rows, int64_t K, int fmt, void* out_bf16,
                   void* stream)
{
    RETURN_IF(check_fmt(fmt));
    RETURN_IF(check_rows_k(rows, K, "dequantize"));
    RETURN_IF(check_ptr(codes, "codes"));
    RETURN_IF(check_ptr(sf, "sf"));
    RETURN_IF(check_ptr(out_bf16, "out"));
    RETURN_IF(check_device());
    snprintf(g_path, sizeof g_path, "dequantize %s", fmt == MXQ_FMT_E4M3 ? "e4m3" : "e2m1");
    return cuda_rc(launch_dequantize(codes, sf, rows, K, fmt, out_bf16, static_cast<cudaStream_t>(stream)),
                   "dequantize launch");
}

int mxq_gemm(const void* a_codes, const void* a_sf, int a_fmt, int64_t M, int64_t K, const void* w_codes,
             const void* w_sf, int64_t N, const void* bias_bf16, void* y_bf16, void* stream)
{
    RETURN_IF(check_gemm(a_codes, a_sf, a_fmt, M, K, w_codes, w_sf, N, bias_bf16, y_bf16));
    RETURN_IF(check_device());
    return run_gemm(a_codes, a_sf, a_fmt, M, K, w_codes, w_sf, N, bias_bf16, y_bf16,
                    static_cast<cudaStream_t>(stream));
}

int mxq_gemm_bf16(const void* a_bf16, int64_t M, int64_t K, const void* b_bf16, int64_t N, const void* bias_bf16,
                  void* y_bf16, void* stream)
{
    RETURN_IF(check_gemm_bf16(a_bf16, M, K, b_bf16, N, bias_bf16, y_bf16));
    RETURN_IF(check_device());
    return run_gemm_bf16(a_bf16, b_bf16, bias_bf16, y_bf16, M, N, K, static_cast<cudaStream_t>(stream));
}

// y = a . b^T + bias in bf16 by the bf16 GEMM kernel, whose extra warps also write a's MX
// quantization (format fmt) as its tiles pass through shared memory: one read of a.
int run_gemm_bf16_quant_a(const void* a, const void* b, const void* bias, void* y, int64_t M, int64_t N, int64_t K,
                          int fmt, void* codes, void* sf, cudaStream_t stream)
{
    GemmArgs g{a, nullptr, MXQ_FMT_E2M1, M, N, K, b, nullptr, bias, y};
    g.bf16 = true;
    g.qa_fmt = fmt;
    g.qa_codes = codes;
    g.qa_sf = sf;
    const char* msg = nullptr;
    int rc = launch_gemm(g, stream, &msg, g_path, sizeof g_path);
    if (rc != MXQ_OK) return fail(rc, "bf16 gemm quantizing a: %s", msg ? msg : "launch failed");
    return ok();
}

int mxq_gemm_bf16_quant_a(const void* a_bf16, int64_t M, int64_t K, const void* b_bf16, int64_t N,
                          const void* bias_bf16, void* y_bf16, int fmt, void* codes, void* sf, void* stream)
{
    RETURN_IF(check_fmt(fmt));
    RETURN_IF(check_rows_k(M, K, "a"));
    RETURN_IF(check_gemm_bf16(a_bf16, M, K, b_bf16, N, bias_bf16, y_bf16));
    if (N > 128) return fail(MXQ_ERR_SHAPE, "bf16 gemm quantizing a: N=%lld is above 128", (long long)N);
    RETURN_IF(check_ptr(codes, "codes"));
    RETURN_IF(check_ptr(sf, "sf"));
    RETURN_IF(check_device());
    return run_gemm_bf16_quant_a(a_bf16, b_bf16, bias_bf16, y_bf16, M, N, K, fmt, codes, sf,
                                 static_cast<cudaStream_t>(stream));
}

int mxq_linear(const void* x_bf16, int64_t M, int64_t K, const void* w_codes, const void* w_sf, int64_t N,
               const void* bias_bf16, int act_fmt, int mode, void* workspace, int64_t ws_bytes, void* y_bf16,
               void* stream)
{
    RETURN_IF(check_mode(mode));
    RETURN_IF(check_ptr(x_bf16, "x"));
    RETURN_IF(check_ptr(workspace, "workspace", kWsAlign));
    // the workspace stands in for the quantized activation in the GEMM checks
    RETURN_IF(check_gemm(workspace, workspace, act_fmt, M, K, w_codes, w_sf, N, bias_bf16, y_bf16));
    RETURN_IF(check_device());
    return run_linear(x_bf16, M, K, w_codes, w_sf, N, bias_bf16, act_fmt, mode, workspace, ws_bytes, y_bf16,
                      static_cast<cudaStream_t>(stream));
}

int64_t mxq_block_workspace_min_bytes(const mxq_wdesc* w, const int64_t* M_in, uint32_t w4a8_bits, int mode)
{
    if (!w || !M_in) return -1;
    int64_t need = 0;
    for (int i = 0; i < 8; ++i) {
        const int fmt = (w4a8_bits >> i) & 1u ? MXQ_FMT_E4M3 : MXQ_FMT_E2M1;
        const int64_t b = mxq_workspace_bytes(M_in[i], w[i].N, w[i].K, fmt, mode);
        if (b < 0) return -1;
        need = std::max(need, b);
    }
    return need;
}

int64_t mxq_block_workspace_bytes(const mxq_wdesc* w, const int64_t* M_in, uint32_t w4a8_bits, int mode)
{
    const int64_t seq = mxq_block_workspace_min_bytes(w, M_in, w4a8_bits, mode);
    if (seq < 0 || mode != MXQ_MODE_NATIVE) return seq;
    int64_t sum = 0;  // one quantized activation per linear
    for (int i = 0; i < 8; ++i)
        sum += round_up(mxq_workspace_bytes(M_in[i], w[i].N, w[i].K, (w4a8_bits >> i) & 1u ? MXQ_FMT_E4M3 : MXQ_FMT_E2M1,
                                            MXQ_MODE_NATIVE),
                        kWsAlign);
    return std::max(seq, sum);
}

}  // extern "C"

namespace {

using PfnCtxGetCurrent = CUresult (*)(CUcontext*);
using PfnCtxGetId = CUresult (*)(CUcontext, unsigned long long*);

// Unique ID of the calling thread's current CUDA context (the runtime's primary context
// of the current device once it has been initialized), through the driver entry points
// the runtime exposes; false if the driver lacks them.
bool current_context_id(unsigned long long* id)
{
    static PfnCtxGetCurrent get_current = nullptr;
    static PfnCtxGetId get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<PfnCtxGetCurrent>(p);
        p = nullptr;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<PfnCtxGetId>(p);
    });
    if (!get_current || !get_id) return false;
    CUcontext ctx = nullptr;
    if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return false;
    return get_id(ctx, id) == CUDA_SUCCESS;
}

// The stream and events the block entry point uses to quantize the next linears' inputs
// while the GEMMs run: one stream (non-blocking) and nine events per device, created on
// first use in each CUDA context (a device reset ends the old context and its handles, and
// the next call creates new ones) and kept until the process exits.  The enqueue sequence
// that uses them holds g_side_mu, so calls from several host threads cannot interleave
// their records and waits.
constexpr int kSideMaxDevices = 64;
struct SideStream {
    cudaStream_t s = nullptr;
    cudaEvent_t ev[9] = {};
    unsigned long long ctx_id = 0;
    bool have_id = false;
};
SideStream g_side[kSideMaxDevices];
std::mutex g_side_mu;

int side_stream(SideStream** out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(MXQ_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kSideMaxDevices) return fail(MXQ_ERR_UNSUPPORTED, "device index %d is too large", dev);
    SideStream& sd = g_side[dev];
    unsigned long long id = 0;
    const bool have_id = current_context_id(&id);
    if (!sd.s || sd.have_id != have_id || (have_id && sd.ctx_id != id)) {
        // first use in this context: the handles of an earlier context died with it
        sd.s = nullptr;
        e = cudaStreamCreateWithFlags(&sd.s, cudaStreamNonBlocking);
        for (int i = 0; i < 9 && e == cudaSuccess; ++i) e = cudaEventCreateWithFlags(&sd.ev[i], cudaEventDisableTiming);
        if (e != cudaSuccess) {
            sd.s = nullptr;
            return fail(MXQ_ERR_CUDA, "creating the block's side stream: %s", cudaGetErrorString(e));
        }
        sd.ctx_id = id;
        sd.have_id = have_id;
    }
    *out = &sd;
    return MXQ_OK;
}

// Native block with one quantized-activation buffer per linear: every input is quantized on
// the side stream, back to back, starting after the caller's earlier work; each GEMM on the
// caller's stream waits only for its own input's quantizer, so the later quantizers run
// while the earlier GEMMs do (the quantizer's CTAs need no shared memory and fit beside the
// GEMM's one CTA per SM).  The last GEMM waits for the last quantizer, so when the caller's
// stream has passed this call, all of it has finished.
int run_block_overlapped(const mxq_wdesc* w, const void* const* x_in, const int64_t* M_in, void* const* y_out,
                         uint32_t w4a8_bits, void* workspace, cudaStream_t stream)
{
    std::lock_guard<std::mutex> g(g_side_mu);
    SideStream* sd = nullptr;
    RETURN_IF(side_stream(&sd));
    uint8_t* buf[8];
    uint8_t* p = static_cast<uint8_t*>(workspace);
    for (int i = 0; i < 8; ++i) {
        const int fmt = (w4a8_bits >> i) & 1u ? MXQ_FMT_E4M3 : MXQ_FMT_E2M1;
        buf[i] = p;
        p += round_up(linear_ws(M_in[i], w[i].N, w[i].K, fmt, MXQ_MODE_NATIVE), kWsAlign);
    }
    RETURN_IF(cuda_rc(cudaEventRecord(sd->ev[8], stream), "event record"));
    RETURN_IF(cuda_rc(cudaStreamWaitEvent(sd->s, sd->ev[8], 0), "stream wait"));
    for (int i = 0; i < 8; ++i) {
        const int fmt = (w4a8_bits >> i) & 1u ? MXQ_FMT_E4M3 : MXQ_FMT_E2M1;
        uint8_t* xc = buf[i];
        uint8_t* xs = xc + round_up(codes_bytes(M_in[i], w[i].K, fmt), kWsAlign);
        RETURN_IF(cuda_rc(launch_quantize(x_in[i], M_in[i], w[i].K, fmt, xc, xs, sd->s), "quantize launch"));
        RETURN_IF(cuda_rc(cudaEventRecord(sd->ev[i], sd->s), "event record"));
    }
    for (int i = 0; i < 8; ++i) {
        const int fmt = (w4a8_bits >> i) & 1u ? MXQ_FMT_E4M3 : MXQ_FMT_E2M1;
        uint8_t* xc = buf[i];
        uint8_t* xs = xc + round_up(codes_bytes(M_in[i], w[i].K, fmt), kWsAlign);
        RETURN_IF(cuda_rc(cudaStreamWaitEvent(stream, sd->ev[i], 0), "stream wait"));
        int rc = run_gemm(xc, xs, fmt, M_in[i], w[i].K, w[i].codes, w[i].sf, w[i].N, w[i].bias, y_out[i], stream);
        if (rc != MXQ_OK) return fail(rc, "block linear %d: %s", i, g_err);
    }
    return MXQ_OK;
}

}  // namespace

extern "C" {

int mxq_dit_block_linears(const mxq_wdesc* w, const void* const* x_in, const int64_t* M_in, void* const* y_out,
                          uint32_t w4a8_bits, int mode, void* workspace, int64_t ws_bytes, void* stream)
{
    if (!w || !x_in || !M_in || !y_out) return fail(MXQ_ERR_INVALID_ARG, "block: NULL array argument");
    if (w4a8_bits > 0xFFu) return fail(MXQ_ERR_INVALID_ARG, "block: w4a8_bits has bits above 7 (0x%x)", w4a8_bits);
    RETURN_IF(check_mode(mode));
    RETURN_IF(check_ptr(workspace, "workspace", kWsAlign));
    for (int i = 0; i < 8; ++i) {
        const int fmt = (w4a8_bits >> i) & 1u ? MXQ_FMT_E4M3 : MXQ_FMT_E2M1;
        RETURN_IF(check_ptr(x_in[i], "block x_in[i]"));
        int rc = check_gemm(workspace, workspace, fmt, M_in[i], w[i].K, w[i].codes, w[i].sf, w[i].N, w[i].bias,
                            y_out[i]);
        if (rc != MXQ_OK) return fail(rc, "block linear %d: %s", i, g_err);
    }
    const int64_t need = mxq_block_workspace_min_bytes(w, M_in, w4a8_bits, mode);
    if (ws_bytes < need)
        return fail(MXQ_ERR_WORKSPACE, "block workspace has %lld bytes, needs %lld", (long long)ws_bytes,
                    (long long)need);
    RETURN_IF(check_device());
    const bool overlap = mode == MXQ_MODE_NATIVE && ws_bytes >= mxq_block_workspace_bytes(w, M_in, w4a8_bits, mode);
    if (overlap) {
        RETURN_IF(run_block_overlapped(w, x_in, M_in, y_out, w4a8_bits, workspace, static_cast<cudaStream_t>(stream)));
    } else {
        for (int i = 0; i < 8; ++i) {
            const int fmt = (w4a8_bits >> i) & 1u ? MXQ_FMT_E4M3 : MXQ_FMT_E2M1;
            int rc = run_linear(x_in[i], M_in[i], w[i].K, w[i].codes, w[i].sf, w[i].N, w[i].bias, fmt, mode,
                                workspace, ws_bytes, y_out[i], static_cast<cudaStream_t>(stream));
            if (rc != MXQ_OK) return fail(rc, "block linear %d: %s", i, g_err);
        }
    }
    snprintf(g_path, sizeof g_path, "block %s%s w4a8_bits 0x%02x", mode == MXQ_MODE_QDQ ? "qdq" : "native",
             overlap ? " overlapped" : "", w4a8_bits);
    return ok();
}

int mxq_gemm_gelu_quant(const void* a_codes, const void* a_sf, int a_fmt, int64_t M, int64_t K,
                        const void* w_codes, const void* w_sf, int64_t N, const void* bias_bf16, int out_fmt,
                        void* out_codes, void* out_sf, void* h_bf16, void* stream)
{
    // out_codes stands in for y in the plain GEMM checks (h is optional)
    RETURN_IF(check_gemm(a_codes, a_sf, a_fmt, M, K, w_codes, w_sf, N, bias_bf16, out_codes));
    RETURN_IF(check_gelu_quant(M, N, out_fmt, out_codes, out_sf, h_bf16));
    RETURN_IF(check_device());
    return run_gemm_gelu_quant(a_codes, a_sf, a_fmt, M, K, w_codes, w_sf, N, bias_bf16, out_fmt, out_codes, out_sf,
                               h_bf16, static_cast<cudaStream_t>(stream));
}

int mxq_gemm_quant(const void* a_codes, const void* a_sf, int a_fmt, int64_t M, int64_t K, const void* w_codes,
                   const void* w_sf, int64_t N, const void* bias_bf16, int act, int out_fmt, void* out_codes,
                   void* out_sf, void* h_bf16, void* stream)
{
    if (act != MXQ_ACT_NONE && act != MXQ_ACT_GELU) return fail(MXQ_ERR_INVALID_ARG, "unknown activation %d", act);
    RETURN_IF(check_gemm(a_codes, a_sf, a_fmt, M, K, w_codes, w_sf, N, bias_bf16, out_codes));
    RETURN_IF(check_gelu_quant(M, N, out_fmt, out_codes, out_sf, h_bf16));
    RETURN_IF(check_device());
    return run_gemm_gelu_quant(a_codes, a_sf, a_fmt, M, K, w_codes, w_sf, N, bias_bf16, out_fmt, out_codes, out_sf,
                               h_bf16, static_cast<cudaStream_t>(stream), act == MXQ_ACT_GELU);
}

int64_t mxq_ffn_workspace_bytes(int64_t M, int64_t K, int64_t H, int up_fmt, int down_fmt)
{
    if (M <= 0 || K <= 0 || H <= 0 || K % 32 != 0 || H % 32 != 0) return -1;
    if ((up_fmt != MXQ_FMT_E2M1 && up_fmt != MXQ_FMT_E4M3) || (down_fmt != MXQ_FMT_E2M1 && down_fmt != MXQ_FMT_E4M3))
        return -1;
    return ffn_ws(M, K, H, up_fmt, down_fmt);
}

int mxq_ffn(const void* x_bf16, int64_t M, int64_t K, const mxq_wdesc* up, const mxq_wdesc* down, int up_fmt,
            int down_fmt, void* workspace, int64_t ws_bytes, void* y_bf16, void* stream)
{
    if (!up || !down) return fail(MXQ_ERR_INVALID_ARG, "ffn: NULL weight descriptor");
    if (up->K != K) return fail(MXQ_ERR_SHAPE, "ffn: up-projection K=%lld but x has K=%lld", (long long)up->K,
                                (long long)K);
    if (down->K != up->N)
        return fail(MXQ_ERR_SHAPE, "ffn: down-projection K=%lld differs from the hidden width %lld",
                    (long long)down->K, (long long)up->N);
    RETURN_IF(check_ptr(x_bf16, "x"));
    RETURN_IF(check_ptr(workspace, "workspace", kWsAlign));
    const int64_t H = up->N;
    RETURN_IF(check_gemm(workspace, workspace, up_fmt, M, K, up->codes, up->sf, H, up->bias, workspace));
    RETURN_IF(check_gelu_quant(M, H, down_fmt, workspace, workspace, nullptr));
    RETURN_IF(check_gemm(workspace, workspace, down_fmt, M, H, down->codes, down->sf, down->N, down->bias, y_bf16));
    const int64_t need = ffn_ws(M, K, H, up_fmt, down_fmt);
    if (ws_bytes < need)
        return fail(MXQ_ERR_WORKSPACE, "ffn workspace has %lld bytes, needs %lld", (long long)ws_bytes,
                    (long long)need);
    RETURN_IF(check_device());
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t* xc = static_cast<uint8_t*>(workspace);
    uint8_t* xs = xc + round_up(codes_bytes(M, K, up_fmt), kWsAlign);
    uint8_t* hc = xs + round_up(sf_bytes(M, K), kWsAlign);
    uint8_t* hs = hc + round_up(codes_bytes(M, H, down_fmt), kWsAlign);
    RETURN_IF(cuda_rc(launch_quantize(x_bf16, M, K, up_fmt, xc, xs, st), "quantize launch"));
    RETURN_IF(run_gemm_gelu_quant(xc, xs, up_fmt, M, K, up->codes, up->sf, H, up->bias, down_fmt, hc, hs, nullptr,
                                  st));
    RETURN_IF(run_gemm(hc, hs, down_fmt, M, H, down->codes, down->sf, down->N, down->bias, y_bf16, st));
    snprintf(g_path, sizeof g_path, "ffn %s -> gelu -> %s fused", up_fmt == MXQ_FMT_E4M3 ? "e4m3" : "e2m1",
             down_fmt == MXQ_FMT_E4M3 ? "e4m3" : "e2m1");
    return ok();
}

int mxq_quantize_act_static(const void* x_bf16, int64_t M, int64_t K, float scale, void* codes, void* sf,
                            void* stream)
{
    if (!(scale > 0.0f) || !std::isfinite(scale))
        return fail(MXQ_ERR_INVALID_ARG, "static scale must be positive and finite (got %g)", (double)scale);
    RETURN_IF(check_rows_k(M, K, "quantize_static"));
    RETURN_IF(check_ptr(x_bf16, "x"));
    RETURN_IF(check_ptr(codes, "codes"));
    RETURN_IF(check_ptr(sf, "sf"));
    RETURN_IF(check_device());
    snprintf(g_path, sizeof g_path, "quantize static e4m3");
    return cuda_rc(launch_quantize_static(x_bf16, M, K, scale, codes, sf,
                                          static_cast<cudaStream_t>(stream)),
                   "quantize launch");
}

int mxq_linear_static(const void* x_bf16, int64_t M, int64_t K, const void* w_codes, const void* w_sf, int64_t N,
                      const void* bias_bf16, float act_scale, void* workspace, int64_t ws_bytes, void* y_bf16,
                      void* stream)
{
    if (!(act_scale > 0.0f) || !std::isfinite(act_scale))
        return fail(MXQ_ERR_INVALID_ARG, "static scale must be positive and finite (got %g)", (double)act_scale);
    RETURN_IF(check_ptr(x_bf16, "x"));
    RETURN_IF(check_ptr(workspace, "workspace", kWsAlign));
    RETURN_IF(check_gemm(workspace, workspace, MXQ_FMT_E4M3, M, K, w_codes, w_sf, N, bias_bf16, y_bf16));
    const int64_t need = linear_ws(M, N, K, MXQ_FMT_E4M3, MXQ_MODE_NATIVE);
    if (ws_bytes < need)
        return fail(MXQ_ERR_WORKSPACE, "workspace has %lld bytes, needs %lld", (long long)ws_bytes, (long long)need);
    RETURN_IF(check_device());
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t* xc = static_cast<uint8_t*>(workspace);
    uint8_t* xs = xc + round_up(codes_bytes(M, K, MXQ_FMT_E4M3), kWsAlign);
    RETURN_IF(cuda_rc(launch_quantize_static(x_bf16, M, K, act_scale, xc, xs, st), "quantize launch"));
    GemmArgs g{xc, xs, MXQ_FMT_E4M3, M, N, K, w_codes, w_sf, bias_bf16, y_bf16};
    g.alpha = act_scale;
    const char* msg = nullptr;
    int rc = launch_gemm(g, st, &msg, g_path, sizeof g_path);
    if (rc != MXQ_OK) return fail(rc, "gemm: %s", msg ? msg : "launch failed");
    snprintf(g_path + strlen(g_path), sizeof g_path - strlen(g_path), " static-scale");
    return ok();
}

int mxq_quantize_act_transformed(const void* x_bf16, int64_t M, int64_t K, int fmt, const float* mul, int block,
                                 void* codes, void* sf, void* stream)
{
    RETURN_IF(check_fmt(fmt));
    RETURN_IF(check_rows_k(M, K, "quantize_transformed"));
    RETURN_IF(check_transform(K, block, mul));
    RETURN_IF(check_ptr(x_bf16, "x"));
    RETURN_IF(check_ptr(codes, "codes"));
    RETURN_IF(check_ptr(sf, "sf"));
    RETURN_IF(check_device());
    snprintf(g_path, sizeof g_path, "quantize %s hadamard%d%s", fmt == MXQ_FMT_E4M3 ? "e4m3" : "e2m1", block,
             mul ? " smooth" : "");
    return cuda_rc(launch_quantize_transform(x_bf16, M, K, fmt, mul, block, hadamard_norm(block), codes, sf,
                                             static_cast<cudaStream_t>(stream)),
                   "quantize launch");
}

int mxq_quantize_weight_transformed(const void* w_bf16, int64_t N, int64_t K, const float* mul, int block, void* codes,
                                    void* sf, void* stream)
{
    return mxq_quantize_act_transformed(w_bf16, N, K, MXQ_FMT_E2M1, mul, block, codes, sf, stream);
}

int mxq_linear_transformed(const void* x_bf16, int64_t M, int64_t K, const void* w_codes, const void* w_sf, int64_t N,
                           const void* bias_bf16, int act_fmt, const float* act_mul, int block, void* workspace,
                           int64_t ws_bytes, void* y_bf16, void* stream)
{
    RETURN_IF(check_ptr(x_bf16, "x"));
    RETURN_IF(check_ptr(workspace, "workspace", kWsAlign));
    RETURN_IF(check_gemm(workspace, workspace, act_fmt, M, K, w_codes, w_sf, N, bias_bf16, y_bf16));
    RETURN_IF(check_transform(K, block, act_mul));
    const int64_t need = linear_ws(M, N, K, act_fmt, MXQ_MODE_NATIVE);
    if (ws_bytes < need)
        return fail(MXQ_ERR_WORKSPACE, "workspace has %lld bytes, needs %lld", (long long)ws_bytes, (long long)need);
    RETURN_IF(check_device());
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t* xc = static_cast<uint8_t*>(workspace);
    uint8_t* xs = xc + round_up(codes_bytes(M, K, act_fmt), kWsAlign);
    RETURN_IF(cuda_rc(launch_quantize_transform(x_bf16, M, K, act_fmt, act_mul, block, hadamard_norm(block), xc, xs, st),
                      "quantize launch"));
    RETURN_IF(run_gemm(xc, xs, act_fmt, M, K, w_codes, w_sf, N, bias_bf16, y_bf16, st));
    snprintf(g_path + strlen(g_path), sizeof g_path - strlen(g_path), " hadamard%d%s", block, act_mul ? " smooth" : "");
    return ok();
}

int64_t mxq_lowrank_workspace_bytes(int64_t M, int64_t N, int64_t K, int fmt, int64_t rank)
{
    const int64_t base = mxq_workspace_bytes(M, N, K, fmt, MXQ_MODE_NATIVE);
    if (base < 0 || rank <= 0 || rank % 64 != 0 || rank > 256) return -1;
    return base + round_up(M * rank * 2, kWsAlign);
}

int mxq_linear_lowrank(const void* x_bf16, int64_t M, int64_t K, const void* r_codes, const void* r_sf, int64_t N,
                       const void* bias_bf16, int act_fmt, const void* l1t_bf16, const void* l2t_bf16, int64_t rank,
                       void* workspace, int64_t ws_bytes, void* y_bf16, void* stream)
{
    if (rank <= 0 || rank % 64 != 0 || rank > 256)
        return fail(MXQ_ERR_INVALID_ARG, "low-rank branch: rank must be 64, 128, 192 or 256 (got %lld)",
                    (long long)rank);
    RETURN_IF(check_ptr(x_bf16, "x"));
    RETURN_IF(check_ptr(l1t_bf16, "l1t"));
    RETURN_IF(check_ptr(l2t_bf16, "l2t"));
    RETURN_IF(check_ptr(workspace, "workspace", kWsAlign));
    RETURN_IF(check_gemm(workspace, workspace, act_fmt, M, K, r_codes, r_sf, N, bias_bf16, y_bf16));
    const int64_t need = mxq_lowrank_workspace_bytes(M, N, K, act_fmt, rank);
    if (ws_bytes < need)
        return fail(MXQ_ERR_WORKSPACE, "workspace has %lld bytes, needs %lld", (long long)ws_bytes, (long long)need);
    RETURN_IF(check_device());
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t* xc = static_cast<uint8_t*>(workspace);
    uint8_t* xs = xc + round_up(codes_bytes(M, K, act_fmt), kWsAlign);
    uint8_t* u = xs + round_up(sf_bytes(M, K), kWsAlign);
    // u = x . l1t^T: [M, K] x [K, rank], the bf16 GEMM with N = rank; up to rank 128 the
    // same launch writes x quantized in act_fmt (xc, xs), so x is read once for both
    int rc;
    if (rank <= 128) {
        rc = run_gemm_bf16_quant_a(x_bf16, l1t_bf16, nullptr, u, M, rank, K, act_fmt, xc, xs, st);
    } else {
        RETURN_IF(cuda_rc(launch_quantize(x_bf16, M, K, act_fmt, xc, xs, st), "quantize launch"));
        rc = run_gemm_bf16(x_bf16, l1t_bf16, nullptr, u, M, rank, K, st);
    }
    if (rc != MXQ_OK) return fail(rc, "low-rank u: %s", g_err);
    GemmArgs g{xc, xs, act_fmt, M, N, K, r_codes, r_sf, bias_bf16, y_bf16};
    g.lr_rank = rank;
    g.lr_u = u;
    g.lr_l2t = l2t_bf16;
    const char* msg = nullptr;
    rc = launch_gemm(g, st, &msg, g_path, sizeof g_path);
    if (rc != MXQ_OK) return fail(rc, "gemm: %s", msg ? msg : "launch failed");
    return ok();
}

int mxq_tier_thresholds(int tier, double* floor_db, double* w4a8_db, double* margin_db)
{
    static const double kTiers[3][3] = {{8.0, 21.0, 0.5}, {10.0, 23.0, 0.5}, {12.0, 25.0, 0.5}};
    if (tier < MXQ_TIER_LOW || tier > MXQ_TIER_HIGH) return fail(MXQ_ERR_INVALID_ARG, "unknown tier %d", tier);
    if (floor_db) *floor_db = kTiers[tier][0];
    if (w4a8_db) *w4a8_db = kTiers[tier][1];
    if (margin_db) *margin_db = kTiers[tier][2];
    return ok();
}

int mxq_select_policy(double sqnr_off, double sqnr_on, int tier)
{
    double floor_db, w4a8_db, margin_db;
    if (mxq_tier_thresholds(tier, &floor_db, &w4a8_db, &margin_db) != MXQ_OK) return -1;
    if (std::isnan(sqnr_off) || std::isnan(sqnr_on)) {
        fail(MXQ_ERR_INVALID_ARG, "NaN SQNR");
        return -1;
    }
    const double best = std::max(sqnr_off, sqnr_on);
    if (best < floor_db) return MXQ_POLICY_BF16;
    if (best < w4a8_db) return MXQ_POLICY_W4A8;
    if (sqnr_on - sqnr_off > margin_db) return MXQ_POLICY_TRANSFORM_ON;
    return MXQ_POLICY_PLAIN_MXFP4;
}

int mxq_absmax(const void* x_bf16, int64_t n, void* out_f32, void* stream)
{
    if (n <= 0 || n % 8 != 0) return fail(MXQ_ERR_SHAPE, "absmax: n=%lld must be a positive multiple of 8", (long long)n);
    RETURN_IF(check_ptr(x_bf16, "x"));
    RETURN_IF(check_ptr(out_f32, "out", 4));
    RETURN_IF(check_device());
    return cuda_rc(launch_absmax(x_bf16, n, static_cast<float*>(out_f32), static_cast<cudaStream_t>(stream)),
                   "absmax launch");
}

int mxq_gelu_bf16(const void* x_bf16, int64_t n, void* y_bf16, void* stream)
{
    if (n <= 0) return fail(MXQ_ERR_INVALID_ARG, "gelu_bf16: n=%lld must be positive", (long long)n);
    RETURN_IF(check_ptr(x_bf16, "x", 2));
    RETURN_IF(check_ptr(y_bf16, "y", 2));
    RETURN_IF(check_device());
    return cuda_rc(launch_gelu_bf16(x_bf16, n, y_bf16, static_cast<cudaStream_t>(stream)), "gelu launch");
}

int mxq_channel_absmax(const void* x_bf16, int64_t rows, int64_t K, float* out_f32, void* stream)
{
    if (rows <= 0 || K <= 0) return fail(MXQ_ERR_INVALID_ARG, "channel_absmax: sizes must be positive");
    if (K % 8 != 0) return fail(MXQ_ERR_SHAPE, "channel_absmax: K=%lld is not a multiple of 8", (long long)K);
    if (rows > (int64_t(1) << 31) - 1 || K > (int64_t(1) << 31) - 1 || rows * K > kMaxElems)
        return fail(MXQ_ERR_SHAPE, "channel_absmax: tensor too large");
    RETURN_IF(check_ptr(x_bf16, "x"));
    RETURN_IF(check_ptr(out_f32, "out", 4));
    RETURN_IF(check_device());
    snprintf(g_path, sizeof g_path, "channel absmax");
    return cuda_rc(launch_channel_absmax(x_bf16, rows, K, out_f32, static_cast<cudaStream_t>(stream)),
                   "channel_absmax launch");
}

int mxq_smooth_scales(const float* amax_x, const float* amax_w, int64_t K, float alpha, float* s, float* inv_s,
                      void* stream)
{
    if (K <= 0 || K > (int64_t(1) << 31) - 1) return fail(MXQ_ERR_INVALID_ARG, "smooth_scales: bad K=%lld", (long long)K);
    if (!(alpha >= 0.0f && alpha <= 1.0f))
        return fail(MXQ_ERR_INVALID_ARG, "smooth_scales: alpha must lie in [0, 1] (got %g)", (double)alpha);
    RETURN_IF(check_ptr(amax_x, "amax_x", 4));
    RETURN_IF(check_ptr(amax_w, "amax_w", 4));
    RETURN_IF(check_ptr(s, "s", 4));
    if (inv_s) RETURN_IF(check_ptr(inv_s, "inv_s", 4));
    RETURN_IF(check_device());
    snprintf(g_path, sizeof g_path, "smooth scales");
    return cuda_rc(launch_smooth_scales(amax_x, amax_w, K, alpha, s, inv_s, static_cast<cudaStream_t>(stream)),
                   "smooth_scales launch");
}

int mxq_sqnr(const void* const* ref_bf16, const void* const* test_bf16, const int64_t* n, int count, double* out_f64,
             void* stream)
{
    if (!ref_bf16 || !test_bf16 || !n || count <= 0) return fail(MXQ_ERR_INVALID_ARG, "sqnr: empty or NULL arrays");
    for (int i = 0; i < count; ++i) {
        if (n[i] <= 0 || n[i] % 8 != 0)
            return fail(MXQ_ERR_SHAPE, "sqnr: tensor %d has n=%lld (a positive multiple of 8 is required)", i,
                        (long long)n[i]);
        RETURN_IF(check_ptr(ref_bf16[i], "ref"));
        RETURN_IF(check_ptr(test_bf16[i], "test"));
    }
    RETURN_IF(check_ptr(out_f64, "out", 8));
    RETURN_IF(check_device());
    snprintf(g_path, sizeof g_path, "sqnr over %d tensors", count);
    return cuda_rc(launch_sqnr(ref_bf16, test_bf16, n, count, out_f64, static_cast<cudaStream_t>(stream)),
                   "sqnr launch");
}

int mxq_lowrank_split(const float* U, int64_t ldu, const float* S, const float* Vh, int64_t ldvh, const void* w_bf16,
                      int64_t N, int64_t K, int64_t rank, void* l2t_bf16, void* l1t_bf16, void* resid_bf16,
                      void* stream)
{
    if (N <= 0 || K <= 0 || rank <= 0) return fail(MXQ_ERR_INVALID_ARG, "lowrank_split: sizes must be positive");
    if (ldu < rank || ldvh < K) return fail(MXQ_ERR_INVALID_ARG, "lowrank_split: row strides too small");
    if (N > (int64_t(1) << 31) - 1 || K > (int64_t(1) << 31) - 1 || rank > 4096 || N * K > kMaxElems)
        return fail(MXQ_ERR_SHAPE, "lowrank_split: sizes above the supported maximum");
    RETURN_IF(check_ptr(U, "U", 4));
    RETURN_IF(check_ptr(S, "S", 4));
    RETURN_IF(check_ptr(Vh, "Vh", 4));
    RETURN_IF(check_ptr(w_bf16, "w"));
    RETURN_IF(check_ptr(l2t_bf16, "l2t"));
    RETURN_IF(check_ptr(l1t_bf16, "l1t"));
    RETURN_IF(check_ptr(resid_bf16, "residual"));
    RETURN_IF(check_device());
    snprintf(g_path, sizeof g_path, "lowrank split rank %lld", (long long)rank);
    return cuda_rc(launch_lowrank_split(U, ldu, S, Vh, ldvh, w_bf16, N, K, rank, l2t_bf16, l1t_bf16, resid_bf16,
                                        static_cast<cudaStream_t>(stream)),
                   "lowrank_split launch");
}

int mxq_sf_to_logical(const void* sf_tiled, int64_t rows, int64_t K, void* sf_rowmajor, void* stream)
{
    RETURN_IF(check_rows_k(rows, K, "sf_to_logical"));
    RETURN_IF(check_ptr(sf_tiled, "sf_tiled"));
    if (!sf_rowmajor) return fail(MXQ_ERR_INVALID_ARG, "sf_rowmajor is NULL");
    RETURN_IF(check_device());
    return cuda_rc(launch_sf_to_logical(sf_tiled, rows, K, sf_rowmajor, static_cast<cudaStream_t>(stream)),
                   "sf_to_logical launch");
}

int mxq_poll_status(void* stream)
{
    uint32_t v = 0, q = 0;
    int rc = read_and_clear_device_status(static_cast<cudaStream_t>(stream), &v);
    if (rc == MXQ_OK) rc = read_and_clear_quant_status(static_cast<cudaStream_t>(stream), &q);
    if (rc != MXQ_OK) return fail(rc, "reading the device status word failed");
    if (v != 0) return fail(static_cast<int>(v), "a GEMM kernel's bounded wait ran out");
    if (q != 0) return fail(static_cast<int>(q), "a quantizer kernel's bounded wait ran out");
    return ok();
}

int mxq_set_debug(uint32_t flags)
{
    set_debug_flags(flags);
    return MXQ_OK;
}

const char* mxq_last_error(void) { return g_err; }
const char* mxq_last_path(void) { return g_path; }

}  // extern "C"

// ----------------------------------------------------------------------------------------
// Linear layer without any allocation.
//
// Some callers cannot allocate device memory at the point where they run a layer: code
// that runs under a memory manager that owns the whole device pool, plugins that are
// handed only the input and output buffers, or code paths that must not call into an
// allocator at all.  mxq_linear_noalloc serves them: the one scratch buffer the native
// linear needs (the quantized activation: element codes and tiled scales) lives in a
// file-scope device array of fixed size instead of a caller-provided workspace.
// ----------------------------------------------------------------------------------------
namespace {

constexpr int64_t kNoAllocScratchBytes = int64_t(32) << 20;  // 32 MiB per device
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kNoAllocMaxDevices = 64;
// Per device: the address found and the CUDA context it belongs to.  A device reset (or
// the primary context being released and created again) loads the module anew, and the
// array can then sit at another address; keying the cache on the context's unique ID
// makes the first call in a new context look the address up again.
struct NoAllocSlot {
    void* ptr = nullptr;
    unsigned long long ctx_id = 0;
    bool have_id = false;
};
NoAllocSlot g_noalloc[kNoAllocMaxDevices];
std::mutex g_noalloc_mu;

// Device address of the scratch array in the current device's context.  In host code the
// array's name is only a stand-in, so the address is looked up (with that device current)
// on the first call in each context and cached.
int noalloc_scratch(void** out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(MXQ_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kNoAllocMaxDevices)
        return fail(MXQ_ERR_UNSUPPORTED, "device index %d is above the supported %d", dev, kNoAllocMaxDevices);
    unsigned long long id = 0;
    bool have_id = current_context_id(&id);
    if (!have_id) {
        // no context current on this thread yet: make the device's primary context current
        // (cudaSetDevice initializes it), then ask again
        e = cudaSetDevice(dev);
        if (e != cudaSuccess) return fail(MXQ_ERR_CUDA, "cudaSetDevice: %s", cudaGetErrorString(e));
        have_id = current_context_id(&id);
    }
    std::lock_guard<std::mutex> g(g_noalloc_mu);
    NoAllocSlot& slot = g_noalloc[dev];
    if (!slot.ptr || slot.have_id != have_id || (have_id && slot.ctx_id != id)) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || !p)
            return fail(MXQ_ERR_CUDA, "cudaGetSymbolAddress of the static scratch: %s", cudaGetErrorString(e));
        slot.ptr = p;
        slot.ctx_id = id;
        slot.have_id = have_id;
    }
    *out = slot.ptr;
    return MXQ_OK;
}

}  // namespace

extern "C" int64_t mxq_linear_noalloc_max_scratch_bytes(void) { return kNoAllocScratchBytes; }

extern "C" int mxq_linear_noalloc(const void* x_bf16, int64_t M, int64_t K, const void* w_codes, const void* w_sf,
                                  int64_t N, const void* bias_bf16, int act_fmt, void* y_bf16, void* stream)
{
    RETURN_IF(check_ptr(x_bf16, "x"));
    // the scratch is 256-byte aligned by its declaration; stand in a non-null aligned value
    const void* scratch_standin = reinterpret_cast<const void*>(uintptr_t(256));
    RETURN_IF(check_gemm(scratch_standin, scratch_standin, act_fmt, M, K, w_codes, w_sf, N, bias_bf16, y_bf16));
    const int64_t need = linear_ws(M, N, K, act_fmt, MXQ_MODE_NATIVE);
    if (need > kNoAllocScratchBytes)
        return fail(MXQ_ERR_WORKSPACE,
                    "mxq_linear_noalloc: M=%lld K=%lld (%s) needs %lld bytes of scratch; the static scratch holds "
                    "%lld bytes (use mxq_linear with a workspace for larger inputs)",
                    (long long)M, (long long)K, act_fmt == MXQ_FMT_E4M3 ? "e4m3" : "e2m1", (long long)need,
                    (long long)kNoAllocScratchBytes);
    RETURN_IF(check_device());
    void* ws = nullptr;
    RETURN_IF(noalloc_scratch(&ws));
    return run_linear(x_bf16, M, K, w_codes, w_sf, N, bias_bf16, act_fmt, MXQ_MODE_NATIVE, ws, kNoAllocScratchBytes,
                      y_bf16, static_cast<cudaStream_t>(stream));
}
