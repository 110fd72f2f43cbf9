/*
 * mxq.h -- C ABI of libmxq.so: the MX block-quantized linear layer on B200 (sm_100a).
 *
 * The operation is the one the blog "Quark Mixed-Precision Quantization for Wan2.2
 * Video Generation on AMD Instinct GPUs" studies:
 *   - W4A4 = OCP MXFP4 weights with dynamic MXFP4 activations, W4A8 = MXFP4 weights
 *     with FP8 E4M3 activations (section "Quantization formats", its table);
 *   - the MX format is the OCP Microscaling spec v1.0 (the blog's reference [7]):
 *     blocks of 32 consecutive elements along K share one E8M0 scale
 *     X = 2^(floor(log2(amax)) - emax) (emax 2 for E2M1, 8 for E4M3; clamped at
 *     2^-127), and each element is stored as round-to-nearest-even(x / X) on the
 *     element grid, saturating at the largest finite element ("RTN" in the
 *     section "Results" tables);
 *   - a block whose input holds Inf or NaN gets scale code 0xFF and zero codes;
 *     a negative value that rounds to zero keeps its sign bit;
 *   - the linear layer is Y = deq(Xq) . deq(Wq)^T (+ bias) with fp32 accumulation
 *     and a bf16 output (section "Quantization formats", "Kernel note": native
 *     MXFP4 GEMM for W4A4; quantize-dequantize emulation for W4A8);
 *   - a per-expert, per-block policy picks W4A4 or W4A8 for each DiT block
 *     (sections "Mixed-Precision selection" and "Practical workflow", step 6).
 *
 * Conventions for every entry point:
 *   - Shapes follow torch.nn.Linear: X is [M, K] (tokens x in-features), W is
 *     [N, K] (out x in-features), Y is [M, N]; all row-major, K contiguous.
 *   - All data pointers are DEVICE pointers the caller allocated and owns (for
 *     example torch tensors); the library never allocates or frees device memory
 *     and never synchronizes.  `stream` is a cudaStream_t (NULL = legacy default
 *     stream); all work is enqueued on it and runs asynchronously.
 *   - Element codes: E2M1 packs two per byte, element 2j in the low nibble of
 *     byte j and element 2j+1 in the high nibble ([rows, K/2] bytes); E4M3 uses one
 *     byte per element ([rows, K] bytes).
 *   - Scale factors (E8M0 bytes) are stored in the tiled layout the tcgen05
 *     block-scaled MMA reads: 512-byte atoms of 128 rows x 4 k-blocks, the byte of
 *     (row r, k-block kb) at offset (r%32)*16 + ((r/32)%4)*4 + kb%4 inside atom
 *     (r/128)*ceil(K/128) + kb/4.  Rows are padded to 128 and k-blocks to a
 *     multiple of 4; the quantizers write the padding as 0.
 *   - Every call returns an mxq_status.  Arguments are validated before anything
 *     is enqueued, so on an error nothing was launched; mxq_last_error() then
 *     describes it.  Kernel launch failures return MXQ_ERR_CUDA.  The internal
 *     waits of the GEMM and of the transform quantizer are bounded; if one ever runs
 *     out, the kernel records MXQ_ERR_TIMEOUT in a device status word that
 *     mxq_poll_status() returns.
 */
#ifndef MXQ_H
#define MXQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MXQ_OK = 0,
    MXQ_ERR_INVALID_ARG = 1, /* null pointer, non-positive size, unknown enum value   */
    MXQ_ERR_SHAPE = 2,       /* K % 32 != 0, N % 8 != 0, W4A8 native with K % 128 != 0 */
    MXQ_ERR_ALIGN = 3,       /* a pointer is not 16-byte aligned (32 for W4A8 weights) */
    MXQ_ERR_UNSUPPORTED = 4, /* the current device is not sm_100                        */
    MXQ_ERR_CUDA = 5,        /* a CUDA runtime or driver call failed                    */
    MXQ_ERR_TIMEOUT = 6,     /* a bounded device-side wait ran out                      */
    MXQ_ERR_WORKSPACE = 7    /* the workspace passed is smaller than required           */
} mxq_status;

typedef enum { MXQ_FMT_E2M1 = 0, MXQ_FMT_E4M3 = 1 } mxq_fmt;      /* activation element format */
typedef enum { MXQ_MODE_NATIVE = 0, MXQ_MODE_QDQ = 1 } mxq_mode;  /* GEMM execution mode       */
typedef enum { MXQ_ACT_NONE = 0, MXQ_ACT_GELU = 1 } mxq_act;       /* quantizing epilogue's activation */

/* Library version (major*10000 + minor*100 + patch). */
int mxq_version(void);

/* Bytes of the element codes of a [rows, K] tensor: rows*K/2 (E2M1) or rows*K (E4M3). */
int64_t mxq_codes_bytes(int64_t rows, int64_t K, int fmt);

/* Bytes of the tiled scale-factor buffer of a [rows, K] tensor:
 * ceil(rows/128)*128 * ceil(K/128)*4. */
int64_t mxq_sf_bytes(int64_t rows, int64_t K);

/* Workspace bytes mxq_linear needs for these sizes, format and mode (native: the
 * quantized activation; QDQ: also both dequantized operands in bf16).  Returns -1 on
 * invalid sizes. */
int64_t mxq_workspace_bytes(int64_t M, int64_t N, int64_t K, int fmt, int mode);

/* Weight quantization (load time), always to MXFP4 (E2M1).
 * Blog section "Quantization formats": "OCP MXFP4 weights", RTN.
 *   w_bf16 [N, K] bf16 (16-byte aligned) -> codes [N, K/2] bytes, sf tiled
 *   (mxq_sf_bytes(N, K) bytes).  Requires K % 32 == 0. */
int mxq_quantize_weight(const void* w_bf16, int64_t N, int64_t K, void* codes, void* sf, void* stream);

/* Dynamic activation quantization to MXFP4 (fmt E2M1) or to E4M3 with 32-element
 * E8M0 block scales (fmt E4M3).
 * Blog section "Quantization formats": "dynamic MXFP4 activations" (W4A4) and
 * "FP8 E4M3 ... activations" (W4A8).
 *   x_bf16 [M, K] -> codes (mxq_codes_bytes(M, K, fmt) bytes), sf tiled.
 *   Requires K % 32 == 0; x, codes and sf 16-byte aligned. */
int mxq_quantize_act(const void* x_bf16, int64_t M, int64_t K, int fmt, void* codes, void* sf, void* stream);

/* Dequantization to bf16 (the "QDQ" of the blog's intro and "Kernel note"):
 *   out[r, k] = bf16(decode(code[r, k]) * 2^(sf[r, k/32] - 127)),
 * the product formed exactly in binary32 and rounded once to nearest even: exact in bf16
 * except that large scales overflow to Inf and E4M3 values under scale codes 0-2 can fall
 * below bf16's 2^-133 step and round.  Scale code 0xFF and E4M3 codes 0x7F / 0xFF give NaN. */
int mxq_dequantize(const void* codes, const void* sf, int64_t rows, int64_t K, int fmt, void* out_bf16,
                   void* stream);

/* GEMM on already-quantized operands (native tcgen05 block-scaled MMA):
 *   y[M, N] = bf16( sum_k deqA[m, k] * deqW[n, k] + bias[n] ), fp32 accumulation.
 * a_fmt E2M1 -> kind::mxf4 (W4A4); E4M3 -> kind::mxf8f6f4 (W4A8, needs K % 128 == 0
 * and a 32-byte aligned w_codes).  bias_bf16 may be NULL.  Requires N % 8 == 0.
 * Blog section "Quantization formats", "Kernel note". */
int mxq_gemm(const void* a_codes, const void* a_sf, int a_fmt, int64_t M, int64_t K, const void* w_codes,
             const void* w_sf, int64_t N, const void* bias_bf16, void* y_bf16, void* stream);

/* Plain bf16 GEMM: y[M, N] = bf16( sum_k a[m, k] * b[n, k] + bias[n] ) with fp32
 * accumulation, a [M, K] and b [N, K] bf16, K contiguous; bias_bf16 may be NULL.  The
 * "standard BF16 GEMM" of the blog's "Kernel note" that the quantize-dequantize emulation
 * runs on the dequantized operands; also the bf16 branch activation of
 * mxq_linear_lowrank and the GEMM of blocks the policy keeps in bf16.  It is the tcgen05
 * kernel of mxq_gemm with kind::f16 MMAs (bf16 x bf16) in 64-element K stages.  Requires
 * K % 8 == 0 and N % 8 == 0; all pointers 16-byte aligned.  Errors as for mxq_gemm. */
int mxq_gemm_bf16(const void* a_bf16, int64_t M, int64_t K, const void* b_bf16, int64_t N, const void* bias_bf16,
                  void* y_bf16, void* stream);

/* mxq_gemm_bf16 for an output of at most 128 columns, which also writes a's MX
 * quantization in format fmt -- codes [M, K/2] (E2M1) or [M, K] (E4M3) and tiled scales,
 * the bits mxq_quantize_act writes -- from the same read of a: its extra warps quantize
 * each 64-column stage of a as it passes through shared memory.  It serves the SVDQuant
 * branch of mxq_linear_lowrank (blog section "Mixed-Precision selection"), whose u =
 * x . l1t^T and whose quantized x both come from x.  Requires 0 < N <= 128, N % 8 == 0,
 * K % 32 == 0 (a's MX blocks); codes and sf as mxq_quantize_act takes them (16-byte
 * aligned, mxq_codes_bytes / mxq_sf_bytes); other arguments and errors as for
 * mxq_gemm_bf16.  Runs on lone CTAs (128-row tiles, six 64-column stages of a in flight)
 * with MMAs as wide as N (rounded up to 16). */
int mxq_gemm_bf16_quant_a(const void* a_bf16, int64_t M, int64_t K, const void* b_bf16, int64_t N,
                          const void* bias_bf16, void* y_bf16, int fmt, void* codes, void* sf, void* stream);

/* The quantized linear layer: quantize x (fmt act_fmt) into the workspace, then
 *   mode NATIVE: mxq_gemm on the quantized operands;
 *   mode QDQ:    dequantize both operands to bf16 and run the bf16 GEMM of
 *                mxq_gemm_bf16, the quantize-dequantize emulation the blog's W4A8
 *                numbers use.
 * workspace: device buffer of at least mxq_workspace_bytes(M, N, K, act_fmt, mode)
 * bytes, 256-byte aligned; its contents are scratch.  Blog sections "Quantization
 * formats" and "Kernel note". */
int mxq_linear(const void* x_bf16, int64_t M, int64_t K, const void* w_codes, const void* w_sf, int64_t N,
               const void* bias_bf16, int act_fmt, int mode, void* workspace, int64_t ws_bytes, void* y_bf16,
               void* stream);

/* One linear layer's quantized weights. */
typedef struct {
    const void* codes; /* E2M1 [N, K/2]            */
    const void* sf;    /* tiled scale factors      */
    const void* bias;  /* bf16 [N] or NULL         */
    int64_t N, K;
} mxq_wdesc;

/* The eight linears of one DiT block, issued in order on one stream:
 *   0 QKV, 1 attn-out, 2 cross-Q, 3 cross-K, 4 cross-V, 5 cross-out, 6 FFN-up,
 *   7 FFN-down.
 * Linear i reads x_in[i] [M_in[i], w[i].K] and writes y_out[i] [M_in[i], w[i].N];
 * bit i of w4a8_bits set -> that linear runs W4A8 (E4M3 activations), else W4A4.
 * The per-expert, per-block policy of the blog (sections "Mixed-Precision
 * selection", "Practical workflow" step 6) is applied by passing 0xFF or 0x00 (or a
 * per-linear refinement) for each (expert, block).  workspace must hold at least
 * mxq_block_workspace_min_bytes(...) bytes; mxq_block_workspace_bytes(...) lets the
 * quantizers overlap the GEMMs (below). */
int mxq_dit_block_linears(const mxq_wdesc* w, const void* const* x_in, const int64_t* M_in,
                          void* const* y_out, uint32_t w4a8_bits, int mode, void* workspace, int64_t ws_bytes,
                          void* stream);

/* Workspace bytes of mxq_dit_block_linears.  mxq_block_workspace_min_bytes: the least it
 * accepts (one linear's workspace, reused; the linears then run one after another).
 * mxq_block_workspace_bytes: in NATIVE mode, a quantized-activation buffer for every
 * linear; with a workspace of at least this size the call quantizes all eight inputs on
 * a stream of the library's own (created with its events on first use in each CUDA
 * context of a device, so a device reset is followed by new ones)
 * while the GEMMs run on `stream`, each GEMM waiting only for its own input.  When
 * `stream` has passed the call, all of its work is done.  In QDQ mode both sizes are the
 * same. */
int64_t mxq_block_workspace_bytes(const mxq_wdesc* w, const int64_t* M_in, uint32_t w4a8_bits, int mode);
int64_t mxq_block_workspace_min_bytes(const mxq_wdesc* w, const int64_t* M_in, uint32_t w4a8_bits, int mode);

/* The native linear layer (as mxq_linear with mode NATIVE) for callers that cannot
 * allocate device memory where they run a layer -- for example code under a memory
 * manager that owns the whole device pool, or a plugin that is handed only its input and
 * output buffers.  The scratch it needs (the quantized activation) lives in a file-scope
 * device array of mxq_linear_noalloc_max_scratch_bytes() bytes (32 MiB) that every GPU
 * loading the library holds until the process exits; the call allocates and frees
 * nothing.  Inputs and outputs are as for mxq_linear.  Inputs whose scratch would not fit
 * (mxq_workspace_bytes(M, N, K, act_fmt, MXQ_MODE_NATIVE) above the array's size: M*K
 * above about 63 million elements for E2M1, 32 million for E4M3) return
 * MXQ_ERR_WORKSPACE and launch nothing.  The first call on a device looks up the array's
 * device address and caches it; make that first call before any stream capture.  The
 * cache is keyed on the device's CUDA context, so after a device reset (or a new primary
 * context) the next call looks the address up again, and that call too should come
 * before any capture.  All calls on a device share the one array, and it keeps the last
 * call's contents (nothing in it needs to start at zero: every byte the GEMM reads is
 * written by the same call's quantizer), so calls that overlap on the GPU -- on
 * different streams or from different threads without ordering -- race and must be
 * avoided.  The blog has no counterpart of this entry point. */
int mxq_linear_noalloc(const void* x_bf16, int64_t M, int64_t K, const void* w_codes, const void* w_sf, int64_t N,
                       const void* bias_bf16, int act_fmt, void* y_bf16, void* stream);

/* Size in bytes of the static scratch used by mxq_linear_noalloc. */
int64_t mxq_linear_noalloc_max_scratch_bytes(void);

/* GEMM whose epilogue produces the next layer's MX-quantized input: the FFN's first
 * linear followed by its GELU, with the hidden activation never written in bf16.
 *   y = acc + bias (fp32) rounded to bf16 (the linear's output type);
 *   h = GELU(y) = y * Phi(y) (the plain erf form) rounded to bf16 -- exactly, once: the
 *       value of mxq_gelu_bf16 on y;
 *   h quantized as mxq_quantize_act would quantize it: per row, each 32 consecutive
 *   columns form one block (the next layer's K = N), E8M0 scale, E2M1 or E4M3 codes.
 * Blog section "Quantization formats" for the formats; the FFN whose hidden activation
 * this is ("WanFeedForward ... GELU") is the one the FP8 page keeps quantized.  The
 * fusion itself has no counterpart in the pages: it saves the bf16 round trip of h.
 *   Inputs as for mxq_gemm.  out_fmt: MXQ_FMT_E2M1 or MXQ_FMT_E4M3.
 *   out_codes: mxq_codes_bytes(M, N, out_fmt) bytes; out_sf: mxq_sf_bytes(M, N) bytes in
 *   the tiled layout, padding written as 0.  h_bf16: NULL, or [M, N] bf16 to also receive
 *   h (for checking).  Requires N % 32 == 0 and N <= 65536 (N is the next layer's K);
 *   all pointers 16-byte aligned.  Errors as for mxq_gemm. */
int mxq_gemm_gelu_quant(const void* a_codes, const void* a_sf, int a_fmt, int64_t M, int64_t K,
                        const void* w_codes, const void* w_sf, int64_t N, const void* bias_bf16, int out_fmt,
                        void* out_codes, void* out_sf, void* h_bf16, void* stream);

/* GELU of n bf16 values, elementwise, as the quantizing epilogue applies it: y[i] =
 * GELU(x[i]) = x[i]/2 erfc(-x[i]/sqrt 2) rounded once to bf16 (nearest, ties to even), the
 * exact value rounded; +Inf gives +Inf, -Inf and NaN give NaN (0x7FC0).  For 2^-10 <= |x|
 * < 16 the kernel looks the result up in a 3584-entry table it builds in shared memory
 * from the fp64 erfc; elsewhere GELU has a closed form at bf16 precision (x/2 rounded,
 * x, or -0).  x, y: n bf16 values on the device, 2-byte aligned (they may be the same
 * buffer).  n > 0, else MXQ_ERR_INVALID_ARG. */
int mxq_gelu_bf16(const void* x_bf16, int64_t n, void* y_bf16, void* stream);

/* mxq_gemm_gelu_quant with the activation chosen: act MXQ_ACT_GELU is that entry point;
 * MXQ_ACT_NONE quantizes the linear's own output, h = bf16(x . deq(w)^T + bias), so the
 * epilogue of any producer linear can emit its consumer's MX-quantized operand (codes and
 * tiled scales equal those of mxq_quantize_act run on mxq_gemm's bf16 output).  Other act
 * values: MXQ_ERR_INVALID_ARG.  Arguments, layouts and errors otherwise as for
 * mxq_gemm_gelu_quant. */
int mxq_gemm_quant(const void* a_codes, const void* a_sf, int a_fmt, int64_t M, int64_t K, const void* w_codes,
                   const void* w_sf, int64_t N, const void* bias_bf16, int act, int out_fmt, void* out_codes,
                   void* out_sf, void* h_bf16, void* stream);

/* The FFN of a DiT block with its hidden activation kept quantized:
 *   y = (GELU(x . up^T + up.bias) quantized to down_fmt) . down^T + down.bias,
 * i.e. quantize x to up_fmt, mxq_gemm_gelu_quant into the workspace, then mxq_gemm.
 * Each linear runs W4A4 or W4A8 as its activation format says (the blog's per-block
 * policy may pick them independently).  x_bf16 [M, K]; up: N = H, K = K; down: K = H;
 * y_bf16 [M, down.N].  down_fmt E4M3 needs H % 128 == 0.  workspace holds
 * mxq_ffn_workspace_bytes(M, K, H, up_fmt, down_fmt) bytes, 256-byte aligned. */
int mxq_ffn(const void* x_bf16, int64_t M, int64_t K, const mxq_wdesc* up, const mxq_wdesc* down, int up_fmt,
            int down_fmt, void* workspace, int64_t ws_bytes, void* y_bf16, void* stream);

/* Workspace bytes of mxq_ffn (the quantized input and hidden activation), or -1. */
int64_t mxq_ffn_workspace_bytes(int64_t M, int64_t K, int64_t H, int up_fmt, int down_fmt);

/* Static per-tensor FP8 E4M3 activations: the blog's W4A8 as its "Quantization formats"
 * table names it ("FP8 E4M3 static activations"), one scale for the whole tensor fixed
 * offline.  codes[m, k] = E4M3 RNE, saturating, of the exact quotient x[m, k] / scale
 * (decided exactly for every bf16 input and every positive finite binary32 scale: no
 * rounding of the quotient to binary32 comes between); sf is written in the tiled layout
 * with every block's scale 127 (x1) and the padding 0, so the codes feed the
 * kind::mxf8f6f4 GEMM unchanged; the tensor scale goes to the GEMM (mxq_linear_static).
 * scale > 0 and finite (MXQ_ERR_INVALID_ARG otherwise); Inf inputs saturate to +-448, NaN
 * gives an E4M3 NaN code.  Sizes and alignment as for mxq_quantize_act with fmt E4M3. */
int mxq_quantize_act_static(const void* x_bf16, int64_t M, int64_t K, float scale, void* codes, void* sf,
                            void* stream);

/* The W4A8 linear with a static per-tensor activation scale:
 *   y = bf16( act_scale * sum_k q[m, k] * deqW[n, k] + bias[n] ),
 * q the static E4M3 codes of x (mxq_quantize_act_static).  Arguments as for mxq_linear
 * with act_fmt E4M3 and mode NATIVE (K % 128 == 0; workspace of
 * mxq_workspace_bytes(M, N, K, MXQ_FMT_E4M3, MXQ_MODE_NATIVE) bytes). */
int mxq_linear_static(const void* x_bf16, int64_t M, int64_t K, const void* w_codes, const void* w_sf, int64_t N,
                      const void* bias_bf16, float act_scale, void* workspace, int64_t ws_bytes, void* y_bf16,
                      void* stream);

/* Calibration of a static scale: out_f32 (one float, device) = max |x| over n bf16
 * values (n % 8 == 0, x 16-byte aligned); the scale is then max / 448.  An Inf or NaN
 * input makes the result Inf or NaN. */
int mxq_absmax(const void* x_bf16, int64_t n, void* out_f32, void* stream);

/* The "transform_on" policy of the blog's section "Mixed-Precision selection": a block is
 * quantized after a fixed transform that spreads its outliers -- per-channel smoothing
 * (SmoothQuant: activations divided by s, weights multiplied by s) and a block Hadamard
 * rotation along K (activations and weights rotated alike, so x . W^T is unchanged).
 *   t[m, k] = fl32(x[m, k] * mul[k])        (mul NULL: t = x; mul = 1/s for activations)
 *   each `block` (32 or 128) consecutive t's along K <- t . H_block * fl32(1/sqrt(block)),
 *     H the Sylvester Hadamard matrix (entries +-1), as a fast Walsh-Hadamard transform in
 *     binary32 (butterflies (a, b) -> (a + b, a - b), h = 1, 2, 4, ..., then the scaling);
 *   t MX-quantized in fmt as by mxq_quantize_act (scale from the block's binary32 abs-max).
 * Each t thus differs from the exact transform (x . diag(mul) . H_block / sqrt(block)) by at
 * most about (log2(block) + 4) 2^-24 sum_i |x_i mul_i| / sqrt(block), and the codes and
 * scales are the exact transform's wherever it lies farther than that from an MX rounding
 * boundary.  mul: NULL or K floats on the device, 16-byte aligned.  Requires
 * K % block == 0.  Other arguments and errors as for mxq_quantize_act. */
int mxq_quantize_act_transformed(const void* x_bf16, int64_t M, int64_t K, int fmt, const float* mul, int block,
                                 void* codes, void* sf, void* stream);

/* Weight side of the transform: as mxq_quantize_act_transformed with fmt E2M1 and
 * mul = s (the SmoothQuant scales; NULL for rotation only).  A linear computes the same
 * product when its weight was quantized with the same block and its activation with
 * mul = 1/s. */
int mxq_quantize_weight_transformed(const void* w_bf16, int64_t N, int64_t K, const float* mul, int block, void* codes,
                                    void* sf, void* stream);

/* Linear layer on the transformed path: mxq_quantize_act_transformed(x, act_mul, block)
 * into the workspace, then the native GEMM against a weight from
 * mxq_quantize_weight_transformed with the same block.  Arguments as for mxq_linear in
 * NATIVE mode plus act_mul and block. */
int mxq_linear_transformed(const void* x_bf16, int64_t M, int64_t K, const void* w_codes, const void* w_sf, int64_t N,
                           const void* bias_bf16, int act_fmt, const float* act_mul, int block, void* workspace,
                           int64_t ws_bytes, void* y_bf16, void* stream);

/* The SVDQuant low-rank branch of the blog's best mixed result (sections "Results",
 * "Calibration-driven block selection"): the weight is split offline into a bf16 rank-r
 * product l2t . l1t (l1t [r, K], l2t [N, r]) and a residual R quantized to MXFP4
 * (r_codes, r_sf as from mxq_quantize_weight), and the layer computes
 *   y = bf16( deq(xq) . deq(Rq)^T + u . l2t^T + bias ),  u = bf16(x . l1t^T) [M, r],
 * x quantized in act_fmt.  Up to rank 128, u and the quantized x come from one launch that
 * reads x once (mxq_gemm_bf16_quant_a); ranks 192 and 256 quantize x and run the bf16 GEMM
 * apart.  u . l2t^T runs as
 * bf16 tensor-core MMAs (kind::f16) into the same TMEM accumulator as the block-scaled
 * product, in stages of 64 along r ahead of it.  rank: 64, 128, 192 or 256; l1t, l2t
 * 16-byte aligned; workspace of mxq_lowrank_workspace_bytes(...) bytes, 256-byte aligned.
 * Other arguments and errors as for mxq_linear in NATIVE mode. */
int mxq_linear_lowrank(const void* x_bf16, int64_t M, int64_t K, const void* r_codes, const void* r_sf, int64_t N,
                       const void* bias_bf16, int act_fmt, const void* l1t_bf16, const void* l2t_bf16, int64_t rank,
                       void* workspace, int64_t ws_bytes, void* y_bf16, void* stream);

/* Workspace bytes of mxq_linear_lowrank (quantized x, u, and the library GEMM's
 * workspace), or -1 for invalid arguments. */
int64_t mxq_lowrank_workspace_bytes(int64_t M, int64_t N, int64_t K, int fmt, int64_t rank);

/* The per-block policy of the blog's section "Calibration-driven block selection": from a
 * block's whole-output SQNR (dB, against the bf16 block) with plain MXFP4 W4A4 (sqnr_off)
 * and with MXFP4 plus a transform (sqnr_on), in this order of precedence:
 *   max(off, on) <  floor      -> MXQ_POLICY_BF16       (keep the block in bf16)
 *   max(off, on) <  w4a8_sqnr  -> MXQ_POLICY_W4A8       (promote to W4A8)
 *   on - off     >  margin     -> MXQ_POLICY_TRANSFORM_ON (W4A4 with the transform)
 *   otherwise                  -> MXQ_POLICY_PLAIN_MXFP4
 * with (floor, w4a8_sqnr, margin) = (8, 21, 0.5) dB for tier LOW, (10, 23, 0.5) for MID and
 * (12, 25, 0.5) for HIGH, the blog's tier table.  Returns the policy, or -1 for an unknown
 * tier or a NaN SQNR.  Runs on the host. */
enum { MXQ_POLICY_PLAIN_MXFP4 = 0, MXQ_POLICY_TRANSFORM_ON = 1, MXQ_POLICY_W4A8 = 2, MXQ_POLICY_BF16 = 3 };
enum { MXQ_TIER_LOW = 0, MXQ_TIER_MID = 1, MXQ_TIER_HIGH = 2 };
int mxq_select_policy(double sqnr_off, double sqnr_on, int tier);

/* The thresholds of a tier (dB); returns MXQ_OK or MXQ_ERR_INVALID_ARG. */
int mxq_tier_thresholds(int tier, double* floor_db, double* w4a8_db, double* margin_db);

/* ---- calibration and load-time preparation of the policy's transforms --------------
 * None of these runs on the layer's path; they prepare its inputs (blog sections
 * "Mixed-Precision selection", "Calibration-driven block selection", "Results"). */

/* Per-channel abs-max: out_f32[k] = max over rows of |x[r, k]| (x bf16 [rows, K], K % 8 ==
 * 0, 16-byte aligned; out K floats, written from zero, so any earlier content is lost).  A
 * NaN in a channel makes its result NaN.  The calibration statistic of SmoothQuant. */
int mxq_channel_absmax(const void* x_bf16, int64_t rows, int64_t K, float* out_f32, void* stream);

/* SmoothQuant's per-channel scales (the smoothing of the "transform_on" policy):
 *   s[k] = max(amax_x[k], 1e-5)^alpha / max(amax_w[k], 1e-5)^(1 - alpha)
 * in fp32 (powf), amax_x / amax_w the channel abs-maxima of the activation and of the
 * weight (mxq_channel_absmax over x [M, K] and over w [N, K]); alpha in [0, 1].  inv_s
 * (may be NULL) receives 1 / s[k].  The activation is then quantized with mul = inv_s and
 * the weight with mul = s.  All arrays K floats on the device. */
int mxq_smooth_scales(const float* amax_x, const float* amax_w, int64_t K, float alpha, float* s, float* inv_s,
                      void* stream);

/* The SQNR of a block's outputs against its reference (the whole-block SQNR the blog's
 * "Calibration-driven block selection" compares against its tier thresholds), over
 * `count` pairs of bf16 tensors (ref[i], test[i]) of n[i] elements each (n[i] % 8 == 0):
 *   out_f64[0] = sum ref^2,  out_f64[1] = sum (ref - test)^2  (fp64, over all pairs),
 *   out_f64[2] = 10 log10(out_f64[0] / out_f64[1])  dB.
 * ref, test, n: host arrays of device pointers and sizes; out_f64: 3 doubles on the device
 * (8-byte aligned), overwritten.  The sums are accumulated with atomics, so their last bits
 * can vary from run to run. */
int mxq_sqnr(const void* const* ref_bf16, const void* const* test_bf16, const int64_t* n, int count, double* out_f64,
             void* stream);

/* The SVDQuant split of a weight W [N, K] (bf16) from its leading singular triplets,
 * U [N, rank] (fp32, row stride ldu >= rank), S [rank], Vh [rank, K] (fp32, row stride
 * ldvh >= K), computed by any factorization:
 *   l2t[n, j] = bf16(U[n, j] * sqrt(S[j])),   l1t[j, k] = bf16(sqrt(S[j]) * Vh[j, k]),
 *   resid[n, k] = bf16(W[n, k] - sum_j l2t[n, j] * l1t[j, k])   (fp32 accumulation);
 * l2t [N, rank], l1t [rank, K] and resid [N, K] bf16, 16-byte aligned.  The residual is
 * then quantized with mxq_quantize_weight and the factors feed mxq_linear_lowrank. */
int mxq_lowrank_split(const float* U, int64_t ldu, const float* S, const float* Vh, int64_t ldvh, const void* w_bf16,
                      int64_t N, int64_t K, int64_t rank, void* l2t_bf16, void* l1t_bf16, void* resid_bf16,
                      void* stream);

/* Tiled scale factors -> logical row-major [rows, K/32] bytes (for tests). */
int mxq_sf_to_logical(const void* sf_tiled, int64_t rows, int64_t K, void* sf_rowmajor, void* stream);

/* Synchronizes `stream`, then returns (and clears) the device status words: MXQ_OK,
 * or MXQ_ERR_TIMEOUT if a bounded wait of a GEMM or transform-quantizer kernel ran out
 * since the last poll. */
int mxq_poll_status(void* stream);

/* Debug flags (0 = none).  Bit 0: the GEMM's producer skips the first stage's load,
 * so the consumer's bounded wait runs out and the kernel reports MXQ_ERR_TIMEOUT.
 * Bit 1: the transform quantizer's first warp skips its first span's copy, with the
 * same outcome. */
int mxq_set_debug(uint32_t flags);

/* Thread-local description of the last error, and of the last path taken
 * (for example "native mxf4 1cta 128x256 grid 148"). */
const char* mxq_last_error(void);
const char* mxq_last_path(void);

#ifdef __cplusplus
}
#endif

#endif /* MXQ_H */
