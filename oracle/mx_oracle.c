/*
 * mx_oracle.c -- plain CPU reference for the MX block-quantized linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU-baseline
 * leg of the benchmark may load this library.  The CUDA library never links it and
 * shares no code, header, table or constant with it.
 *
 * What it computes (blog "Quark Mixed-Precision Quantization for Wan2.2 Video
 * Generation on AMD Instinct GPUs", section "Quantization formats": W4A4 = OCP MXFP4
 * weights with dynamic MXFP4 activations, W4A8 = MXFP4 weights with FP8 E4M3
 * activations; the MX format itself is the OCP Microscaling spec v1.0, the blog's
 * reference [7]):
 *
 *   * a tensor is cut into blocks of 32 consecutive elements along K;
 *   * every block shares one E8M0 scale X = 2^(floor(log2(amax)) - emax)
 *     (emax = 2 for E2M1, 8 for E4M3), clamped at E8M0's smallest value 2^-127;
 *   * every element x is stored as RTN(x / X) on the element grid, with ties to
 *     even and saturation at the largest finite element;
 *   * the linear layer is Y = deq(Xq) . deq(Wq)^T (+ bias), here in fp64.
 *
 * Readings taken where the pages are silent:
 *   R1 scale = floor rule above (OCP v1.0);  R2 zero / subnormal amax -> scale code 0;
 *   R3 a block holding Inf or NaN -> scale code 0xFF and all element codes 0;
 *   R4 "RTN" = IEEE round-to-nearest-even, saturating to +-max;
 *   R5 a negative value that rounds to zero keeps its sign bit;
 *   R6 E2M1 element 2j sits in the low nibble of byte j, 2j+1 in the high nibble;
 *   R7 tiled scale layout: 512-byte atoms of 128 rows x 4 k-blocks,
 *      offset = (r%32)*16 + ((r/32)%4)*4 + kb%4, atoms ordered row-tile major;
 *   R8 tolerance row norm = infinity norm of the oracle's output row.
 *
 * Everything is computed in double precision.  Every step is written out on its
 * own; nothing is blocked, fused or reordered beyond splitting independent rows
 * across host threads.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define MXO_E2M1 0
#define MXO_E4M3 1

/* Element format parameters.  E2M1: 2 exponent bits (bias 1), 1 mantissa bit,
 * no Inf/NaN, largest magnitude 6.  E4M3 (the "FN" variant of OCP FP8): 4
 * exponent bits (bias 7), 3 mantissa bits, only NaN is S.1111.111, largest
 * magnitude 448 = S.1111.110.  emax is the exponent of the largest normal. */
typedef struct {
    int ebits, mbits, bias, emax;
    double maxval;
} mxo_fmt;

static const mxo_fmt FMTS[2] = {
    {2, 1, 1, 2, 6.0},
    {4, 3, 7, 8, 448.0},
};

static const mxo_fmt *fmt_of(int f) { return (f == MXO_E4M3) ? &FMTS[1] : &FMTS[0]; }

/* ---- bf16 ------------------------------------------------------------------ */

/* bf16 is the upper half of an IEEE binary32; widen and convert exactly. */
double mxo_bf16_to_double(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* ---- element grid ------------------------------------------------------------ */

/* Magnitude bits (exponent field | mantissa field) of a value v that is already
 * exactly on the format's grid and not above its largest finite value. */
static int grid_bits(double v, const mxo_fmt *f)
{
    if (v == 0.0) return 0;
    int e2;
    frexp(v, &e2);              /* v = m * 2^e2, m in [0.5, 1) */
    int e = e2 - 1;             /* v = (1.f) * 2^e             */
    int emin = 1 - f->bias;
    if (e < emin) {             /* subnormal: value = mant * 2^(emin - mbits) */
        return (int)(v / ldexp(1.0, emin - f->mbits));
    }
    int mant = (int)(v / ldexp(1.0, e - f->mbits)) - (1 << f->mbits);
    return ((e + f->bias) << f->mbits) | mant;
}

/* Round y to the element grid: round-to-nearest, ties-to-even (R4), saturating
 * at +-max, sign kept on a zero result (R5).  Returns the element code. */
int mxo_encode_elem(double y, int fmt)
{
    const mxo_fmt *f = fmt_of(fmt);
    int nbits = f->ebits + f->mbits;
    int sign = signbit(y) ? 1 : 0;
    double a = fabs(y);
    double v;
    if (a >= f->maxval) {
        v = f->maxval;
    } else if (a == 0.0) {
        v = 0.0;
    } else {
        int e2;
        frexp(a, &e2);
        int e = e2 - 1;
        int emin = 1 - f->bias;
        if (e < emin) e = emin;                 /* subnormal spacing below the min normal */
        double q = ldexp(1.0, e - f->mbits);    /* grid spacing around a                  */
        double n = nearbyint(a / q);            /* default rounding mode: ties to even    */
        v = n * q;
        if (v > f->maxval) v = f->maxval;       /* rounding up past max saturates         */
    }
    return (sign << nbits) | grid_bits(v, f);
}

/* Value of an element code; E4M3's S.1111.111 is NaN. */
double mxo_decode_elem(int code, int fmt)
{
    const mxo_fmt *f = fmt_of(fmt);
    int nbits = f->ebits + f->mbits;
    int sign = (code >> nbits) & 1;
    int ef = (code >> f->mbits) & ((1 << f->ebits) - 1);
    int mf = code & ((1 << f->mbits) - 1);
    if (fmt == MXO_E4M3 && ef == 15 && mf == 7) return NAN;
    double mag;
    if (ef == 0)
        mag = ldexp((double)mf, 1 - f->bias - f->mbits);
    else
        mag = ldexp((double)((1 << f->mbits) + mf), ef - f->bias - f->mbits);
    return sign ? -mag : mag;
}

/* ---- shared scale ------------------------------------------------------------ */

/* E8M0 scale code of a block with absolute maximum amax (R1, R2, R3). */
int mxo_scale_code(double amax, int nonfinite, int fmt)
{
    const mxo_fmt *f = fmt_of(fmt);
    if (nonfinite) return 255;
    if (amax == 0.0) return 0;
    int e2;
    frexp(amax, &e2);                    /* floor(log2(amax)) = e2 - 1 */
    int sc = (e2 - 1) + 127 - f->emax;
    return sc < 0 ? 0 : sc;
}

/* Value of an E8M0 scale code. */
double mxo_scale_value(int sc)
{
    if (sc == 255) return NAN;
    return ldexp(1.0, sc - 127);
}

/* ---- block and tensor quantization ------------------------------------------- */

/* Quantize one block of 32 values into 32 element codes and a scale code. */
static int quantize_values(const double *v, int fmt, int codes[32])
{
    double amax = 0.0;
    int nonfinite = 0;
    for (int i = 0; i < 32; ++i) {
        if (isnan(v[i]) || isinf(v[i])) nonfinite = 1;
        else if (fabs(v[i]) > amax) amax = fabs(v[i]);
    }
    int sc = mxo_scale_code(amax, nonfinite, fmt);
    for (int i = 0; i < 32; ++i) {
        if (sc == 255) codes[i] = 0;
        else codes[i] = mxo_encode_elem(v[i] / mxo_scale_value(sc), fmt);
    }
    return sc;
}

/* One block of 32 bf16 values. */
static int quantize_block(const uint16_t *x, int fmt, int codes[32])
{
    double v[32];
    for (int i = 0; i < 32; ++i) v[i] = mxo_bf16_to_double(x[i]);
    return quantize_values(v, fmt, codes);
}

/* Place the 32 codes of block kb into a row of element codes (R6). */
static void store_block_codes(uint8_t *out, int64_t kb, const int codes[32], int fmt)
{
    for (int i = 0; i < 32; ++i) {
        int64_t k = kb * 32 + i;
        if (fmt == MXO_E4M3) {
            out[k] = (uint8_t)codes[i];
        } else if ((k & 1) == 0) {
            out[k / 2] = (uint8_t)(codes[i] & 0xF);
        } else {
            out[k / 2] |= (uint8_t)((codes[i] & 0xF) << 4);
        }
    }
}

/* Bytes of element codes per row: K/2 (E2M1, two per byte, R6) or K (E4M3). */
int64_t mxo_codes_row_bytes(int64_t K, int fmt) { return fmt == MXO_E4M3 ? K : K / 2; }

typedef struct {
    const uint16_t *x;
    int64_t r0, r1, K;
    int fmt;
    uint8_t *codes;
    uint8_t *sf;
} quant_job;

static void *quant_rows(void *arg)
{
    quant_job *j = (quant_job *)arg;
    int64_t KB = j->K / 32;
    int64_t rb = mxo_codes_row_bytes(j->K, j->fmt);
    int codes[32];
    for (int64_t r = j->r0; r < j->r1; ++r) {
        for (int64_t kb = 0; kb < KB; ++kb) {
            int sc = quantize_block(j->x + r * j->K + kb * 32, j->fmt, codes);
            j->sf[r * KB + kb] = (uint8_t)sc;
            store_block_codes(j->codes + r * rb, kb, codes, j->fmt);
        }
    }
    return NULL;
}

/* Split rows [0, rows) into nthreads contiguous ranges and run fn on each. */
static void run_rows(void *(*fn)(void *), void *jobs, size_t job_size, int64_t rows, int nthreads,
                     void (*set_range)(void *, int64_t, int64_t))
{
    if (nthreads < 1) nthreads = 1;
    if (nthreads > rows) nthreads = (int)(rows > 0 ? rows : 1);
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    int64_t per = (rows + nthreads - 1) / nthreads;
    for (int t = 0; t < nthreads; ++t) {
        void *job = (char *)jobs + (size_t)t * job_size;
        int64_t r0 = t * per, r1 = r0 + per;
        if (r1 > rows) r1 = rows;
        if (r0 > rows) r0 = rows;
        set_range(job, r0, r1);
        if (nthreads == 1) fn(job);
        else pthread_create(&th[t], NULL, fn, job);
    }
    if (nthreads > 1)
        for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
    free(th);
}

static void set_quant_range(void *j, int64_t r0, int64_t r1)
{
    ((quant_job *)j)->r0 = r0;
    ((quant_job *)j)->r1 = r1;
}

/* x: bf16 bits [rows, K] row-major.  codes: [rows, K/2] (E2M1) or [rows, K] (E4M3).
 * sf: logical scale codes [rows, K/32] row-major.  K must be a multiple of 32. */
int mxo_quantize(const uint16_t *x, int64_t rows, int64_t K, int fmt,
                 uint8_t *codes, uint8_t *sf, int nthreads)
{
    if (K % 32 != 0 || rows < 0) return -1;
    if (nthreads < 1) nthreads = 1;
    quant_job *jobs = (quant_job *)calloc((size_t)nthreads, sizeof(quant_job));
    for (int t = 0; t < nthreads; ++t) {
        jobs[t].x = x; jobs[t].K = K; jobs[t].fmt = fmt; jobs[t].codes = codes; jobs[t].sf = sf;
    }
    run_rows(quant_rows, jobs, sizeof(quant_job), rows, nthreads, set_quant_range);
    free(jobs);
    return 0;
}

/* Element code k of a row of packed codes. */
static int code_at(const uint8_t *row, int64_t k, int fmt)
{
    if (fmt == MXO_E4M3) return row[k];
    uint8_t b = row[k / 2];
    return (k & 1) ? (b >> 4) : (b & 0xF);
}

/* Dequantize: out[r, k] = decode(code[r, k]) * 2^(sf[r, k/32] - 127). */
int mxo_dequantize(const uint8_t *codes, const uint8_t *sf, int64_t rows, int64_t K, int fmt,
                   double *out)
{
    if (K % 32 != 0) return -1;
    int64_t KB = K / 32, rb = mxo_codes_row_bytes(K, fmt);
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t k = 0; k < K; ++k)
            out[r * K + k] = mxo_decode_elem(code_at(codes + r * rb, k, fmt), fmt) *
                             mxo_scale_value(sf[r * KB + k / 32]);
    return 0;
}

/* ---- tiled scale layout (R7) ------------------------------------------------- */

/* Bytes of the tiled scale buffer: rows padded to 128, k-blocks padded to 4. */
int64_t mxo_sf_tiled_bytes(int64_t rows, int64_t K)
{
    int64_t KB = K / 32;
    return ((rows + 127) / 128) * 128 * ((KB + 3) / 4) * 4;
}

/* Byte offset of logical scale (r, kb) in the tiled layout. */
int64_t mxo_sf_tiled_offset(int64_t r, int64_t kb, int64_t K)
{
    int64_t KB = K / 32;
    int64_t atoms_k = (KB + 3) / 4;
    int64_t atom = (r / 128) * atoms_k + kb / 4;
    return atom * 512 + (r % 32) * 16 + ((r / 32) % 4) * 4 + (kb % 4);
}

/* Scatter a logical [rows, K/32] scale array into the tiled layout; padding is 0. */
int mxo_sf_to_tiled(const uint8_t *sf, int64_t rows, int64_t K, uint8_t *tiled)
{
    int64_t KB = K / 32;
    memset(tiled, 0, (size_t)mxo_sf_tiled_bytes(rows, K));
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t kb = 0; kb < KB; ++kb)
            tiled[mxo_sf_tiled_offset(r, kb, K)] = sf[r * KB + kb];
    return 0;
}

/* ---- the linear layer ---------------------------------------------------------- */

typedef struct {
    const uint8_t *a_codes, *a_sf;
    int a_fmt;
    const int64_t *rows;
    int64_t i0, i1, K, N;
    const double *wdeq;   /* [N, K] dequantized weights */
    const uint16_t *bias; /* [N] bf16 or NULL */
    double *y;            /* [nrows, N] */
} lin_job;

static void *lin_rows(void *arg)
{
    lin_job *j = (lin_job *)arg;
    int64_t K = j->K, KB = K / 32, rb = mxo_codes_row_bytes(K, j->a_fmt);
    double *a = (double *)malloc(sizeof(double) * (size_t)K);
    for (int64_t i = j->i0; i < j->i1; ++i) {
        int64_t m = j->rows[i];
        for (int64_t k = 0; k < K; ++k)
            a[k] = mxo_decode_elem(code_at(j->a_codes + m * rb, k, j->a_fmt), j->a_fmt) *
                   mxo_scale_value(j->a_sf[m * KB + k / 32]);
        for (int64_t n = 0; n < j->N; ++n) {
            const double *w = j->wdeq + n * K;
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) acc += a[k] * w[k];
            if (j->bias) acc += mxo_bf16_to_double(j->bias[n]);
            j->y[i * j->N + n] = acc;
        }
    }
    free(a);
    return NULL;
}

static void set_lin_range(void *j, int64_t r0, int64_t r1)
{
    ((lin_job *)j)->i0 = r0;
    ((lin_job *)j)->i1 = r1;
}

/* y[i, n] = sum_k deqA[rows[i], k] * deqW[n, k] + bias[n], in fp64.
 * A: activation codes in fmt a_fmt with logical scales [M, K/32]; W: E2M1 codes
 * [N, K/2] with logical scales [N, K/32]; rows: the nrows output rows wanted. */
int mxo_linear_rows(const uint8_t *a_codes, const uint8_t *a_sf, int a_fmt,
                    const int64_t *rows, int64_t nrows, int64_t K,
                    const uint8_t *w_codes, const uint8_t *w_sf, int64_t N,
                    const uint16_t *bias, double *y, int nthreads)
{
    if (K % 32 != 0) return -1;
    double *wdeq = (double *)malloc(sizeof(double) * (size_t)(N * K));
    if (!wdeq) return -2;
    mxo_dequantize(w_codes, w_sf, N, K, MXO_E2M1, wdeq);
    if (nthreads < 1) nthreads = 1;
    lin_job *jobs = (lin_job *)calloc((size_t)nthreads, sizeof(lin_job));
    for (int t = 0; t < nthreads; ++t) {
        lin_job *j = &jobs[t];
        j->a_codes = a_codes; j->a_sf = a_sf; j->a_fmt = a_fmt; j->rows = rows;
        j->K = K; j->N = N; j->wdeq = wdeq; j->bias = bias; j->y = y;
    }
    run_rows(lin_rows, jobs, sizeof(lin_job), nrows, nthreads, set_lin_range);
    free(jobs);
    free(wdeq);
    return 0;
}

/* ---- the FFN hidden activation: bf16 rounding and GELU --------------------------- */

/* Round v to the nearest bf16 value, ties to even, returned as bf16 bits.  bf16 is
 * binary32 with its fraction cut to 7 bits: 8 significant bits, exponent bias 127,
 * subnormals below 2^-126.  As for any IEEE binary format, a result whose rounded
 * magnitude (with an unbounded exponent) exceeds the largest finite value is Inf.
 * NaN stays NaN (the quiet pattern 0x7FC0 with v's sign). */
uint16_t mxo_double_to_bf16(double v)
{
    uint16_t sign = signbit(v) ? 0x8000u : 0u;
    if (isnan(v)) return (uint16_t)(sign | 0x7FC0u);
    double a = fabs(v);
    if (isinf(a)) return (uint16_t)(sign | 0x7F80u);
    if (a == 0.0) return sign;
    int e2;
    frexp(a, &e2);
    int e = e2 - 1;                          /* a = 1.f * 2^e                    */
    if (e < -126) e = -126;                  /* subnormal spacing below 2^-126   */
    double q = ldexp(1.0, e - 7);            /* spacing of the bf16 grid near a  */
    double r = nearbyint(a / q) * q;         /* default rounding: ties to even   */
    if (r >= ldexp(1.0, 128)) return (uint16_t)(sign | 0x7F80u);
    float f = (float)r;                      /* exact: every bf16 value is a binary32 value */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(sign | (u >> 16));
}

/* GELU in its plain form, x * Phi(x) = x/2 * (1 + erf(x / sqrt 2)), in fp64.  The
 * same function is evaluated as x/2 * erfc(-x / sqrt 2): 1 + erf(t) cancels to
 * nothing for t below about -6, where erfc keeps full relative accuracy. */
double mxo_gelu(double x) { return 0.5 * x * erfc(-x / sqrt(2.0)); }

/* n elements: y (fp64) -> bf16 bits, the rounding of a linear layer's output. */
void mxo_round_bf16(const double *y, int64_t n, uint16_t *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = mxo_double_to_bf16(y[i]);
}

/* n elements: h = bf16(GELU(y)) for bf16 inputs y, the activation between the FFN's
 * two linears as a bf16 network computes it (GELU of the bf16 linear output,
 * rounded back to bf16). */
void mxo_gelu_bf16(const uint16_t *y, int64_t n, uint16_t *h)
{
    for (int64_t i = 0; i < n; ++i) h[i] = mxo_double_to_bf16(mxo_gelu(mxo_bf16_to_double(y[i])));
}

/* ---- static per-tensor E4M3 activations ------------------------------------------- */

/* The W4A8 of the blog's "Quantization formats" table names "FP8 E4M3 static
 * activations": one scale s for the whole tensor, fixed offline (calibration: s = amax /
 * 448, the largest E4M3 magnitude).  Each element becomes RNE_sat(x / s) on the E4M3
 * grid, x / s the exact quotient.  The block scales the MMA reads are all 127 (x1) and
 * the linear layer multiplies its sums by s.
 *
 * The quotient is taken as one IEEE double division of the exact operands (x is bf16, s
 * binary32), so it carries a relative rounding error below 2^-53.  That never moves it
 * across an E4M3 decision boundary: a boundary m (a midpoint between grid values, at most
 * 5 significant bits) equals x / s only if x = s * m exactly, and otherwise x - s * m is a
 * nonzero multiple of the coarser of x's and s*m's last-bit weights, which puts x / s more
 * than 2^-30 |m| away from m.  So the double lands on the same side of every boundary as
 * the exact quotient, and on a boundary only when x / s is one. */
int mxo_quantize_static_e4m3(const uint16_t *x, int64_t n, float scale, uint8_t *codes)
{
    for (int64_t i = 0; i < n; ++i) {
        double q = mxo_bf16_to_double(x[i]) / (double)scale;
        if (isnan(q)) codes[i] = (uint8_t)((signbit(q) ? 0x80 : 0x00) | 0x7F);
        else codes[i] = (uint8_t)mxo_encode_elem(q, MXO_E4M3);
    }
    return 0;
}

/* y[i, n] = alpha * sum_k deqA[rows[i], k] * deqW[n, k] + bias[n] in fp64: the linear layer
 * whose activation carries a per-tensor scale alpha on top of its block scales. */
int mxo_linear_rows_scaled(const uint8_t *a_codes, const uint8_t *a_sf, int a_fmt,
                           const int64_t *rows, int64_t nrows, int64_t K,
                           const uint8_t *w_codes, const uint8_t *w_sf, int64_t N,
                           const uint16_t *bias, double alpha, double *y, int nthreads)
{
    int rc = mxo_linear_rows(a_codes, a_sf, a_fmt, rows, nrows, K, w_codes, w_sf, N, NULL, y, nthreads);
    if (rc != 0) return rc;
    for (int64_t i = 0; i < nrows; ++i)
        for (int64_t j = 0; j < N; ++j)
            y[i * N + j] = alpha * y[i * N + j] + (bias ? mxo_bf16_to_double(bias[j]) : 0.0);
    return 0;
}

/* ---- transform_on: per-channel smoothing and block Hadamard rotation --------------- */

/* The third policy value of the blog's "Mixed-Precision selection": the activation is
 * transformed before it is quantized -- divided per channel by SmoothQuant scales (the
 * weights carry the scales instead) and rotated by a fixed block Hadamard matrix (the
 * weights rotated the same way offline), so x . W^T is unchanged while outliers spread
 * over a block.  The definition, taken here in fp64:
 *   a_k = x_k * mul_k                 (mul = 1/s for activations, s for weights; NULL: a = x)
 *   each block of B consecutive a's:  t = a . H_B / sqrt(B),  H_B the Sylvester Hadamard
 *                                      matrix, H_B[j][k] = (-1)^popcount(j & k)
 *   t MX-quantized exactly as mxo_quantize quantizes a row.
 * a_k is exact in fp64 (8 + 24 significant bits), each t is a sum of B exact terms, so its
 * fp64 error is below B * 2^-53 * L1 / sqrt(B), L1 = sum_k |a_k| over the rotation block.
 *
 * Evaluating t in binary32 (as a GPU does) moves it by more than that.  For any evaluation
 * that rounds each product a_k once, each of the log2(B) butterfly sums and differences
 * once (in any stage order) and the scaling by fl32(1/sqrt B) and by the power-of-two block
 * scale at most twice, the standard error bounds of summation (N. J. Higham, "Accuracy and
 * Stability of Numerical Algorithms", 2nd ed., section 4.2; products and quotients add their
 * own relative u and, in the subnormal range, an absolute 2^-150) give
 *   |t_binary32 - t| <= delta = 1.01 * ((log2(B) + 4) * u * L1 + (B + 2) * 2^-150) / sqrt(B),
 * u = 2^-24.  So this oracle also reports, per MX block, whether the scale could differ
 * (the codes of max |t| - delta and max |t| + delta differ, or L1 >= 2^127 so that a
 * binary32 evaluation could overflow), and per element the two codes of t -+ delta under
 * the definition's scale: an element whose two codes differ lies within delta of a
 * decision boundary of the element grid (or of zero), and any binary32 evaluation may
 * take either code there.  The codes reported as `codes` are always the definition's. */
typedef struct {
    const uint16_t *x;
    int64_t r0, r1, K;
    const float *mul;
    int B, fmt;
    uint8_t *codes, *sf, *code_lo, *code_hi, *blk_amb;
    double *t_out;
} transform_job;

static void *transform_rows(void *arg)
{
    const transform_job *jb = (const transform_job *)arg;
    const uint16_t *x = jb->x;
    const int64_t K = jb->K;
    const float *mul = jb->mul;
    const int B = jb->B, fmt = jb->fmt;
    uint8_t *codes = jb->codes, *sf = jb->sf, *code_lo = jb->code_lo, *code_hi = jb->code_hi;
    uint8_t *blk_amb = jb->blk_amb;
    double *t_out = jb->t_out;
    int d = 0;
    while ((1 << d) < B) ++d;
    const double inv_sqrt_b = 1.0 / sqrt((double)B);
    const double u = ldexp(1.0, -24);
    const int64_t KB = K / 32, rb = mxo_codes_row_bytes(K, fmt);
    double *a = (double *)malloc(sizeof(double) * (size_t)K);
    double *t = (double *)malloc(sizeof(double) * (size_t)K);
    double *delta = (double *)malloc(sizeof(double) * (size_t)K);
    double *l1 = (double *)malloc(sizeof(double) * (size_t)K);
    int cd[32];
    for (int64_t r = jb->r0; r < jb->r1; ++r) {
        for (int64_t k = 0; k < K; ++k) {
            double xk = mxo_bf16_to_double(x[r * K + k]);
            a[k] = mul ? xk * (double)mul[k] : xk;
        }
        for (int64_t b0 = 0; b0 < K; b0 += B) {
            double s1 = 0.0;
            for (int k = 0; k < B; ++k) s1 += fabs(a[b0 + k]);
            for (int j = 0; j < B; ++j) {
                double acc = 0.0;
                for (int k = 0; k < B; ++k) {
                    double h = (__builtin_popcount((unsigned)(j & k)) & 1) ? -1.0 : 1.0;
                    acc += h * a[b0 + k];
                }
                t[b0 + j] = acc * inv_sqrt_b;
                l1[b0 + j] = s1;
                delta[b0 + j] = 1.01 * ((d + 4) * u * s1 + (B + 2) * ldexp(1.0, -150)) * inv_sqrt_b;
            }
        }
        if (t_out) memcpy(t_out + r * K, t, sizeof(double) * (size_t)K);
        for (int64_t kb = 0; kb < KB; ++kb) {
            const double *tb = t + kb * 32;
            int sc = quantize_values(tb, fmt, cd);
            sf[r * KB + kb] = (uint8_t)sc;
            store_block_codes(codes + r * rb, kb, cd, fmt);
            int amb = 0;
            if (sc != 255) {
                double lo = 0.0, hi = 0.0;
                for (int i = 0; i < 32; ++i) {
                    double dl = fabs(tb[i]) - delta[kb * 32 + i], dh = fabs(tb[i]) + delta[kb * 32 + i];
                    if (dl > lo) lo = dl;
                    if (dh > hi) hi = dh;
                    if (l1[kb * 32 + i] >= ldexp(1.0, 127)) amb = 2;
                }
                if (!amb && mxo_scale_code(lo, 0, fmt) != mxo_scale_code(hi, 0, fmt)) amb = 1;
            }
            if (blk_amb) blk_amb[r * KB + kb] = (uint8_t)amb;
            for (int i = 0; i < 32; ++i) {
                int c_lo = cd[i], c_hi = cd[i];
                if (sc != 255) {
                    double X = mxo_scale_value(sc), dv = delta[kb * 32 + i];
                    c_lo = mxo_encode_elem((tb[i] - dv) / X, fmt);
                    c_hi = mxo_encode_elem((tb[i] + dv) / X, fmt);
                }
                if (code_lo) code_lo[r * K + kb * 32 + i] = (uint8_t)c_lo;
                if (code_hi) code_hi[r * K + kb * 32 + i] = (uint8_t)c_hi;
            }
        }
    }
    free(a);
    free(t);
    free(delta);
    free(l1);
    return NULL;
}

static void set_transform_range(void *j, int64_t r0, int64_t r1)
{
    ((transform_job *)j)->r0 = r0;
    ((transform_job *)j)->r1 = r1;
}

/* x: bf16 bits [rows, K]; mul: K floats or NULL; B: 32 or a larger power of two dividing K.
 * Outputs: codes (packed as mxo_quantize packs them) and logical scales [rows, K/32] of the
 * definition; optionally t [rows, K] (fp64), the two candidate codes per element
 * code_lo / code_hi [rows, K] (one byte each), and blk_amb [rows, K/32] (0: the scale is
 * certain; 1: a binary32 evaluation could take a neighbouring scale; 2: it could overflow). */
int mxo_quantize_transformed(const uint16_t *x, int64_t rows, int64_t K, const float *mul, int B, int fmt,
                             uint8_t *codes, uint8_t *sf, double *t_out, uint8_t *code_lo, uint8_t *code_hi,
                             uint8_t *blk_amb, int nthreads)
{
    if (K % 32 != 0 || B < 32 || (B & (B - 1)) != 0 || K % B != 0 || rows < 0) return -1;
    if (nthreads < 1) nthreads = 1;
    transform_job *jobs = (transform_job *)calloc((size_t)nthreads, sizeof(transform_job));
    for (int t = 0; t < nthreads; ++t) {
        transform_job *j = &jobs[t];
        j->x = x; j->K = K; j->mul = mul; j->B = B; j->fmt = fmt; j->codes = codes; j->sf = sf;
        j->code_lo = code_lo; j->code_hi = code_hi; j->blk_amb = blk_amb; j->t_out = t_out;
    }
    run_rows(transform_rows, jobs, sizeof(transform_job), rows, nthreads, set_transform_range);
    free(jobs);
    return 0;
}

/* ---- SVDQuant low-rank branch ---------------------------------------------------- */

/* The blog's best mixed configuration adds SVDQuant ("Results", "Calibration-driven block
 * selection"): a weight W [N, K] is split offline into a rank-r product B . A kept in 16-bit
 * (A = l1t [r, K], B = l2t [N, r], bf16) and a residual R = W - B . A quantized to MXFP4.
 * The linear layer is
 *   y = deq(xq) . deq(Rq)^T + u . B^T + bias,   u = bf16(x . A^T)  [rows, r],
 * the branch's activation u being a 16-bit tensor like any linear output (rounded once to
 * bf16), everything else in fp64.  x_bits are the layer's bf16 inputs [M, K]; the rows
 * listed are the output rows wanted. */
int mxo_linear_lowrank_rows(const uint8_t *a_codes, const uint8_t *a_sf, int a_fmt, const int64_t *rows,
                            int64_t nrows, int64_t K, const uint8_t *r_codes, const uint8_t *r_sf, int64_t N,
                            const uint16_t *x_bits, const uint16_t *l1t, const uint16_t *l2t, int64_t r,
                            const uint16_t *bias, double *y, int nthreads)
{
    int rc = mxo_linear_rows(a_codes, a_sf, a_fmt, rows, nrows, K, r_codes, r_sf, N, NULL, y, nthreads);
    if (rc != 0) return rc;
    double *u = (double *)malloc(sizeof(double) * (size_t)r);
    for (int64_t i = 0; i < nrows; ++i) {
        const int64_t m = rows[i];
        for (int64_t j = 0; j < r; ++j) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k)
                acc += mxo_bf16_to_double(x_bits[m * K + k]) * mxo_bf16_to_double(l1t[j * K + k]);
            u[j] = mxo_bf16_to_double(mxo_double_to_bf16(acc));
        }
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int64_t j = 0; j < r; ++j) acc += u[j] * mxo_bf16_to_double(l2t[n * r + j]);
            y[i * N + n] += acc + (bias ? mxo_bf16_to_double(bias[n]) : 0.0);
        }
    }
    free(u);
    return 0;
}
