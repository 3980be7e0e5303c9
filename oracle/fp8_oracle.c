/*
 * Plain CPU oracle for the blockwise-E4M3 FP8 linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or
 * calls this file: only tests/, the package's smoke check and the
 * benchmark's CPU-baseline leg may.  It shares no code, header, table or
 * constant with the CUDA library.
 *
 * What it follows
 * ---------------
 * The Puro-2B-Base model card (friendli.ai), training-setup paragraph below
 * the Phase 1 / Phase 2 setting table, states that the main Transformer
 * linear-layer GEMMs run in blockwise E4M3 FP8 while numerically sensitive
 * operations, master weights and optimizer state stay in BF16 or FP32; the
 * alphaneural.io model card repeats it.  The tech report's related-work
 * section (part 7/7, section 5) places this in the FP8 mixed-precision line
 * of DeepSeek-V3.  The pages give no block size, scale format or rounding
 * rule, so this oracle fixes the plainest definition consistent with them:
 *
 *   - E4M3 is the OCP FP8 E4M3FN format: bias 7, no infinities, largest
 *     finite magnitude 448, codes 0x7F/0xFF are NaN.
 *   - Activations are quantized in groups of 128 consecutive elements along
 *     the contraction dimension; weights in 128x128 blocks.
 *   - The scale is the FP32 number s = amax / 448 (IEEE single division),
 *     stored as the dequantization multiplier.
 *   - A code is E4M3(x / s): single-precision division first, then
 *     round-to-nearest-even onto the E4M3 grid, saturating at +-448 and
 *     keeping the sign (a negative value that rounds to zero gives 0x80).
 *     A group whose amax is zero stores s = 0 and all codes 0x00.
 *   - The GEMM dequantizes (code value times scale) and accumulates in FP64.
 *     For each output element and each 128-wide contraction slab t it forms
 *     the slab sum P_t of decoded-code products, which is exact in FP64
 *     (each decoded code times 2^9 is an integer below 2^18, so a slab sum
 *     of 128 products stays below 2^53 in units of 2^-18), and adds
 *     (s_a,t * s_b,t) * P_t.  It also returns the bound
 *     S = sum_t |s_a,t s_b,t| * sum_k |a_k||b_k| that the acceptance test
 *     |gpu - oracle| <= 2e-3 * S + 1e-6 uses.
 *
 * Layouts (all row-major, element [i][j] at i*ld + j):
 *   activation x      bf16 bits [rows, cols]
 *   row-wise codes    u8  [rows, cols]       scales f32 [cols/128, rows]
 *   col-wise codes    u8  [cols, rows]       scales f32 [rows/128, cols]
 *                     (groups of 128 consecutive rows, output transposed)
 *   weight w          bf16 bits [n, k]
 *   weight codes      u8  [n, k]             scales f32 [n/128, k/128]
 *
 * Every function that fills arrays returns 0 on success and a negative
 * number on a bad argument or a non-finite input (non-finite inputs are
 * outside the definition); the scalar codec and rounding functions return
 * their result.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define GROUP 128

/* ---------------------------------------------------------------- codec */

/* Widen a bfloat16 bit pattern to float: bf16 is the top half of a float. */
float orc_bf16_to_float(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Value of an E4M3FN code: sign bit, 4 exponent bits (bias 7), 3 mantissa
 * bits.  Exponent field 0 encodes subnormals m * 2^-9; S.1111.111 is NaN. */
double orc_e4m3_decode(uint8_t code)
{
    int sign = code >> 7;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    double mag;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        mag = ldexp((double)m, -9);
    else
        mag = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -mag : mag;
}

/* Round a finite float onto the E4M3 grid: nearest value, ties to the even
 * mantissa, magnitudes at or above 448 saturate to 448, sign kept. */
uint8_t orc_e4m3_encode(float v)
{
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs((double)v);
    double quantum, t, fl, frac, n, r, f;
    int e;

    if (a >= 448.0)
        return sign | 0x7E;

    /* Grid spacing at a: 2^-9 in the subnormal range [0, 2^-6); otherwise
     * 2^(E-3) where 2^E <= a < 2^(E+1). */
    if (a < ldexp(1.0, -6)) {
        quantum = ldexp(1.0, -9);
    } else {
        frexp(a, &e);                 /* a in [2^(e-1), 2^e) */
        quantum = ldexp(1.0, (e - 1) - 3);
    }

    t = a / quantum;                  /* exact: quantum is a power of two */
    fl = floor(t);
    frac = t - fl;
    if (frac > 0.5)
        n = fl + 1.0;
    else if (frac < 0.5)
        n = fl;
    else
        n = (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
    r = n * quantum;                  /* rounded magnitude, exact */

    if (r == 0.0)
        return sign;
    if (r < ldexp(1.0, -6))           /* subnormal: r = m * 2^-9, m in 1..7 */
        return sign | (uint8_t)(r / ldexp(1.0, -9));
    f = frexp(r, &e);                 /* r = (2f) * 2^(e-1), 2f in [1, 2) */
    {
        int E = e - 1;                /* -6 .. 8 */
        int m = (int)((2.0 * f - 1.0) * 8.0);
        return sign | (uint8_t)(((E + 7) << 3) | m);
    }
}

/* Element-wise forms of the two functions above, for arrays. */
void orc_e4m3_encode_array(const float *v, int64_t n, uint8_t *codes)
{
    for (int64_t i = 0; i < n; ++i)
        codes[i] = orc_e4m3_encode(v[i]);
}

void orc_e4m3_decode_array(const uint8_t *codes, int64_t n, double *v)
{
    for (int64_t i = 0; i < n; ++i)
        v[i] = orc_e4m3_decode(codes[i]);
}

/* ------------------------------------------------------------ quantizers */

/* Scale of one group: s = amax / 448 in single precision. */
static float group_scale(float amax)
{
    volatile float s = amax / 448.0f;
    return s;
}

/* Code of one element of a group with scale s. */
static uint8_t element_code(float x, float s)
{
    if (s == 0.0f)
        return 0x00;
    volatile float ratio = x / s;
    return orc_e4m3_encode(ratio);
}

/* 1x128 groups along each row (the contraction dimension of fprop/dgrad). */
int orc_quant_act_rowwise(const uint16_t *x, int64_t rows, int64_t cols,
                          uint8_t *q, float *s)
{
    if (rows < 0 || cols < 0 || cols % GROUP != 0)
        return -1;
    int64_t groups = cols / GROUP;
    int bad = 0;
#pragma omp parallel for schedule(static) reduction(| : bad)
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t g = 0; g < groups; ++g) {
            const uint16_t *xg = x + r * cols + g * GROUP;
            float amax = 0.0f;
            for (int j = 0; j < GROUP; ++j) {
                float v = orc_bf16_to_float(xg[j]);
                if (!isfinite(v))
                    bad = 1;
                if (fabsf(v) > amax)
                    amax = fabsf(v);
            }
            float sc = group_scale(amax);
            s[g * rows + r] = sc;
            for (int j = 0; j < GROUP; ++j)
                q[r * cols + g * GROUP + j] =
                    element_code(orc_bf16_to_float(xg[j]), sc);
        }
    }
    return bad ? -2 : 0;
}

/* Groups of 128 consecutive rows in each column (the token dimension, which
 * wgrad contracts over); codes are written transposed, [cols, rows]. */
int orc_quant_act_colwise(const uint16_t *x, int64_t rows, int64_t cols,
                          uint8_t *qT, float *s)
{
    if (rows < 0 || cols < 0 || rows % GROUP != 0)
        return -1;
    int64_t rgroups = rows / GROUP;
    int bad = 0;
#pragma omp parallel for schedule(static) reduction(| : bad)
    for (int64_t c = 0; c < cols; ++c) {
        for (int64_t rb = 0; rb < rgroups; ++rb) {
            float amax = 0.0f;
            for (int j = 0; j < GROUP; ++j) {
                float v = orc_bf16_to_float(x[(rb * GROUP + j) * cols + c]);
                if (!isfinite(v))
                    bad = 1;
                if (fabsf(v) > amax)
                    amax = fabsf(v);
            }
            float sc = group_scale(amax);
            s[rb * cols + c] = sc;
            for (int j = 0; j < GROUP; ++j) {
                int64_t r = rb * GROUP + j;
                qT[c * rows + r] =
                    element_code(orc_bf16_to_float(x[r * cols + c]), sc);
            }
        }
    }
    return bad ? -2 : 0;
}

/* 128x128 blocks of a weight matrix [n, k]. */
int orc_quant_weight(const uint16_t *w, int64_t n, int64_t k, uint8_t *q,
                     float *s)
{
    if (n < 0 || k < 0 || n % GROUP != 0 || k % GROUP != 0)
        return -1;
    int64_t nb_count = n / GROUP, kb_count = k / GROUP;
    int bad = 0;
#pragma omp parallel for schedule(static) reduction(| : bad)
    for (int64_t nb = 0; nb < nb_count; ++nb) {
        for (int64_t kb = 0; kb < kb_count; ++kb) {
            float amax = 0.0f;
            for (int i = 0; i < GROUP; ++i)
                for (int j = 0; j < GROUP; ++j) {
                    float v = orc_bf16_to_float(
                        w[(nb * GROUP + i) * k + kb * GROUP + j]);
                    if (!isfinite(v))
                        bad = 1;
                    if (fabsf(v) > amax)
                        amax = fabsf(v);
                }
            float sc = group_scale(amax);
            s[nb * kb_count + kb] = sc;
            for (int i = 0; i < GROUP; ++i)
                for (int j = 0; j < GROUP; ++j) {
                    int64_t idx = (nb * GROUP + i) * k + kb * GROUP + j;
                    q[idx] = element_code(orc_bf16_to_float(w[idx]), sc);
                }
        }
    }
    return bad ? -2 : 0;
}

/* ----------------------------------------------------------------- GEMMs */

/* Decode an array of codes to doubles (no scale applied). */
static double *decode_all(const uint8_t *codes, int64_t count)
{
    double *out = (double *)malloc((size_t)(count > 0 ? count : 1) * sizeof(double));
    if (!out)
        return NULL;
    for (int64_t i = 0; i < count; ++i)
        out[i] = orc_e4m3_decode(codes[i]);
    return out;
}

/* One output element: sum over slabs t of (sa[t] * sb[t]) * P_t where
 * P_t = sum_{k in slab t} a[k] * b[k]; a and b are contiguous decoded rows
 * of length kc (a multiple of 128); sa and sb are read with strides. */
static void slab_dot(const double *a, const double *b, int64_t kc,
                     const float *sa, int64_t sa_stride, const float *sb,
                     int64_t sb_stride, double *y, double *bound)
{
    double acc = 0.0, abs_acc = 0.0;
    for (int64_t t = 0; t < kc / GROUP; ++t) {
        double p = 0.0, p_abs = 0.0;
        for (int64_t k = t * GROUP; k < (t + 1) * GROUP; ++k) {
            p += a[k] * b[k];
            p_abs += fabs(a[k]) * fabs(b[k]);
        }
        double c = (double)sa[t * sa_stride] * (double)sb[t * sb_stride];
        acc += c * p;
        abs_acc += fabs(c) * p_abs;
    }
    *y = acc;
    *bound = abs_acc;
}

/* fprop: Y[m, n] = sum_k X[m, k] W[n, k].
 * xq [M, K] with row-wise scales sx [K/128, M]; wq [N, K] with block scales
 * sw [N/128, K/128].  rows selects which output rows to compute (all when
 * NULL); y and bound are [nrows, N]. */
int orc_gemm_fprop(const uint8_t *xq, const float *sx, const uint8_t *wq,
                   const float *sw, int64_t M, int64_t N, int64_t K,
                   const int64_t *rows, int64_t nrows, double *y,
                   double *bound)
{
    if (M < 0 || N % GROUP || K % GROUP || N < 0 || K < 0)
        return -1;
    if (!rows)
        nrows = M;
    double *wd = decode_all(wq, N * K);
    if (!wd)
        return -3;
    int64_t kb_count = K / GROUP;
#pragma omp parallel
    {
        double *xrow = (double *)malloc((size_t)(K > 0 ? K : 1) * sizeof(double));
#pragma omp for schedule(dynamic, 1)
        for (int64_t i = 0; i < nrows; ++i) {
            int64_t m = rows ? rows[i] : i;
            for (int64_t k = 0; k < K; ++k)
                xrow[k] = orc_e4m3_decode(xq[m * K + k]);
            for (int64_t n = 0; n < N; ++n)
                slab_dot(xrow, wd + n * K, K, sx + m, M,
                         sw + (n / GROUP) * kb_count, 1, &y[i * N + n],
                         &bound[i * N + n]);
        }
        free(xrow);
    }
    free(wd);
    return 0;
}

/* dgrad: dX[m, k] = sum_n dY[m, n] W[n, k].
 * dyq [M, N] with row-wise scales sdy [N/128, M] (groups along n); wq and sw
 * are the same [N, K] codes and [N/128, K/128] scales fprop uses.  The slab
 * index runs over n; the weight scale of slab t for output column k is
 * sw[t][k/128].  dx and bound are [nrows, K]. */
int orc_gemm_dgrad(const uint8_t *dyq, const float *sdy, const uint8_t *wq,
                   const float *sw, int64_t M, int64_t N, int64_t K,
                   const int64_t *rows, int64_t nrows, double *dx,
                   double *bound)
{
    if (M < 0 || N % GROUP || K % GROUP || N < 0 || K < 0)
        return -1;
    if (!rows)
        nrows = M;
    /* Decoded weight, stored column by column so that the n-contraction of
     * one output column is contiguous: wt[k][n] = dec(wq[n][k]). */
    double *wt = (double *)malloc((size_t)(N * K > 0 ? N * K : 1) * sizeof(double));
    if (!wt)
        return -3;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            wt[k * N + n] = orc_e4m3_decode(wq[n * K + k]);
    int64_t kb_count = K / GROUP;
#pragma omp parallel
    {
        double *dyrow = (double *)malloc((size_t)(N > 0 ? N : 1) * sizeof(double));
#pragma omp for schedule(dynamic, 1)
        for (int64_t i = 0; i < nrows; ++i) {
            int64_t m = rows ? rows[i] : i;
            for (int64_t n = 0; n < N; ++n)
                dyrow[n] = orc_e4m3_decode(dyq[m * N + n]);
            for (int64_t k = 0; k < K; ++k)
                slab_dot(dyrow, wt + k * N, N, sdy + m, M, sw + k / GROUP,
                         kb_count, &dx[i * K + k], &bound[i * K + k]);
        }
        free(dyrow);
    }
    free(wt);
    return 0;
}

/* wgrad: dW[n, k] = sum_m dY[m, n] X[m, k], contracting over the M tokens.
 * dyqT [N, M] and xqT [K, M] are the column-wise (along-token) codes, with
 * scales sdyT [M/128, N] and sxT [M/128, K].  rows selects output rows n;
 * dw and bound are [nrows, K]. */
int orc_gemm_wgrad(const uint8_t *dyqT, const float *sdyT, const uint8_t *xqT,
                   const float *sxT, int64_t N, int64_t K, int64_t M,
                   const int64_t *rows, int64_t nrows, double *dw,
                   double *bound)
{
    if (M % GROUP || M < 0 || N < 0 || K < 0)
        return -1;
    if (!rows)
        nrows = N;
    double *xd = decode_all(xqT, K * M);
    if (!xd)
        return -3;
#pragma omp parallel
    {
        double *dyrow = (double *)malloc((size_t)(M > 0 ? M : 1) * sizeof(double));
#pragma omp for schedule(dynamic, 1)
        for (int64_t i = 0; i < nrows; ++i) {
            int64_t n = rows ? rows[i] : i;
            for (int64_t m = 0; m < M; ++m)
                dyrow[m] = orc_e4m3_decode(dyqT[n * M + m]);
            for (int64_t k = 0; k < K; ++k)
                slab_dot(dyrow, xd + k * M, M, sdyT + n, N, sxT + k, K,
                         &dw[i * K + k], &bound[i * K + k]);
        }
        free(dyrow);
    }
    free(xd);
    return 0;
}

/* wgrad accumulated into a main gradient kept across micro-batches: the
 * Puro-2B-Base model card (friendli.ai), training-setup paragraph, keeps
 * master weights and optimizer state in FP32, and one optimizer step sums
 * the weight gradients of its micro-batches (setting table: global batch
 * 1536 sequences, micro-batch 2).  dw_out[i, k] = dw_in[n, k] + dW[n, k]
 * for output row n = rows[i] (all rows when rows is NULL), with dW exactly
 * as orc_gemm_wgrad computes it and the sum taken in FP64.  dw_in is the
 * running main gradient [N, K] in FP64 (an FP32 array converts to it
 * exactly; NULL means zeros), so chained calls accumulate without rounding
 * to FP32 in between.  bound is the wgrad bound of this call's product. */
int orc_gemm_wgrad_accum(const uint8_t *dyqT, const float *sdyT,
                         const uint8_t *xqT, const float *sxT, int64_t N,
                         int64_t K, int64_t M, const int64_t *rows,
                         int64_t nrows, const double *dw_in, double *dw_out,
                         double *bound)
{
    int rc = orc_gemm_wgrad(dyqT, sdyT, xqT, sxT, N, K, M, rows, nrows,
                            dw_out, bound);
    if (rc != 0)
        return rc;
    if (!dw_in)
        return 0;
    if (!rows)
        nrows = N;
    for (int64_t i = 0; i < nrows; ++i) {
        int64_t n = rows ? rows[i] : i;
        for (int64_t k = 0; k < K; ++k) {
            double v = dw_in[n * K + k];
            if (!isfinite(v))
                return -2;
            dw_out[i * K + k] = v + dw_out[i * K + k];
        }
    }
    return 0;
}

/* Threads the parallel loops above use. */
int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* --------------------------------------------------------------- SwiGLU
 *
 * The feed-forward block of the Qwen3-1.7B configuration (named in the
 * friendli.ai model card's model property table) is a gated SiLU unit:
 * H = silu(gate) * up, with gate and up the two halves of the fused
 * gate_up projection.  With activations kept in BF16 (model card,
 * training-setup paragraph), the unfused path rounds twice:
 * h = bf16(bf16(silu(g)) * u).  This oracle takes exactly that, with each
 * rounding to nearest even and silu evaluated in double precision before
 * its single rounding to bfloat16.  It is the definition a fused
 * quantize-on-output kernel has to reproduce before its 1x128 groups are
 * quantized as above.
 */

/* Nearest bfloat16 of the finite value hi + lo, where lo is either zero or
 * too small to move hi across a bfloat16 rounding boundary and matters only
 * when hi lies exactly on one (a midpoint between two bfloat16 values): then
 * its sign says on which side the value lies.  Otherwise ties go to the even
 * significand.  8 significant bits, float32's exponent range including its
 * subnormals; beyond the largest finite bfloat16 the result is infinity.
 * Returns the bit pattern. */
static uint16_t bf16_round_split(double hi, double lo)
{
    uint16_t sgn = signbit(hi) ? 0x8000 : 0x0000;
    double mag = fabs(hi);
    int ex;
    if (mag == 0.0)
        return sgn;
    (void)frexp(mag, &ex);                 /* mag in [2^(ex-1), 2^ex) */
    int lead = ex - 1 < -126 ? -126 : ex - 1;
    double step = ldexp(1.0, lead - 7);    /* bfloat16 spacing at mag */
    double units = mag / step;             /* exact: a power-of-two divisor */
    double below = floor(units);
    double frac = units - below;
    int up;
    if (frac != 0.5)
        up = frac > 0.5;
    else if (lo != 0.0)
        up = (lo > 0.0) == (hi > 0.0);     /* the value lies beyond the midpoint */
    else
        up = fmod(below, 2.0) == 1.0;      /* a true tie: to the even one */
    double rounded = (below + (up ? 1.0 : 0.0)) * step;
    if (rounded >= ldexp(1.0, 128))
        return sgn | 0x7F80;
    float as_float = (float)rounded;       /* exact: at most 8 significant bits */
    uint32_t u;
    memcpy(&u, &as_float, sizeof u);
    return sgn | (uint16_t)((u >> 16) & 0x7FFF);
}

/* Nearest bfloat16 of a finite double, ties to even. */
uint16_t orc_bf16_from_double(double v)
{
    return bf16_round_split(v, 0.0);
}

/* silu(g) = g / (1 + e^-g) for a bfloat16 g, rounded once to bfloat16.
 * For |g| < 2^-30 the series g/2 + g^2/4 + O(g^4) is used instead: in
 * double, 1 + e^-g rounds to 2 - g or to 2 and the quotient loses the g^2/4
 * term, which is what decides the rounding when g/2 is a bfloat16 midpoint
 * (g an odd multiple of the smallest subnormal).  There g/2 is exact and the
 * higher terms cannot reach a rounding boundary.  Elsewhere the double
 * quotient is within a few units in its last place of silu(g), far from any
 * bfloat16 boundary for every bfloat16 g. */
uint16_t orc_silu_bf16(uint16_t g_bits)
{
    double g = (double)orc_bf16_to_float(g_bits);
    if (fabs(g) < 0x1p-30)
        return bf16_round_split(g / 2.0, g * g / 4.0);
    return orc_bf16_from_double(g / (1.0 + exp(-g)));
}

/* H [rows, ffn] from a gate_up activation [rows, 2 * ffn] whose columns
 * [0, ffn) are the gate and [ffn, 2 * ffn) the up projection.  The product
 * of two bfloat16 values is exact in double, so h has one rounding after
 * silu's. */
int orc_swiglu_bf16(const uint16_t *gate_up, int64_t rows, int64_t ffn,
                    uint16_t *h)
{
    if (rows < 0 || ffn < 0)
        return -1;
    int bad = 0;
#pragma omp parallel for schedule(static) reduction(| : bad)
    for (int64_t r = 0; r < rows; ++r) {
        const uint16_t *gate = gate_up + r * 2 * ffn;
        const uint16_t *up = gate + ffn;
        for (int64_t j = 0; j < ffn; ++j) {
            float gf = orc_bf16_to_float(gate[j]);
            float uf = orc_bf16_to_float(up[j]);
            if (!isfinite(gf) || !isfinite(uf))
                bad = 1;
            double s = (double)orc_bf16_to_float(orc_silu_bf16(gate[j]));
            h[r * ffn + j] = orc_bf16_from_double(s * (double)uf);
        }
    }
    return bad ? -2 : 0;
}

/* -------------------------------------------------------------- RMSNorm
 *
 * The Qwen3-1.7B configuration (friendli.ai model card, model property
 * table; the card's export class is Qwen3ForCausalLM) normalizes the input
 * of the attention and feed-forward blocks with RMSNorm.  The linear
 * layers' X is its BF16 output (training-setup paragraph: activations stay
 * BF16), so a quantizer fused into the norm has to reproduce
 *
 *   r    = 1 / sqrt(mean_k x[k]^2 + eps)          per row, rounded to FP32
 *   t[k] = fp32(x[k] * r)                         one FP32 multiply
 *   y[k] = bf16(gamma[k] * bf16(t[k]))            each rounding to nearest even
 *
 * (the order of the Transformers Qwen3 RMSNorm: normalize in FP32, round to
 * the activation type, then scale by the BF16 weight).  r is split off as
 * its own function: the fused quantizer takes it as an input, computed by
 * the row reduction that precedes it.
 */

/* r[i] for each row of x [rows, cols]: the squares of bfloat16 values are
 * exact in double and their sum is taken in double in index order (for the
 * row lengths of the path its relative error is below 2^-40); the mean is
 * that sum / cols, eps is added in double, and 1 / sqrt(.) is rounded once
 * from double to FP32. */
int orc_rmsnorm_rstd(const uint16_t *x, int64_t rows, int64_t cols, float eps,
                     float *r)
{
    if (rows < 0 || cols <= 0 || !(eps >= 0.0f))
        return -1;
    int bad = 0;
#pragma omp parallel for schedule(static) reduction(| : bad)
    for (int64_t i = 0; i < rows; ++i) {
        double sum = 0.0;
        for (int64_t k = 0; k < cols; ++k) {
            double v = (double)orc_bf16_to_float(x[i * cols + k]);
            if (!isfinite(v))
                bad = 1;
            sum += v * v;
        }
        double ms = sum / (double)cols + (double)eps;
        r[i] = (float)(1.0 / sqrt(ms));
    }
    return bad ? -2 : 0;
}

/* y [rows, cols] = bf16(gamma * bf16(fp32(x * r))) with r per row (FP32)
 * and gamma [cols] (bfloat16).  The FP32 product is a C float multiply
 * (one IEEE rounding); the product of two bfloat16 values is exact in
 * double, so each bfloat16 result has one rounding. */
int orc_rmsnorm_apply(const uint16_t *x, int64_t rows, int64_t cols,
                      const float *r, const uint16_t *gamma, uint16_t *y)
{
    if (rows < 0 || cols < 0)
        return -1;
    int bad = 0;
#pragma omp parallel for schedule(static) reduction(| : bad)
    for (int64_t i = 0; i < rows; ++i) {
        for (int64_t k = 0; k < cols; ++k) {
            float xf = orc_bf16_to_float(x[i * cols + k]);
            float gf = orc_bf16_to_float(gamma[k]);
            if (!isfinite(xf) || !isfinite(gf) || !isfinite(r[i]))
                bad = 1;
            volatile float t = xf * r[i];
            double b = (double)orc_bf16_to_float(orc_bf16_from_double((double)t));
            y[i * cols + k] = orc_bf16_from_double((double)gf * b);
        }
    }
    return bad ? -2 : 0;
}
