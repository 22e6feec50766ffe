/*
 * wq_oracle.c -- plain, slow, single-threaded CPU oracle for the quantization
 * hot path.  TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the
 * benchmark's CPU-baseline leg are the only callers.  It shares no code with
 * the CUDA library (no headers, helpers or tables) and never calls it.
 *
 * Every routine is the plain definition from the source pages, written as
 * scalar loops in the order the pages state the steps:
 *
 *   [P1] "How quantization works" (AI-infra handbook): section "The math of
 *        quantization" (symmetric s = max|x|/(2^(b-1)-1), q = clamp(round(x/s)),
 *        x^ = q*s), the quant.py listing (absmax clamped at 1e-8), section
 *        "Activation quantization and outliers" (per-row INT8, SmoothQuant
 *        s_j = max|X_j|^a / max|W_j|^(1-a) with 1e-5 clamps, X/s and W*s),
 *        exercise 2 (fp16 scale + 4-bit zero point per group of 128).
 *   [P2] "Quantization" (engine-room ch. 15), section "The Mathematics":
 *        SmoothQuant Y = (X diag(s)^-1)(diag(s) W).
 *   [P3] "Quantization from Scratch: Scale, Zero-Point, GPTQ and AWQ":
 *        section "Scale and zero-point" (w^ = (q - z) s) and the round-to-
 *        nearest quantize() in "Measured on two real layers" (scale 0 -> 1).
 *   [P4] "Quantization: Smaller Weights, Same Answers (Mostly)": section
 *        "How does quantized matrix multiplication actually run on the GPU?"
 *        (integer products summed exactly in a 32-bit accumulator).
 *   [P5] "Quantization Explained: INT8, INT4, GPTQ and AWQ for LLMs":
 *        "Uniform Affine Quantization" (x_q = round(x/s) + z,
 *        x^ = s (x_q - z)), "Scale and Zero-Point" (s = (max-min)/(2^b-1),
 *        z = round(-min/s)), "Manual Group-Wise Quantizer" (clamp to [0,15]).
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *   - round() is round-half-to-even (the pages' code uses torch/np.round);
 *     here nearbyint() in the default FE_TONEAREST mode.
 *   - x/s is an IEEE fp32 division (no reciprocal, no fused multiply-add);
 *     build with -ffp-contract=off -fno-fast-math.
 *   - the INT4 group scale is rounded to fp16 (the stored format) BEFORE z
 *     and the codes are computed, so quantizer and dequantizer share one grid.
 *   - the INT4 group range is widened to contain 0 (lo = min(min,0),
 *     hi = max(max,0)) so that z lands in [0,15] and 0 maps to an exact code.
 *   - INT4 codes: element k of a row is nibble (k mod 8) of word k/8; the
 *     zero point of group j is nibble (j mod 8) of zero word j/8.
 *   - INT8 scales are fp32; smoothing never rounds X/s or W*s to fp16.
 *   - inputs must be finite.
 *
 * Floating-point matmul references are computed in fp64.
 */
#include <fenv.h>
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* IEEE 754 binary16, written from the format definition:                    */
/*   normal:    (-1)^s * 2^(e-15) * (1 + m/1024),  1 <= e <= 30              */
/*   subnormal: (-1)^s * 2^(-14)  * (m/1024),      e == 0                    */
/* ------------------------------------------------------------------------ */

float orc_half_to_float(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int m = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);                 /* 2^-14 * m/1024 */
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + m), e - 25);     /* 2^(e-15) * (1024+m)/1024 */
    return (float)(sign ? -v : v);
}

/* Nearest binary16 value, ties to even mantissa; overflow to infinity. */
uint16_t orc_float_to_half(float f)
{
    uint16_t sign = signbit(f) ? 0x8000 : 0;
    double a = fabs((double)f);
    if (isnan(f))
        return 0x7e00;
    /* 65520 is the midpoint between 65504 (largest finite) and 2^16; it and
       everything above round to infinity. */
    if (a >= 65520.0)
        return sign | 0x7c00;
    if (a < ldexp(1.0, -14)) {
        /* subnormal grid: multiples of 2^-24 */
        double m = nearbyint(a / ldexp(1.0, -24));
        return sign | (uint16_t)m;                 /* m == 1024 is the smallest normal */
    }
    int E;
    frexp(a, &E);                                  /* a = f * 2^E, f in [0.5, 1) */
    int e = E - 1;                                 /* a in [2^e, 2^(e+1)) */
    double m = nearbyint(a / ldexp(1.0, e - 10));  /* in [1024, 2048] */
    if (m == 2048.0) {
        m = 1024.0;
        e += 1;
    }
    return sign | (uint16_t)(((e + 15) << 10) | ((int)m - 1024));
}

static int rne_to_int(float v)
{
    return (int)nearbyintf(v);                     /* FE_TONEAREST: half to even */
}

static int clampi(int v, int lo, int hi)
{
    return v < lo ? lo : (v > hi ? hi : v);
}

int orc_rounding_mode_is_nearest(void)
{
    return fegetround() == FE_TONEAREST;
}

/* ------------------------------------------------------------------------ */
/* Asymmetric INT4 per-group quantizer  ([P5] "Scale and Zero-Point",        */
/* [P3] quantize(), [P1] exercise 2 for the stored format).                  */
/* w: [N][K] fp32 (w_is_f16 == 0) or fp16 bits (w_is_f16 == 1), row-major.   */
/* Outputs: qweight [N][K/8], scales fp16 bits [N][K/g],                     */
/*          qzeros [N][ceil(K/g/8)].  Returns 0, or -1 on bad arguments.     */
/* ------------------------------------------------------------------------ */
static float load_w(const void *w, int w_is_f16, size_t idx)
{
    return w_is_f16 ? orc_half_to_float(((const uint16_t *)w)[idx]) : ((const float *)w)[idx];
}

int orc_quantize_group_int4(const void *w, int w_is_f16, int N, int K, int g,
                            uint32_t *qweight, uint16_t *scales, uint32_t *qzeros)
{
    if (N <= 0 || K <= 0 || g <= 0 || K % g != 0 || K % 8 != 0)
        return -1;
    const int G = K / g;
    const int ZW = (G + 7) / 8;
    memset(qweight, 0, sizeof(uint32_t) * (size_t)N * (K / 8));
    memset(qzeros, 0, sizeof(uint32_t) * (size_t)N * ZW);
    for (int n = 0; n < N; ++n) {
        for (int j = 0; j < G; ++j) {
            const size_t base = (size_t)n * K + (size_t)j * g;
            /* range of the group, widened to contain 0 */
            float lo = 0.0f, hi = 0.0f;
            for (int t = 0; t < g; ++t) {
                float v = load_w(w, w_is_f16, base + t);
                if (v < lo) lo = v;
                if (v > hi) hi = v;
            }
            /* s = (max - min) / (2^4 - 1), stored as fp16; a zero scale becomes 1 */
            float s32 = (hi - lo) / 15.0f;
            uint16_t s16 = orc_float_to_half(s32);
            if (s16 == 0)
                s16 = 0x3c00;                       /* 1.0 */
            float s = orc_half_to_float(s16);
            /* z = round(-min / s), kept in the 4-bit range */
            int z = clampi(rne_to_int(-lo / s), 0, 15);
            scales[(size_t)n * G + j] = s16;
            qzeros[(size_t)n * ZW + j / 8] |= (uint32_t)z << (4 * (j % 8));
            /* q = clamp(round(w / s) + z, 0, 15) */
            for (int t = 0; t < g; ++t) {
                int k = j * g + t;
                float v = load_w(w, w_is_f16, base + t);
                int q = clampi(rne_to_int(v / s) + z, 0, 15);
                qweight[(size_t)n * (K / 8) + k / 8] |= (uint32_t)q << (4 * (k % 8));
            }
        }
    }
    return 0;
}

/* Unpack helpers for the stored INT4 layout. */
int orc_int4_code(const uint32_t *qweight, int K, int n, int k)
{
    return (int)((qweight[(size_t)n * (K / 8) + k / 8] >> (4 * (k % 8))) & 0xf);
}

int orc_int4_zero(const uint32_t *qzeros, int K, int g, int n, int j)
{
    const int ZW = (K / g + 7) / 8;
    return (int)((qzeros[(size_t)n * ZW + j / 8] >> (4 * (j % 8))) & 0xf);
}

/* w^[n][k] = s * (q - z) in fp64  ([P3] "Scale and zero-point", [P5]). */
void orc_dequant_int4(const uint32_t *qweight, const uint16_t *scales,
                      const uint32_t *qzeros, int N, int K, int g, double *what)
{
    const int G = K / g;
    for (int n = 0; n < N; ++n)
        for (int k = 0; k < K; ++k) {
            int j = k / g;
            double s = (double)orc_half_to_float(scales[(size_t)n * G + j]);
            int q = orc_int4_code(qweight, K, n, k);
            int z = orc_int4_zero(qzeros, K, g, n, j);
            what[(size_t)n * K + k] = s * (double)(q - z);
        }
}

/* ------------------------------------------------------------------------ */
/* Symmetric b-bit per row ([P1] "The math of quantization", quant.py       */
/* fake_quant_int, q8_per_row; SmoothQuant's Xs = X / s, Ws = W * s first).  */
/* x: fp16 bits [R][K].  mode 0: no smoothing; 1: multiply column k by       */
/* smooth[k] (weights, diag(s) W); 2: divide column k by smooth[k]           */
/* (activations, X diag(s)^-1).  bits in [2, 8]: s = max|x| / (2^(b-1) - 1), */
/* codes clamped to [-2^(b-1), 2^(b-1) - 1].  Outputs q [R][K] int8 and      */
/* scales [R] fp32.  INT8 per channel / per token is bits == 8.              */
/* ------------------------------------------------------------------------ */
static float smoothed(float v, const float *smooth, int mode, int k)
{
    if (mode == 1) return v * smooth[k];
    if (mode == 2) return v / smooth[k];
    return v;
}

int orc_quantize_sym_rows(const uint16_t *x, int R, int K, const float *smooth, int mode,
                          int bits, int8_t *q, float *scales)
{
    if (R <= 0 || K <= 0 || mode < 0 || mode > 2 || (mode != 0 && !smooth) || bits < 2 || bits > 8)
        return -1;
    const int qmax = (1 << (bits - 1)) - 1;
    for (int r = 0; r < R; ++r) {
        const uint16_t *row = x + (size_t)r * K;
        float a = 0.0f;
        for (int k = 0; k < K; ++k) {
            float v = fabsf(smoothed(orc_half_to_float(row[k]), smooth, mode, k));
            if (v > a) a = v;
        }
        if (a < 1e-8f) a = 1e-8f;                   /* absmax.clamp(min=1e-8) */
        float s = a / (float)qmax;                  /* s = max|x| / (2^(b-1) - 1) */
        scales[r] = s;
        for (int k = 0; k < K; ++k) {
            float v = smoothed(orc_half_to_float(row[k]), smooth, mode, k);
            q[(size_t)r * K + k] = (int8_t)clampi(rne_to_int(v / s), -qmax - 1, qmax);
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* SmoothQuant factors ([P1] "Activation quantization and outliers",         */
/* [P2] "The Mathematics"): s_j = max|X_j|^a / max|W_j|^(1-a), both maxima   */
/* clamped at 1e-5, X: fp16 [M][K], W: fp16 [N][K] (nn.Linear layout, so    */
/* column j of both is input channel j).  For a == 0.5 the powers are        */
/* square roots (correctly rounded); otherwise pow() in fp64 rounded to fp32.*/
/* ------------------------------------------------------------------------ */
int orc_smooth(const uint16_t *X, int M, const uint16_t *W, int N, int K,
               double alpha, float *s)
{
    if (M <= 0 || N <= 0 || K <= 0)
        return -1;
    for (int j = 0; j < K; ++j) {
        float ax = 0.0f, aw = 0.0f;
        for (int m = 0; m < M; ++m) {
            float v = fabsf(orc_half_to_float(X[(size_t)m * K + j]));
            if (v > ax) ax = v;
        }
        for (int n = 0; n < N; ++n) {
            float v = fabsf(orc_half_to_float(W[(size_t)n * K + j]));
            if (v > aw) aw = v;
        }
        if (ax < 1e-5f) ax = 1e-5f;
        if (aw < 1e-5f) aw = 1e-5f;
        float num, den;
        if (alpha == 0.5) {
            num = sqrtf(ax);
            den = sqrtf(aw);
        } else {
            num = (float)pow((double)ax, alpha);
            den = (float)pow((double)aw, 1.0 - alpha);
        }
        s[j] = num / den;
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* W4A16 matmul reference in fp64 ([P1] "Inference view": weights unpacked,  */
/* multiplied by their scales and accumulated): y[b][n] = sum_k w^[n][k]     */
/* x[b][k], plus bound[b][n] = sum_k |w^[n][k] x[b][k]|.  rows (nullable)    */
/* selects output rows; results are [B][nrows].                              */
/* ------------------------------------------------------------------------ */
/* bfloat16: the upper 16 bits of an IEEE binary32 (1 sign, 8 exponent, 7 mantissa bits). */
float orc_bf16_to_float(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

static void matmul_w4a16(const uint16_t *x, float (*load_x)(uint16_t), int B, const uint32_t *qweight,
                         const uint16_t *scales, const uint32_t *qzeros, int N, int K, int g,
                         const int *rows, int nrows, double *y, double *bound);

void orc_matmul_w4a16_ref(const uint16_t *x, int B, const uint32_t *qweight,
                          const uint16_t *scales, const uint32_t *qzeros, int N, int K,
                          int g, const int *rows, int nrows, double *y, double *bound)
{
    matmul_w4a16(x, orc_half_to_float, B, qweight, scales, qzeros, N, K, g, rows, nrows, y, bound);
}

/* The same reference with bf16 activations. */
void orc_matmul_w4a16_ref_bf16(const uint16_t *x, int B, const uint32_t *qweight,
                               const uint16_t *scales, const uint32_t *qzeros, int N, int K,
                               int g, const int *rows, int nrows, double *y, double *bound)
{
    matmul_w4a16(x, orc_bf16_to_float, B, qweight, scales, qzeros, N, K, g, rows, nrows, y, bound);
}

static void matmul_w4a16(const uint16_t *x, float (*load_x)(uint16_t), int B, const uint32_t *qweight,
                         const uint16_t *scales, const uint32_t *qzeros, int N, int K, int g,
                         const int *rows, int nrows, double *y, double *bound)
{
    const int G = K / g;
    if (!rows) nrows = N;
    for (int i = 0; i < nrows; ++i) {
        int n = rows ? rows[i] : i;
        for (int b = 0; b < B; ++b) {
            double acc = 0.0, bnd = 0.0;
            for (int k = 0; k < K; ++k) {
                int j = k / g;
                double s = (double)orc_half_to_float(scales[(size_t)n * G + j]);
                int q = orc_int4_code(qweight, K, n, k);
                int z = orc_int4_zero(qzeros, K, g, n, j);
                double t = s * (double)(q - z) * (double)load_x(x[(size_t)b * K + k]);
                acc += t;
                bnd += fabs(t);
            }
            y[(size_t)b * nrows + i] = acc;
            bound[(size_t)b * nrows + i] = bnd;
        }
    }
}

/* W8A16 reference: w^[n][k] = sw[n] * q[n][k] ([P1] per-channel INT8). */
void orc_matmul_w8a16_ref(const uint16_t *x, int B, const int8_t *wq, const float *sw,
                          int N, int K, const int *rows, int nrows, double *y, double *bound)
{
    if (!rows) nrows = N;
    for (int i = 0; i < nrows; ++i) {
        int n = rows ? rows[i] : i;
        for (int b = 0; b < B; ++b) {
            double acc = 0.0, bnd = 0.0;
            for (int k = 0; k < K; ++k) {
                double t = (double)sw[n] * (double)wq[(size_t)n * K + k] *
                           (double)orc_half_to_float(x[(size_t)b * K + k]);
                acc += t;
                bnd += fabs(t);
            }
            y[(size_t)b * nrows + i] = acc;
            bound[(size_t)b * nrows + i] = bnd;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* W8A8 reference ([P4] quantized matmul on the GPU; [P1] W8A8 scheme):      */
/* acc[m][n] = sum_k xq[m][k] wq[n][k] exactly (int64, checked to fit int32),*/
/* y = acc * sx[m] * sw[n] in fp64, bound = sx sw sum |xq wq|.               */
/* ms/ns select rows of X and rows of W (columns of y); results [nm][nn].    */
/* Returns 0, or -2 if an accumulator leaves the int32 range.                */
/* ------------------------------------------------------------------------ */
int orc_gemm_w8a8_ref(const int8_t *xq, const float *sx, const int8_t *wq, const float *sw,
                      int M, int N, int K, const int *ms, int nm, const int *ns, int nn,
                      int64_t *acc, double *y, double *bound)
{
    int rc = 0;
    if (!ms) nm = M;
    if (!ns) nn = N;
    for (int a = 0; a < nm; ++a) {
        int m = ms ? ms[a] : a;
        for (int c = 0; c < nn; ++c) {
            int n = ns ? ns[c] : c;
            int64_t s = 0, sa = 0;
            for (int k = 0; k < K; ++k) {
                int64_t p = (int64_t)xq[(size_t)m * K + k] * (int64_t)wq[(size_t)n * K + k];
                s += p;
                sa += p < 0 ? -p : p;
            }
            if (s > INT32_MAX || s < INT32_MIN)
                rc = -2;
            acc[(size_t)a * nn + c] = s;
            y[(size_t)a * nn + c] = (double)s * (double)sx[m] * (double)sw[n];
            bound[(size_t)a * nn + c] = (double)sa * (double)sx[m] * (double)sw[n];
        }
    }
    return rc;
}

/* ------------------------------------------------------------------------ */
/* FP8 E4M3 ([P3] "Formats": 4 exponent bits, 3 mantissa bits, up to 448;   */
/* [P4] "What about FP8, MXFP4, NVFP4 and GGUF?": E4M3 reaches +-448), the  */
/* variant without infinities:                                               */
/*   exponent field e in 1..15: (-1)^s * 2^(e-7) * (1 + m/8)                 */
/*   e == 0 (subnormal):        (-1)^s * 2^(-6)  * (m/8)                     */
/*   e == 15 and m == 7:        NaN  (so the largest finite value is 448)    */
/* ------------------------------------------------------------------------ */
float orc_e4m3_to_float(uint8_t c)
{
    int sign = (c >> 7) & 1;
    int e = (c >> 3) & 0xf;
    int m = c & 7;
    double v;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);                  /* 2^-6 * m/8 */
    else
        v = ldexp((double)(8 + m), e - 10);        /* 2^(e-7) * (8+m)/8 */
    return (float)(sign ? -v : v);
}

/* Nearest E4M3 value, ties to even mantissa; magnitudes beyond 448 saturate
   to 448 (reading: the format has no infinity, and every quantizer below
   chooses its scale so that |x/s| <= 448 up to one rounding).  The sign of a
   value that rounds to zero is kept. */
uint8_t orc_float_to_e4m3(float f)
{
    uint8_t sign = signbit(f) ? 0x80 : 0;
    double a = fabs((double)f);
    if (isnan(f))
        return 0x7f;
    if (a >= 448.0)
        return sign | 0x7e;
    if (a < ldexp(1.0, -6)) {
        /* subnormal grid: multiples of 2^-9; m == 8 is the smallest normal */
        double m = nearbyint(a / ldexp(1.0, -9));
        return sign | (uint8_t)m;
    }
    int E;
    frexp(a, &E);                                  /* a in [2^(E-1), 2^E) */
    int e = E - 1;
    double m = nearbyint(a / ldexp(1.0, e - 3));   /* in [8, 16] */
    if (m == 16.0) {
        m = 8.0;
        e += 1;
    }
    int field = e + 7;
    if (field > 15 || (field == 15 && (int)m - 8 == 7))
        return sign | 0x7e;                        /* rounds past 448: saturate */
    return sign | (uint8_t)((field << 3) | ((int)m - 8));
}

/* ------------------------------------------------------------------------ */
/* FP8 E4M3 quantizer ([P1] quant.py fake_quant_fp8: scale = max|w| / 448,  */
/* codes = (w / scale) cast to E4M3).  x: fp16 bits [R][K].  per_row != 0:  */
/* one scale per row (per output channel for weights, per token for          */
/* activations; scales [R]); per_row == 0: one scale for the whole tensor   */
/* (scales [1]), as in the listing.  The absmax is clamped at 1e-8 (the     */
/* same guard as the listing's integer quantizer) so that an all-zero input */
/* gets a finite scale.  w / scale is one IEEE fp32 division, then rounded  */
/* to E4M3.                                                                  */
/* ------------------------------------------------------------------------ */
int orc_quantize_fp8_e4m3(const uint16_t *x, int R, int K, int per_row, uint8_t *q, float *scales)
{
    if (R <= 0 || K <= 0)
        return -1;
    float tensor_a = 0.0f;
    if (!per_row) {
        for (size_t i = 0; i < (size_t)R * K; ++i) {
            float v = fabsf(orc_half_to_float(x[i]));
            if (v > tensor_a) tensor_a = v;
        }
        if (tensor_a < 1e-8f) tensor_a = 1e-8f;
        scales[0] = tensor_a / 448.0f;
    }
    for (int r = 0; r < R; ++r) {
        const uint16_t *row = x + (size_t)r * K;
        float s;
        if (per_row) {
            float a = 0.0f;
            for (int k = 0; k < K; ++k) {
                float v = fabsf(orc_half_to_float(row[k]));
                if (v > a) a = v;
            }
            if (a < 1e-8f) a = 1e-8f;
            s = a / 448.0f;
            scales[r] = s;
        } else {
            s = scales[0];
        }
        for (int k = 0; k < K; ++k)
            q[(size_t)r * K + k] = orc_float_to_e4m3(orc_half_to_float(row[k]) / s);
    }
    return 0;
}

/* FP8 W8A8 reference: y[m][n] = sx * sw * sum_k e4m3(xq[m][k]) e4m3(wq[n][k])
   in fp64 (every product and partial sum is exact in fp64 for K <= 2^20),
   bound = sx * sw * sum_k |products|.  sx_per_row / sw_per_row == 0 means one
   scale for the whole operand (element 0).  ms/ns select rows of X and W. */
void orc_gemm_fp8_ref(const uint8_t *xq, const float *sx, int sx_per_row, const uint8_t *wq,
                      const float *sw, int sw_per_row, int M, int N, int K, const int *ms, int nm,
                      const int *ns, int nn, double *y, double *bound)
{
    if (!ms) nm = M;
    if (!ns) nn = N;
    for (int a = 0; a < nm; ++a) {
        int m = ms ? ms[a] : a;
        double sxm = (double)sx[sx_per_row ? m : 0];
        for (int c = 0; c < nn; ++c) {
            int n = ns ? ns[c] : c;
            double swn = (double)sw[sw_per_row ? n : 0];
            double acc = 0.0, abs_acc = 0.0;
            for (int k = 0; k < K; ++k) {
                double p = (double)orc_e4m3_to_float(xq[(size_t)m * K + k]) *
                           (double)orc_e4m3_to_float(wq[(size_t)n * K + k]);
                acc += p;
                abs_acc += fabs(p);
            }
            y[(size_t)a * nn + c] = acc * sxm * swn;
            bound[(size_t)a * nn + c] = abs_acc * sxm * swn;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* LLM.int8() mixed-precision decomposition ([P2] "The Mathematics":        */
/* C ~= S_out (.) (X_q W_q) + X_16 W_16, the outlier feature dimensions     */
/* removed from the integer path and multiplied in 16-bit; [P2] "The         */
/* Breakthrough": vector-wise scales per row and per column; [P4] outlier  */
/* schemes: LLM.int8()-style mixed precision keeps the outlier dimensions  */
/* in FP16 and quantizes the rest).                                          */
/* Readings: an outlier dimension is an input column j with                  */
/* max_m |X[m][j]| >= threshold (the threshold is a parameter; the pages do */
/* not give its value); at most `cap` of them, the lowest column indices,   */
/* are carved out; the weights are stored once, as per-output-channel INT8 */
/* (the method halves weight memory, so no 16-bit copy exists) and W_16 is  */
/* their dequantized outlier columns s_w[n] * W_q[n][j].                     */
/* ------------------------------------------------------------------------ */

/* Outlier columns of X [M][K] (fp16 bits): writes the first min(total, cap)
   qualifying column indices in increasing order to idx and returns the
   total number that qualify. */
int orc_outlier_columns(const uint16_t *X, int M, int K, float threshold, int cap, int *idx)
{
    int total = 0;
    for (int j = 0; j < K; ++j) {
        float a = 0.0f;
        for (int m = 0; m < M; ++m) {
            float v = fabsf(orc_half_to_float(X[(size_t)m * K + j]));
            if (v > a) a = v;
        }
        if (a >= threshold) {
            if (total < cap)
                idx[total] = j;
            ++total;
        }
    }
    return total;
}

/* The decomposed product for the carved-out columns idx[0..n_out):
     keep[j] = 0 for carved columns, 1 otherwise
     X_q, s_x = per-row symmetric INT8 of X * keep   (orc_quantize_sym_rows)
     y[m][n]  = s_w[n] * ( s_x[m] * sum_{j not carved} X_q[m][j] W_q[n][j]
                           + sum_{j carved} X[m][j] W_q[n][j] )       (fp64)
   bound = s_w (s_x sum |X_q W_q| + sum |X W_q|).  xq/sx receive X_q and s_x
   (both [M][K] / [M], required).  ms/ns select rows of X and of W. */
int orc_llm_int8_ref(const uint16_t *X, int M, int K, const int8_t *wq, const float *sw, int N,
                     const int *idx, int n_out, const int *ms, int nm, const int *ns, int nn,
                     int8_t *xq, float *sx, double *y, double *bound)
{
    if (M <= 0 || N <= 0 || K <= 0 || n_out < 0 || n_out > K)
        return -1;
    float *keep = (float *)malloc(sizeof(float) * (size_t)K);
    char *carved = (char *)calloc((size_t)K, 1);
    if (!keep || !carved) {
        free(keep);
        free(carved);
        return -1;
    }
    for (int j = 0; j < K; ++j)
        keep[j] = 1.0f;
    for (int i = 0; i < n_out; ++i) {
        keep[idx[i]] = 0.0f;
        carved[idx[i]] = 1;
    }
    int rc = orc_quantize_sym_rows(X, M, K, keep, 1, 8, xq, sx);
    if (!ms) nm = M;
    if (!ns) nn = N;
    for (int a = 0; rc == 0 && a < nm; ++a) {
        int m = ms ? ms[a] : a;
        for (int c = 0; c < nn; ++c) {
            int n = ns ? ns[c] : c;
            double acc8 = 0.0, abs8 = 0.0, acc16 = 0.0, abs16 = 0.0;
            for (int k = 0; k < K; ++k) {
                double w = (double)wq[(size_t)n * K + k];
                if (carved[k]) {
                    double p = (double)orc_half_to_float(X[(size_t)m * K + k]) * w;
                    acc16 += p;
                    abs16 += fabs(p);
                } else {
                    double p = (double)xq[(size_t)m * K + k] * w;
                    acc8 += p;
                    abs8 += fabs(p);
                }
            }
            y[(size_t)a * nn + c] = (double)sw[n] * ((double)sx[m] * acc8 + acc16);
            bound[(size_t)a * nn + c] = (double)sw[n] * ((double)sx[m] * abs8 + abs16);
        }
    }
    free(keep);
    free(carved);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Block-scaled FP4 ([P4] "What about FP8, MXFP4, NVFP4 and GGUF?": MXFP4   */
/* stores blocks of 32 four-bit floats (E2M1) sharing one 8-bit power-of-two */
/* scale; NVFP4 uses blocks of 16 with an FP8 scale per block plus one FP32 */
/* scale per tensor; [P3] "Formats": blocks of 32 share one 8-bit           */
/* power-of-two scale; [P1] "Mainstream schemes": FP4 (NVFP4 / MXFP4) on    */
/* Blackwell).                                                               */
/* E2M1: 1 sign, 2 exponent bits (bias 1), 1 mantissa bit, no inf/NaN:       */
/*   e in 1..3: (-1)^s * 2^(e-1) * (1 + m/2);  e == 0: (-1)^s * m/2          */
/*   i.e. 0, 0.5, 1, 1.5, 2, 3, 4, 6.                                        */
/* Readings (the pages name the formats, not their rounding rules):          */
/*  - MXFP4 follows the microscaling specification the pages cite: shared    */
/*    exponent floor(log2(max|v|)) - 2 (2 = the exponent of E2M1's largest   */
/*    value 6), stored as E8M0 = exponent + 127 (an all-zero block gets 0,   */
/*    i.e. 2^-127); elements v / 2^e rounded to nearest even, saturating at  */
/*    +-6.                                                                   */
/*  - NVFP4: tensor scale S = max(max|v|, 1e-8) / (6 * 448); block scale     */
/*    E4M3 code of (max_block|v| / 6) / S (positive); elements               */
/*    e2m1_rn(v / (e4m3(block) * S)), all zero when the block code is 0.     */
/*  - two elements per byte, element 2i in the low nibble.                   */
/* ------------------------------------------------------------------------ */
float orc_e2m1_to_float(uint8_t c)
{
    int sign = (c >> 3) & 1;
    int e = (c >> 1) & 3;
    int m = c & 1;
    double v = e == 0 ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return (float)(sign ? -v : v);
}

/* Nearest E2M1 value, ties to even mantissa, magnitudes beyond 6 saturate. */
uint8_t orc_float_to_e2m1(float f)
{
    uint8_t sign = signbit(f) ? 8 : 0;
    double a = fabs((double)f);
    if (a >= 6.0)
        return sign | 7;
    if (a < 1.0) {                                 /* subnormal grid: multiples of 0.5 */
        double m = nearbyint(a / 0.5);             /* 0, 1 or 2 (2 = the value 1.0) */
        return sign | (uint8_t)m;
    }
    int E;
    frexp(a, &E);                                  /* a in [2^(E-1), 2^E) */
    int e = E - 1;                                 /* 0..2 */
    double m = nearbyint(a / ldexp(1.0, e - 1));   /* in [2, 4] */
    if (m == 4.0) {
        m = 2.0;
        e += 1;
    }
    if (e + 1 > 3)
        return sign | 7;
    return sign | (uint8_t)(((e + 1) << 1) | ((int)m - 2));
}

float orc_e8m0_to_float(uint8_t c)
{
    return (float)ldexp(1.0, (int)c - 127);        /* 255 would be NaN; never produced */
}

static void put_nibble(uint8_t *q, size_t k, uint8_t v)
{
    if (k % 2 == 0)
        q[k / 2] = (uint8_t)((q[k / 2] & 0xf0) | (v & 0xf));
    else
        q[k / 2] = (uint8_t)((q[k / 2] & 0x0f) | ((v & 0xf) << 4));
}

uint8_t orc_fp4_code(const uint8_t *q, size_t k)
{
    return (k % 2 == 0) ? (q[k / 2] & 0xf) : (q[k / 2] >> 4);
}

/* MXFP4: x fp16 [R][K], K % 32 == 0 -> q [R][K/2], scales E8M0 [R][K/32]. */
int orc_quantize_mxfp4(const uint16_t *x, int R, int K, uint8_t *q, uint8_t *scales)
{
    if (R <= 0 || K <= 0 || K % 32 != 0)
        return -1;
    for (int r = 0; r < R; ++r) {
        for (int b = 0; b < K / 32; ++b) {
            const uint16_t *blk = x + (size_t)r * K + (size_t)b * 32;
            float a = 0.0f;
            for (int i = 0; i < 32; ++i) {
                float v = fabsf(orc_half_to_float(blk[i]));
                if (v > a) a = v;
            }
            int e;
            if (a == 0.0f) {
                e = -127;
            } else {
                int E;
                frexp((double)a, &E);              /* floor(log2 a) = E - 1 */
                e = (E - 1) - 2;
                if (e < -127) e = -127;
                if (e > 127) e = 127;
            }
            scales[(size_t)r * (K / 32) + b] = (uint8_t)(e + 127);
            for (int i = 0; i < 32; ++i) {
                float v = orc_half_to_float(blk[i]);
                float t = (float)ldexp((double)v, -e); /* exact: a power-of-two scaling */
                put_nibble(q + (size_t)r * (K / 2), (size_t)b * 32 + i, a == 0.0f ? 0 : orc_float_to_e2m1(t));
            }
        }
    }
    return 0;
}

/* NVFP4: x fp16 [R][K], K % 16 == 0 -> q [R][K/2], scales E4M3 [R][K/16], tensor scale [1]. */
int orc_quantize_nvfp4(const uint16_t *x, int R, int K, uint8_t *q, uint8_t *scales, float *tensor_scale)
{
    if (R <= 0 || K <= 0 || K % 16 != 0)
        return -1;
    float at = 0.0f;
    for (size_t i = 0; i < (size_t)R * K; ++i) {
        float v = fabsf(orc_half_to_float(x[i]));
        if (v > at) at = v;
    }
    if (at < 1e-8f) at = 1e-8f;
    const float S = at / 2688.0f;                  /* 6 * 448 */
    tensor_scale[0] = S;
    for (int r = 0; r < R; ++r) {
        for (int b = 0; b < K / 16; ++b) {
            const uint16_t *blk = x + (size_t)r * K + (size_t)b * 16;
            float a = 0.0f;
            for (int i = 0; i < 16; ++i) {
                float v = fabsf(orc_half_to_float(blk[i]));
                if (v > a) a = v;
            }
            const float e = (a / 6.0f) / S;
            const uint8_t sb = orc_float_to_e4m3(e);
            scales[(size_t)r * (K / 16) + b] = sb;
            const float d = orc_e4m3_to_float(sb) * S;
            for (int i = 0; i < 16; ++i) {
                float v = orc_half_to_float(blk[i]);
                put_nibble(q + (size_t)r * (K / 2), (size_t)b * 16 + i, sb == 0 ? 0 : orc_float_to_e2m1(v / d));
            }
        }
    }
    return 0;
}

/* Block-scaled FP4 GEMM reference: y[m][n] = ta * tb * sum_k dec(a[m][k]) sa(m, k/bs)
   dec(b[n][k]) sb(n, k/bs) in fp64 (bs = 32 with E8M0 scales for MXFP4, 16 with E4M3
   scales for NVFP4; ta/tb are the tensor scales, 1 for MXFP4), bound = the same with
   absolute values.  ms/ns select rows of A and B. */
void orc_gemm_fp4_ref(int nvfp4, const uint8_t *a, const uint8_t *sa, float ta, const uint8_t *b,
                      const uint8_t *sb, float tb, int M, int N, int K, const int *ms, int nm,
                      const int *ns, int nn, double *y, double *bound)
{
    const int bs = nvfp4 ? 16 : 32;
    const int nb = K / bs;
    if (!ms) nm = M;
    if (!ns) nn = N;
    for (int i = 0; i < nm; ++i) {
        int m = ms ? ms[i] : i;
        for (int j = 0; j < nn; ++j) {
            int n = ns ? ns[j] : j;
            double acc = 0.0, abs_acc = 0.0;
            for (int k = 0; k < K; ++k) {
                uint8_t ca = sa[(size_t)m * nb + k / bs], cb = sb[(size_t)n * nb + k / bs];
                double fa = nvfp4 ? (double)orc_e4m3_to_float(ca) : (double)orc_e8m0_to_float(ca);
                double fb = nvfp4 ? (double)orc_e4m3_to_float(cb) : (double)orc_e8m0_to_float(cb);
                double p = (double)orc_e2m1_to_float(orc_fp4_code(a + (size_t)m * (K / 2), k)) * fa *
                           (double)orc_e2m1_to_float(orc_fp4_code(b + (size_t)n * (K / 2), k)) * fb;
                acc += p;
                abs_acc += fabs(p);
            }
            y[(size_t)i * nn + j] = acc * (double)ta * (double)tb;
            bound[(size_t)i * nn + j] = abs_acc * (double)ta * (double)tb;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Calibration-driven INT4: GPTQ and AWQ's scaling search ([P3] "GPTQ:      */
/* rounding with error compensation", "AWQ: protect the channels that      */
/* matter" and the gptq()/awq() routines of "Measured on two real layers"; */
/* [P2] "The Mathematics": H = 2 X^T X; [P5] GPTQ and AWQ sections).        */
/* Both produce the stored INT4 format of orc_quantize_group_int4; readings:*/
/*  - a group's grid is the stored-format rule of orc_quantize_group_int4   */
/*    (range widened to contain 0, fp16 scale, zero clamped to [0,15]),     */
/*    applied to the fp32 values of the weights it quantizes;               */
/*  - GPTQ's blocks are the groups (block = group size), its per-element    */
/*    rounding is that rule's fp32 decision on the compensated weight       */
/*    rounded to fp32; compensation runs in fp64;                           */
/*  - H's damping adds damp * mean(diag H) to the diagonal.                 */
/* ------------------------------------------------------------------------ */

/* One group's stored-format grid from n fp32 values: *s16 (fp16 bits), *z. */
static void group_grid(const float *v, int n, uint16_t *s16_out, int *z_out)
{
    float lo = 0.0f, hi = 0.0f;
    for (int t = 0; t < n; ++t) {
        if (v[t] < lo) lo = v[t];
        if (v[t] > hi) hi = v[t];
    }
    uint16_t s16 = orc_float_to_half((hi - lo) / 15.0f);
    if (s16 == 0) s16 = 0x3c00;
    float s = orc_half_to_float(s16);
    *s16_out = s16;
    *z_out = clampi(rne_to_int(-lo / s), 0, 15);
}

static int group_code(float w, float s, int z)
{
    return clampi(rne_to_int(w / s) + z, 0, 15);
}

/* H = 2 X^T X in fp64, X fp16 bits [T][K]; H [K][K]. */
void orc_hessian(const uint16_t *X, int T, int K, double *H)
{
    memset(H, 0, sizeof(double) * (size_t)K * K);
    for (int t = 0; t < T; ++t)
        for (int i = 0; i < K; ++i) {
            double xi = (double)orc_half_to_float(X[(size_t)t * K + i]);
            if (xi == 0.0) continue;
            for (int j = 0; j < K; ++j)
                H[(size_t)i * K + j] += 2.0 * xi * (double)orc_half_to_float(X[(size_t)t * K + j]);
        }
}

/* In-place lower Cholesky factor of the SPD matrix A [n][n] (upper part untouched). */
static int cholesky_lower(double *A, int n)
{
    for (int j = 0; j < n; ++j) {
        double d = A[(size_t)j * n + j];
        for (int k = 0; k < j; ++k) d -= A[(size_t)j * n + k] * A[(size_t)j * n + k];
        if (!(d > 0.0)) return -1;
        d = sqrt(d);
        A[(size_t)j * n + j] = d;
        for (int i = j + 1; i < n; ++i) {
            double v = A[(size_t)i * n + j];
            for (int k = 0; k < j; ++k) v -= A[(size_t)i * n + k] * A[(size_t)j * n + k];
            A[(size_t)i * n + j] = v / d;
        }
    }
    return 0;
}

/* U = upper Cholesky factor of (H + damp * mean(diag H) * I)^{-1}: U^T U = H'^{-1}.
   Written as the inverse of H' via its Cholesky factor, then the Cholesky factor of
   that inverse.  H, U: [K][K] fp64.  Returns 0, or -1 if H' is not positive definite. */
int orc_gptq_hinv_chol(const double *H, int K, double damp, double *U)
{
    double *A = (double *)malloc(sizeof(double) * (size_t)K * K);
    double *Li = (double *)calloc((size_t)K * K, sizeof(double));
    if (!A || !Li) { free(A); free(Li); return -1; }
    double mean = 0.0;
    for (int i = 0; i < K; ++i) mean += H[(size_t)i * K + i];
    mean /= K;
    memcpy(A, H, sizeof(double) * (size_t)K * K);
    for (int i = 0; i < K; ++i) A[(size_t)i * K + i] += damp * mean;
    int rc = cholesky_lower(A, K);                 /* H' = L L^T */
    if (rc == 0) {
        /* Li = L^{-1} (lower), column by column by forward substitution */
        for (int c = 0; c < K; ++c) {
            for (int i = c; i < K; ++i) {
                double v = (i == c) ? 1.0 : 0.0;
                for (int k = c; k < i; ++k) v -= A[(size_t)i * K + k] * Li[(size_t)k * K + c];
                Li[(size_t)i * K + c] = v / A[(size_t)i * K + i];
            }
        }
        /* H'^{-1} = Li^T Li into A (full) */
        for (int i = 0; i < K; ++i)
            for (int j = 0; j < K; ++j) {
                double v = 0.0;
                for (int k = (i > j ? i : j); k < K; ++k) v += Li[(size_t)k * K + i] * Li[(size_t)k * K + j];
                A[(size_t)i * K + j] = v;
            }
        rc = cholesky_lower(A, K);                 /* H'^{-1} = C C^T, U = C^T */
        if (rc == 0)
            for (int i = 0; i < K; ++i)
                for (int j = 0; j < K; ++j)
                    U[(size_t)i * K + j] = j >= i ? A[(size_t)j * K + i] : 0.0;
    }
    free(A);
    free(Li);
    return rc;
}

/* GPTQ: W fp16 bits [N][K] -> the stored INT4 format, quantizing one column at a time within
   blocks of g columns (one group) and pushing each column's error onto the later columns through
   U (from orc_gptq_hinv_chol):
     for each block [i1, i2): grid of every row from its current (compensated) block values;
       for i in block: q = code of fl32(W[n][i]); e = (W[n][i] - (q - z) s) / U[i][i];
                       W[n][j] -= e U[i][j] for i < j < i2;  E[n][i] = e
     then W[n][j] -= sum_i E[n][i] U[i][j] for j >= i2.
   Returns 0, or -1 on bad arguments. */
int orc_gptq(const uint16_t *W, int N, int K, int g, const double *U, uint32_t *qweight,
             uint16_t *scales, uint32_t *qzeros)
{
    if (N <= 0 || K <= 0 || g <= 0 || K % g != 0 || K % 8 != 0)
        return -1;
    const int G = K / g, ZW = (G + 7) / 8;
    double *Wd = (double *)malloc(sizeof(double) * (size_t)N * K);
    double *E = (double *)malloc(sizeof(double) * (size_t)N * g);
    float *blk = (float *)malloc(sizeof(float) * (size_t)g);
    if (!Wd || !E || !blk) { free(Wd); free(E); free(blk); return -1; }
    for (size_t i = 0; i < (size_t)N * K; ++i) Wd[i] = (double)orc_half_to_float(W[i]);
    memset(qweight, 0, sizeof(uint32_t) * (size_t)N * (K / 8));
    memset(qzeros, 0, sizeof(uint32_t) * (size_t)N * ZW);
    for (int b = 0; b < G; ++b) {
        const int i1 = b * g, i2 = i1 + g;
        for (int n = 0; n < N; ++n) {
            double *row = Wd + (size_t)n * K;
            for (int t = 0; t < g; ++t) blk[t] = (float)row[i1 + t];
            uint16_t s16;
            int z;
            group_grid(blk, g, &s16, &z);
            const float s = orc_half_to_float(s16);
            scales[(size_t)n * G + b] = s16;
            qzeros[(size_t)n * ZW + b / 8] |= (uint32_t)z << (4 * (b % 8));
            for (int i = i1; i < i2; ++i) {
                const int q = group_code((float)row[i], s, z);
                qweight[(size_t)n * (K / 8) + i / 8] |= (uint32_t)q << (4 * (i % 8));
                const double e = (row[i] - (double)(q - z) * (double)s) / U[(size_t)i * K + i];
                for (int j = i + 1; j < i2; ++j) row[j] -= e * U[(size_t)i * K + j];
                E[(size_t)n * g + (i - i1)] = e;
            }
            for (int j = i2; j < K; ++j) {
                double v = 0.0;
                for (int i = i1; i < i2; ++i) v += E[(size_t)n * g + (i - i1)] * U[(size_t)i * K + j];
                row[j] -= v;
            }
        }
    }
    free(Wd);
    free(E);
    free(blk);
    return 0;
}

/* AWQ's scaling search.  mag[j] = mean_t |X[t][j]|; for each alpha of the grid:
     s_j = mag_j^alpha, s /= sqrt(max s * min s)            (fp64, then rounded to fp32)
     codes = stored-format RTN of the fp32 products W[n][j] * s_j
     D = W - dequant(codes) / s;  err(alpha) = sum_n D[n] H D[n]^T  (fp64)
   and keeps the first alpha with the smallest error.  Writes that alpha's codes,
   s [K] (fp32) and err[grid] (all errors); returns the index of the chosen alpha,
   or -1 on bad arguments. */
int orc_awq(const uint16_t *W, int N, int K, int g, const uint16_t *X, int T, const double *H,
            const double *grid, int ngrid, uint32_t *qweight, uint16_t *scales, uint32_t *qzeros,
            float *s_out, double *err)
{
    if (N <= 0 || K <= 0 || T <= 0 || ngrid <= 0 || K % g != 0 || K % 8 != 0)
        return -1;
    const int G = K / g, ZW = (G + 7) / 8;
    double *mag = (double *)calloc((size_t)K, sizeof(double));
    float *s = (float *)malloc(sizeof(float) * (size_t)K);
    float *ws = (float *)malloc(sizeof(float) * (size_t)N * K);
    uint32_t *qw = (uint32_t *)malloc(sizeof(uint32_t) * (size_t)N * (K / 8));
    uint16_t *sc = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)N * G);
    uint32_t *qz = (uint32_t *)malloc(sizeof(uint32_t) * (size_t)N * ZW);
    double *D = (double *)malloc(sizeof(double) * (size_t)K);
    double *what = (double *)malloc(sizeof(double) * (size_t)N * K);
    int best = -1;
    if (!mag || !s || !ws || !qw || !sc || !qz || !D || !what) goto done;
    for (int t = 0; t < T; ++t)
        for (int j = 0; j < K; ++j) mag[j] += fabs((double)orc_half_to_float(X[(size_t)t * K + j]));
    for (int j = 0; j < K; ++j) mag[j] /= T;
    for (int a = 0; a < ngrid; ++a) {
        double smax = 0.0, smin = INFINITY;
        double *sd = D;                             /* reuse D as the fp64 scales */
        for (int j = 0; j < K; ++j) {
            sd[j] = pow(mag[j], grid[a]);
            if (sd[j] > smax) smax = sd[j];
            if (sd[j] < smin) smin = sd[j];
        }
        const double norm = sqrt(smax * smin);
        for (int j = 0; j < K; ++j) s[j] = (float)(sd[j] / norm);
        for (int n = 0; n < N; ++n)
            for (int j = 0; j < K; ++j)
                ws[(size_t)n * K + j] = orc_half_to_float(W[(size_t)n * K + j]) * s[j];
        orc_quantize_group_int4(ws, 0, N, K, g, qw, sc, qz);
        orc_dequant_int4(qw, sc, qz, N, K, g, what);
        double e = 0.0;
        for (int n = 0; n < N; ++n) {
            for (int j = 0; j < K; ++j)
                D[j] = (double)orc_half_to_float(W[(size_t)n * K + j]) - what[(size_t)n * K + j] / (double)s[j];
            for (int i = 0; i < K; ++i) {
                if (D[i] == 0.0) continue;
                double hd = 0.0;
                for (int j = 0; j < K; ++j) hd += H[(size_t)i * K + j] * D[j];
                e += D[i] * hd;
            }
        }
        err[a] = e;
        if (best < 0 || e < err[best]) {
            best = a;
            memcpy(qweight, qw, sizeof(uint32_t) * (size_t)N * (K / 8));
            memcpy(scales, sc, sizeof(uint16_t) * (size_t)N * G);
            memcpy(qzeros, qz, sizeof(uint32_t) * (size_t)N * ZW);
            memcpy(s_out, s, sizeof(float) * (size_t)K);
        }
    }
done:
    free(mag); free(s); free(ws); free(qw); free(sc); free(qz); free(D); free(what);
    return best;
}
