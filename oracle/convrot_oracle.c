/*
 * CPU oracle for the ConvRot256 INT8 linear path.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the package's smoke check and the
 * benchmark's CPU-baseline leg may load this library. The product path (the
 * CUDA library) shares no code with it and never calls it.
 *
 * It is deliberately plain and slow: every step is written out in the order of
 * the method's definition, in IEEE single precision with round-to-nearest-even
 * and no operation fused or reordered (compile with -ffp-contract=off and
 * without -ffast-math). Where the definition is the bf16 rounding of an exact
 * real value (the input activation, the input RMSNorm), that value is
 * evaluated in double precision and rounded once. Rows are spread over OpenMP
 * threads; that changes no arithmetic, because every output element is
 * computed by one thread alone.
 *
 * Sources for what is computed:
 *  - comfy-kitchen 0.2.40 (PyPI page), "Huawei Ascend backend" and "HIP
 *    backend": quantize_int8_rowwise (dynamic per-row INT8),
 *    quantize_and_rotate_rowwise (rotation fused with the per-row quantiser),
 *    int8_linear (activation quantisation then INT8 matmul).
 *  - sglang PR "Tune Kitchen INT8 row splitting for SM120", "Accuracy Test":
 *    BF16 activations and bias, INT8 weights, FP32 row scales, ConvRot256.
 *  - ComfyUI-AppleSilicon-FP8 README, "What it fixes" table, row 17: rotate
 *    the activation online, per-row quantise it, INT8 x INT8 -> INT32, then a
 *    per-row rescale plus bias in the store epilogue; row 12: the INT32 sums
 *    stay well inside the int32 range.
 * The pages name ConvRot256 and call it a Hadamard rotation but print no
 * formula. The reading taken here: the normalised 256-point Walsh-Hadamard
 * transform (Sylvester order, no random signs), as 8 butterfly stages with
 * h = 1, 2, 4, ..., 128 followed by an exact multiply by 1/16. Scale
 * s = absmax / 127 (IEEE division), code = round-half-even(y / s) clamped to
 * [-127, 127]; an all-zero row gets s = 0 and all-zero codes. Epilogue:
 * y = bf16_rne(((float(acc) * s_x) * s_w) + float(bias)), each step rounded
 * to fp32; a missing bias adds +0.0f.
 *
 * The last section holds ConvRot NVFP4 (FP4 E2M1 codes with E4M3 block
 * scales), with its own sources and readings stated there.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ROT_N 256

/* BF16 -> fp32 is exact: the bf16 bits are the upper half of the fp32 bits. */
float oracle_bf16_to_f32(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* fp32 -> BF16 by the definition of round-to-nearest-even on the upper 16
 * bits: keep the upper half, and add one unit in its last place when the
 * discarded lower half is above one half, or exactly one half with an odd
 * kept part. Overflow carries into the exponent and gives infinity, as IEEE
 * rounding does. NaN is never produced by this path's arithmetic. */
uint16_t oracle_f32_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    uint32_t kept = u >> 16;
    uint32_t rest = u & 0xFFFFu;
    if (rest > 0x8000u || (rest == 0x8000u && (kept & 1u)))
        kept += 1u;
    return (uint16_t)kept;
}

/* ---------------------------------------------------------------- input_act
 * comfy-kitchen 0.2.40, "HIP backend": int8_linear(input_act=...) applies an
 * activation to the linear's input inside the quantiser's load, so
 * linear(act(proj(x))) never stores act's output. The pages do not list the
 * activations nor their formulas; the readings taken: relu, silu
 * x / (1 + e^-x) and the tanh form of gelu
 * 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3))). Each bf16 input x becomes
 * the bf16 value nearest to the exact act(x) (ties to even), which is what an
 * unfused activation stored in bf16 would hold at best; that value then goes
 * through the rotation and the quantiser.
 *
 * The exact value is evaluated here in double precision (libm exp), the gelu
 * as x / (1 + e^(-2u)), u = sqrt(2/pi) (x + 0.044715 x^3): the same number as
 * 0.5 x (1 + tanh(u)) without its cancellation where tanh(u) is near -1.
 * Rounding the double result once to bf16 gives the exact value's bf16
 * rounding unless that value lies within the double evaluation's error
 * (about |2u| * 2^-52 relative) of a rounding midpoint. For x != 0 act(x) is
 * transcendental and never a midpoint itself. One case needs care: for
 * |x| < 2^-120 the double evaluation returns x/2 exactly (1 + e^-x rounds to
 * 2), which can be a midpoint between two bf16 subnormals, while the exact
 * value is strictly above x/2 (act(x) - x/2 = x (sigma(.) - 1/2) > 0, with
 * sigma(.) - 1/2 of the sign of x) by less than x^2 / 2, far below the
 * spacing; so there x/2 is rounded with ties going up. */
#define ACT_NONE 0
#define ACT_RELU 1
#define ACT_SILU 2
#define ACT_GELU_TANH 3

/* float64 -> bf16 by the definition of round-to-nearest-even, from the double
 * value directly (no intermediate fp32 rounding): bf16 keeps 8 significant
 * bits, with spacing 2^(e-8) for |v| in [2^(e-1), 2^e) and 2^-133 below
 * 2^-126 (subnormals); |v| at or above 2^128 - 2^119 overflows to infinity. */
uint16_t oracle_f64_to_bf16_rne(double v) {
    uint16_t sign = signbit(v) ? 0x8000u : 0u;
    double a = fabs(v);
    if (a != a)
        return 0x7FC0u;
    if (a == 0.0)
        return sign;
    if (isinf(a))
        return (uint16_t)(sign | 0x7F80u);
    int e;
    frexp(a, &e); /* a = f * 2^e, f in [0.5, 1) */
    int qe = e - 8;
    if (qe < -133)
        qe = -133;
    double q = nearbyint(ldexp(a, -qe)); /* exact scaling, then ties to even */
    double r = ldexp(q, qe);
    if (r >= 0x1p128)
        return (uint16_t)(sign | 0x7F80u);
    float f = (float)r; /* exact: r has at most 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(sign | (u >> 16));
}

double oracle_act_f64(int act, double x) {
    switch (act) {
    case ACT_RELU:
        return x > 0.0 ? x : 0.0;
    case ACT_SILU:
        return x / (1.0 + exp(-x));
    case ACT_GELU_TANH: {
        double u = sqrt(2.0 / 3.14159265358979323846) * (x + 0.044715 * (x * x * x));
        return x / (1.0 + exp(-2.0 * u));
    }
    default:
        return x;
    }
}

/* The activation of one bf16 input, as bf16 bits. */
uint16_t oracle_act_bf16(int act, uint16_t xb) {
    double x = (double)oracle_bf16_to_f32(xb);
    if (act == ACT_NONE)
        return xb;
    if ((act == ACT_SILU || act == ACT_GELU_TANH) && x != 0.0 && fabs(x) < 0x1p-120) {
        double t = ldexp(x / 2.0, 133); /* x/2 in units of the subnormal spacing */
        double lo = floor(t);
        double q = (t - lo == 0.5) ? lo + 1.0 : nearbyint(t);
        return oracle_f64_to_bf16_rne(copysign(ldexp(q, -133), x)); /* -0 stays -0 */
    }
    return oracle_f64_to_bf16_rne(oracle_act_f64(act, x));
}

void oracle_act_bf16_array(int act, const uint16_t *x, int64_t n, uint16_t *y) {
    for (int64_t i = 0; i < n; ++i)
        y[i] = oracle_act_bf16(act, x[i]);
}

/* ConvRot256 on one block of 256 values, in place. */
void oracle_rot256(float *v) {
    for (int h = 1; h < ROT_N; h <<= 1) {
        for (int i = 0; i < ROT_N; ++i) {
            if ((i & h) == 0) {
                float a = v[i];
                float c = v[i + h];
                v[i] = a + c;
                v[i + h] = a - c;
            }
        }
    }
    for (int i = 0; i < ROT_N; ++i)
        v[i] = v[i] * 0.0625f;
}

/* Dynamic symmetric per-row quantisation of one row y[0..K) to codes in
 * [-qmax, qmax]: qmax = 127 for INT8, 7 for signed INT4 (codes kept in int8
 * storage). */
void oracle_quant_row_q(const float *y, int64_t K, float qmax, int8_t *q, float *s_out);

/* Dynamic symmetric per-row INT8 quantisation of one row y[0..K). */
void oracle_quant_row(const float *y, int64_t K, int8_t *q, float *s_out) {
    oracle_quant_row_q(y, K, 127.0f, q, s_out);
}

void oracle_quant_row_q(const float *y, int64_t K, float qmax, int8_t *q, float *s_out) {
    float amax = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
        float a = fabsf(y[k]);
        if (a > amax)
            amax = a;
    }
    float s = amax / qmax;
    *s_out = s;
    if (amax == 0.0f) {
        memset(q, 0, (size_t)K);
        return;
    }
    for (int64_t k = 0; k < K; ++k) {
        float t = y[k] / s;
        float r = nearbyintf(t); /* default rounding mode: ties to even */
        if (r > qmax)
            r = qmax;
        if (r < -qmax)
            r = -qmax;
        q[k] = (int8_t)r;
    }
}

/* quantize_and_rotate_rowwise on BF16 rows: widen, ConvRot256 every 256-block
 * of the row, then quantise the whole rotated row. X has row stride ldx
 * (elements). rotate == 0 skips the rotation (plain quantize_int8_rowwise). */
int oracle_quantize_rows_bf16_act(const uint16_t *X, int64_t M, int64_t K, int64_t ldx,
                                  int rotate, int act, int8_t *Qx, float *s_x);

int oracle_quantize_rows_bf16(const uint16_t *X, int64_t M, int64_t K, int64_t ldx,
                              int rotate, int8_t *Qx, float *s_x) {
    return oracle_quantize_rows_bf16_act(X, M, K, ldx, rotate, ACT_NONE, Qx, s_x);
}

int oracle_quantize_rows_bf16_q(const uint16_t *X, int64_t M, int64_t K, int64_t ldx,
                                int rotate, int act, float qmax, int8_t *Qx, float *s_x);

/* The same, with the input activation applied first (ACT_NONE: none). */
int oracle_quantize_rows_bf16_act(const uint16_t *X, int64_t M, int64_t K, int64_t ldx,
                                  int rotate, int act, int8_t *Qx, float *s_x) {
    return oracle_quantize_rows_bf16_q(X, M, K, ldx, rotate, act, 127.0f, Qx, s_x);
}

/* ... and with codes in [-qmax, qmax] (7: convrot_w4a4_linear's INT4). */
int oracle_quantize_rows_bf16_q(const uint16_t *X, int64_t M, int64_t K, int64_t ldx,
                                int rotate, int act, float qmax, int8_t *Qx, float *s_x) {
    if (K % ROT_N != 0 || ldx < K)
        return 1;
    int err = 0;
#pragma omp parallel
    {
        float *buf = (float *)malloc((size_t)K * sizeof(float));
        if (!buf) {
#pragma omp atomic write
            err = 2;
        } else {
#pragma omp for schedule(static)
            for (int64_t m = 0; m < M; ++m) {
                const uint16_t *row = X + m * ldx;
                for (int64_t k = 0; k < K; ++k) {
                    buf[k] = oracle_bf16_to_f32(oracle_act_bf16(act, row[k]));
                }
                if (rotate)
                    for (int64_t b = 0; b < K; b += ROT_N)
                        oracle_rot256(buf + b);
                oracle_quant_row_q(buf, K, qmax, Qx + m * K, s_x + m);
            }
            free(buf);
        }
    }
    return err;
}

/* Offline weight preparation: fp32 W [N,K] (row stride K), rotated along K
 * with the same ConvRot256, then quantised per output row. */
int oracle_rotate_quant_weight(const float *W, int64_t N, int64_t K, int8_t *Qw, float *s_w) {
    if (K % ROT_N != 0)
        return 1;
    int err = 0;
#pragma omp parallel
    {
        float *buf = (float *)malloc((size_t)K * sizeof(float));
        if (!buf) {
#pragma omp atomic write
            err = 2;
        } else {
#pragma omp for schedule(static)
            for (int64_t n = 0; n < N; ++n) {
                memcpy(buf, W + n * K, (size_t)K * sizeof(float));
                for (int64_t b = 0; b < K; b += ROT_N)
                    oracle_rot256(buf + b);
                oracle_quant_row(buf, K, Qw + n * K, s_w + n);
            }
            free(buf);
        }
    }
    return err;
}

/* convrot_w4a4_linear's weights (comfy-kitchen 0.2.40, "Huawei Ascend
 * backend": ConvRot then signed INT4 quantisation; packed weights are
 * unpacked to INT8 for INT32 accumulation): each fp32 row rotated, quantised
 * to [-7, 7] with s = absmax / 7, then packed two codes per byte, element 2j
 * in the low nibble and 2j + 1 in the high nibble, each nibble the 4-bit
 * two's complement of its code (the packing order is a reading). */
int oracle_rotate_quant_weight_int4(const float *W, int64_t N, int64_t K, uint8_t *Qw4,
                                    float *s_w) {
    if (K % ROT_N != 0)
        return 1;
    int err = 0;
#pragma omp parallel
    {
        float *buf = (float *)malloc((size_t)K * sizeof(float));
        int8_t *q = (int8_t *)malloc((size_t)K);
        if (!buf || !q) {
#pragma omp atomic write
            err = 2;
        } else {
#pragma omp for schedule(static)
            for (int64_t n = 0; n < N; ++n) {
                memcpy(buf, W + n * K, (size_t)K * sizeof(float));
                for (int64_t b = 0; b < K; b += ROT_N)
                    oracle_rot256(buf + b);
                oracle_quant_row_q(buf, K, 7.0f, q, s_w + n);
                for (int64_t j = 0; j < K / 2; ++j)
                    Qw4[n * (K / 2) + j] =
                        (uint8_t)(((uint8_t)q[2 * j] & 0xFu) | (((uint8_t)q[2 * j + 1] & 0xFu) << 4));
            }
        }
        free(buf);
        free(q);
    }
    return err;
}

/* Packed INT4 [rows, K/2] -> int8 codes [rows, K] (sign-extended nibbles). */
void oracle_unpack_int4(const uint8_t *Q4, int64_t rows, int64_t K, int8_t *Q8) {
    for (int64_t i = 0; i < rows * (K / 2); ++i) {
        int lo = Q4[i] & 0xF, hi = Q4[i] >> 4;
        Q8[2 * i] = (int8_t)(lo >= 8 ? lo - 16 : lo);
        Q8[2 * i + 1] = (int8_t)(hi >= 8 ? hi - 16 : hi);
    }
}

/* dequantize_int8_simple / dequantize_int8_simple_dtype (comfy-kitchen 0.2.40,
 * "Huawei Ascend backend"): y = float(q) * s, one fp32 rounding, with s one
 * scale for the tensor (per_row == 0: s[0]) or one per row (s[m]); the dtype
 * form rounds y to bf16. Yf and/or Yb may be NULL. (Readings: the page lists
 * the names only.) */
void oracle_dequantize_int8(const int8_t *Q, const float *s, int64_t rows, int64_t K, int per_row,
                            float *Yf, uint16_t *Yb) {
    for (int64_t m = 0; m < rows; ++m) {
        float sc = per_row ? s[m] : s[0];
        for (int64_t k = 0; k < K; ++k) {
            float y = (float)Q[m * K + k] * sc;
            if (Yf)
                Yf[m * K + k] = y;
            if (Yb)
                Yb[m * K + k] = oracle_f32_to_bf16_rne(y);
        }
    }
}

/* quantize_int8_tensorwise (same page): one scale s = absmax(X) / 127 for the
 * whole tensor, q = round-half-even(x / s) clamped to [-127, 127]; a zero
 * tensor gets s = 0 and zero codes. No rotation. */
void oracle_quantize_int8_tensorwise(const uint16_t *X, int64_t M, int64_t K, int64_t ldx,
                                     int8_t *Q, float *s_out) {
    float amax = 0.0f;
    for (int64_t m = 0; m < M; ++m)
        for (int64_t k = 0; k < K; ++k) {
            float a = fabsf(oracle_bf16_to_f32(X[m * ldx + k]));
            if (a > amax)
                amax = a;
        }
    float s = amax / 127.0f;
    *s_out = s;
    for (int64_t m = 0; m < M; ++m)
        for (int64_t k = 0; k < K; ++k) {
            float r = 0.0f;
            if (amax != 0.0f) {
                r = nearbyintf(oracle_bf16_to_f32(X[m * ldx + k]) / s);
                if (r > 127.0f)
                    r = 127.0f;
                if (r < -127.0f)
                    r = -127.0f;
            }
            Q[m * K + k] = (int8_t)r;
        }
}

/* acc[m][n] = sum_k Qx[m][k] * Qw[n][k], exact in int32 while K * 127^2 < 2^31. */
void oracle_gemm_i32(const int8_t *Qx, const int8_t *Qw, int64_t M, int64_t N, int64_t K,
                     int32_t *acc) {
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        const int8_t *a = Qx + m * K;
        for (int64_t n = 0; n < N; ++n) {
            const int8_t *b = Qw + n * K;
            int32_t s = 0;
            for (int64_t k = 0; k < K; ++k)
                s += (int32_t)a[k] * (int32_t)b[k];
            acc[m * N + n] = s;
        }
    }
}

/* Y[m][n] = bf16_rne(((float(acc) * s_x[m]) * s_w[n]) + float(bias[n])). */
static uint16_t epilogue_one(int32_t acc, float sx, float sw, float b) {
    float f = (float)acc; /* int32 -> fp32, round to nearest even */
    f = f * sx;
    f = f * sw;
    f = f + b;
    return oracle_f32_to_bf16_rne(f);
}

void oracle_epilogue(const int32_t *acc, const float *s_x, const float *s_w, const uint16_t *bias,
                     int64_t M, int64_t N, uint16_t *Y) {
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            float b = bias ? oracle_bf16_to_f32(bias[n]) : 0.0f;
            Y[m * N + n] = epilogue_one(acc[m * N + n], s_x[m], s_w[n], b);
        }
}

/* Rows of the linear computed one by one from already-quantised activations:
 * Y_rows[i][n] for row index rows[i] of Qx. Used to check sampled rows of a
 * full-size output without forming the whole INT32 product. */
void oracle_linear_rows(const int8_t *Qx, const float *s_x, const int8_t *Qw, const float *s_w,
                        const uint16_t *bias, int64_t N, int64_t K, const int64_t *rows,
                        int64_t nrows, uint16_t *Y_rows) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < nrows; ++i) {
        const int8_t *a = Qx + rows[i] * K;
        for (int64_t n = 0; n < N; ++n) {
            const int8_t *b = Qw + n * K;
            int32_t s = 0;
            for (int64_t k = 0; k < K; ++k)
                s += (int32_t)a[k] * (int32_t)b[k];
            float bb = bias ? oracle_bf16_to_f32(bias[n]) : 0.0f;
            Y_rows[i * N + n] = epilogue_one(s, s_x[rows[i]], s_w[n], bb);
        }
    }
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ============================================================ input RMSNorm
 * comfy-kitchen 0.2.40 (PyPI page), "Huawei Ascend backend": int8_linear
 * accepts the input RMSNorm and residual arguments and applies them with the
 * shared device-side helpers, apart from its GEMM. The page prints no
 * formula. The reading here is the usual add-then-normalise form:
 *   h   = bf16_rne(fl32(x + r))   the residual add as a bf16 tensor addition
 *                                 stores it (h = x when there is no residual);
 *                                 the residual output is h
 *   y_k = the bf16 value nearest to h_k g_k / sqrt(mean_k(h_k^2) + eps)
 *         (ties to even; without g, g_k = 1), the exact real value.
 * The exact value is evaluated in double precision: every h_k^2 and h_k g_k
 * is exact in double (8-bit significands), the sum of squares is
 * compensated (Neumaier's variant of Kahan summation, error about 2^-52
 * relative), then one division, one square root and two products. Where
 * that value lies within 2^-34 (relative) of a bf16 rounding midpoint, both
 * neighbours count as correct: an evaluation in double precision whose sum
 * of squares runs in any order (relative error below K 2^-53 <= 2^-36 for
 * K <= 2^17) may land on either side. Yalt receives the other neighbour for
 * those elements and y itself elsewhere. eps must be > 0 (a zero row then
 * gives y = 0). */
static double sum_squares_bf16(const uint16_t *h, int64_t K) {
    double s = 0.0, c = 0.0;
    for (int64_t k = 0; k < K; ++k) {
        double v = (double)oracle_bf16_to_f32(h[k]);
        double t = v * v; /* exact */
        double n = s + t;
        if (fabs(s) >= fabs(t))
            c += (s - n) + t;
        else
            c += (t - n) + s;
        s = n;
    }
    return s + c;
}

/* Round v to bf16 and report the other neighbour when v lies within
 * tol * |v| of the midpoint between the two (alt = the rounding otherwise). */
static uint16_t bf16_round_with_alt(double v, double tol, uint16_t *alt) {
    uint16_t r = oracle_f64_to_bf16_rne(v);
    *alt = r;
    double rv = (double)oracle_bf16_to_f32(r);
    if (rv == v || isinf(rv))
        return r;
    /* the neighbour on v's other side of r */
    uint16_t o = (uint16_t)((fabs(v) > fabs(rv)) ? r + 1u : r - 1u);
    if (fabs(rv) == 0.0)
        o = (uint16_t)((v > 0) ? 0x0001u : 0x8001u);
    double ov = (double)oracle_bf16_to_f32(o);
    double mid = 0.5 * (rv + ov); /* exact: both have 8 significant bits */
    if (fabs(v - mid) <= tol * fabs(v))
        *alt = o;
    return r;
}

int oracle_rmsnorm_rows(const uint16_t *X, int64_t ldx, const uint16_t *R, int64_t ldr,
                        const uint16_t *g, float eps, int64_t M, int64_t K, uint16_t *Y,
                        uint16_t *Rout, uint16_t *Yalt) {
    if (K % ROT_N != 0) return -1;
    int err = 0;
#pragma omp parallel
    {
        uint16_t *h = (uint16_t *)malloc((size_t)K * sizeof(uint16_t));
        if (!h) {
#pragma omp atomic write
            err = -2;
        }
#pragma omp for schedule(static)
        for (int64_t m = 0; m < M; ++m) {
            if (!h) continue;
            for (int64_t k = 0; k < K; ++k) {
                float x = oracle_bf16_to_f32(X[m * ldx + k]);
                h[k] = R ? oracle_f32_to_bf16_rne(x + oracle_bf16_to_f32(R[m * ldr + k]))
                         : X[m * ldx + k];
            }
            if (Rout)
                for (int64_t k = 0; k < K; ++k) Rout[m * K + k] = h[k];
            double ss = sum_squares_bf16(h, K);
            double inv = 1.0 / sqrt(ss / (double)K + (double)eps);
            for (int64_t k = 0; k < K; ++k) {
                double v = (double)oracle_bf16_to_f32(h[k]);
                if (g) v = v * (double)oracle_bf16_to_f32(g[k]);
                v = v * inv;
                uint16_t a;
                Y[m * K + k] = bf16_round_with_alt(v, 0x1p-34, &a);
                if (Yalt) Yalt[m * K + k] = a;
            }
        }
        free(h);
    }
    return err;
}

/* ===================================================================== NVFP4
 * ConvRot NVFP4 (ComfyUI-HSWQ-Loader-and-Tools, "NVFP4 torch.compile Fix",
 * section 5-1, nvfp4_gemm.py): FP4 E2M1 codes with one scale per 16 values
 * along K, the block scales kept in the cuBLAS 128 x 4 blocked layout that
 * from_blocked undoes, and a per-tensor scale; dequantisation is the code's
 * value times (per-tensor scale x block scale), and the linear is
 * a_dq @ w_dq.T (+ bias). The pages print no quantiser; the reading here is
 * the usual two-level NVFP4 one, on the ConvRot256-rotated rows:
 *   s_t = amax(tensor) / 2688            (6 = largest E2M1, 448 = largest E4M3)
 *   b   = E4M3_rne_sat((amax(block) / 6) / s_t)       (0 when s_t == 0)
 *   d   = float(b) * s_t
 *   q   = E2M1_rne_sat(y / d)            (+0 when d == 0)
 * Two codes per byte, element 2j in the low nibble (the tensor cores' order;
 * the page's decoder also reads the high nibble first, hi_first). */

/* E2M1: sign bit 3, exponent bits 2-1 (bias 1), mantissa bit 0; exponent 0
 * holds 0 and 0.5. Values 0, 0.5, 1, 1.5, 2, 3, 4, 6 and their negatives. */
float oracle_e2m1_to_f32(uint8_t c) {
    int s = (c >> 3) & 1, e = (c >> 1) & 3, m = c & 1;
    float mag = (e == 0) ? 0.5f * (float)m : ldexpf(1.0f + 0.5f * (float)m, e - 1);
    return s ? -mag : mag;
}

/* Nearest E2M1 value, ties to the even mantissa, magnitudes above 6 saturate
 * to 6; the sign is kept (a negative value that rounds to zero gives -0).
 * The distances to the two nearest candidates are exact (Sterbenz), so ties
 * are seen exactly. */
uint8_t oracle_f32_to_e2m1_rne(float v) {
    uint8_t sign = signbit(v) ? 8u : 0u;
    float a = fabsf(v);
    if (a >= 6.0f)
        return (uint8_t)(sign | 7u);
    uint8_t best = 0;
    float bestd = a;
    for (uint8_t c = 1; c < 8; ++c) {
        float d = fabsf(a - oracle_e2m1_to_f32(c));
        if (d < bestd || (d == bestd && (c & 1u) == 0)) {
            best = c;
            bestd = d;
        }
    }
    return (uint8_t)(sign | best);
}

/* E4M3 (the finite-only variant): sign bit 7, exponent bits 6-3 (bias 7),
 * mantissa bits 2-0; exponent 0 is subnormal (m * 2^-9); largest 448. */
float oracle_e4m3_to_f32(uint8_t b) {
    int s = (b >> 7) & 1, e = (b >> 3) & 15, m = b & 7;
    float mag = (e == 0) ? ldexpf((float)m, -9) : ldexpf(1.0f + (float)m / 8.0f, e - 7);
    return s ? -mag : mag;
}

/* Non-negative v to the nearest E4M3 value, ties to the even mantissa,
 * saturating at 448: with 2^E the leading power of two of v (E >= -6, the
 * subnormals sharing the spacing of the first binade), the spacing is
 * u = 2^(E-3), v / u is exact and rounding it to the nearest even integer k
 * gives the value k * u. */
uint8_t oracle_f32_to_e4m3_rne(float v) {
    if (!(v > 0.0f))
        return 0;
    if (v >= 448.0f)
        return 0x7E;
    int e;
    frexpf(v, &e);
    int E = e - 1;
    if (E < -6)
        E = -6;
    float u = ldexpf(1.0f, E - 3);
    float k = nearbyintf(v / u);
    float r = k * u;
    if (r == 0.0f)
        return 0;
    frexpf(r, &e);
    E = e - 1;
    if (E < -6)
        return (uint8_t)(r / ldexpf(1.0f, -9)); /* subnormal: m * 2^-9 */
    int m = (int)(r / ldexpf(1.0f, E - 3)) - 8;
    return (uint8_t)(((E + 7) << 3) | m);
}

/* Byte offset of the scale of row r, scale column c (= k / 16) among C
 * columns, in the blocked layout: 512-byte tiles of 128 rows x 4 columns,
 * tiles in row-block-major order with the column blocks fastest; inside a
 * tile, rows r, r + 32, r + 64, r + 96 share the 16-byte line r % 32. */
int64_t oracle_nvfp4_sf_offset(int64_t r, int64_t c, int64_t C) {
    int64_t tiles_c = (C + 3) / 4;
    int64_t tile = (r / 128) * tiles_c + c / 4;
    return tile * 512 + (r % 32) * 16 + ((r % 128) / 32) * 4 + c % 4;
}

/* Bytes of the blocked scales of a [R, K] tensor (rows padded to 128, scale
 * columns to 4; padding bytes are zero). */
int64_t oracle_nvfp4_sf_bytes(int64_t R, int64_t K) {
    return ((R + 127) / 128) * 128 * (((K / 16) + 3) / 4) * 4;
}

static void nvfp4_load_rotated(const void *X, int bf16, int64_t ldx, int64_t r, int64_t K,
                               float *buf) {
    for (int64_t k = 0; k < K; ++k)
        buf[k] = bf16 ? oracle_bf16_to_f32(((const uint16_t *)X)[r * ldx + k])
                      : ((const float *)X)[r * ldx + k];
    for (int64_t b = 0; b < K; b += ROT_N)
        oracle_rot256(buf + b);
}

/* ConvRot NVFP4 quantisation of R rows (bf16 when bf16 != 0, else fp32) with
 * row stride ldx: Q [R, K/2] packed codes, S the blocked block scales
 * (oracle_nvfp4_sf_bytes(R, K) bytes), *s_t the per-tensor scale. Two passes
 * over the rows: the tensor's absmax first, then the codes. */
static int nvfp4_rows(const void *X, int bf16, int64_t R, int64_t K, int64_t ldx, uint8_t *Q,
                      uint8_t *S, float *s_t_out) {
    if (K % ROT_N != 0 || ldx < K)
        return 1;
    float amax = 0.0f;
    int err = 0;
#pragma omp parallel reduction(max : amax)
    {
        float *buf = (float *)malloc((size_t)K * sizeof(float));
        if (!buf) {
#pragma omp atomic write
            err = 2;
        } else {
#pragma omp for schedule(static)
            for (int64_t r = 0; r < R; ++r) {
                nvfp4_load_rotated(X, bf16, ldx, r, K, buf);
                for (int64_t k = 0; k < K; ++k)
                    if (fabsf(buf[k]) > amax)
                        amax = fabsf(buf[k]);
            }
            free(buf);
        }
    }
    if (err)
        return err;
    const float s_t = amax / 2688.0f;
    *s_t_out = s_t;
    const int64_t C = K / 16;
    memset(S, 0, (size_t)oracle_nvfp4_sf_bytes(R, K));
#pragma omp parallel
    {
        float *buf = (float *)malloc((size_t)K * sizeof(float));
        if (!buf) {
#pragma omp atomic write
            err = 2;
        } else {
#pragma omp for schedule(static)
            for (int64_t r = 0; r < R; ++r) {
                nvfp4_load_rotated(X, bf16, ldx, r, K, buf);
                uint8_t *q = Q + r * (K / 2);
                memset(q, 0, (size_t)(K / 2));
                for (int64_t c = 0; c < C; ++c) {
                    const float *y = buf + 16 * c;
                    float ab = 0.0f;
                    for (int i = 0; i < 16; ++i)
                        if (fabsf(y[i]) > ab)
                            ab = fabsf(y[i]);
                    uint8_t b = 0;
                    if (s_t > 0.0f) {
                        float t = ab / 6.0f;
                        t = t / s_t;
                        b = oracle_f32_to_e4m3_rne(t);
                    }
                    S[oracle_nvfp4_sf_offset(r, c, C)] = b;
                    const float d = oracle_e4m3_to_f32(b) * s_t;
                    for (int i = 0; i < 16; ++i) {
                        uint8_t code = 0;
                        if (d != 0.0f)
                            code = oracle_f32_to_e2m1_rne(y[i] / d);
                        int64_t k = 16 * c + i;
                        q[k / 2] = (uint8_t)(q[k / 2] | (code << (4 * (k & 1))));
                    }
                }
            }
            free(buf);
        }
    }
    return err;
}

int oracle_quantize_rotate_nvfp4_bf16(const uint16_t *X, int64_t M, int64_t K, int64_t ldx,
                                      uint8_t *Q, uint8_t *S, float *s_t) {
    return nvfp4_rows(X, 1, M, K, ldx, Q, S, s_t);
}

int oracle_rotate_quant_weight_nvfp4(const float *W, int64_t N, int64_t K, uint8_t *Q,
                                     uint8_t *S, float *s_t) {
    return nvfp4_rows(W, 0, N, K, K, Q, S, s_t);
}

/* Dequantisation as the page's decoder does it, in fp32: value =
 * e2m1(code) * (s_t * e4m3(block scale)); hi_first reads the high nibble of
 * each byte as the first of its two elements. */
void oracle_dequantize_nvfp4(const uint8_t *Q, const uint8_t *S, float s_t, int64_t R, int64_t K,
                             int hi_first, float *out) {
    const int64_t C = K / 16;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; ++r)
        for (int64_t k = 0; k < K; ++k) {
            uint8_t byte = Q[r * (K / 2) + k / 2];
            int first = (k & 1) == 0;
            uint8_t code = (first == hi_first) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 15u);
            float scale = s_t * oracle_e4m3_to_f32(S[oracle_nvfp4_sf_offset(r, k / 16, C)]);
            out[r * K + k] = oracle_e2m1_to_f32(code) * scale;
        }
}

/* Rows of the NVFP4 linear: for each listed row m of A and every n,
 * acc = sum_k (e2m1(qa) e4m3(ba)) (e2m1(qw) e4m3(bw)) summed in double (each
 * term is exact), Y = bf16_rne(fl(fl(float(acc) * alpha) + bias)) with
 * alpha = fl(s_ta * s_tw); mag = sum_k |term| * alpha (for error bounds of a
 * float accumulation). */
void oracle_nvfp4_linear_rows(const uint8_t *Qa, const uint8_t *Sa, float s_ta, int64_t M,
                              const uint8_t *Qw, const uint8_t *Sw, float s_tw, int64_t N,
                              const uint16_t *bias, int64_t K, const int64_t *rows, int64_t nrows,
                              uint16_t *Y, double *mag) {
    const int64_t C = K / 16;
    const float alpha = s_ta * s_tw;
    (void)M;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < nrows; ++i) {
        const int64_t m = rows[i];
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0, am = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                uint8_t ca = (uint8_t)((Qa[m * (K / 2) + k / 2] >> (4 * (k & 1))) & 15u);
                uint8_t cw = (uint8_t)((Qw[n * (K / 2) + k / 2] >> (4 * (k & 1))) & 15u);
                double a = (double)oracle_e2m1_to_f32(ca) *
                           (double)oracle_e4m3_to_f32(Sa[oracle_nvfp4_sf_offset(m, k / 16, C)]);
                double w = (double)oracle_e2m1_to_f32(cw) *
                           (double)oracle_e4m3_to_f32(Sw[oracle_nvfp4_sf_offset(n, k / 16, C)]);
                acc += a * w;
                am += fabs(a * w);
            }
            float f = (float)acc;
            f = f * alpha;
            f = f + (bias ? oracle_bf16_to_f32(bias[n]) : 0.0f);
            Y[i * N + n] = oracle_f32_to_bf16_rne(f);
            if (mag)
                mag[i * N + n] = am * (double)alpha;
        }
    }
}
