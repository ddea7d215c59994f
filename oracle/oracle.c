/*
 * CPU oracle for the Hadamard-rotated ("ConvRot") INT8 linear layer.
 *
 * TEST INFRASTRUCTURE. This file is the slow, plain reference that the CUDA
 * library is checked against. Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load it; the product path never does.
 * It shares no code, header, table or helper with the CUDA library.
 *
 * Build: gcc -std=c11 -O2 -ffp-contract=off -fno-fast-math -fopenmp -shared -fPIC
 * (contraction off: every fp32 operation below is one IEEE-754 round-to-nearest-even
 * step, in the order written). OpenMP is used only across independent rows, so the
 * results do not depend on the thread count.
 *
 * Sources (web pages on the method; cited by page title and section):
 *  [CR]   "ConvRot / Hadamard SDNQ" (SimpleTuner docs): Quick Setup, What The Options Do,
 *         PEFT Behavior.
 *  [SD]   "SDNQ: SD.Next Quantization Engine" (README): feature list (Hadamard on both
 *         quantized weights and quantized matmul; INT8 quantized matmul), SDNQConfig example
 *         (group_size -1 = row-wise; hadamard_group_size; dequantize_fp32 = FP32 scales and
 *         FP32 de-quant steps).
 *  [HS]   "Hybrid-Sensitivity-Weighted-Quantization" README: Rigorous grid / pack simulation
 *         (ConvRot = Hadamard rotate, then channelwise absmax onto the symmetric INT8 grid).
 *
 * Readings taken where the pages are silent (each one is listed in the design notes):
 *  - H_g is the Sylvester Hadamard matrix in natural order, H[i][j] = (-1)^popcount(i&j),
 *    applied block-diagonally along K in groups of g columns, normalised by 1/sqrt(g).
 *  - The butterfly runs in fp32 with stages h = 1, 2, 4, ..., g/2 in that order; each
 *    stage replaces (a, b) = (v[j], v[j+h]) for (j & h) == 0 by (a + b, a - b).
 *  - Codes come from the unnormalised rotation z; the 1/sqrt(g) factor is folded into the
 *    stored scale: s = fp32(amax / 127) * fp32(1/sqrt(g)).
 *  - Scale granularity: one scale per row of the operand (full row for weights, per token
 *    for activations), absmax over all K/g groups of the row.
 *  - Rounding to integer is half-to-even on the IEEE fp32 quotient z / s_z; codes are
 *    clamped to the symmetric range [-127, 127]. An all-zero row gives s = 0 and codes 0.
 *  - Epilogue, fp32: t = s_x*s_w; v = float(acc)*t; v = v + bias; v = v + lora_scale*L;
 *    out = bf16_rne(v).
 *  - LoRA: u = bf16_rne(sum_k x*A) summed in fp64; L = fp32(sum_r u*B) summed in fp64;
 *    x is the unrotated bf16 input (the adapter sits beside the frozen base, [CR] PEFT
 *    Behavior).
 *  - GELU (MLP glue between the up and down projections): exact erf form
 *    x * Phi(x) = 0.5 * x * erfc(-x / sqrt(2)) in fp64, rounded once to bf16.
 *  - Input gradient of the frozen base: dy * sW quantized per token (no rotation on that
 *    operand), int8 matmul against the stored codes, then v = fp32(acc) * s, the fp32
 *    butterfly, times fp32(1/sqrt(g)), bf16_rne.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_ERR_ARG 1
#define ORACLE_ERR_NOMEM 2

/* ---- bf16 <-> binary32 / binary64, written out from the IEEE-754 formats ---- */

static float bf16_bits_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16; /* bf16 is the top half of a binary32 */
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* binary32 -> bf16, round to nearest, ties to even. */
static uint16_t f32_to_bf16_rne(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7fffffffu) > 0x7f800000u) /* NaN: keep it a quiet NaN */
        return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

/* binary64 -> bf16 with a single rounding (nearest, ties to even). */
static uint16_t f64_to_bf16_rne(double d)
{
    if (isnan(d))
        return 0x7fc0u;
    uint16_t sign = signbit(d) ? 0x8000u : 0u;
    if (isinf(d))
        return (uint16_t)(sign | 0x7f80u);
    double a = fabs(d);
    double r;
    if (a < 0x1p-126) {
        /* bf16 subnormal range: the grid step is 2^-133 */
        r = nearbyint(a * 0x1p133) * 0x1p-133;
    } else {
        /* keep 1 + 7 significand bits: drop the low 45 of binary64's 52 */
        uint64_t u;
        memcpy(&u, &a, sizeof u);
        uint64_t lsb = (u >> 45) & 1u;
        u += (((uint64_t)1) << 44) - 1u + lsb;
        u &= ~((((uint64_t)1) << 45) - 1u);
        memcpy(&r, &u, sizeof r);
    }
    float f = (float)r; /* exact (8 significant bits), or +inf past the bf16 range */
    uint32_t fu;
    memcpy(&fu, &f, sizeof fu);
    return (uint16_t)(sign | (uint16_t)(fu >> 16));
}

void oracle_bf16_to_f32(const uint16_t *in, int64_t n, float *out)
{
    for (int64_t i = 0; i < n; i++)
        out[i] = bf16_bits_to_f32(in[i]);
}

void oracle_f32_to_bf16(const float *in, int64_t n, uint16_t *out)
{
    for (int64_t i = 0; i < n; i++)
        out[i] = f32_to_bf16_rne(in[i]);
}

void oracle_f64_to_bf16(const double *in, int64_t n, uint16_t *out)
{
    for (int64_t i = 0; i < n; i++)
        out[i] = f64_to_bf16_rne(in[i]);
}

static int is_pow2(int64_t g) { return g >= 1 && (g & (g - 1)) == 0; }

/* ---- Walsh-Hadamard butterfly ([SD] feature list; [CR] What The Options Do) ----
 * Unnormalised transform of one group of g values, fp32, ascending stages. */
static void fwht_group_f32(float *v, int64_t g)
{
    for (int64_t h = 1; h < g; h <<= 1) {
        for (int64_t j = 0; j < g; j++) {
            if ((j & h) == 0) {
                float a = v[j];
                float b = v[j + h];
                v[j] = a + b;
                v[j + h] = a - b;
            }
        }
    }
}

/* Block-diagonal butterfly over n values (n a multiple of g), in place. */
int oracle_fwht_f32(float *v, int64_t n, int64_t g)
{
    if (!v || !is_pow2(g) || n < 0 || n % g != 0)
        return ORACLE_ERR_ARG;
    for (int64_t k0 = 0; k0 < n; k0 += g)
        fwht_group_f32(v + k0, g);
    return ORACLE_OK;
}

/* The same butterfly in binary64: used only for quality reports and pins. */
int oracle_fwht_f64(double *v, int64_t n, int64_t g)
{
    if (!v || !is_pow2(g) || n < 0 || n % g != 0)
        return ORACLE_ERR_ARG;
    for (int64_t k0 = 0; k0 < n; k0 += g) {
        double *w = v + k0;
        for (int64_t h = 1; h < g; h <<= 1)
            for (int64_t j = 0; j < g; j++)
                if ((j & h) == 0) {
                    double a = w[j], b = w[j + h];
                    w[j] = a + b;
                    w[j + h] = a - b;
                }
    }
    return ORACLE_OK;
}

/* ---- Rotate + quantize one row per scale ([SD] SDNQConfig; [CR] What The Options Do;
 * [HS] Rigorous grid / pack simulation) ----
 * x:  bf16 bits [rows, K], row stride ldx elements.
 * q:  int8 codes [rows, K], dense.  s: fp32 scale per row (scale of the normalised
 * rotation, so that x_rot[r][k] ~= s[r] * q[r][k]).  Works for weights (one scale per
 * output row, static) and activations (one scale per token, dynamic) alike. */
int oracle_rotate_quantize(const uint16_t *x, int64_t rows, int64_t K, int64_t ldx,
                           int64_t g, int8_t *q, float *s, int nthreads)
{
    if (!x || !q || !s || rows < 0 || K <= 0 || ldx < K || !is_pow2(g) || K % g != 0)
        return ORACLE_ERR_ARG;
    const float c_g = (float)(1.0 / sqrt((double)g));
    int err = 0;
#pragma omp parallel for num_threads(nthreads > 0 ? nthreads : 1) schedule(static)
    for (int64_t r = 0; r < rows; r++) {
        float *z = (float *)malloc((size_t)K * sizeof(float));
        if (!z) {
#pragma omp atomic write
            err = 1;
            continue;
        }
        const uint16_t *xr = x + r * ldx;
        for (int64_t k = 0; k < K; k++)
            z[k] = bf16_bits_to_f32(xr[k]);
        for (int64_t k0 = 0; k0 < K; k0 += g)
            fwht_group_f32(z + k0, g);
        float amax = 0.0f;
        for (int64_t k = 0; k < K; k++) {
            float a = fabsf(z[k]);
            if (a > amax)
                amax = a;
        }
        const float s_z = amax / 127.0f;
        int8_t *qr = q + r * K;
        for (int64_t k = 0; k < K; k++) {
            int code = 0;
            if (amax != 0.0f) {
                float t = z[k] / s_z;      /* IEEE fp32 quotient */
                float n = nearbyintf(t);   /* half-to-even */
                if (n > 127.0f)
                    n = 127.0f;
                if (n < -127.0f)
                    n = -127.0f;
                code = (n == n) ? (int)n : 0;
            }
            qr[k] = (int8_t)code;
        }
        s[r] = s_z * c_g;
        free(z);
    }
    return err ? ORACLE_ERR_NOMEM : ORACLE_OK;
}

/* ---- INT8 x INT8 -> INT32 matmul ([SD] feature list: INT8 quantized matmul) ----
 * acc[m][n] = sum_k a[m][k] * b[n][k]; both operands K-contiguous, dense. */
int oracle_gemm_s8(const int8_t *a, const int8_t *b, int64_t M, int64_t N, int64_t K,
                   int32_t *acc, int nthreads)
{
    if (!a || !b || !acc || M < 0 || N < 0 || K <= 0)
        return ORACLE_ERR_ARG;
#pragma omp parallel for num_threads(nthreads > 0 ? nthreads : 1) schedule(static)
    for (int64_t m = 0; m < M; m++) {
        const int8_t *am = a + m * K;
        for (int64_t n = 0; n < N; n++) {
            const int8_t *bn = b + n * K;
            int32_t sum = 0;
            for (int64_t k = 0; k < K; k++)
                sum += (int32_t)am[k] * (int32_t)bn[k];
            acc[m * N + n] = sum;
        }
    }
    return ORACLE_OK;
}

/* ---- FP32 de-quant epilogue ([SD] SDNQConfig dequantize_fp32) ----
 * out[m][n] = bf16( ((float)acc * (s_x[m]*s_w[n])) + bias[n] + lora_scale*L[m][n] ).
 * bias (bf16 bits [N]) and L (fp32 [M,N]) may be NULL. */
int oracle_dequant_epilogue(const int32_t *acc, const float *sx, const float *sw,
                            const uint16_t *bias, const float *L, float lora_scale,
                            int64_t M, int64_t N, uint16_t *out, int nthreads)
{
    if (!acc || !sx || !sw || !out || M < 0 || N < 0)
        return ORACLE_ERR_ARG;
#pragma omp parallel for num_threads(nthreads > 0 ? nthreads : 1) schedule(static)
    for (int64_t m = 0; m < M; m++) {
        for (int64_t n = 0; n < N; n++) {
            float t = sx[m] * sw[n];
            float v = (float)acc[m * N + n] * t;
            if (bias)
                v = v + bf16_bits_to_f32(bias[n]);
            if (L) {
                float l = lora_scale * L[m * N + n];
                v = v + l;
            }
            out[m * N + n] = f32_to_bf16_rne(v);
        }
    }
    return ORACLE_OK;
}

/* ---- LoRA side path on the frozen base ([CR] PEFT Behavior: adapters stay bf16) ----
 * u[m][j] = bf16( sum_k x[m][k] * A[k][j] ), summed in fp64. x row stride ldx. */
int oracle_lora_down(const uint16_t *x, int64_t M, int64_t K, int64_t ldx,
                     const uint16_t *A, int64_t rank, uint16_t *u, int nthreads)
{
    if (!x || !A || !u || M < 0 || K <= 0 || ldx < K || rank <= 0)
        return ORACLE_ERR_ARG;
#pragma omp parallel for num_threads(nthreads > 0 ? nthreads : 1) schedule(static)
    for (int64_t m = 0; m < M; m++) {
        for (int64_t j = 0; j < rank; j++) {
            double sum = 0.0;
            for (int64_t k = 0; k < K; k++)
                sum += (double)bf16_bits_to_f32(x[m * ldx + k]) *
                       (double)bf16_bits_to_f32(A[k * rank + j]);
            u[m * rank + j] = f64_to_bf16_rne(sum);
        }
    }
    return ORACLE_OK;
}

/* L[m][n] = fp32( sum_j u[m][j] * B[j][n] ), summed in fp64. */
int oracle_lora_up(const uint16_t *u, const uint16_t *B, int64_t M, int64_t N, int64_t rank,
                   float *L, int nthreads)
{
    if (!u || !B || !L || M < 0 || N < 0 || rank <= 0)
        return ORACLE_ERR_ARG;
#pragma omp parallel for num_threads(nthreads > 0 ? nthreads : 1) schedule(static)
    for (int64_t m = 0; m < M; m++) {
        for (int64_t n = 0; n < N; n++) {
            double sum = 0.0;
            for (int64_t j = 0; j < rank; j++)
                sum += (double)bf16_bits_to_f32(u[m * rank + j]) *
                       (double)bf16_bits_to_f32(B[j * N + n]);
            L[m * N + n] = (float)sum;
        }
    }
    return ORACLE_OK;
}

/* ---- GELU between the MLP projections (exact erf form), bf16 -> bf16 ---- */
int oracle_gelu_bf16(const uint16_t *in, int64_t n, uint16_t *out, int nthreads)
{
    if (!in || !out || n < 0)
        return ORACLE_ERR_ARG;
#pragma omp parallel for num_threads(nthreads > 0 ? nthreads : 1) schedule(static)
    for (int64_t i = 0; i < n; i++) {
        double x = (double)bf16_bits_to_f32(in[i]);
        double y = 0.5 * x * erfc(-x / sqrt(2.0));
        out[i] = f64_to_bf16_rne(y);
    }
    return ORACLE_OK;
}

/* ---- Input gradient through the frozen rotated int8 base ----
 * [SD] quantized training example (the quantized matmul runs on the forward and on the
 * backward pass); [CR] PEFT Behavior (the base is frozen under bf16 adapters, so the only
 * gradient it passes on is the one with respect to its input).
 * The weight the layer holds is W_hat = W_rot H with W_rot[n][k] = sW[n] * qW[n][k] (the
 * rotated, normalised rows) and H the normalised block-diagonal Hadamard matrix, which is
 * symmetric and its own inverse. So dx = dy W_hat = ((dy * sW) qW) H, computed in three
 * steps: a per-token int8 quantization of dy * sW (sW varies along the contraction, so it is
 * folded into dy before the integer matmul), the int8 matmul against the stored codes qW
 * read as [N][K], and an epilogue that applies the row scale, the butterfly and 1/sqrt(g). */

/* Step 1: c[m][n] = fp32(dy[m][n]) * sw[n]; amax over the row; s = amax / 127;
 * codes rne(c / s) clamped to [-127, 127]; stored scale s. dy row stride ld. */
int oracle_colscale_quantize(const uint16_t *dy, int64_t rows, int64_t N, int64_t ld,
                             const float *sw, int8_t *q, float *s, int nthreads)
{
    if (!dy || !sw || !q || !s || rows < 0 || N <= 0 || ld < N)
        return ORACLE_ERR_ARG;
    int err = 0;
#pragma omp parallel for num_threads(nthreads > 0 ? nthreads : 1) schedule(static)
    for (int64_t r = 0; r < rows; r++) {
        float *c = (float *)malloc((size_t)N * sizeof(float));
        if (!c) {
#pragma omp atomic write
            err = 1;
            continue;
        }
        float amax = 0.0f;
        for (int64_t n = 0; n < N; n++) {
            c[n] = bf16_bits_to_f32(dy[r * ld + n]) * sw[n];
            float a = fabsf(c[n]);
            if (a > amax)
                amax = a;
        }
        const float s_c = amax / 127.0f;
        for (int64_t n = 0; n < N; n++) {
            int code = 0;
            if (amax != 0.0f) {
                float n_ = nearbyintf(c[n] / s_c);
                if (n_ > 127.0f)
                    n_ = 127.0f;
                if (n_ < -127.0f)
                    n_ = -127.0f;
                code = (n_ == n_) ? (int)n_ : 0;
            }
            q[r * N + n] = (int8_t)code;
        }
        s[r] = s_c;
        free(c);
    }
    return err ? ORACLE_ERR_NOMEM : ORACLE_OK;
}

/* Step 2: acc[m][k] = sum_n a[m][n] * b[n][k] in int32; a [M][N] and b [N][K] dense. */
int oracle_gemm_s8_nn(const int8_t *a, const int8_t *b, int64_t M, int64_t N, int64_t K,
                      int32_t *acc, int nthreads)
{
    if (!a || !b || !acc || M < 0 || N <= 0 || K < 0)
        return ORACLE_ERR_ARG;
#pragma omp parallel for num_threads(nthreads > 0 ? nthreads : 1) schedule(static)
    for (int64_t m = 0; m < M; m++) {
        for (int64_t k = 0; k < K; k++) {
            int32_t sum = 0;
            for (int64_t n = 0; n < N; n++)
                sum += (int32_t)a[m * N + n] * (int32_t)b[n * K + k];
            acc[m * K + k] = sum;
        }
    }
    return ORACLE_OK;
}

/* Step 3: v[m][k] = fp32(acc[m][k]) * s[m]; the fp32 butterfly of each group of g columns
 * (ascending stages, as in the forward rotation); dx[m][k] = bf16_rne(z[k] * c_g) with
 * c_g = fp32(1/sqrt(g)). */
int oracle_grad_input_epilogue(const int32_t *acc, const float *s, int64_t M, int64_t K,
                               int64_t g, uint16_t *dx, int nthreads)
{
    if (!acc || !s || !dx || M < 0 || K <= 0 || !is_pow2(g) || K % g != 0)
        return ORACLE_ERR_ARG;
    const float c_g = (float)(1.0 / sqrt((double)g));
    int err = 0;
#pragma omp parallel for num_threads(nthreads > 0 ? nthreads : 1) schedule(static)
    for (int64_t m = 0; m < M; m++) {
        float *z = (float *)malloc((size_t)K * sizeof(float));
        if (!z) {
#pragma omp atomic write
            err = 1;
            continue;
        }
        for (int64_t k = 0; k < K; k++)
            z[k] = (float)acc[m * K + k] * s[m];
        for (int64_t k0 = 0; k0 < K; k0 += g)
            fwht_group_f32(z + k0, g);
        for (int64_t k = 0; k < K; k++)
            dx[m * K + k] = f32_to_bf16_rne(z[k] * c_g);
        free(z);
    }
    return err ? ORACLE_ERR_NOMEM : ORACLE_OK;
}

/* ---- FP8 (e4m3) variant of the rotated quantized matmul ----
 * [SD] feature list and SDNQConfig (FP8 weights and FP8 quantized matmul beside INT8); the
 * rotation is the same. e4m3 ("fn" flavour, as used for FP8 matmuls): 1 sign bit, 4 exponent
 * bits with bias 7, 3 mantissa bits; normal values (1 + m/8) 2^(e-7) for e = 1..15 except
 * e = 15, m = 7 (NaN), so the largest finite value is 448; subnormals (m/8) 2^-6; no
 * infinities. Encoding rounds to nearest with ties to the even code and saturates finite
 * values beyond 448 to +-448. */

static uint8_t e4m3_encode(double v)
{
    if (v != v)
        return 0x7f;
    const uint8_t sign = (v < 0.0 || (v == 0.0 && signbit(v))) ? 0x80 : 0x00;
    double a = fabs(v);
    if (a >= 448.0)
        return sign | 0x7e; /* saturate */
    int e;
    frexp(a, &e);               /* a = f 2^e with f in [0.5, 1): a in [2^(e-1), 2^e) */
    int E = e - 1;              /* a in [2^E, 2^(E+1)) */
    if (E < -6)
        E = -6;                 /* subnormal range shares the quantum of binade -6 */
    const double quantum = ldexp(1.0, E - 3);
    double q = nearbyint(a / quantum) * quantum; /* exact scaling; ties to even multiple */
    if (q >= 448.0)
        q = 448.0;
    if (q == 0.0)
        return sign;
    /* q is representable: split into exponent / mantissa fields */
    int qe;
    double qf = frexp(q, &qe);  /* q = qf 2^qe, qf in [0.5, 1) */
    int biased = qe - 1 + 7;
    if (biased >= 1) {
        int m = (int)(qf * 16.0) - 8; /* (1 + m/8) = 2 qf */
        return sign | (uint8_t)(biased << 3) | (uint8_t)m;
    }
    int m = (int)(q / ldexp(1.0, -9));  /* subnormal: q = m 2^-9 */
    return sign | (uint8_t)m;
}

static double e4m3_decode(uint8_t c)
{
    const int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
    double v;
    if (e == 15 && m == 7)
        v = NAN;
    else if (e == 0)
        v = ldexp((double)m, -9);
    else
        v = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -v : v;
}

void oracle_e4m3_encode(const float *in, int64_t n, uint8_t *out)
{
    for (int64_t i = 0; i < n; i++)
        out[i] = e4m3_encode((double)in[i]);
}

void oracle_e4m3_decode(const uint8_t *in, int64_t n, float *out)
{
    for (int64_t i = 0; i < n; i++)
        out[i] = (float)e4m3_decode(in[i]);
}

/* Rotate + quantize to e4m3: the same butterfly and row absmax as the int8 path, then
 * s_z = fp32(amax / 448), codes e4m3(fp32(z / s_z)), stored scale fp32(s_z * fp32(1/sqrt g)).
 * An all-zero row gives s = 0 and codes +0. */
int oracle_rotate_quantize_fp8(const uint16_t *x, int64_t rows, int64_t K, int64_t ldx,
                               int64_t g, uint8_t *q, float *s, int nthreads)
{
    if (!x || !q || !s || rows < 0 || K <= 0 || ldx < K || !is_pow2(g) || K % g != 0)
        return ORACLE_ERR_ARG;
    const float c_g = (float)(1.0 / sqrt((double)g));
    int err = 0;
#pragma omp parallel for num_threads(nthreads > 0 ? nthreads : 1) schedule(static)
    for (int64_t r = 0; r < rows; r++) {
        float *z = (float *)malloc((size_t)K * sizeof(float));
        if (!z) {
#pragma omp atomic write
            err = 1;
            continue;
        }
        for (int64_t k = 0; k < K; k++)
            z[k] = bf16_bits_to_f32(x[r * ldx + k]);
        for (int64_t k0 = 0; k0 < K; k0 += g)
            fwht_group_f32(z + k0, g);
        float amax = 0.0f;
        for (int64_t k = 0; k < K; k++) {
            float a = fabsf(z[k]);
            if (a > amax)
                amax = a;
        }
        const float s_z = amax / 448.0f;
        for (int64_t k = 0; k < K; k++) {
            float t = (amax != 0.0f) ? z[k] / s_z : 0.0f; /* IEEE fp32 quotient */
            q[r * K + k] = e4m3_encode((double)t);
        }
        s[r] = s_z * c_g;
        free(z);
    }
    return err ? ORACLE_ERR_NOMEM : ORACLE_OK;
}

/* acc[m][n] = fp32( sum_k dec(a[m][k]) * dec(b[n][k]) ): every product is exact, the sum is
 * taken in binary64 and rounded once. */
int oracle_gemm_fp8(const uint8_t *a, const uint8_t *b, int64_t M, int64_t N, int64_t K,
                    float *acc, int nthreads)
{
    if (!a || !b || !acc || M < 0 || N < 0 || K <= 0)
        return ORACLE_ERR_ARG;
    double lut[256];
    for (int c = 0; c < 256; c++)
        lut[c] = e4m3_decode((uint8_t)c);
#pragma omp parallel for num_threads(nthreads > 0 ? nthreads : 1) schedule(static)
    for (int64_t m = 0; m < M; m++) {
        for (int64_t n = 0; n < N; n++) {
            double sum = 0.0;
            for (int64_t k = 0; k < K; k++)
                sum += lut[a[m * K + k]] * lut[b[n * K + k]];
            acc[m * N + n] = (float)sum;
        }
    }
    return ORACLE_OK;
}

/* The fp32 de-quant epilogue on fp32 accumulators (same op order as the int8 one):
 * t = sx*sw; v = acc*t; v = v + bias; out = bf16_rne(v). */
int oracle_dequant_epilogue_f32(const float *acc, const float *sx, const float *sw,
                                const uint16_t *bias, int64_t M, int64_t N, uint16_t *out,
                                int nthreads)
{
    if (!acc || !sx || !sw || !out || M < 0 || N < 0)
        return ORACLE_ERR_ARG;
#pragma omp parallel for num_threads(nthreads > 0 ? nthreads : 1) schedule(static)
    for (int64_t m = 0; m < M; m++) {
        for (int64_t n = 0; n < N; n++) {
            float t = sx[m] * sw[n];
            float v = acc[m * N + n] * t;
            if (bias)
                v = v + bf16_bits_to_f32(bias[n]);
            out[m * N + n] = f32_to_bf16_rne(v);
        }
    }
    return ORACLE_OK;
}

/* ---- Hadamard-rotated int8 QK inside attention ----
 * [SD] SDNQ attention example (an SDPA replacement: int8 QK matmul, smooth_k, use_hadamard,
 * hadamard_group_size; the PV matmul left unquantized). Per batch b and head h, with Q
 * [Lq][D], K and V [Lk][D] (bf16, stored [B][L][H][D]):
 *   mu[d]    = fp32( sum_j K[j][d] / Lk ), the sum in binary64 (smooth_k);
 *   K'[j][d] = fp32( K[j][d] - mu[d] )   (softmax is unchanged: q.mu is constant per row);
 *   Q and K' rows rotated by the butterfly over groups of min(g, D) and quantized per row
 *   exactly as the linear path's activations (codes, stored scale s = fp32(amax/127) * c);
 *   logit[i][j] = fp32( fp32( fp32(acc) * fp32(s_q[i] * s_k[j]) ) * scale ),
 *   acc = sum_d qQ[i][d] qK[j][d] in int32 (the rotation cancels in the product);
 *   O[i] = sum_j softmax_j(logit[i][j]) V[j] in binary64, rounded once to bf16. */

/* K' rows from bf16 K and the per-(b, h) channel means: kq [B][Lk][H][D] int8, sk [B][H][Lk]. */
static void quantize_rows_f32(float *z, int64_t K, int64_t g, int8_t *q, float *s, float c_g)
{
    for (int64_t k0 = 0; k0 < K; k0 += g)
        fwht_group_f32(z + k0, g);
    float amax = 0.0f;
    for (int64_t k = 0; k < K; k++) {
        float a = fabsf(z[k]);
        if (a > amax)
            amax = a;
    }
    const float s_z = amax / 127.0f;
    for (int64_t k = 0; k < K; k++) {
        int code = 0;
        if (amax != 0.0f) {
            float n_ = nearbyintf(z[k] / s_z);
            if (n_ > 127.0f)
                n_ = 127.0f;
            if (n_ < -127.0f)
                n_ = -127.0f;
            code = (n_ == n_) ? (int)n_ : 0;
        }
        q[k] = (int8_t)code;
    }
    *s = s_z * c_g;
}

int oracle_attn_prep(const uint16_t *q, const uint16_t *k, int64_t B, int64_t Lq, int64_t Lk,
                     int64_t H, int64_t D, int64_t g, int smooth_k, int8_t *qq, float *sq,
                     int8_t *kq, float *sk, float *mu, int nthreads)
{
    if (!q || !k || !qq || !sq || !kq || !sk || !mu || B <= 0 || Lq <= 0 || Lk <= 0 || H <= 0 ||
        D <= 0 || !is_pow2(g) || !is_pow2(D))
        return ORACLE_ERR_ARG;
    const int64_t ge = g < D ? g : D;
    const float c_g = (float)(1.0 / sqrt((double)ge));
    for (int64_t b = 0; b < B; b++)
        for (int64_t h = 0; h < H; h++)
            for (int64_t d = 0; d < D; d++) {
                double sum = 0.0;
                if (smooth_k)
                    for (int64_t j = 0; j < Lk; j++)
                        sum += (double)bf16_bits_to_f32(k[((b * Lk + j) * H + h) * D + d]);
                mu[(b * H + h) * D + d] = (float)(sum / (double)Lk);
            }
    int err = 0;
#pragma omp parallel for num_threads(nthreads > 0 ? nthreads : 1) schedule(static)
    for (int64_t r = 0; r < B * Lq * H; r++) {
        float z[1024];
        if (D > 1024) {
#pragma omp atomic write
            err = 1;
            continue;
        }
        const int64_t b = r / (Lq * H), i = (r / H) % Lq, h = r % H;
        for (int64_t d = 0; d < D; d++)
            z[d] = bf16_bits_to_f32(q[r * D + d]);
        quantize_rows_f32(z, D, ge, qq + r * D, sq + (b * H + h) * Lq + i, c_g);
    }
#pragma omp parallel for num_threads(nthreads > 0 ? nthreads : 1) schedule(static)
    for (int64_t r = 0; r < B * Lk * H; r++) {
        float z[1024];
        if (D > 1024)
            continue;
        const int64_t b = r / (Lk * H), j = (r / H) % Lk, h = r % H;
        for (int64_t d = 0; d < D; d++)
            z[d] = bf16_bits_to_f32(k[r * D + d]) - mu[(b * H + h) * D + d];
        quantize_rows_f32(z, D, ge, kq + r * D, sk + (b * H + h) * Lk + j, c_g);
    }
    return err ? ORACLE_ERR_ARG : ORACLE_OK;
}

/* logits [B][H][Lq][Lk] (fp32) from the prepared codes and scales. */
int oracle_attn_logits(const int8_t *qq, const float *sq, const int8_t *kq, const float *sk,
                       int64_t B, int64_t Lq, int64_t Lk, int64_t H, int64_t D, float scale,
                       float *logits, int nthreads)
{
    if (!qq || !sq || !kq || !sk || !logits || B <= 0 || Lq <= 0 || Lk <= 0 || H <= 0 || D <= 0)
        return ORACLE_ERR_ARG;
#pragma omp parallel for num_threads(nthreads > 0 ? nthreads : 1) schedule(static)
    for (int64_t bhi = 0; bhi < B * H * Lq; bhi++) {
        const int64_t b = bhi / (H * Lq), h = (bhi / Lq) % H, i = bhi % Lq;
        const int8_t *qr = qq + ((b * Lq + i) * H + h) * D;
        for (int64_t j = 0; j < Lk; j++) {
            const int8_t *kr = kq + ((b * Lk + j) * H + h) * D;
            int32_t acc = 0;
            for (int64_t d = 0; d < D; d++)
                acc += (int32_t)qr[d] * (int32_t)kr[d];
            float t = sq[(b * H + h) * Lq + i] * sk[(b * H + h) * Lk + j];
            float v = (float)acc * t;
            logits[bhi * Lk + j] = v * scale;
        }
    }
    return ORACLE_OK;
}

/* O [B][Lq][H][D] bf16 = softmax(logits) V, in binary64. */
int oracle_attn_softmax_pv(const float *logits, const uint16_t *v, int64_t B, int64_t Lq,
                           int64_t Lk, int64_t H, int64_t D, uint16_t *o, int nthreads)
{
    if (!logits || !v || !o || B <= 0 || Lq <= 0 || Lk <= 0 || H <= 0 || D <= 0)
        return ORACLE_ERR_ARG;
    int err = 0;
#pragma omp parallel for num_threads(nthreads > 0 ? nthreads : 1) schedule(static)
    for (int64_t bhi = 0; bhi < B * H * Lq; bhi++) {
        const int64_t b = bhi / (H * Lq), h = (bhi / Lq) % H, i = bhi % Lq;
        const float *lr = logits + bhi * Lk;
        double m = -INFINITY;
        for (int64_t j = 0; j < Lk; j++)
            if ((double)lr[j] > m)
                m = (double)lr[j];
        double *acc = (double *)calloc((size_t)D, sizeof(double));
        if (!acc) {
#pragma omp atomic write
            err = 1;
            continue;
        }
        double l = 0.0;
        for (int64_t j = 0; j < Lk; j++) {
            const double p = exp((double)lr[j] - m);
            l += p;
            const uint16_t *vr = v + ((b * Lk + j) * H + h) * D;
            for (int64_t d = 0; d < D; d++)
                acc[d] += p * (double)bf16_bits_to_f32(vr[d]);
        }
        uint16_t *orow = o + ((b * Lq + i) * H + h) * D;
        for (int64_t d = 0; d < D; d++)
            orow[d] = f64_to_bf16_rne(acc[d] / l);
        free(acc);
    }
    return err ? ORACLE_ERR_NOMEM : ORACLE_OK;
}
