/*
 * Oracle for the SmoothQuant-smoothed INT8 W8A8 linear path.
 *
 * TEST INFRASTRUCTURE ONLY. This is a plain, slow, single-purpose CPU restatement of
 * what the path computes, written to be checked against the pages by eye. Only the
 * test-suite, the smoke check and the benchmark's CPU-baseline leg may load it; the
 * library never calls it, and it shares no code, header, table or helper with the
 * CUDA library.
 *
 * Arithmetic conventions (a reading where the pages are silent; see the design notes):
 *   - IEEE binary32 with round-to-nearest-even for every float operation, no FMA
 *     contraction (built with -ffp-contract=off) except where fmaf() is written out.
 *   - bf16 values travel as raw 16-bit patterns; widening is exact, narrowing is RN-even.
 *
 * Sources (page title, section):
 *   [P1] "Optimizing Llama 3 Inference Speed Using INT8 Quantization via AutoGPTQ"
 *        (promptcube3), "Crucial Config Tips for Performance" -- GPTQ's dampening factor.
 *   [P2] "INT8 W8A8 ... using SmoothQuant and GPTQ" (arc-codex article 3619...):
 *        "At its core, quantizing a weight involves 2 steps" -- scale = max|col|/127,
 *        q = round(w/scale); "The problem with naive quantization" -- per-channel RTN and
 *        its worked example; "Why activation quantization is hard" -- one dynamic scale per
 *        token, worked example [1.32, 0.75, 0.91, 153.0]; "How SmoothQuant prevents
 *        outliers" -- RMSNorm = divide by RMS then multiply by gamma, gamma folding;
 *        "How the SmoothQuant smoothing factor is computed" -- s_j from max|A_j|, max|W_j|,
 *        alpha (formula lost in the extract; the SmoothQuant paper's form is used); "The
 *        solution: How GPTQ improves on naive quantization" -- quantize a weight, measure the
 *        error, redistribute it over the remaining weights guided by the Hessian.
 *   [P3] "INT8 Post-Training Quantization for LLM Inference on NVIDIA GPUs", section
 *        "1. Min-Max Calibration" -- S = max(|min|,|max|)/127, range [-127, 127].
 *   [P4] "W8A8 ... accuracy and serving results" (Red Hat developer article), section
 *        "Inter-token latency (ITL)" -- per layer: measure the range, compute a scale,
 *        convert to INT8, multiply, convert back to BF16; "When W8A8 INT8 quantization is a
 *        good fit" and "What to explore next" -- W8A8 FP8 as the variant for Hopper and
 *        Blackwell GPUs.
 *   [P5] "05 Quantization AWQ GPTQ FP8", section "Ladder" -- FP8 as the near-lossless
 *        8-bit step. Neither page fixes the FP8 encoding; the FP8 functions take the OCP
 *        E4M3 format with per-token / per-channel scales absmax / 448 (the largest E4M3
 *        value), the analogue of the INT8 scales absmax / 127.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ bf16 <-> f32 */

/* Widen a bf16 bit pattern: the 16 bits are the top half of a binary32. */
float oracle_bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Narrow binary32 to bf16 with round-to-nearest, ties to even. NaN stays NaN. */
uint16_t oracle_f32_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu) != 0u)
        return (uint16_t)((u >> 16) | 0x0040u); /* quiet NaN */
    uint32_t lsb = (u >> 16) & 1u;             /* ties go to the even neighbour */
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

/* ------------------------------------------------------------ per-token quantization */

/*
 * Symmetric per-token quantization of one row of fp32 values [P2 "Why activation
 * quantization is hard"; P3 "1. Min-Max Calibration"]:
 *   amax = max_j |y_j|,  s = amax / 127,  q_j = clamp(round_half_even(y_j / s), -127, 127).
 * An all-zero row has no range; it gets s = 0 and q = 0 (the pages are silent).
 */
void oracle_quantize_row_f32(const float *y, int64_t K, int8_t *q, float *s_out)
{
    float amax = 0.0f;
    for (int64_t j = 0; j < K; ++j) {
        float a = fabsf(y[j]);
        if (a > amax)
            amax = a;
    }
    if (amax == 0.0f) {
        *s_out = 0.0f;
        for (int64_t j = 0; j < K; ++j)
            q[j] = 0;
        return;
    }
    float s = amax / 127.0f;
    *s_out = s;
    for (int64_t j = 0; j < K; ++j) {
        float t = rintf(y[j] / s); /* default rounding mode: nearest, ties to even */
        if (t > 127.0f)
            t = 127.0f;
        if (t < -127.0f)
            t = -127.0f;
        q[j] = (int8_t)t;
    }
}

/* ------------------------------------------------------------------ parallel rows */

typedef void (*row_fn)(void *ctx, int64_t row);
struct par_job {
    row_fn fn;
    void *ctx;
    int64_t begin, end;
};

static void *par_worker(void *arg)
{
    struct par_job *j = (struct par_job *)arg;
    for (int64_t r = j->begin; r < j->end; ++r)
        j->fn(j->ctx, r);
    return NULL;
}

/* Runs fn(ctx, r) for r in [0, n). Rows are independent, so splitting them across threads
 * changes no arithmetic. */
static void parallel_rows(row_fn fn, void *ctx, int64_t n, int nthreads)
{
    if (nthreads < 1)
        nthreads = 1;
    if (nthreads > 256)
        nthreads = 256;
    if ((int64_t)nthreads > n)
        nthreads = (int)(n > 0 ? n : 1);
    if (nthreads == 1) {
        for (int64_t r = 0; r < n; ++r)
            fn(ctx, r);
        return;
    }
    pthread_t tid[256];
    struct par_job jobs[256];
    for (int t = 0; t < nthreads; ++t) {
        jobs[t].fn = fn;
        jobs[t].ctx = ctx;
        jobs[t].begin = n * t / nthreads;
        jobs[t].end = n * (t + 1) / nthreads;
        pthread_create(&tid[t], NULL, par_worker, &jobs[t]);
    }
    for (int t = 0; t < nthreads; ++t)
        pthread_join(tid[t], NULL);
}

/* ------------------------------------------------------------------- quantize_rows */

struct qrows_ctx {
    const uint16_t *x;
    const float *sinv;
    int64_t K;
    int8_t *q;
    float *s;
};

static void qrows_row(void *vctx, int64_t m)
{
    struct qrows_ctx *c = (struct qrows_ctx *)vctx;
    float *y = (float *)malloc((size_t)c->K * sizeof(float));
    for (int64_t j = 0; j < c->K; ++j) {
        y[j] = oracle_bf16_to_f32(c->x[m * c->K + j]);
        if (c->sinv)
            y[j] = y[j] * c->sinv[j]; /* smoothing folded into X: X' = X diag(1/s) */
    }
    oracle_quantize_row_f32(y, c->K, c->q + m * c->K, c->s + m);
    free(y);
}

/*
 * Per-token dynamic quantization of a bf16 activation [M, K] (row-major), optionally
 * after multiplying channel j by sinv[j] = 1/s_j (SmoothQuant applied to X directly).
 * [P2 "Why activation quantization is hard"; P3 "1. Min-Max Calibration"]
 */
int oracle_quantize_rows(const uint16_t *x, const float *sinv, int64_t M, int64_t K, int8_t *q,
                         float *s, int nthreads)
{
    struct qrows_ctx c = {x, sinv, K, q, s};
    parallel_rows(qrows_row, &c, M, nthreads);
    return 0;
}

/* ------------------------------------------------- static per-tensor quantization */

/*
 * Symmetric min-max calibration of one tensor [P3 "1. Min-Max Calibration"]: the observed
 * range [min, max] of the calibration values maps onto [-127, 127] with
 * S = max(|min|, |max|) / 127 (binary32 division). Returns 0 for an empty or all-zero set.
 */
float oracle_minmax_scale(const float *v, int64_t n)
{
    if (n <= 0)
        return 0.0f;
    float lo = v[0], hi = v[0];
    for (int64_t j = 1; j < n; ++j) {
        if (v[j] < lo)
            lo = v[j];
        if (v[j] > hi)
            hi = v[j];
    }
    float a = fabsf(lo) > fabsf(hi) ? fabsf(lo) : fabsf(hi);
    return a / 127.0f;
}

struct qstatic_ctx {
    const uint16_t *x;
    const float *sinv;
    float S;
    int64_t K;
    int8_t *q;
};

static void qstatic_row(void *vctx, int64_t m)
{
    struct qstatic_ctx *c = (struct qstatic_ctx *)vctx;
    for (int64_t j = 0; j < c->K; ++j) {
        float y = oracle_bf16_to_f32(c->x[m * c->K + j]);
        if (c->sinv)
            y = y * c->sinv[j];
        float t = rintf(y / c->S); /* ties to even */
        if (t > 127.0f)
            t = 127.0f;
        if (t < -127.0f)
            t = -127.0f;
        c->q[m * c->K + j] = (int8_t)t;
    }
}

/*
 * Static per-tensor activation quantization [P3 "1. Min-Max Calibration"]: one scale S > 0,
 * fixed offline by calibration, for every token; q = clamp(round_half_even(y / S), -127,
 * 127) with y = x (or x * sinv[j]). Values beyond the calibrated range saturate at +-127.
 */
int oracle_quantize_rows_static(const uint16_t *x, const float *sinv, float S, int64_t M,
                                int64_t K, int8_t *q, int nthreads)
{
    if (!(S > 0.0f))
        return -1;
    struct qstatic_ctx c = {x, sinv, S, K, q};
    parallel_rows(qstatic_row, &c, M, nthreads);
    return 0;
}

/* ------------------------------------------------------------ FP8 (E4M3) variant */

/*
 * OCP 8-bit floating point E4M3 (the "FN" form: no infinities, S.1111.111 is NaN): sign, 4
 * exponent bits (bias 7), 3 fraction bits. Normal values 2^(e-7) (1 + f/8), e = 1..15;
 * subnormals 2^-6 (f/8); largest finite 448. Encoding rounds to nearest, ties to even, and
 * saturates to +-448 (the conversion used for W8A8 FP8 codes).
 */
float oracle_e4m3_to_f32(uint8_t b)
{
    const int sign = b >> 7, e = (b >> 3) & 15, f = b & 7;
    if (e == 15 && f == 7)
        return NAN;
    const double v = e == 0 ? ldexp((double)f, -9) : ldexp(8.0 + f, e - 10);
    return (float)(sign ? -v : v);
}

uint8_t oracle_f32_to_e4m3(float v)
{
    if (v != v)
        return 0x7F;
    const uint8_t sign = signbit(v) ? 0x80 : 0x00;
    const double a = fabs((double)v);
    if (a >= 448.0)
        return sign | 0x7E; /* saturate */
    if (a == 0.0)
        return sign;
    /* quantum of the binade of a (subnormal binade below 2^-6), then round the significand
     * a / quantum to the nearest integer, ties to even */
    int E;
    frexp(a, &E);          /* a = m 2^E, m in [0.5, 1): binade exponent E - 1 */
    int be = E - 1;
    if (be < -6)
        be = -6;
    const double q = ldexp(1.0, be - 3);
    const double n = rint(a / q); /* a / q is exact; rint: ties to even */
    const double r = n * q;
    if (r >= 448.0)
        return sign | 0x7E;
    if (r < ldexp(1.0, -6)) /* subnormal (or rounded up to the smallest normal below) */
        return sign | (uint8_t)(r / ldexp(1.0, -9));
    int E2;
    frexp(r, &E2);
    const int e = (E2 - 1) + 7;
    const int f = (int)(r / ldexp(1.0, E2 - 1) * 8.0) - 8;
    return sign | (uint8_t)((e << 3) | f);
}

/* Per-token FP8 quantization of one fp32 row: s = amax / 448, q_j = e4m3(y_j / s) (binary32
 * division, then the rounding above); an all-zero row gets s = 0 and q = 0. */
void oracle_quantize_row_f32_fp8(const float *y, int64_t K, uint8_t *q, float *s_out)
{
    float amax = 0.0f;
    for (int64_t j = 0; j < K; ++j)
        if (fabsf(y[j]) > amax)
            amax = fabsf(y[j]);
    if (amax == 0.0f) {
        *s_out = 0.0f;
        memset(q, 0, (size_t)K);
        return;
    }
    const float s = amax / 448.0f;
    *s_out = s;
    for (int64_t j = 0; j < K; ++j)
        q[j] = oracle_f32_to_e4m3(y[j] / s);
}

struct qrows8_ctx {
    const uint16_t *x;
    const float *sinv;
    int64_t K;
    uint8_t *q;
    float *s;
};

static void qrows8_row(void *vctx, int64_t m)
{
    struct qrows8_ctx *c = (struct qrows8_ctx *)vctx;
    float *y = (float *)malloc((size_t)c->K * sizeof(float));
    for (int64_t j = 0; j < c->K; ++j) {
        y[j] = oracle_bf16_to_f32(c->x[m * c->K + j]);
        if (c->sinv)
            y[j] = y[j] * c->sinv[j];
    }
    oracle_quantize_row_f32_fp8(y, c->K, c->q + m * c->K, c->s + m);
    free(y);
}

/* Per-token FP8 quantization of bf16 activations [M, K] (optionally times sinv). */
int oracle_quantize_rows_fp8(const uint16_t *x, const float *sinv, int64_t M, int64_t K,
                             uint8_t *q, float *s, int nthreads)
{
    struct qrows8_ctx c = {x, sinv, K, q, s};
    parallel_rows(qrows8_row, &c, M, nthreads);
    return 0;
}

struct qf8_ctx {
    const float *y;
    int64_t K;
    uint8_t *q;
    float *s;
};

static void qf8_row(void *vctx, int64_t m)
{
    struct qf8_ctx *c = (struct qf8_ctx *)vctx;
    oracle_quantize_row_f32_fp8(c->y + m * c->K, c->K, c->q + m * c->K, c->s + m);
}

/* Per-row FP8 quantization of fp32 rows [M, K] (normalized activations, SiLU*up, or
 * smoothed weights, whose rows are output channels). */
int oracle_quantize_rows_f32_fp8(const float *y, int64_t M, int64_t K, uint8_t *q, float *s,
                                 int nthreads)
{
    struct qf8_ctx c = {y, K, q, s};
    parallel_rows(qf8_row, &c, M, nthreads);
    return 0;
}

/* The FP8 epilogue applied to given binary32 accumulators [M, N]: y = bf16_RN((acc s_tok)
 * s_ch). Used to check a device's epilogue against its own accumulators, whose rounding
 * order is the tensor cores'. */
int oracle_dequant_f32acc(const float *acc, const float *s_tok, const float *s_ch, int64_t M,
                          int64_t N, uint16_t *y)
{
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            float f = acc[m * N + n] * s_tok[m];
            f = f * s_ch[n];
            y[m * N + n] = oracle_f32_to_bf16(f);
        }
    return 0;
}

/*
 * FP8 GEMM reference: acc[m,n] = sum_k e4m3(xq[m,k]) e4m3(wq[n,k]) computed exactly (each
 * product is exact in binary64 and the sum stays exact for K <= 2^15: the terms are
 * multiples of 2^-18 below 2^18), also sum_k |products| (the scale of the rounding error of
 * any binary32 accumulation), and y = bf16_RN((float(acc) s_tok) s_ch).
 */
struct gemm8_ctx {
    const float *xd, *wd;
    const float *s_tok, *s_ch;
    int64_t N, K;
    double *acc, *absacc;
    uint16_t *y;
};

static void gemm8_row(void *vctx, int64_t m)
{
    struct gemm8_ctx *c = (struct gemm8_ctx *)vctx;
    const int64_t N = c->N, K = c->K;
    for (int64_t n = 0; n < N; ++n) {
        double a = 0.0, b = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            const double p = (double)c->xd[m * K + k] * (double)c->wd[n * K + k];
            a += p;
            b += fabs(p);
        }
        c->acc[m * N + n] = a;
        c->absacc[m * N + n] = b;
        float f = (float)a;
        f = f * c->s_tok[m];
        f = f * c->s_ch[n];
        c->y[m * N + n] = oracle_f32_to_bf16(f);
    }
}

int oracle_gemm_fp8(const uint8_t *xq, const float *s_tok, const uint8_t *wq, const float *s_ch,
                    int64_t M, int64_t N, int64_t K, double *acc, double *absacc, uint16_t *y,
                    int nthreads)
{
    float *xd = (float *)malloc((size_t)(M * K) * sizeof(float));
    float *wd = (float *)malloc((size_t)(N * K) * sizeof(float));
    for (int64_t i = 0; i < M * K; ++i)
        xd[i] = oracle_e4m3_to_f32(xq[i]);
    for (int64_t i = 0; i < N * K; ++i)
        wd[i] = oracle_e4m3_to_f32(wq[i]);
    struct gemm8_ctx c = {xd, wd, s_tok, s_ch, N, K, acc, absacc, y};
    parallel_rows(gemm8_row, &c, M, nthreads);
    free(xd);
    free(wd);
    return 0;
}

/* --------------------------------------------------------- smoothed RMSNorm + quant */

struct rms_ctx {
    const uint16_t *x, *r;
    uint16_t *h_out;
    const float *gamma;
    float eps;
    int64_t K;
    int8_t *q;
    float *s, *ms_out, *y_out;
    uint8_t *ambiguous;
    const float *ms_override;
};

static void rms_row(void *vctx, int64_t m)
{
    struct rms_ctx *c = (struct rms_ctx *)vctx;
    const int64_t K = c->K;
    float *h = (float *)malloc((size_t)K * sizeof(float));
    float *y = (float *)malloc((size_t)K * sizeof(float));

    /* Optional residual add; the sum is rounded to bf16 (it is the next residual). */
    for (int64_t j = 0; j < K; ++j) {
        float v = oracle_bf16_to_f32(c->x[m * K + j]);
        if (c->r) {
            uint16_t hb = oracle_f32_to_bf16(v + oracle_bf16_to_f32(c->r[m * K + j]));
            if (c->h_out)
                c->h_out[m * K + j] = hb;
            v = oracle_bf16_to_f32(hb);
        }
        h[j] = v;
    }

    /* Mean of squares. Each square of a bf16 value is exact in binary32; the sum is
     * accumulated in binary64 in index order. The order of a binary64 sum is not fixed by
     * the method, so any order is acceptable: the row is flagged when another order could
     * round the mean to a different binary32 value. */
    double sum = 0.0;
    for (int64_t j = 0; j < K; ++j)
        sum += (double)(h[j] * h[j]);
    float ms = (float)(sum / (double)K);
    if (c->ambiguous) {
        /* |any-order sum - this sum| <= 2 (K-1) u sum with u = 2^-53 (recursive summation
         * bound for non-negative terms, applied to both orders); widened by 2x. */
        double delta = 4.0 * (double)K * ldexp(1.0, -53) * sum;
        float lo = (float)((sum - delta) / (double)K);
        float hi = (float)((sum + delta) / (double)K);
        c->ambiguous[m] = (lo != hi) ? 1 : 0;
    }
    if (c->ms_override)
        ms = c->ms_override[m];
    if (c->ms_out)
        c->ms_out[m] = ms;

    float rstd = 1.0f / sqrtf(ms + c->eps);
    /* [P2 "How SmoothQuant prevents outliers"]: divide by the RMS, then multiply channel
     * by channel by gamma; here gamma already carries the smoothing (gamma' = gamma / s). */
    for (int64_t j = 0; j < K; ++j) {
        float t = h[j] * rstd;
        y[j] = t * c->gamma[j];
    }
    if (c->y_out)
        memcpy(c->y_out + m * K, y, (size_t)K * sizeof(float));
    if (c->q)
        oracle_quantize_row_f32(y, K, c->q + m * K, c->s + m);
    free(h);
    free(y);
}

/*
 * h = bf16(x + residual) (if residual), rstd = 1/sqrt(mean(h^2) + eps), y = h*rstd*gamma',
 * then per-token quantization of y. Optional outputs: ms_out (the binary32 mean of
 * squares used), ambiguous (1 where another summation order could change ms), y_out (the
 * fp32 normalized row before quantization). ms_override forces ms per row (used to
 * evaluate the other admissible ms of an ambiguous row). q may be NULL (y_out only).
 */
int oracle_smooth_rmsnorm_quant(const uint16_t *x, const uint16_t *residual, uint16_t *h_out,
                                const float *gamma, float eps, int64_t M, int64_t K, int8_t *q,
                                float *s, float *ms_out, uint8_t *ambiguous,
                                const float *ms_override, float *y_out, int nthreads)
{
    struct rms_ctx c = {x, residual, h_out, gamma, eps, K, q, s, ms_out, y_out, ambiguous,
                        ms_override};
    parallel_rows(rms_row, &c, M, nthreads);
    return 0;
}

/* ------------------------------------------------------------ exp and SiLU(gate)*up */

/*
 * exp for binary32, fixed so that two independent implementations agree bit for bit:
 * Cody & Waite argument reduction (x = k ln2 + r, ln2 split into a 16-bit head and a
 * binary32 tail), the degree-7 Taylor polynomial of e^r evaluated by Horner's rule with
 * fused multiply-adds, and an exact scaling by 2^k done as two power-of-two factors so
 * that overflow and gradual underflow round once, in the last multiply.
 *   x > 89 -> +inf;  x < -104 -> +0;  NaN -> NaN.
 */
float oracle_exp(float x)
{
    if (x != x)
        return x;
    if (x > 89.0f)
        return INFINITY;
    if (x < -104.0f)
        return 0.0f;
    const float log2e = 1.44269502162933349609375f;     /* RN_binary32(1/ln 2) */
    const float ln2_hi = 0.693145751953125f;            /* ln 2 to 16 significant bits */
    const float ln2_lo = 1.428606765330187045037746429443359375e-06f; /* RN(ln2 - ln2_hi) */
    float kf = rintf(x * log2e);
    int k = (int)kf;
    float r = fmaf(-kf, ln2_hi, x);
    r = fmaf(-kf, ln2_lo, r);
    /* Taylor coefficients 1/i!, i = 7 .. 0, each rounded to binary32. */
    const float c7 = 1.0f / 5040.0f, c6 = 1.0f / 720.0f, c5 = 1.0f / 120.0f,
                c4 = 1.0f / 24.0f, c3 = 1.0f / 6.0f, c2 = 0.5f, c1 = 1.0f, c0 = 1.0f;
    float p = c7;
    p = fmaf(p, r, c6);
    p = fmaf(p, r, c5);
    p = fmaf(p, r, c4);
    p = fmaf(p, r, c3);
    p = fmaf(p, r, c2);
    p = fmaf(p, r, c1);
    p = fmaf(p, r, c0);
    int k1 = k / 2; /* truncation toward zero; k1 and k - k1 are both in [-75, 65] */
    int k2 = k - k1;
    return (p * ldexpf(1.0f, k1)) * ldexpf(1.0f, k2);
}

/* silu(g) = g * sigmoid(g) = g / (1 + e^-g), in binary32 with oracle_exp. */
float oracle_silu(float g)
{
    return g / (1.0f + oracle_exp(-g));
}

struct silu_ctx {
    const uint16_t *gu;
    int64_t I;
    int8_t *q;
    float *s;
    float *a_out;
};

static void silu_row(void *vctx, int64_t m)
{
    struct silu_ctx *c = (struct silu_ctx *)vctx;
    const int64_t I = c->I;
    float *a = c->a_out ? c->a_out + m * I : (float *)malloc((size_t)I * sizeof(float));
    for (int64_t j = 0; j < I; ++j) {
        float g = oracle_bf16_to_f32(c->gu[m * 2 * I + j]);     /* gate half */
        float u = oracle_bf16_to_f32(c->gu[m * 2 * I + I + j]); /* up half */
        a[j] = oracle_silu(g) * u;
    }
    if (c->q)
        oracle_quantize_row_f32(a, I, c->q + m * I, c->s + m);
    if (!c->a_out)
        free(a);
}

/*
 * Llama MLP activation before the down projection, a = silu(gate) * up on the
 * concatenated [M, 2I] gate|up output, then per-token quantization of a (fp32, never
 * rounded to bf16).
 */
int oracle_silu_mul_quant(const uint16_t *gate_up, int64_t M, int64_t I, int8_t *q, float *s,
                          int nthreads)
{
    struct silu_ctx c = {gate_up, I, q, s, NULL};
    parallel_rows(silu_row, &c, M, nthreads);
    return 0;
}

/* The activation alone: a = silu(gate) * up in binary32, [M, I] (what oracle_silu_mul_quant
 * quantizes). */
int oracle_silu_mul(const uint16_t *gate_up, int64_t M, int64_t I, float *a, int nthreads)
{
    struct silu_ctx c = {gate_up, I, NULL, NULL, a};
    parallel_rows(silu_row, &c, M, nthreads);
    return 0;
}

/* -------------------------------------------------------------- GEMM and dequant */

/* Dequantize one accumulator [P2 "applied and reversed after accumulation"; P4 "converting
 * back to BF16"]: y = bf16( (float(acc) * s_tok) * s_ch ). */
uint16_t oracle_dequant(int32_t acc, float s_tok, float s_ch)
{
    float f = (float)acc; /* round to nearest even: |acc| may exceed 2^24 */
    f = f * s_tok;
    f = f * s_ch;
    return oracle_f32_to_bf16(f);
}

struct gemm_ctx {
    const int8_t *xq;
    const float *s_tok;
    const int8_t *wq;
    const float *s_ch;
    int64_t N, K;
    uint16_t *y;
    int32_t *acc;
};

static void gemm_row(void *vctx, int64_t m)
{
    struct gemm_ctx *c = (struct gemm_ctx *)vctx;
    for (int64_t n = 0; n < c->N; ++n) {
        int32_t a = 0;
        for (int64_t k = 0; k < c->K; ++k)
            a += (int32_t)c->xq[m * c->K + k] * (int32_t)c->wq[n * c->K + k];
        if (c->acc)
            c->acc[m * c->N + n] = a;
        if (c->y)
            c->y[m * c->N + n] = oracle_dequant(a, c->s_tok[m], c->s_ch[n]);
    }
}

/*
 * y[m,n] = bf16( (float(sum_k xq[m,k] wq[n,k]) * s_tok[m]) * s_ch[n] ).
 * xq [M,K] and wq [N,K] are int8, both K-contiguous; the int32 sum is exact for
 * K <= 2^31 / 127^2 = 133,144. acc (optional) receives the int32 sums [M,N].
 */
int oracle_gemm_dequant(const int8_t *xq, const float *s_tok, const int8_t *wq,
                        const float *s_ch, int64_t M, int64_t N, int64_t K, uint16_t *y,
                        int32_t *acc, int nthreads)
{
    struct gemm_ctx c = {xq, s_tok, wq, s_ch, N, K, y, acc};
    parallel_rows(gemm_row, &c, M, nthreads);
    return 0;
}

/* The same output at `count` chosen (m, n) positions only, for shapes too large to do whole. */
int oracle_gemm_dequant_sampled(const int8_t *xq, const float *s_tok, const int8_t *wq,
                                const float *s_ch, int64_t K, const int64_t *ms,
                                const int64_t *ns, int64_t count, uint16_t *y, int32_t *acc)
{
    for (int64_t i = 0; i < count; ++i) {
        int64_t m = ms[i], n = ns[i];
        int32_t a = 0;
        for (int64_t k = 0; k < K; ++k)
            a += (int32_t)xq[m * K + k] * (int32_t)wq[n * K + k];
        if (acc)
            acc[i] = a;
        if (y)
            y[i] = oracle_dequant(a, s_tok[m], s_ch[n]);
    }
    return 0;
}

/* ------------------------------------------------------------- offline preparation */

/* max_m |A[m, j]| over the rows of a fp32 [M, K] matrix (the calibration statistic of
 * [P2 "How the SmoothQuant smoothing factor is computed"]). */
int oracle_column_absmax_f32(const float *a, int64_t M, int64_t K, float *amax)
{
    for (int64_t j = 0; j < K; ++j)
        amax[j] = 0.0f;
    for (int64_t m = 0; m < M; ++m)
        for (int64_t j = 0; j < K; ++j) {
            float v = fabsf(a[m * K + j]);
            if (v > amax[j])
                amax[j] = v;
        }
    return 0;
}

/* max over rows of |B[m, j]| for a bf16 matrix, e.g. the weight W [N, K] whose input
 * channel j is column j (the page's "row j" refers to the transposed [K, N] layout). */
int oracle_column_absmax_bf16(const uint16_t *b, int64_t M, int64_t K, float *amax)
{
    for (int64_t j = 0; j < K; ++j)
        amax[j] = 0.0f;
    for (int64_t m = 0; m < M; ++m)
        for (int64_t j = 0; j < K; ++j) {
            float v = fabsf(oracle_bf16_to_f32(b[m * K + j]));
            if (v > amax[j])
                amax[j] = v;
        }
    return 0;
}

/*
 * Smoothing factor per input channel, s_j = max|A_j|^alpha / max|W_j|^(1 - alpha),
 * evaluated in binary64 and rounded once to binary32. A channel with no activation or no
 * weight range keeps s_j = 1 (the page is silent).
 */
int oracle_smoothing_factors(const float *a_max, const float *w_max, int64_t K, double alpha,
                             float *s)
{
    for (int64_t j = 0; j < K; ++j) {
        if (a_max[j] == 0.0f || w_max[j] == 0.0f) {
            s[j] = 1.0f;
            continue;
        }
        double v = pow((double)a_max[j], alpha) / pow((double)w_max[j], 1.0 - alpha);
        s[j] = (float)v;
    }
    return 0;
}

/* gamma'_j = gamma_j / s_j and the reciprocal 1/s_j used when smoothing X directly
 * [P2 "How the SmoothQuant smoothing factor is computed", last paragraph]. */
int oracle_fold_gamma(const float *gamma, const float *s, int64_t K, float *gamma_folded,
                      float *s_inv)
{
    for (int64_t j = 0; j < K; ++j) {
        if (gamma_folded)
            gamma_folded[j] = gamma[j] / s[j];
        if (s_inv)
            s_inv[j] = 1.0f / s[j];
    }
    return 0;
}

/* W'[n, j] = W[n, j] * s_j: the receiving linear's input channel j scaled up by s_j
 * [P2 "How the SmoothQuant smoothing factor is computed", last paragraph]. fp32 out. */
int oracle_smooth_weight(const uint16_t *w, const float *s, int64_t N, int64_t K, float *out)
{
    for (int64_t n = 0; n < N; ++n)
        for (int64_t j = 0; j < K; ++j)
            out[n * K + j] = oracle_bf16_to_f32(w[n * K + j]) * s[j];
    return 0;
}

struct rtn_ctx {
    const uint16_t *w;
    const float *s;
    int64_t K;
    int8_t *wq;
    float *s_ch;
};

static void rtn_row(void *vctx, int64_t n)
{
    struct rtn_ctx *c = (struct rtn_ctx *)vctx;
    float *v = (float *)malloc((size_t)c->K * sizeof(float));
    for (int64_t j = 0; j < c->K; ++j) {
        v[j] = oracle_bf16_to_f32(c->w[n * c->K + j]);
        if (c->s)
            v[j] = v[j] * c->s[j]; /* W' = W diag(s): input channel j scaled up by s_j */
    }
    oracle_quantize_row_f32(v, c->K, c->wq + n * c->K, c->s_ch + n);
    free(v);
}

/*
 * Per-output-channel round-to-nearest weight quantization of the smoothed weight
 * [P2 "The problem with naive quantization"]: for each output channel n (a row of the
 * [N, K] weight), s_ch[n] = max_j |W'[n, j]| / 127 and wq = round(W' / s_ch).
 * s may be NULL (no smoothing).
 */
int oracle_rtn_weights(const uint16_t *w, const float *s, int64_t N, int64_t K, int8_t *wq,
                       float *s_ch, int nthreads)
{
    struct rtn_ctx c = {w, s, K, wq, s_ch};
    parallel_rows(rtn_row, &c, N, nthreads);
    return 0;
}

/* ------------------------------------------------------------------ GPTQ weights */

/*
 * GPTQ weight quantization [P2 "The solution: How GPTQ improves on naive quantization": after
 * rounding each weight, measure the error it introduced and redistribute it over the weights
 * not yet quantized, guided by a Hessian computed from the calibration activations; P1
 * "Crucial Config Tips for Performance": a dampening factor]. The pages give the steps in
 * prose only; the arithmetic is the GPTQ paper's (Frantar et al., 2022), which the pages
 * follow: per output channel (a row of W [N, K]), columns in order j = 0 .. K-1,
 *   q_j = clamp(rint(w_j / s), -127, 127)                (s: the row's RTN scale, kept fixed)
 *   e_j = (w_j - q_j s) / U[j][j]
 *   w_k = w_k - e_j U[j][k]  for every k > j             (the compensation)
 * with U the upper-triangular Cholesky factor of H^-1 (H^-1 = U^T U), whose row j is the
 * inverse Hessian of the columns not yet quantized, scaled, that the compensation needs.
 * Everything is binary64 here; H is built, dampened and factored by the three functions
 * below, in this order.
 */

/* Steps 1-3: H = (2 / T) X^T X from the calibration activations X [T, K] (binary32, as the
 * layer receives them); a column with H_jj = 0 (an input channel that is always zero) gets
 * H_jj = 1 and is flagged dead (its weights are zeroed before quantization); then
 * H_jj += damp * mean_j(H_jj). H: [K, K] row-major. */
int oracle_gptq_hessian(const float *x, int64_t T, int64_t K, double damp, double *H,
                        uint8_t *dead)
{
    for (int64_t i = 0; i < K; ++i)
        for (int64_t j = 0; j < K; ++j) {
            double acc = 0.0;
            for (int64_t t = 0; t < T; ++t)
                acc += (double)x[t * K + i] * (double)x[t * K + j];
            H[i * K + j] = 2.0 * acc / (double)T;
        }
    double mean = 0.0;
    for (int64_t j = 0; j < K; ++j) {
        dead[j] = H[j * K + j] == 0.0;
        if (dead[j])
            H[j * K + j] = 1.0;
        mean += H[j * K + j];
    }
    mean /= (double)K;
    for (int64_t j = 0; j < K; ++j)
        H[j * K + j] += damp * mean;
    return 0;
}

/* Step 4: U with H^-1 = U^T U, U upper triangular, positive diagonal; computed as written:
 * L = Cholesky factor of H (H = L L^T), H^-1 = L^-T L^-1, then the Cholesky factorization
 * of H^-1 in the U^T U form. Returns -1 if H is not positive definite. */
int oracle_gptq_hinv_chol(const double *H, int64_t K, double *U)
{
    double *L = (double *)calloc((size_t)(K * K), sizeof(double));
    double *Li = (double *)calloc((size_t)(K * K), sizeof(double));
    double *Hi = (double *)calloc((size_t)(K * K), sizeof(double));
    int rc = 0;
    for (int64_t j = 0; j < K && rc == 0; ++j) {
        double d = H[j * K + j];
        for (int64_t k = 0; k < j; ++k)
            d -= L[j * K + k] * L[j * K + k];
        if (!(d > 0.0)) {
            rc = -1;
            break;
        }
        L[j * K + j] = sqrt(d);
        for (int64_t i = j + 1; i < K; ++i) {
            double v = H[i * K + j];
            for (int64_t k = 0; k < j; ++k)
                v -= L[i * K + k] * L[j * K + k];
            L[i * K + j] = v / L[j * K + j];
        }
    }
    if (rc == 0) {
        /* L^-1 by forward substitution, one unit vector (column c) at a time */
        for (int64_t c = 0; c < K; ++c)
            for (int64_t i = c; i < K; ++i) {
                double v = i == c ? 1.0 : 0.0;
                for (int64_t k = c; k < i; ++k)
                    v -= L[i * K + k] * Li[k * K + c];
                Li[i * K + c] = v / L[i * K + i];
            }
        /* H^-1 = (L^-1)^T L^-1 */
        for (int64_t i = 0; i < K; ++i)
            for (int64_t j = 0; j < K; ++j) {
                double v = 0.0;
                for (int64_t k = (i > j ? i : j); k < K; ++k)
                    v += Li[k * K + i] * Li[k * K + j];
                Hi[i * K + j] = v;
            }
        /* H^-1 = U^T U */
        memset(U, 0, (size_t)(K * K) * sizeof(double));
        for (int64_t i = 0; i < K && rc == 0; ++i) {
            double d = Hi[i * K + i];
            for (int64_t k = 0; k < i; ++k)
                d -= U[k * K + i] * U[k * K + i];
            if (!(d > 0.0)) {
                rc = -1;
                break;
            }
            U[i * K + i] = sqrt(d);
            for (int64_t j = i + 1; j < K; ++j) {
                double v = Hi[i * K + j];
                for (int64_t k = 0; k < i; ++k)
                    v -= U[k * K + i] * U[k * K + j];
                U[i * K + j] = v / U[i * K + i];
            }
        }
    }
    free(L);
    free(Li);
    free(Hi);
    return rc;
}

struct gptq_ctx {
    const float *w;
    int64_t K;
    const uint8_t *dead;
    const double *U;
    int8_t *q;
    float *s_ch;
    double *wcomp;
    const int8_t *q_follow;
    double tie_tol;
    uint8_t *status;
};

static void gptq_row(void *vctx, int64_t n)
{
    struct gptq_ctx *c = (struct gptq_ctx *)vctx;
    const int64_t K = c->K;
    /* the row's scale, from the weight as given (RTN's scale) */
    float amax = 0.0f;
    for (int64_t j = 0; j < K; ++j)
        if (fabsf(c->w[n * K + j]) > amax)
            amax = fabsf(c->w[n * K + j]);
    const float s = amax / 127.0f;
    c->s_ch[n] = s;
    double *w = (double *)malloc((size_t)K * sizeof(double));
    for (int64_t j = 0; j < K; ++j)
        w[j] = c->dead[j] ? 0.0 : (double)c->w[n * K + j];
    for (int64_t j = 0; j < K; ++j) {
        if (c->wcomp)
            c->wcomp[n * K + j] = w[j];
        double qd = 0.0, r = 0.0;
        if (s > 0.0f) {
            r = w[j] / (double)s;
            qd = rint(r);
            qd = qd > 127.0 ? 127.0 : (qd < -127.0 ? -127.0 : qd);
        }
        if (c->q_follow) {
            /* follow given codes: judge each against this step's own decision */
            const double qf = (double)c->q_follow[n * K + j];
            uint8_t st = 0;
            if (qf != qd) {
                /* admissible only across a rounding tie: |qf - qd| = 1 and r within tie_tol
                 * of the half-integer between them */
                const double mid = 0.5 * (qf + qd);
                st = (fabs(qf - qd) == 1.0 && fabs(r - mid) <= c->tie_tol) ? 1 : 2;
            }
            c->status[n * K + j] = st;
            qd = qf;
        }
        c->q[n * K + j] = (int8_t)qd;
        const double e = (w[j] - qd * (double)s) / c->U[j * K + j];
        for (int64_t k = j + 1; k < K; ++k)
            w[k] -= e * c->U[j * K + k];
    }
    free(w);
}

/* Steps 5-6 for the rows of W [N, K] (binary32, the smoothed weight) given dead and U.
 * wcomp (optional): the compensated value of every weight at the moment it is quantized.
 * q_follow (optional): codes from elsewhere to propagate instead of this function's own;
 * status[n, j] then says whether code j of row n equals the own decision (0), differs from
 * it by one across a rounding tie within tie_tol (1), or differs otherwise (2). */
int oracle_gptq_quantize(const float *w, int64_t N, int64_t K, const uint8_t *dead,
                         const double *U, int8_t *q, float *s_ch, double *wcomp,
                         const int8_t *q_follow, double tie_tol, uint8_t *status, int nthreads)
{
    struct gptq_ctx c = {w, K, dead, U, q, s_ch, wcomp, q_follow, tie_tol, status};
    parallel_rows(gptq_row, &c, N, nthreads);
    return 0;
}
