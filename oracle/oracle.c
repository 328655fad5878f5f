/*
 * oracle.c -- plain, slow CPU oracle of the W8A8 linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the tests, the smoke check and the CPU-baseline leg
 * of the benchmark use it.  It shares no code, header or table with the CUDA
 * library.
 *
 * Source of the method: "Realizing Native INT8 Compute for Diffusion
 * Transformers on Consumer GPUs: A Fused INT8 GEMM Kernel for Ideogram 4.0"
 * (arXiv 2606.14598), abstract.  The abstract describes W8A8 post-training
 * quantization, an int8 x int8 -> int32 GEMM, and a per-token x per-channel
 * dequantization plus bias folded into the GEMM epilogue, with bf16 output.
 * The page on themodelwire.com restates the same epilogue ("per-token,
 * per-channel dequantization").  The pages give no formulas; the readings
 * taken here are the plainest ones and are listed in the design notes:
 *
 *   scale[r]  = fl32( max_k |x[r,k]| / 127 )           symmetric absmax
 *   q[r,k]    = clamp( rne( fl32(x[r,k] / scale[r]) ), -127, 127 )
 *               (a row whose scale is 0 -- all zeros, or fp32 weights so
 *               small that absmax/127 underflows -- gets q 0, no division)
 *   acc[m,n]  = sum_k q_x[m,k] * q_w[n,k]              exact integer
 *   out[m,n]  = bf16_rne( fl32( fl32( fl32(acc)*s_a[m] ) * s_w[n] ) + bias[n] )
 *
 * Every floating-point step is one IEEE binary32 operation in the order
 * written; the file must be compiled with -ffp-contract=off so that no
 * multiply-add is fused, and without -ffast-math (subnormals, exact
 * division).  Rounding-mode dependent calls (nearbyintf) rely on the
 * default round-to-nearest-even mode.
 *
 * FP8 variant (the paper's comparison baseline and its "native FP8 path" on
 * B200): the same per-token / per-channel symmetric scheme with OCP FP8
 * E4M3 codes (1 sign, 4 exponent bits with bias 7, 3 mantissa bits; largest
 * finite value 448; no infinities):
 *
 *   scale[r]  = fl32( max_k |x[r,k]| / 448 )
 *   q[r,k]    = e4m3_rne( clamp( fl32(x[r,k] / scale[r]), -448, 448 ) )
 *   acc[m,n]  = sum_k e4m3(q_x[m,k]) * e4m3(q_w[n,k])   (exact, here in binary64)
 *   out[m,n]  = bf16_rne( fl32( fl32( fl32(acc)*s_a[m] ) * s_w[n] ) + bias[n] )
 *
 * GELU before a linear layer (the producer of its input, fused with the
 * per-token quantizer on the GPU).  The pages name no activation; the one
 * taken is the tanh form of GELU (Hendrycks & Gimpel, "Gaussian Error
 * Linear Units"), as DiT MLPs use it, rounded once to bf16 -- what a GELU
 * kernel stores for the next linear layer:
 *
 *   gelu(h)   = 0.5 h (1 + tanh(u)),   u = sqrt(2/pi) (h + 0.044715 h^3)
 *   g[r,k]    = bf16_rne( gelu(h[r,k]) ),  then the quantizer above on g
 *
 * gelu is evaluated in binary64 through the equal form h / (1 + exp(-2u))
 * (0.5 (1 + tanh u) = 1 / (1 + exp(-2u))), which, unlike 1 + tanh(u), does
 * not cancel for negative h, with the C library's exp, and the binary64
 * value is rounded once to bf16 (no intermediate binary32 rounding).
 *
 * Parity pins (what this file is checked against, other than itself):
 * brute force and closed forms in the CPU test suite -- numpy float32
 * division and rint for the quantizer, numpy int64 matmul and exact
 * integer closed forms for the accumulator, torch's bf16 conversion for
 * the rounding helper, and an fp64 recomputation bounding the epilogue;
 * for GELU, the correctly rounded bf16 value of the exact function
 * (60-digit decimal arithmetic) on every bf16 input, exact rational
 * rounding for the binary64 -> bf16 step, and torch's float64 GELU.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------- bf16 */

/* bf16 is the upper half of a binary32; widening is exact. */
float oracle_bf16_to_f32(uint16_t h) {
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Round a binary32 to the nearest bf16, ties to even (IEEE 754 RNE). */
uint16_t oracle_f32_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if (isnan(f)) return (uint16_t)((u >> 16) | 0x0040u); /* stay NaN */
    uint32_t kept = u >> 16;          /* truncated bf16 */
    uint32_t dropped = u & 0xffffu;   /* discarded low half */
    int round_up;
    if (dropped > 0x8000u) round_up = 1;
    else if (dropped < 0x8000u) round_up = 0;
    else round_up = (int)(kept & 1u); /* exact tie: go to even */
    /* A carry out of the mantissa moves into the exponent, which is the
     * correct next representable value (up to and including infinity). */
    return (uint16_t)(kept + (uint32_t)round_up);
}

/* ------------------------------------------------------------ fp8 e4m3 */

/* Value of an E4M3 code: sign, exponent e (bias 7), mantissa m (3 bits);
 * e == 0 is subnormal (m/8 * 2^-6); 0x7F / 0xFF are NaN. */
double oracle_e4m3_to_f64(uint8_t c) {
    int sign = (c >> 7) & 1;
    int e = (c >> 3) & 0xF;
    int m = c & 7;
    double v;
    if (e == 0xF && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m / 8.0, -6);
    else v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

/* Values of the non-negative finite codes 0x00..0x7E (filled once). */
static double e4m3_pos[0x7F];
static pthread_once_t e4m3_once = PTHREAD_ONCE_INIT;
static void e4m3_fill(void) {
    for (int c = 0; c < 0x7F; ++c) e4m3_pos[c] = oracle_e4m3_to_f64((uint8_t)c);
}

/* The E4M3 code nearest to f (ties to the even mantissa), |f| <= 448
 * (callers clamp).  Found by scanning the 127 non-negative finite codes in
 * increasing order of value, which is the definition of round to nearest. */
uint8_t oracle_f32_to_e4m3_rne(float f) {
    pthread_once(&e4m3_once, e4m3_fill);
    double a = fabs((double)f);
    uint8_t sign = (f < 0.0f || (f == 0.0f && signbit(f))) ? 0x80 : 0x00;
    uint8_t best = 0;
    for (uint8_t c = 1; c < 0x7F; ++c) {        /* codes 0x00..0x7E are finite, increasing */
        double lo = e4m3_pos[c - 1];
        double hi = e4m3_pos[c];
        if (a < lo) break;
        if (a >= hi) { best = c; continue; }
        /* lo <= a < hi */
        double mid = 0.5 * (lo + hi);
        if (a > mid) best = c;
        else if (a < mid) best = (uint8_t)(c - 1);
        else best = ((c & 1) == 0) ? c : (uint8_t)(c - 1);  /* tie: even code */
        break;
    }
    return (uint8_t)(sign | best);
}

static void quantize_row_fp8(const float* v, int64_t K, uint8_t* q, float* scale) {
    float peak = 0.0f;
    for (int64_t k = 0; k < K; ++k) peak = fmaxf(peak, fabsf(v[k]));
    float sc = peak / 448.0f;
    *scale = sc;
    for (int64_t k = 0; k < K; ++k) {
        if (sc == 0.0f) { q[k] = 0; continue; }
        float u = v[k] / sc;         /* one IEEE binary32 division */
        u = fminf(fmaxf(u, -448.0f), 448.0f);
        q[k] = oracle_f32_to_e4m3_rne(u);
    }
}

/* Per-token FP8 quantizer: bf16 X [M, K] -> E4M3 codes [M, K] + fp32 scales. */
int oracle_quantize_rows_bf16_fp8(const uint16_t* x, int64_t M, int64_t K, int64_t ldx,
                                  uint8_t* q, int64_t ldq, float* scale) {
    if (M < 0 || K < 1 || ldx < K || ldq < K) return 1;
    float* row = (float*)malloc((size_t)K * sizeof(float));
    if (!row) return 2;
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t k = 0; k < K; ++k) row[k] = oracle_bf16_to_f32(x[m * ldx + k]);
        quantize_row_fp8(row, K, q + m * ldq, scale + m);
    }
    free(row);
    return 0;
}

/* Per-channel FP8 quantizer of fp32 W [N, K]. */
int oracle_quantize_rows_f32_fp8(const float* w, int64_t N, int64_t K, int64_t ldw,
                                 uint8_t* q, int64_t ldq, float* scale) {
    if (N < 0 || K < 1 || ldw < K || ldq < K) return 1;
    for (int64_t n = 0; n < N; ++n) quantize_row_fp8(w + n * ldw, K, q + n * ldq, scale + n);
    return 0;
}

/* acc[m, n] = sum_k e4m3(a[m,k]) * e4m3(b[n,k]), in binary64: each product of
 * two 4-significant-bit values is exact, and for the value ranges of scaled
 * codes (|q| <= 448, K <= 2^17) the running sum stays exact to far below
 * binary32's precision. */
int oracle_gemm_fp8_f64(const uint8_t* a, const uint8_t* b, int64_t M, int64_t N, int64_t K, double* acc) {
    if (M < 0 || N < 0 || K < 1) return 1;
    double lut[256];
    for (int c = 0; c < 256; ++c) lut[c] = oracle_e4m3_to_f64((uint8_t)c);
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double s = 0.0;
            for (int64_t k = 0; k < K; ++k) s += lut[a[m * K + k]] * lut[b[n * K + k]];
            acc[m * N + n] = s;
        }
    return 0;
}

/* The epilogue of the FP8 variant: the accumulator rounded once to binary32,
 * then the same operations as the int8 epilogue. */
int oracle_epilogue_fp8(const double* acc, const float* scale_a, const float* scale_w,
                        const uint16_t* bias, int64_t M, int64_t N, uint16_t* out) {
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            float d = (float)acc[m * N + n];      /* the one rounding of the sum */
            d *= scale_a[m];
            d *= scale_w[n];
            float bn = bias ? oracle_bf16_to_f32(bias[n]) : 0.0f;
            out[m * N + n] = oracle_f32_to_bf16_rne(d + bn);
        }
    return 0;
}

/* ------------------------------------------------- GELU, the producer of X */

/* Round a binary64 to the nearest bf16, ties to even, in one step (a
 * binary64 -> binary32 -> bf16 route would round twice).  bf16 has an
 * 8-bit significand and binary32's exponent range: on [2^E, 2^(E+1)),
 * E >= -126, its values are the multiples of 2^(E-7); below 2^-126 the
 * subnormal ones are the multiples of 2^-133.  The quotient by that spacing
 * is exact (a power-of-two scaling), nearbyint rounds it to an integer with
 * ties to even, and the product back is a bf16 value (2^128 and beyond is
 * +-inf). */
uint16_t oracle_f64_to_bf16_rne(double d) {
    uint16_t sign = signbit(d) ? 0x8000u : 0x0000u;
    if (isnan(d)) return (uint16_t)(sign | 0x7FC0u);
    double a = fabs(d);
    if (a == 0.0) return sign;
    if (isinf(a)) return (uint16_t)(sign | 0x7F80u);
    int e;
    frexp(a, &e);                  /* a in [2^(e-1), 2^e) */
    int E = e - 1;
    if (E < -126) E = -126;        /* the subnormal spacing */
    double n = nearbyint(ldexp(a, 7 - E));
    double v = ldexp(n, E - 7);
    if (v >= 0x1p128) return (uint16_t)(sign | 0x7F80u);
    float f = (float)v;            /* exact: v is a bf16 value */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(sign | (u >> 16));
}

/* GELU of h, tanh form, in binary64 (each operation rounded in the order
 * written; -ffp-contract=off keeps the products and sums separate). */
static const double GELU_C0 = 0.79788456080286535587989211986876373695;  /* sqrt(2 / pi) */
static const double GELU_C1 = 0.044715;

double oracle_gelu_f64(double h) {
    double h3 = (h * h) * h;
    double inner = h + GELU_C1 * h3;
    double u = GELU_C0 * inner;
    double e = exp(-2.0 * u);      /* +inf for very negative h: h / inf = -0 */
    return h / (1.0 + e);
}

/* Element-wise over arrays (for the checks of these two functions). */
void oracle_gelu_f64_array(const double* x, int64_t n, double* y) {
    for (int64_t i = 0; i < n; ++i) y[i] = oracle_gelu_f64(x[i]);
}

void oracle_f64_to_bf16_array(const double* x, int64_t n, uint16_t* y) {
    for (int64_t i = 0; i < n; ++i) y[i] = oracle_f64_to_bf16_rne(x[i]);
}

/* g = bf16_rne(GELU(h)) for bf16 rows h [M, K] (row stride ldh) into g
 * (row stride ldg): what a GELU kernel writes for the next linear layer. */
int oracle_gelu_rows(const uint16_t* h, int64_t M, int64_t K, int64_t ldh, uint16_t* g, int64_t ldg) {
    if (M < 0 || K < 0 || ldh < K || ldg < K) return 1;
    for (int64_t m = 0; m < M; ++m)
        for (int64_t k = 0; k < K; ++k) {
            double hv = (double)oracle_bf16_to_f32(h[m * ldh + k]);
            g[m * ldg + k] = oracle_f64_to_bf16_rne(oracle_gelu_f64(hv));
        }
    return 0;
}

/* --------------------------------------------------- symmetric quantizer */

/* One row: absmax scale and int8 codes, as described in the header. */
static void quantize_row(const float* v, int64_t K, int8_t* q, float* scale) {
    float amax = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
        float a = fabsf(v[k]);
        if (a > amax) amax = a;
    }
    float s = amax / 127.0f;
    *scale = s;
    for (int64_t k = 0; k < K; ++k) {
        if (s == 0.0f) { q[k] = 0; continue; }
        float t = v[k] / s;          /* one IEEE binary32 division */
        float r = nearbyintf(t);     /* ties to even */
        if (r > 127.0f) r = 127.0f;
        if (r < -127.0f) r = -127.0f;
        q[k] = (int8_t)r;
    }
}

/* Per-token activation quantizer: bf16 X [M, K] (row stride ldx elements)
 * -> int8 Xq [M, K] (row stride ldq) and fp32 scale_a [M]. */
int oracle_quantize_rows_bf16(const uint16_t* x, int64_t M, int64_t K, int64_t ldx,
                              int8_t* q, int64_t ldq, float* scale) {
    if (M < 0 || K < 1 || ldx < K || ldq < K) return 1;
    float* row = (float*)malloc((size_t)K * sizeof(float));
    if (!row) return 2;
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t k = 0; k < K; ++k) row[k] = oracle_bf16_to_f32(x[m * ldx + k]);
        quantize_row(row, K, q + m * ldq, scale + m);
    }
    free(row);
    return 0;
}

/* Per-output-channel weight quantizer: fp32 W [N, K] -> int8 Wq [N, K] and
 * fp32 scale_w [N].  Same rule as the activation quantizer, one row per
 * output channel. */
int oracle_quantize_rows_f32(const float* w, int64_t N, int64_t K, int64_t ldw,
                             int8_t* q, int64_t ldq, float* scale) {
    if (N < 0 || K < 1 || ldw < K || ldq < K) return 1;
    for (int64_t n = 0; n < N; ++n) quantize_row(w + n * ldw, K, q + n * ldq, scale + n);
    return 0;
}

/* ----------------------------------------------------- exact int GEMM */

typedef struct {
    const int8_t* a;   /* [M, K] */
    const int8_t* b;   /* [N, K] */
    int64_t* acc;      /* [M, N] */
    int64_t M, N, K;
    int64_t row_begin, row_end;
} gemm_job;

static void* gemm_rows(void* arg) {
    gemm_job* j = (gemm_job*)arg;
    for (int64_t m = j->row_begin; m < j->row_end; ++m) {
        const int8_t* ar = j->a + m * j->K;
        for (int64_t n = 0; n < j->N; ++n) {
            const int8_t* br = j->b + n * j->K;
            int64_t s = 0;
            for (int64_t k = 0; k < j->K; ++k) s += (int64_t)ar[k] * (int64_t)br[k];
            j->acc[m * j->N + n] = s;
        }
    }
    return NULL;
}

/* acc[m, n] = sum_k a[m, k] * b[n, k] in int64 (both operands K-contiguous,
 * i.e. acc = A . B^T as in a linear layer).  Rows are split over nthreads
 * POSIX threads; the arithmetic of each output is the plain loop above. */
int oracle_gemm_i64(const int8_t* a, const int8_t* b, int64_t M, int64_t N, int64_t K,
                    int64_t* acc, int nthreads) {
    if (M < 0 || N < 0 || K < 1) return 1;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if ((int64_t)nthreads > M) nthreads = (int)(M > 0 ? M : 1);
    pthread_t tid[256];
    int spawned[256];
    gemm_job job[256];
    int64_t per = (M + nthreads - 1) / nthreads;
    for (int t = 0; t < nthreads; ++t) {
        job[t].a = a; job[t].b = b; job[t].acc = acc;
        job[t].M = M; job[t].N = N; job[t].K = K;
        job[t].row_begin = (int64_t)t * per;
        job[t].row_end = job[t].row_begin + per < M ? job[t].row_begin + per : M;
        spawned[t] = 0;
        if (job[t].row_begin >= job[t].row_end) continue;
        if (nthreads > 1 && pthread_create(&tid[t], NULL, gemm_rows, &job[t]) == 0)
            spawned[t] = 1;
        else
            gemm_rows(&job[t]);
    }
    for (int t = 0; t < nthreads; ++t)
        if (spawned[t]) pthread_join(tid[t], NULL);
    return 0;
}

/* ------------------------------------------------ dequant + bias epilogue */

/* out[m, n] = bf16_rne( (fl32(acc) * s_a[m]) * s_w[n] + bias[n] ), each op a
 * separate binary32 operation.  bias may be NULL (treated as zero).
 * Returns 3 if an accumulator does not fit in int32 (the GEMM's contract). */
int oracle_epilogue(const int64_t* acc, const float* scale_a, const float* scale_w,
                    const uint16_t* bias, int64_t M, int64_t N, uint16_t* out) {
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            int64_t a = acc[m * N + n];
            if (a > INT32_MAX || a < INT32_MIN) return 3;
            /* int32 -> double is exact; double -> float rounds to nearest
             * even, which is the single rounding of int32 -> float. */
            float t = (float)(double)a;
            t = t * scale_a[m];
            t = t * scale_w[n];
            float b = bias ? oracle_bf16_to_f32(bias[n]) : 0.0f;
            float y = t + b;
            out[m * N + n] = oracle_f32_to_bf16_rne(y);
        }
    }
    return 0;
}

/* The same epilogue carried out in binary64 without rounding to bf16: used
 * only to bound the binary32 oracle's own rounding error. */
int oracle_epilogue_f64(const int64_t* acc, const float* scale_a, const float* scale_w,
                        const uint16_t* bias, int64_t M, int64_t N, double* out) {
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double b = bias ? (double)oracle_bf16_to_f32(bias[n]) : 0.0;
            out[m * N + n] = (double)acc[m * N + n] * (double)scale_a[m] * (double)scale_w[n] + b;
        }
    return 0;
}

/* ------------------------------------------------------- whole layer */

/* The W8A8 linear layer, step by step: per-token quantization of X, exact
 * integer GEMM against the pre-quantized weight, dequant + bias epilogue.
 * xq / scale_a / acc receive the intermediates (acc may be NULL). */
int oracle_linear(const uint16_t* x, const int8_t* wq, const float* scale_w,
                  const uint16_t* bias, int64_t M, int64_t N, int64_t K,
                  uint16_t* out, int8_t* xq, float* scale_a, int64_t* acc, int nthreads) {
    int rc = oracle_quantize_rows_bf16(x, M, K, K, xq, K, scale_a);
    if (rc) return rc;
    int64_t* tmp = acc;
    if (!tmp) {
        tmp = (int64_t*)malloc((size_t)(M * N > 0 ? M * N : 1) * sizeof(int64_t));
        if (!tmp) return 2;
    }
    rc = oracle_gemm_i64(xq, wq, M, N, K, tmp, nthreads);
    if (!rc) rc = oracle_epilogue(tmp, scale_a, scale_w, bias, M, N, out);
    if (!acc) free(tmp);
    return rc;
}
