/*
 * svdq_oracle.c -- plain, slow, obviously correct CPU oracle of the SVDQuant
 * W4A4 linear layer.  TEST INFRASTRUCTURE ONLY: nothing in the product path
 * (the CUDA library and its Python binding) may link, load or call this file;
 * only the tests, the smoke check and the benchmark's CPU-baseline leg do.
 * It shares no code, header, table or constant generator with the CUDA path.
 *
 * What it computes (the layer of the SVDQuant paper that the Diffusers docs
 * page "Nunchaku Lite" links to and names `svdq_w4a4`):
 *
 *     y = dequant(Q4(x/lambda)) . dequant(Q4(R))^T + ((x/lambda) . L_down) . L_up + b
 *
 *   x [M,K] bf16 activations (tokens x in-features), lambda [K] fp32 > 0 the
 *   per-input-channel smoothing divisor, R [N,K] bf16 the residual weight,
 *   L_down [K,r] and L_up [r,N] bf16 the rank-r branch, b [N] bf16.
 *
 * Schemes (Diffusers docs "Nunchaku Lite", "Supported quantization types"
 * table): svdq_w4a4 / nvfp4 / group 16 and svdq_w4a4 / int4 / group 64, both
 * "with SVDQ low-rank correction"; the config schema in the section
 * "NunchakuLiteQuantizationConfig" gives rank 32 and compute dtype bfloat16.
 *
 * Bit-level readings (the pages give the format names only):
 *   - fl32(.) is one IEEE binary32 operation rounded to nearest-even.  This
 *     file must be compiled without -ffast-math and with -ffp-contract=off.
 *   - E2M1 (FP4): grid {0, .5, 1, 1.5, 2, 3, 4, 6}; round to nearest, ties to
 *     the even code; |v| > 6 saturates to 6; the sign bit is kept (so a
 *     negative value that rounds to zero is code 0x8).
 *   - E4M3 (OCP FP8 E4M3FN): bias 7, subnormal step 2^-9, max 448, round to
 *     nearest-even, saturate to 448.
 *   - nvfp4 tensor scale S = fl32(amax / 2688) (2688 = 6 * 448); an all-zero
 *     tensor gets S = 1 so that every later reciprocal stays finite.
 *   - nvfp4 group of 16: e = E4M3(fl32(a / fl32(6 S))), dec = fl32(e S),
 *     inv = (dec == 0 ? 0 : fl32(1 / dec)), code = E2M1(fl32(v * inv)).
 *   - int4 group of 64: s = bf16_RN(fl32(a / 7)), inv = (s == 0 ? 0 :
 *     fl32(1 / s)), q = clamp(rint_even(fl32(v * inv)), -8, 7).
 *   - smoothing: v = fl32(x * fl32(1 / lambda)); the weight side uses v = R.
 *   - the GEMM, the rank-r branch and the bias are accumulated in fp64; the
 *     output is rounded once to bf16 (nearest-even).
 *
 * Layouts here are the plain logical ones (row-major; two FP4/INT4 codes per
 * byte, low nibble = even k; one scale per (row, group), row-major).  They are
 * NOT the CUDA library's MMA layouts; tests translate with their own index map.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#include <float.h>
#include <fenv.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------ bf16 */

/* bf16 bit pattern -> value (exact). */
double oracle_bf16_to_double(uint16_t h)
{
    uint32_t bits = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &bits, 4);
    return (double)f;
}

/* Round a double to the nearest bf16 (ties to even), directly (one rounding).
 * bf16 keeps 8 significant bits; normal exponents down to 2^-126, subnormal
 * step 2^-133; overflow goes to infinity as IEEE round-to-nearest does. */
uint16_t oracle_bf16_from_double(double d)
{
    double r;
    if (isnan(d)) return 0x7FC0;
    if (d == 0.0) return signbit(d) ? 0x8000 : 0x0000;
    double a = fabs(d);
    if (a < ldexp(1.0, -126)) {
        r = nearbyint(a * ldexp(1.0, 133)) * ldexp(1.0, -133);
    } else {
        int e;
        double f = frexp(a, &e);               /* a = f * 2^e, f in [0.5, 1) */
        r = ldexp(nearbyint(ldexp(f, 8)), e - 8);  /* keep 8 significant bits */
    }
    float fr;
    if (r >= ldexp(1.0, 128)) fr = INFINITY;
    else fr = (float)r;                        /* exact: r has <= 8 bits */
    if (signbit(d)) fr = -fr;
    uint32_t bits;
    memcpy(&bits, &fr, 4);
    return (uint16_t)(bits >> 16);
}

/* ------------------------------------------------------------------ E2M1 */

static const double kE2M1Grid[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double oracle_e2m1_decode(int code)
{
    double v = kE2M1Grid[code & 7];
    return (code & 8) ? -v : v;
}

/* Nearest grid point, ties to the even code.  Each test below is the
 * midpoint between two neighbouring grid values; ">" means the tie stays on
 * the lower (even) code, ">=" means the tie moves up to the (even) upper code. */
int oracle_e2m1_encode(float v)
{
    int sign = signbit(v) ? 8 : 0;
    float a = fabsf(v);
    int idx = 0;
    if (a > 0.25f) idx = 1;   /* 0 (even) | 0.5          */
    if (a >= 0.75f) idx = 2;  /* 0.5      | 1 (even)     */
    if (a > 1.25f) idx = 3;   /* 1 (even) | 1.5          */
    if (a >= 1.75f) idx = 4;  /* 1.5      | 2 (even)     */
    if (a > 2.5f) idx = 5;    /* 2 (even) | 3            */
    if (a >= 3.5f) idx = 6;   /* 3        | 4 (even)     */
    if (a > 5.0f) idx = 7;    /* 4 (even) | 6; above 6 saturates to 6 */
    return sign | idx;
}

/* ------------------------------------------------------------------ E4M3 */

double oracle_e4m3_decode(int byte)
{
    int s = (byte >> 7) & 1, e = (byte >> 3) & 15, m = byte & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);               /* subnormal: m * 2^-9 */
    else v = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -v : v;
}

/* Round to nearest-even E4M3FN, saturating to +-448 (never NaN for finite v). */
int oracle_e4m3_encode(float v)
{
    int sign = signbit(v) ? 0x80 : 0;
    double a = fabs((double)v);
    int code;
    if (isnan(v)) return 0x7F;
    if (a > 448.0) return sign | 0x7E;                  /* satfinite */
    if (a < ldexp(1.0, -6)) {
        /* subnormal range: integer multiples of 2^-9; m == 8 is the smallest
         * normal 2^-6, whose bit pattern is exactly 0x08 */
        code = (int)nearbyint(a * 512.0);
    } else {
        int e;
        double f = frexp(a, &e);                        /* a = (2f) * 2^(e-1) */
        int ex = e - 1;                                 /* in [-6, 8] */
        int m = (int)nearbyint((2.0 * f - 1.0) * 8.0);  /* 3 mantissa bits */
        if (m == 8) { m = 0; ex += 1; }
        code = ((ex + 7) << 3) | m;
        if (code > 0x7E) code = 0x7E;
    }
    return sign | code;
}

/* ------------------------------------------------------------ smoothing */

/* v = fl32(x * fl32(1/lambda[k])); lambda == NULL means no smoothing (v = x). */
static float smoothed(const uint16_t* x, const float* lambda, long row, long K, long k)
{
    float xv = (float)oracle_bf16_to_double(x[row * K + k]);
    if (!lambda) return xv;
    float inv = 1.0f / lambda[k];
    return xv * inv;
}

/* ----------------------------------------------------------- nvfp4 side */

/* S = fl32(amax|v| / 2688) over the whole tensor, or 1 for an all-zero one. */
float oracle_nvfp4_tensor_scale(const uint16_t* x, const float* lambda, long rows, long K)
{
    float amax = 0.0f;
    for (long m = 0; m < rows; ++m)
        for (long k = 0; k < K; ++k) {
            float a = fabsf(smoothed(x, lambda, m, K, k));
            if (a > amax) amax = a;
        }
    float S = amax / 2688.0f;
    if (!(S > 0.0f)) S = 1.0f;
    return S;
}

/* Per row, per group of 16: E4M3 group scale and E2M1 codes.
 *   codes  [rows, K/2]  (low nibble = even k)
 *   scales [rows, K/16] E4M3 bytes */
void oracle_nvfp4_quantize(const uint16_t* x, const float* lambda, long rows, long K,
                           float S, uint8_t* codes, uint8_t* scales)
{
    const long G = 16;
    float six_s = 6.0f * S;
#pragma omp parallel for schedule(static)
    for (long m = 0; m < rows; ++m) {
        for (long g = 0; g < K / G; ++g) {
            float v[16];
            float a = 0.0f;
            for (long i = 0; i < G; ++i) {
                v[i] = smoothed(x, lambda, m, K, g * G + i);
                if (fabsf(v[i]) > a) a = fabsf(v[i]);
            }
            int e = (six_s == 0.0f) ? 0 : oracle_e4m3_encode(a / six_s);
            float dec = (float)oracle_e4m3_decode(e) * S;
            float inv = (dec == 0.0f) ? 0.0f : 1.0f / dec;
            scales[m * (K / G) + g] = (uint8_t)e;
            for (long i = 0; i < G; i += 2) {
                int lo = oracle_e2m1_encode(v[i] * inv);
                int hi = oracle_e2m1_encode(v[i + 1] * inv);
                codes[m * (K / 2) + (g * G + i) / 2] = (uint8_t)(lo | (hi << 4));
            }
        }
    }
}

/* deq[m,k] = E2M1(code) * E4M3(scale) * S, exact in fp64. */
void oracle_nvfp4_dequant(const uint8_t* codes, const uint8_t* scales, float S,
                          long rows, long K, double* out)
{
#pragma omp parallel for schedule(static)
    for (long m = 0; m < rows; ++m)
        for (long k = 0; k < K; ++k) {
            int byte = codes[m * (K / 2) + k / 2];
            int c = (k & 1) ? (byte >> 4) : (byte & 15);
            out[m * K + k] = oracle_e2m1_decode(c) * oracle_e4m3_decode(scales[m * (K / 16) + k / 16]) * (double)S;
        }
}

/* ------------------------------------------------------------ int4 side */

/* Per row, per group of 64: bf16 scale s = bf16(amax/7), codes in [-8,7].
 *   codes  [rows, K/2] two's-complement nibbles (low nibble = even k)
 *   scales [rows, K/64] bf16 bit patterns */
void oracle_int4_quantize(const uint16_t* x, const float* lambda, long rows, long K,
                          uint8_t* codes, uint16_t* scales)
{
    const long G = 64;
#pragma omp parallel for schedule(static)
    for (long m = 0; m < rows; ++m) {
        for (long g = 0; g < K / G; ++g) {
            float v[64];
            float a = 0.0f;
            for (long i = 0; i < G; ++i) {
                v[i] = smoothed(x, lambda, m, K, g * G + i);
                if (fabsf(v[i]) > a) a = fabsf(v[i]);
            }
            uint16_t sb = oracle_bf16_from_double((double)(a / 7.0f));
            float s = (float)oracle_bf16_to_double(sb);
            float inv = (s == 0.0f) ? 0.0f : 1.0f / s;
            scales[m * (K / G) + g] = sb;
            for (long i = 0; i < G; i += 2) {
                int q[2];
                for (int j = 0; j < 2; ++j) {
                    float t = rintf(v[i + j] * inv);     /* ties to even */
                    if (t < -8.0f) t = -8.0f;
                    if (t > 7.0f) t = 7.0f;
                    q[j] = (int)t;
                }
                codes[m * (K / 2) + (g * G + i) / 2] = (uint8_t)((q[0] & 15) | ((q[1] & 15) << 4));
            }
        }
    }
}

static int int4_code(const uint8_t* codes, long K, long m, long k)
{
    int byte = codes[m * (K / 2) + k / 2];
    int c = (k & 1) ? (byte >> 4) : (byte & 15);
    return (c & 8) ? c - 16 : c;
}

/* --------------------------------------------------------- rank-r branch */

/* L[m,j] = sum_k (x[m,k] / lambda[k]) * L_down[k,j], in fp64. */
void oracle_lowrank_down(const uint16_t* x, const float* lambda, long M, long K,
                         const uint16_t* L_down, long r, double* L)
{
#pragma omp parallel for schedule(static)
    for (long m = 0; m < M; ++m)
        for (long j = 0; j < r; ++j) {
            double acc = 0.0;
            for (long k = 0; k < K; ++k) {
                double xs = oracle_bf16_to_double(x[m * K + k]) / (double)lambda[k];
                acc += xs * oracle_bf16_to_double(L_down[k * r + j]);
            }
            L[m * r + j] = acc;
        }
}

/* ------------------------------------------------------------------ GEMM */

/* One output row: y[n] = sum_k xd[k] wd[n,k] + sum_j L[j] L_up[j,n] + b[n]. */
static void lowrank_bias_row(const double* Lrow, const uint16_t* L_up, long r, const uint16_t* bias,
                             long N, double* yrow)
{
    for (long n = 0; n < N; ++n) {
        double acc = 0.0;
        for (long j = 0; j < r; ++j) acc += Lrow[j] * oracle_bf16_to_double(L_up[j * N + n]);
        if (bias) acc += oracle_bf16_to_double(bias[n]);
        yrow[n] += acc;
    }
}

/* nvfp4 linear for the selected rows of x (rows == NULL: rows 0..nrows-1).
 *   xd [*, K]   dequantized activations (fp64), indexed by the row id
 *   wd [N, K]   dequantized weight (fp64)
 *   L  [*, r]   rank-r activations (fp64) or NULL when r == 0
 *   y  [nrows, N] fp64 result, ybf [nrows, N] its bf16 rounding */
void oracle_nvfp4_linear(const double* xd, const long* rows, long nrows, long K,
                         const double* wd, long N, const double* L, const uint16_t* L_up, long r,
                         const uint16_t* bias, double* y, uint16_t* ybf)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (long i = 0; i < nrows; ++i) {
        long m = rows ? rows[i] : i;
        const double* xr = xd + m * K;
        double* yr = y + i * N;
        for (long n = 0; n < N; ++n) {
            const double* wr = wd + n * K;
            double acc = 0.0;
            for (long k = 0; k < K; ++k) acc += xr[k] * wr[k];
            yr[n] = acc;
        }
        lowrank_bias_row(r ? L + m * r : NULL, L_up, r, bias, N, yr);
        for (long n = 0; n < N; ++n) ybf[i * N + n] = oracle_bf16_from_double(yr[n]);
    }
}

/* int4 linear: per group of 64 an exact integer dot product, times the two
 * bf16 group scales, summed in fp64; plus the rank-r branch and the bias. */
void oracle_int4_linear(const uint8_t* xc, const uint16_t* xs, const long* rows, long nrows, long K,
                        const uint8_t* wc, const uint16_t* ws, long N,
                        const double* L, const uint16_t* L_up, long r,
                        const uint16_t* bias, double* y, uint16_t* ybf)
{
    const long G = 64;
#pragma omp parallel for schedule(dynamic, 1)
    for (long i = 0; i < nrows; ++i) {
        long m = rows ? rows[i] : i;
        double* yr = y + i * N;
        for (long n = 0; n < N; ++n) {
            double acc = 0.0;
            for (long g = 0; g < K / G; ++g) {
                long dot = 0;
                for (long k = g * G; k < (g + 1) * G; ++k)
                    dot += (long)int4_code(xc, K, m, k) * (long)int4_code(wc, K, n, k);
                acc += oracle_bf16_to_double(xs[m * (K / G) + g]) *
                       oracle_bf16_to_double(ws[n * (K / G) + g]) * (double)dot;
            }
            yr[n] = acc;
        }
        lowrank_bias_row(r ? L + m * r : NULL, L_up, r, bias, N, yr);
        for (long n = 0; n < N; ++n) ybf[i * N + n] = oracle_bf16_from_double(yr[n]);
    }
}

/* ------------------------------------------- fused QKV + RMSNorm + RoPE */
/*
 * The fused attention-input path of the original Nunchaku engine (the
 * tutorial page's "structural rewrite" section, the fused_qkv_norm_rottary
 * operator on one to_qkv projection; the Diffusers docs page "Nunchaku Lite",
 * section "Fused kernels": "QKV+norm+RoPE" fusion).  Readings (the pages name
 * the fusion but fix none of its details; these follow the split path the
 * tutorial prints -- norm_q / norm_k per head, then apply_rotary_emb -- with
 * the FLUX-class DiT's choices):
 *   - y [rows, N] is the to_qkv output with N = 3 * H * D: columns [0, HD) are
 *     Q, [HD, 2HD) are K, [2HD, 3HD) are V; head h of Q (or K) is its columns
 *     [hD, (h+1)D);
 *   - RMSNorm per head of Q and of K: v / sqrt(mean_d(v^2) + eps) * w[d], with
 *     its own weight w (D values) for Q and for K;
 *   - RoPE on Q and K: the pairs (2i, 2i+1) of a head rotate by the token's
 *     angle theta[i] (given as cos and sin, D/2 per token):
 *         out[2i]   = v[2i] cos - v[2i+1] sin
 *         out[2i+1] = v[2i+1] cos + v[2i] sin;
 *   - V is passed through; everything in fp64, rounded once to bf16.
 */

/* RMSNorm of one head vector v[D] with weight w (bf16 bits), in place. */
void oracle_rms_norm_head(double* v, long D, const uint16_t* w, double eps)
{
    double ss = 0.0;
    for (long d = 0; d < D; ++d) ss += v[d] * v[d];
    double inv = 1.0 / sqrt(ss / (double)D + eps);
    for (long d = 0; d < D; ++d) v[d] = v[d] * inv * oracle_bf16_to_double(w[d]);
}

/* Rotary embedding of one head vector v[D] in place: pair i by (cos[i], sin[i]). */
void oracle_rope_head(double* v, long D, const double* cs, const double* sn)
{
    for (long i = 0; i < D / 2; ++i) {
        double a = v[2 * i], b = v[2 * i + 1];
        v[2 * i] = a * cs[i] - b * sn[i];
        v[2 * i + 1] = b * cs[i] + a * sn[i];
    }
}

/* The whole epilogue on fp64 rows of y:
 *   y, out [rows, N] (N = 3 H D); cs, sn [rows, D/2] per-token cos / sin;
 *   wq, wk [D] bf16 norm weights; out_bf16 [rows, N] the bf16 rounding of out. */
void oracle_qkv_norm_rope(const double* y, long rows, long H, long D, const uint16_t* wq, const uint16_t* wk,
                          double eps, const double* cs, const double* sn, double* out, uint16_t* out_bf16)
{
    const long N = 3 * H * D;
#pragma omp parallel for schedule(static)
    for (long m = 0; m < rows; ++m) {
        const double* yr = y + m * N;
        double* o = out + m * N;
        for (long n = 0; n < N; ++n) o[n] = yr[n];
        for (long part = 0; part < 2; ++part)          /* Q, then K */
            for (long h = 0; h < H; ++h) {
                double* v = o + part * H * D + h * D;
                oracle_rms_norm_head(v, D, part == 0 ? wq : wk, eps);
                oracle_rope_head(v, D, cs + m * (D / 2), sn + m * (D / 2));
            }
        for (long n = 0; n < N; ++n) out_bf16[m * N + n] = oracle_bf16_from_double(o[n]);
    }
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Weight-only int4 linear (the awq_w4a16 scheme of the Diffusers docs page
 * "Nunchaku Lite", section "Supported quantization types"): the bf16
 * activation is used as it is; each weight is its int4 code times its bf16
 * group-64 scale; the products and their sum are taken in fp64, then the bias
 * is added and the result rounded once to bf16. */
void oracle_w4a16_linear(const uint16_t* x, const long* rows, long nrows, long K,
                         const uint8_t* wc, const uint16_t* ws, long N,
                         const uint16_t* bias, double* y, uint16_t* ybf)
{
    const long G = 64;
#pragma omp parallel for schedule(dynamic, 1)
    for (long i = 0; i < nrows; ++i) {
        long m = rows ? rows[i] : i;
        double* yr = y + i * N;
        for (long n = 0; n < N; ++n) {
            double acc = 0.0;
            for (long k = 0; k < K; ++k) {
                double w = (double)int4_code(wc, K, n, k) * oracle_bf16_to_double(ws[n * (K / G) + k / G]);
                acc += oracle_bf16_to_double(x[m * K + k]) * w;
            }
            yr[n] = acc + (bias ? oracle_bf16_to_double(bias[n]) : 0.0);
            ybf[i * N + n] = oracle_bf16_from_double(yr[n]);
        }
    }
}

/* GELU, the activation between the two linear layers of the DiT MLP that the
 * fused GELU-MLP kernel of the Diffusers docs page "Nunchaku Lite" (section
 * "Fused kernels") targets.  approx = 0: the exact form x Phi(x), written
 * with erfc so that the tail for negative x keeps its relative accuracy;
 * approx = 1: the tanh form 0.5 x (1 + tanh(u)), u = sqrt(2/pi)(x + 0.044715
 * x^3), written as x / (1 + exp(-2u)), the same function without the
 * cancellation of 1 + tanh(u) for negative u. */
double oracle_gelu(double x, int approx)
{
    if (approx == 0) return 0.5 * x * erfc(-x / sqrt(2.0));
    const double u = sqrt(2.0 / 3.14159265358979323846) * (x + 0.044715 * x * x * x);
    return x / (1.0 + exp(-2.0 * u));
}

/* bf16 in -> GELU in fp64 -> one rounding to bf16. */
void oracle_gelu_bf16(const uint16_t* in, long n, int approx, uint16_t* out)
{
#pragma omp parallel for schedule(static)
    for (long i = 0; i < n; ++i) out[i] = oracle_bf16_from_double(oracle_gelu(oracle_bf16_to_double(in[i]), approx));
}
