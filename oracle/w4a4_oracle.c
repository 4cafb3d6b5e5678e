/*
 * w4a4_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, fp64 / int64 CPU statement of what the DSFQ (Dual-Smoothed
 * Fine-Grained Quantization) W4A4 linear layer computes at inference time.
 * It exists to check the CUDA library against; nothing in the product path
 * may load it.  Only tests/, __graft_entry__.smoke() and bench.py's CPU
 * baseline / reference arm use it.  It shares no code, header, table or
 * helper with the CUDA library.
 *
 * Sources (the method is described on web pages; formulas were stripped from
 * the page text, so each step states which passage it follows and how it is
 * read):
 *   [PTQ]   page "十亿参数的三维重建模型，能塞进手机吗？" (Chinese translation of
 *           the QuantVGGT paper), section "训练后量化（PTQ）": symmetric
 *           quantizer, "round" is rounding, clamp keeps codes in
 *           [-2^(N-1), 2^(N-1)-1].
 *   [ROT]   same page, section "双平滑细粒度量化（DSFQ）" / "预全局旋转
 *           （Pre-Global-Rotation）": Hadamard matrix with H H^T = I, rotation
 *           of both activations and weights keeps the matrix product unchanged.
 *   [SMOOTH] same page, "后局部平滑（Post-Local-Smooth）": per-channel scaling
 *           factors computed from the rotated distributions, alpha (usually
 *           0.5) balances activation and weight difficulty; rotate first,
 *           then scale.
 *   [GRAN]  same page, "细粒度量化粒度（Fine-Grained Quantization
 *           Granularity）" (text truncated on the page): read as per-token
 *           activation scales and per-output-channel weight scales.
 *
 * Conventions: row-major arrays; bf16 values arrive as raw uint16 bit patterns
 * and are widened exactly to double.  Every function returns 0 on success and a
 * negative number on a bad argument.
 *
 * Pins: tests/test_oracle_pins.py checks each function against closed forms,
 * library routines and brute force (see that file's header).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static int is_pow2(int64_t d) { return d >= 1 && (d & (d - 1)) == 0; }

void oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* bf16 -> double, exact: a bf16 value is the upper half of an IEEE binary32. */
int oracle_bf16_to_double(const uint16_t *x, int64_t n, double *y)
{
    if (!x || !y || n < 0) return -1;
    for (int64_t i = 0; i < n; ++i) {
        uint32_t u = (uint32_t)x[i] << 16;
        float f;
        memcpy(&f, &u, sizeof f);
        y[i] = (double)f;
    }
    return 0;
}

/* Round a double to the nearest bf16 (8 significant bits), ties to even, in
 * one step (no detour through binary32).  Finite, normal-range inputs only
 * (the generated data never leaves that range). */
static uint16_t double_to_bf16_rne(double v)
{
    if (v == 0.0) return signbit(v) ? 0x8000u : 0u;
    int e;
    double m = frexp(v, &e);            /* v = m * 2^e, 0.5 <= |m| < 1 */
    double r = nearbyint(m * 256.0);    /* 8 significant bits, default mode = ties-to-even */
    double q = ldexp(r, e - 8);         /* exact */
    float f = (float)q;                 /* exact: q has 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(u >> 16);
}

int oracle_double_to_bf16(const double *x, int64_t n, uint16_t *y)
{
    if (!x || !y || n < 0) return -1;
    for (int64_t i = 0; i < n; ++i) y[i] = double_to_bf16_rne(x[i]);
    return 0;
}

/* GELU applied to bf16 activations before an MLP's second linear (exact erf
 * form), result rounded to bf16.  Not on the pages: the plainest reading of
 * "fc1 output goes through GELU in bf16". */
int oracle_gelu_bf16(const uint16_t *x, int64_t n, uint16_t *y)
{
    if (!x || !y || n < 0) return -1;
    for (int64_t i = 0; i < n; ++i) {
        double v;
        oracle_bf16_to_double(&x[i], 1, &v);
        double g = 0.5 * v * (1.0 + erf(v / sqrt(2.0)));
        y[i] = double_to_bf16_rne(g);
    }
    return 0;
}

/* [ROT] Sylvester Hadamard matrix of order d (d a power of two), natural
 * order, entries +-1 (unnormalised):  H_1 = [1],  H_2n = [[H_n, H_n],
 * [H_n, -H_n]].  Built by that recursion, in place in a d x d array. */
int oracle_hadamard(int32_t d, double *H)
{
    if (!H || !is_pow2(d)) return -1;
    H[0] = 1.0;
    for (int32_t n = 1; n < d; n *= 2) {
        for (int32_t i = 0; i < n; ++i) {
            for (int32_t j = 0; j < n; ++j) {
                double h = H[(int64_t)i * d + j];
                H[(int64_t)i * d + (j + n)] = h;
                H[(int64_t)(i + n) * d + j] = h;
                H[(int64_t)(i + n) * d + (j + n)] = -h;
            }
        }
    }
    return 0;
}

/* [ROT] Pre-global rotation along the feature dimension:
 *   out[r, :] = X[r, :] . (H / sqrt(d))
 * with the dense matrix product (H / sqrt(d) is orthonormal).  Used for the
 * activations X [rows, d] and, row by row, for the weights W [N, d] (the
 * rotation acts on the input-feature dimension of both). */
int oracle_rotate(const double *X, int64_t rows, int32_t d, double *out)
{
    if (!X || !out || rows < 0 || !is_pow2(d)) return -1;
    double *H = (double *)malloc(sizeof(double) * (size_t)d * (size_t)d);
    if (!H) return -2;
    oracle_hadamard(d, H);
    const double inv_sqrt_d = 1.0 / sqrt((double)d);
    int bad = 0;
#pragma omp parallel
    {
        double *acc = (double *)malloc(sizeof(double) * (size_t)d);
        if (!acc) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for schedule(static)
            for (int64_t r = 0; r < rows; ++r) {
                const double *x = X + r * d;
                for (int32_t j = 0; j < d; ++j) acc[j] = 0.0;
                for (int32_t i = 0; i < d; ++i) {
                    const double xi = x[i];
                    const double *h = H + (int64_t)i * d;
                    for (int32_t j = 0; j < d; ++j) acc[j] += xi * h[j];
                }
                for (int32_t j = 0; j < d; ++j) out[r * d + j] = acc[j] * inv_sqrt_d;
            }
            free(acc);
        }
    }
    free(H);
    return bad ? -2 : 0;
}

/* [SMOOTH] Post-local channel smoothing factors, computed in the rotated
 * space from the rotated calibration activations Xt [Mc, K] and the rotated
 * weights Wt [N, K]:
 *   s_j = (max_i |Xt[i, j]|)^alpha / (max_n |Wt[n, j]|)^(1 - alpha)
 * (SmoothQuant form; alpha = 0.5 on the page).  Reading for a channel whose
 * activation or weight maximum is zero: s_j = 1. */
int oracle_smooth_factors(const double *Xt, int64_t Mc, const double *Wt, int32_t N, int32_t K,
                          double alpha, double *s)
{
    if (!Xt || !Wt || !s || Mc < 1 || N < 1 || K < 1) return -1;
    for (int32_t j = 0; j < K; ++j) {
        double ax = 0.0, aw = 0.0;
        for (int64_t i = 0; i < Mc; ++i) ax = fmax(ax, fabs(Xt[i * K + j]));
        for (int32_t n = 0; n < N; ++n) aw = fmax(aw, fabs(Wt[(int64_t)n * K + j]));
        if (ax > 0.0 && aw > 0.0)
            s[j] = pow(ax, alpha) / pow(aw, 1.0 - alpha);
        else
            s[j] = 1.0;
    }
    return 0;
}

/* [PTQ] + [GRAN] Symmetric uniform quantization of each row of Y [rows, K]
 * with its own step (per token for activations, per output channel for
 * weights):
 *   delta = max_j |Y[r, j]| / (2^(bits-1) - 1)
 *   q     = clamp(round(Y / delta), -2^(bits-1), 2^(bits-1) - 1)
 * "round" is read as round-half-to-even.  A row that is all zero gets
 * delta = 0 and all-zero codes.  bits = 4 gives codes in [-8, 7] and
 * delta = absmax / 7. */
int oracle_quantize_rows(const double *Y, int64_t rows, int32_t K, int32_t bits, int8_t *q,
                         double *delta)
{
    if (!Y || !q || !delta || rows < 0 || K < 1 || bits < 2 || bits > 8) return -1;
    const double qmax = (double)((1 << (bits - 1)) - 1);
    const double qmin = -(double)(1 << (bits - 1));
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        const double *y = Y + r * K;
        double amax = 0.0;
        for (int32_t j = 0; j < K; ++j) amax = fmax(amax, fabs(y[j]));
        const double d = amax / qmax;
        delta[r] = d;
        for (int32_t j = 0; j < K; ++j) {
            double v = (d > 0.0) ? nearbyint(y[j] / d) : 0.0;   /* ties to even */
            if (v < qmin) v = qmin;
            if (v > qmax) v = qmax;
            q[r * K + j] = (int8_t)v;
        }
    }
    return 0;
}

/* Storage of int4 codes: two per byte, element 2i in the low nibble and 2i+1
 * in the high nibble, each nibble the 4-bit two's complement of its code.
 * (The pages do not fix a packing; this is the library's documented format.) */
int oracle_pack_int4(const int8_t *q, int64_t rows, int32_t K, uint8_t *packed)
{
    if (!q || !packed || rows < 0 || K < 2 || (K & 1)) return -1;
    for (int64_t r = 0; r < rows; ++r) {
        for (int32_t i = 0; i < K / 2; ++i) {
            int lo = q[r * K + 2 * i], hi = q[r * K + 2 * i + 1];
            if (lo < -8 || lo > 7 || hi < -8 || hi > 7) return -3;
            packed[r * (K / 2) + i] = (uint8_t)(((unsigned)lo & 0xFu) | (((unsigned)hi & 0xFu) << 4));
        }
    }
    return 0;
}

int oracle_unpack_int4(const uint8_t *packed, int64_t rows, int32_t K, int8_t *q)
{
    if (!q || !packed || rows < 0 || K < 2 || (K & 1)) return -1;
    for (int64_t r = 0; r < rows; ++r) {
        for (int32_t i = 0; i < K / 2; ++i) {
            unsigned b = packed[r * (K / 2) + i];
            int lo = (int)(b & 0xFu), hi = (int)(b >> 4);
            q[r * K + 2 * i] = (int8_t)(lo >= 8 ? lo - 16 : lo);
            q[r * K + 2 * i + 1] = (int8_t)(hi >= 8 ? hi - 16 : hi);
        }
    }
    return 0;
}

/* Integer GEMM of the quantized linear: acc[m, n] = sum_k A[m, k] * B[n, k]
 * (activation codes times weight codes, the weight matrix stored [N, K]),
 * accumulated exactly in int64. */
int oracle_int_gemm(const int8_t *A, const int8_t *B, int64_t M, int32_t N, int32_t K, int64_t *acc)
{
    if (!A || !B || !acc || M < 0 || N < 1 || K < 1) return -1;
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        const int8_t *a = A + m * K;
        for (int32_t n = 0; n < N; ++n) {
            const int8_t *b = B + (int64_t)n * K;
            int64_t s = 0;
            for (int32_t k = 0; k < K; ++k) s += (int64_t)a[k] * (int64_t)b[k];
            acc[m * N + n] = s;
        }
    }
    return 0;
}

/* Dequantization of the integer product back to real values:
 *   Y[m, n] = acc[m, n] * delta_tok[m] * delta_ch[n] + bias[n]
 * (per-token times per-channel step, the product of the two symmetric
 * quantizers' scales [PTQ][GRAN]); bias may be NULL (zero). */
int oracle_dequant(const int64_t *acc, const double *delta_tok, const double *delta_ch,
                   const double *bias, int64_t M, int32_t N, double *Y)
{
    if (!acc || !delta_tok || !delta_ch || !Y || M < 0 || N < 1) return -1;
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int32_t n = 0; n < N; ++n)
            Y[m * N + n] = (double)acc[m * N + n] * delta_tok[m] * delta_ch[n] + (bias ? bias[n] : 0.0);
    return 0;
}

/* Plain real matrix product Y = X . W^T + bias (fp64), the unquantized
 * layer used as the reference for SQNR. */
int oracle_matmul_nt(const double *X, const double *W, const double *bias, int64_t M, int32_t N,
                     int32_t K, double *Y)
{
    if (!X || !W || !Y || M < 0 || N < 1 || K < 1) return -1;
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int32_t n = 0; n < N; ++n) {
            double s = 0.0;
            for (int32_t k = 0; k < K; ++k) s += X[m * K + k] * W[(int64_t)n * K + k];
            Y[m * N + n] = s + (bias ? bias[n] : 0.0);
        }
    }
    return 0;
}
