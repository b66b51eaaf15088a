/*
 * zt_q4_oracle.c -- the plain, slow CPU oracle for the q4f16 dequantizing
 * matrix-vector product.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the library's product path may link,
 * load or call this file; only the tests, the smoke check and the bench's
 * CPU-baseline leg do.  It shares no code, header, table or constant generator
 * with the CUDA library: every step here is written out from the definition.
 *
 * What it computes (all arithmetic in IEEE double):
 *
 *   The pages (Zero-TVM forum write-up, section "完整的推理流水线") name the
 *   compute core "int4 反量化矩阵乘法" -- an int4 dequantizing matrix product --
 *   with a plain variant, and an f32-output variant for the LM head "for
 *   sampling stability"; the same page's performance section names the
 *   weights "Phi-3-mini-q4f16_1": 4-bit weights, fp16 scales, fp16
 *   activations.  The pages do not spell out the bit format.  This library
 *   fixes it as follows (the plainest reading consistent with the pages):
 *
 *     weights   W is N x K (out x in).  qw is uint32 [N][K/8]; element (n,k)
 *               is bits 4*(k%8) .. 4*(k%8)+3 of qw[n][k/8]  (low nibble first)
 *     scales    fp16 [N][K/32], one per group of 32 consecutive k (the
 *               functions take the group size: 64 or 128 k per scale, the
 *               usual GPTQ / AWQ groupings, are the same formula)
 *     dequant   w[n][k] = (q[n][k] - 7) * s[n][k/32]
 *     product   y[m][n] = sum_k w[n][k] * x[m][k], summed in plain k order
 *
 *   fused FFN ("fused_ffn.wgsl": gate, up and SiLU in one pass, section
 *   "内核融合"): weight rows [0,N) are gate, rows [N,2N) are up;
 *   out[m][n] = SiLU(g) * u with SiLU(g) = g / (1 + exp(-g)).
 *
 *   LM head + greedy sampling (section "完整的推理流水线": f32 LM head and "a
 *   simple argmax dispatch"): logits = y kept in double; argmax = the lowest
 *   index among the maxima, NaN treated as -infinity.
 *
 *   rotary position embedding (section "完整的推理流水线": RoPE computed in
 *   place inside the fused QKV kernel; no formula given, the standard
 *   rotation is read): within each head of d features, feature pair
 *   (i, i + d/2) of token m turns by pos[m] * theta^(-2i/d).
 *
 *   batched prefill (limitations section, item on sequential prefill: the
 *   project ships batched-prefill shaders without wiring them in; its
 *   shaders need WebGPU's shader-f16, i.e. they compute in f16): for M
 *   tokens at once the weights are first dequantized to binary16 the way an
 *   f16 shader forms them, w16[n][k] = fp16((q[n][k] - 7) * s) -- the
 *   product is exact in double, so this is one correct rounding -- and then
 *   y[m][n] = sum_k w16[n][k] * x[m][k] in plain k order.
 *
 *   residual add + RMSNorm ("add_norm.wgsl": the residual connection and
 *   RMSNorm in one step, section "内核融合"; the pages give no formula, so
 *   the standard RMSNorm is read): per row m, h = fp16(residual + delta)
 *   (the residual stream stays fp16), x = fp16(h * gamma / sqrt(mean_k h^2 +
 *   eps)).  x is then the input of the next projection.
 *
 * Every function computes each output row with the same fixed sequence of
 * operations, so the optional OpenMP split over rows (threads > 1) returns
 * bit-identical results to the single-threaded run.
 */
#include <math.h>
#include <stddef.h>
#include <stdlib.h>
#include <stdint.h>

#define ZTO_GROUP 32   /* k values per fp16 scale in the q4f16 format (callers pass it; larger groups also work) */
#define ZTO_ZERO 7     /* the zero point subtracted from every 4-bit code */

/* IEEE-754 binary16 bit pattern -> double, written out from the format:
 * 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double zto_half_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int expo = (h >> 10) & 0x1F;
    int frac = h & 0x3FF;
    double v;
    if (expo == 0) {
        v = ldexp((double)frac, -24);                 /* zero / subnormal */
    } else if (expo == 31) {
        v = frac ? NAN : INFINITY;                    /* inf / NaN */
    } else {
        v = ldexp((double)(1024 + frac), expo - 25);  /* normal */
    }
    return sign ? -v : v;
}

/* The 4-bit code of element (n,k): the (k%8)-th nibble, counted from the
 * least significant end, of word qw[n][k/8]. */
static int zto_code(const uint32_t *qw, int64_t K, int64_t n, int64_t k)
{
    uint32_t word = qw[n * (K / 8) + k / 8];
    return (int)((word >> (4 * (k % 8))) & 0xFu);
}

/* Dequantized weight w[n][k] = (q - 7) * s, exact in double. */
static double zto_weight(const uint32_t *qw, const uint16_t *scales, int64_t K, int64_t group,
                         int64_t n, int64_t k)
{
    double s = zto_half_to_double(scales[n * (K / group) + k / group]);
    return (double)(zto_code(qw, K, n, k) - ZTO_ZERO) * s;
}

/* One dot product: sum over k = 0..K-1, in that order, of w[n][k] * x[m][k]. */
static double zto_row_dot(const uint32_t *qw, const uint16_t *scales,
                          const uint16_t *x, int64_t K, int64_t group, int64_t m, int64_t n)
{
    double acc = 0.0;
    for (int64_t k = 0; k < K; ++k)
        acc += zto_weight(qw, scales, K, group, n, k) * zto_half_to_double(x[m * K + k]);
    return acc;
}

/* Shapes: K a multiple of 8 (whole words) and of the group size (whole
 * groups); the format's group is ZTO_GROUP = 32, larger groups share one
 * scale among group / 32 consecutive blocks of 32. */
static int zto_shape_ok(int M, int N, int K, int group)
{
    return M >= 1 && N >= 1 && group >= 1 && K >= group && K % group == 0 && K % 8 == 0;
}

/* Unpack codes: q[n][k] (one byte each, 0..15) from qw[n][K/8]. */
int zto_unpack(const uint32_t *qw, int N, int K, uint8_t *q)
{
    if (!qw || !q || N < 1 || K < 8 || K % 8) return -1;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            q[n * K + k] = (uint8_t)zto_code(qw, K, n, k);
    return 0;
}

/* Pack codes 0..15 into words, low nibble first. Codes above 15 are an error. */
int zto_pack(const uint8_t *q, int N, int K, uint32_t *qw)
{
    if (!qw || !q || N < 1 || K < 8 || K % 8) return -1;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t w = 0; w < K / 8; ++w) {
            uint32_t word = 0;
            for (int j = 0; j < 8; ++j) {
                uint8_t c = q[n * K + 8 * w + j];
                if (c > 15) return -1;
                word |= (uint32_t)c << (4 * j);
            }
            qw[n * (K / 8) + w] = word;
        }
    }
    return 0;
}

/* y[m][i] = sum_k w[row_i][k] x[m][k].  rows == NULL computes every row
 * (n_rows must equal N and row_i = i); otherwise only the listed rows, and y is
 * [M][n_rows].  Output in double, no rounding to fp16. */
int zto_gemv(const uint32_t *qw, const uint16_t *scales, const uint16_t *x,
             int M, int N, int K, int group, const int32_t *rows, int n_rows,
             double *y, int threads)
{
    if (!qw || !scales || !x || !y || !zto_shape_ok(M, N, K, group)) return -1;
    if (!rows) n_rows = N;
    for (int i = 0; rows && i < n_rows; ++i)
        if (rows[i] < 0 || rows[i] >= N) return -1;
    if (threads < 1) threads = 1;
#pragma omp parallel for schedule(static) num_threads(threads)
    for (int i = 0; i < n_rows; ++i) {
        int64_t n = rows ? rows[i] : i;
        for (int64_t m = 0; m < M; ++m)
            y[m * n_rows + i] = zto_row_dot(qw, scales, x, K, group, m, n);
    }
    return 0;
}

/* SiLU(g) = g * sigmoid(g) = g / (1 + exp(-g)). */
double zto_silu(double g)
{
    return g / (1.0 + exp(-g));
}

/* Fused gate/up + SiLU.  qw and scales hold 2N rows: rows 0..N-1 are the gate
 * projection, rows N..2N-1 the up projection.  out[m][i] = SiLU(g) * u with
 * g = dot(gate row n), u = dot(up row n), n = rows[i] (or i), all in double. */
int zto_gate_up_silu(const uint32_t *qw, const uint16_t *scales, const uint16_t *x,
                     int M, int N, int K, int group, const int32_t *rows, int n_rows,
                     double *out, int threads)
{
    if (!qw || !scales || !x || !out || !zto_shape_ok(M, N, K, group)) return -1;
    if (!rows) n_rows = N;
    for (int i = 0; rows && i < n_rows; ++i)
        if (rows[i] < 0 || rows[i] >= N) return -1;
    if (threads < 1) threads = 1;
#pragma omp parallel for schedule(static) num_threads(threads)
    for (int i = 0; i < n_rows; ++i) {
        int64_t n = rows ? rows[i] : i;
        for (int64_t m = 0; m < M; ++m) {
            double g = zto_row_dot(qw, scales, x, K, group, m, n);
            double u = zto_row_dot(qw, scales, x, K, group, m, n + N);
            out[m * n_rows + i] = zto_silu(g) * u;
        }
    }
    return 0;
}

/* Greedy sampling over one row of logits: the lowest index among the maxima.
 * NaN compares as -infinity, so a row of NaNs (or of -inf) returns 0. */
int32_t zto_argmax(const double *v, int N)
{
    int32_t best = 0;
    double best_v = isnan(v[0]) ? -INFINITY : v[0];
    for (int32_t n = 1; n < N; ++n) {
        double c = isnan(v[n]) ? -INFINITY : v[n];
        if (c > best_v) {   /* strict: an equal later value never wins */
            best_v = c;
            best = n;
        }
    }
    return best;
}

/* LM head: logits[m][n] (double, never rounded to fp16) and argmax[m]. */
int zto_lmhead_argmax(const uint32_t *qw, const uint16_t *scales, const uint16_t *x,
                      int M, int N, int K, int group, double *logits, int32_t *argmax,
                      int threads)
{
    if (!qw || !scales || !x || !logits || !argmax || !zto_shape_ok(M, N, K, group)) return -1;
    int rc = zto_gemv(qw, scales, x, M, N, K, group, NULL, N, logits, threads);
    if (rc) return rc;
    for (int64_t m = 0; m < M; ++m)
        argmax[m] = zto_argmax(logits + m * N, N);
    return 0;
}

/* double -> IEEE-754 binary16 bit pattern, round to nearest, ties to even,
 * written out from the format: in the binade [2^e, 2^(e+1)) (e >= -14; below
 * that the subnormal spacing 2^-24 continues) representable values are
 * spaced 2^(e-10), so the value is rounded to an integer count of spacings.
 * Values that round above 65504 (the largest finite) become infinity; NaN
 * becomes the quiet NaN 0x7E00. */
uint16_t zto_double_to_half(double v)
{
    const uint16_t sign = signbit(v) ? 0x8000 : 0;
    if (isnan(v)) return 0x7E00;
    const double a = fabs(v);
    if (isinf(a)) return sign | 0x7C00;
    if (a == 0.0) return sign;
    int E;
    (void)frexp(a, &E);                 /* a in [2^(E-1), 2^E) */
    int e = E - 1;
    if (e < -14) e = -14;               /* subnormals share the spacing of binade -14 */
    const double units = ldexp(a, 10 - e);          /* a / 2^(e-10), exact */
    double r = floor(units);
    const double frac = units - r;                  /* exact */
    if (frac > 0.5 || (frac == 0.5 && fmod(r, 2.0) != 0.0)) r += 1.0;
    if (ldexp(r, e - 10) > 65504.0) return sign | 0x7C00;
    int64_t ri = (int64_t)r;
    if (ri == 2048) {                   /* rounded up into the next binade */
        ri = 1024;
        e += 1;
    }
    if (ri < 1024) return sign | (uint16_t)ri;      /* subnormal (e == -14) */
    return sign | (uint16_t)((e + 15) << 10) | (uint16_t)(ri - 1024);
}

/* Residual add + RMSNorm over rows of [M][K] fp16:
 *   h[m][k] = fp16(residual[m][k] + delta[m][k])     (delta == NULL: h = residual)
 *   r[m]    = 1 / sqrt((sum_k h[m][k]^2) / K + eps)   (k in plain order, double)
 *   x[m][k] = fp16(h[m][k] * r[m] * gamma[k])
 * h_out (may be NULL) receives h, x_out receives x (fp16 bit patterns). */
int zto_add_rmsnorm(const uint16_t *residual, const uint16_t *delta, const uint16_t *gamma,
                    int M, int K, double eps, uint16_t *h_out, uint16_t *x_out)
{
    if (!residual || !gamma || !x_out || M < 1 || K < 1 || !(eps >= 0.0)) return -1;
    for (int64_t m = 0; m < M; ++m) {
        double ss = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            double h = zto_half_to_double(residual[m * K + k]);
            if (delta) h += zto_half_to_double(delta[m * K + k]);   /* exact: two fp16 values */
            const uint16_t hb = zto_double_to_half(h);
            if (h_out) h_out[m * K + k] = hb;
            const double hd = zto_half_to_double(hb);
            ss += hd * hd;
        }
        const double r = 1.0 / sqrt(ss / (double)K + eps);
        for (int64_t k = 0; k < K; ++k) {
            double h = zto_half_to_double(residual[m * K + k]);
            if (delta) h += zto_half_to_double(delta[m * K + k]);
            const double hd = zto_half_to_double(zto_double_to_half(h));
            x_out[m * K + k] = zto_double_to_half(hd * r * zto_half_to_double(gamma[k]));
        }
    }
    return 0;
}

/* Projection + rotary position embedding.  y = W x as zto_gemv (double, all N
 * rows), then for every head h (d = head_dim features, N % d == 0), every
 * i < d/2 and every token m, with n = h*d + i, n2 = n + d/2 and
 * phi = pos[m] * theta^(-2i/d):
 *   out[m][n]  = y[m][n] cos(phi) - y[m][n2] sin(phi)
 *   out[m][n2] = y[m][n2] cos(phi) + y[m][n] sin(phi)            */
int zto_gemv_rope(const uint32_t *qw, const uint16_t *scales, const uint16_t *x,
                  int M, int N, int K, int group, const int32_t *pos, int head_dim, double theta,
                  double *out, int threads)
{
    if (!qw || !scales || !x || !pos || !out || !zto_shape_ok(M, N, K, group)) return -1;
    if (head_dim < 2 || head_dim % 2 || N % head_dim || !(theta > 0.0)) return -1;
    const int half = head_dim / 2;
    if (threads < 1) threads = 1;
#pragma omp parallel for schedule(static) num_threads(threads)
    for (int p = 0; p < N / 2; ++p) {
        const int64_t h = p / half, i = p % half;
        const int64_t n = h * head_dim + i, n2 = n + half;
        const double inv_freq = pow(theta, -2.0 * (double)i / (double)head_dim);
        for (int64_t m = 0; m < M; ++m) {
            const double a = zto_row_dot(qw, scales, x, K, group, m, n);
            const double b = zto_row_dot(qw, scales, x, K, group, m, n2);
            const double phi = (double)pos[m] * inv_freq;
            out[m * N + n] = a * cos(phi) - b * sin(phi);
            out[m * N + n2] = b * cos(phi) + a * sin(phi);
        }
    }
    return 0;
}

/* Dequantize to binary16: w16[n][k] = fp16((q[n][k] - 7) * s[n][k/group]),
 * round to nearest even (zto_double_to_half); the product itself is exact in
 * double (a 4-bit integer times an 11-bit significand). */
int zto_dequant_f16(const uint32_t *qw, const uint16_t *scales, int N, int K, int group, uint16_t *w16)
{
    if (!qw || !scales || !w16 || !zto_shape_ok(1, N, K, group)) return -1;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            w16[n * K + k] = zto_double_to_half(zto_weight(qw, scales, K, group, n, k));
    return 0;
}

/* Batched product on the binary16 weights: y[m][i] = sum_k w16[row_i][k] x[m][k]
 * with w16 as zto_dequant_f16 forms it, summed in double in plain k order.
 * Each row's w16 values are formed once into a scratch row and then used for
 * every token.  rows / n_rows / y as in zto_gemv. */
int zto_gemm_f16w(const uint32_t *qw, const uint16_t *scales, const uint16_t *x,
                  int M, int N, int K, int group, const int32_t *rows, int n_rows,
                  double *y, int threads)
{
    if (!qw || !scales || !x || !y || !zto_shape_ok(M, N, K, group)) return -1;
    if (!rows) n_rows = N;
    for (int i = 0; rows && i < n_rows; ++i)
        if (rows[i] < 0 || rows[i] >= N) return -1;
    if (threads < 1) threads = 1;
    int bad = 0;
#pragma omp parallel for schedule(static) num_threads(threads) reduction(| : bad)
    for (int i = 0; i < n_rows; ++i) {
        const int64_t n = rows ? rows[i] : i;
        double *w = (double *)malloc(sizeof(double) * (size_t)K);
        if (!w) {
            bad = 1;
            continue;
        }
        for (int64_t k = 0; k < K; ++k)
            w[k] = zto_half_to_double(zto_double_to_half(zto_weight(qw, scales, K, group, n, k)));
        for (int64_t m = 0; m < M; ++m) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k)
                acc += w[k] * zto_half_to_double(x[m * K + k]);
            y[m * n_rows + i] = acc;
        }
        free(w);
    }
    return bad ? -1 : 0;
}

/* Fused gate/up + SiLU on the binary16 weights: qw and scales hold 2N rows
 * (gate rows 0..N-1, up rows N..2N-1); with g = sum_k w16[n][k] x[m][k] and
 * u = sum_k w16[N + n][k] x[m][k] (double, plain k order, w16 as
 * zto_dequant_f16 forms it), out[m][i] = SiLU(g) * u for n = rows[i] (or i). */
int zto_gate_up_silu_f16w(const uint32_t *qw, const uint16_t *scales, const uint16_t *x,
                          int M, int N, int K, int group, const int32_t *rows, int n_rows,
                          double *out, int threads)
{
    if (!qw || !scales || !x || !out || !zto_shape_ok(M, N, K, group)) return -1;
    if (!rows) n_rows = N;
    for (int i = 0; rows && i < n_rows; ++i)
        if (rows[i] < 0 || rows[i] >= N) return -1;
    if (threads < 1) threads = 1;
    int bad = 0;
#pragma omp parallel for schedule(static) num_threads(threads) reduction(| : bad)
    for (int i = 0; i < n_rows; ++i) {
        const int64_t n = rows ? rows[i] : i;
        double *wg = (double *)malloc(sizeof(double) * 2 * (size_t)K);
        if (!wg) {
            bad = 1;
            continue;
        }
        double *wu = wg + K;
        for (int64_t k = 0; k < K; ++k) {
            wg[k] = zto_half_to_double(zto_double_to_half(zto_weight(qw, scales, K, group, n, k)));
            wu[k] = zto_half_to_double(zto_double_to_half(zto_weight(qw, scales, K, group, N + n, k)));
        }
        for (int64_t m = 0; m < M; ++m) {
            double g = 0.0, u = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                const double xv = zto_half_to_double(x[m * K + k]);
                g += wg[k] * xv;
                u += wu[k] * xv;
            }
            out[m * n_rows + i] = zto_silu(g) * u;
        }
        free(wg);
    }
    return bad ? -1 : 0;
}
