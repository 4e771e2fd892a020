/*
 * rrs_oracle.c -- plain, slow CPU oracle for the Rotated Runtime Smooth (RRS)
 * W4A4 linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may load this library.  The product path
 * (the CUDA library and its binding) never calls it, and this file shares no
 * code, header, table or constant with the CUDA sources.
 *
 * Sources (web pages on Rotated Runtime Smooth, by page title and section):
 *  [RRS-summary]  "Rotated Runtime Smooth: Training-Free Activation Smoother
 *                 for accurate INT4 inference" (AI summary page), "Approach":
 *                 Runtime Smooth divides activations by group-wise channel
 *                 maxima computed at inference after reordering channels, and
 *                 is applied after a Hadamard rotation.
 *  [RRS-rebuttal] the same paper's OpenReview rebuttal page: "Novelty"
 *                 (reorder, then a group-wise smoothing scale aligned with the
 *                 hardware GEMM), "Description of the reorder process"
 *                 (Y = X W^T = sum_i X_i W_i^T, X and W permuted alike).
 *  [L2Rot]        "Understanding LLM Quantization through Activation-Guided
 *                 Compensation and Orthogonal Residuals": Sec. 3.1 (per-token
 *                 symmetric quantiser Delta_t * round(Z / Delta_t)), Sec. 3.2
 *                 (normalised Hadamard, entries of magnitude 1/sqrt(d),
 *                 O(d log d) fast transform), Appendix B.1 (Delta_t =
 *                 ||Z_t||_inf / q_A with q_A = 2^(b-1) - 1), Sec. 5
 *                 "Quantization and calibration" (per-output-channel symmetric
 *                 weights).
 *
 * Where the pages are silent the readings are:
 *  R1  Hadamard arithmetic: fp32, iterative radix-2 stages h = 1, 2, 4, ...,
 *      pair (j, j+h) -> (a+b, a-b) with a the lower index.
 *  R2  normalisation: one multiply by c_n = (float)(1/sqrt((double)n)) after
 *      the transform.
 *  R3  rotation first, then the reorder X'[:, j] = X_rot[:, perm[j]].
 *  R4  zero guards: a group whose max is 0 is divided by 1; a token whose
 *      quantisation scale is 0 gets all-zero codes.
 *  R5  smoothing is an IEEE fp32 division by s_g (not a reciprocal multiply).
 *  R6  4-bit symmetric quantiser: scale = amax / 7 (q_A = 7), fp32.
 *  R7  round half to even (rintf in the default rounding mode).
 *  R8  no clipping ratio.
 *  R14 KV cache (the "4-4-4" setting): each head vector rotated by the
 *      normalised Hadamard transform of its length D, then the per-token
 *      symmetric INT4 quantiser; no runtime smoothing (see orc_kv_quant).
 *  R9  packing: byte i = (q[2i] & 0xF) | (q[2i+1] & 0xF) << 4, two's
 *      complement nibbles.
 *  Y   sum_g s_g * P_g accumulated in double, times scale_t and scale_w in
 *      double, rounded once to fp32.
 *
 * Build: gcc -O2 -ffp-contract=off -fno-fast-math -shared -fPIC.  On x86-64
 * float arithmetic is SSE single precision (FLT_EVAL_METHOD 0), so every
 * '+', '-', '*', '/' below is one IEEE fp32 operation rounded to nearest.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------- Hadamard */

/* In-place unnormalised fast Walsh-Hadamard transform of v[0..n), n a power
 * of two, in the stage order of reading R1 ([L2Rot] Sec. 3.2: the normalised
 * Hadamard admits an O(d log d) fast transform).  The Sylvester matrix it
 * applies has H[i][j] = (-1)^popcount(i & j). */
void orc_fwht(float *v, int n)
{
    for (int h = 1; h < n; h *= 2) {
        for (int i = 0; i < n; i += 2 * h) {
            for (int j = i; j < i + h; ++j) {
                float a = v[j];
                float b = v[j + h];
                v[j] = a + b;
                v[j + h] = a - b;
            }
        }
    }
}

/* c_n of reading R2. */
float orc_hadamard_scale(int n)
{
    return (float)(1.0 / sqrt((double)n));
}

static int is_pow2(int n) { return n > 0 && (n & (n - 1)) == 0; }

/* X_rot = blockdiag(H_n, ..., H_n) applied to each row, then times c_n
 * ([RRS-summary] "Approach": the activations are Hadamard-rotated online; the
 * block-diagonal form covers K = B * n).  n = 1 is the identity (plain
 * Runtime Smooth).  X, out: fp32 [rows, K], X holding fp16 values exactly. */
int orc_rotate(const float *X, int64_t rows, int K, int n, float *out)
{
    if (!is_pow2(n) || K % n != 0) return -1;
    float c = orc_hadamard_scale(n);
    float *row = (float *)malloc(sizeof(float) * (size_t)K);
    if (!row) return -2;
    for (int64_t t = 0; t < rows; ++t) {
        memcpy(row, X + t * (int64_t)K, sizeof(float) * (size_t)K);
        for (int b = 0; b < K / n; ++b) orc_fwht(row + (int64_t)b * n, n);
        for (int j = 0; j < K; ++j) out[t * (int64_t)K + j] = row[j] * c;
    }
    free(row);
    return 0;
}

/* X'[t][j] = X_rot[t][perm[j]] ([RRS-rebuttal] "Description of the reorder
 * process": the channels of X and W are rearranged by the same index). */
int orc_reorder(const float *Xrot, int64_t rows, int K, const int32_t *perm, float *Xp)
{
    for (int j = 0; j < K; ++j)
        if (perm[j] < 0 || perm[j] >= K) return -1;
    for (int64_t t = 0; t < rows; ++t)
        for (int j = 0; j < K; ++j)
            Xp[t * (int64_t)K + j] = Xrot[t * (int64_t)K + perm[j]];
    return 0;
}

/* s[g] = max over all tokens t and channels j of group g of |X'[t][j]|
 * ([RRS-summary] "Approach": group-wise channel maxima computed at inference;
 * [RRS-rebuttal] "Novelty": the smoothing scale is applied group-wise). */
int orc_group_max(const float *Xp, int64_t M, int K, int G, float *s)
{
    if (G <= 0 || K % G != 0) return -1;
    for (int g = 0; g < K / G; ++g) s[g] = 0.0f;
    for (int64_t t = 0; t < M; ++t)
        for (int j = 0; j < K; ++j) {
            float a = fabsf(Xp[t * (int64_t)K + j]);
            if (a > s[j / G]) s[j / G] = a;
        }
    return 0;
}

/* Pack signed 4-bit codes, reading R9. */
static void pack_row(const int8_t *q, int K, uint8_t *out)
{
    for (int i = 0; i < K / 2; ++i)
        out[i] = (uint8_t)(((uint8_t)q[2 * i] & 0x0Fu) | (((uint8_t)q[2 * i + 1] & 0x0Fu) << 4));
}

/* Per-row symmetric INT4 quantiser ([L2Rot] Sec. 3.1 and Appendix B.1 with
 * b = 4: Delta = ||z||_inf / 7, code = round(z / Delta); readings R4, R6-R8).
 * Writes the codes (one int8 per element) and returns the scale. */
static float quant_row(const float *z, int K, int8_t *q)
{
    float amax = 0.0f;
    for (int j = 0; j < K; ++j) {
        float a = fabsf(z[j]);
        if (a > amax) amax = a;
    }
    float scale = amax / 7.0f;
    for (int j = 0; j < K; ++j) {
        if (scale == 0.0f) { q[j] = 0; continue; }
        float r = rintf(z[j] / scale);
        if (r > 7.0f) r = 7.0f;
        if (r < -8.0f) r = -8.0f;
        q[j] = (int8_t)r;
    }
    return scale;
}

/* Runtime Smooth + per-token quantisation of already rotated and reordered
 * activations X' [M, K]:  X~ = X' / s_g (R4, R5), then quant_row per token.
 * unit_scales != 0 replaces s by 1 everywhere (the A4W4 per-channel scheme
 * without smoothing, [RRS-rebuttal] "complete efficiency metrics" list).
 * Outputs: codes int8 [M, K] (optional, may be NULL), packed qX [M, K/2],
 * s [K/G] (the group maxima, or 1 under unit_scales), scale_t [M]. */
int orc_smooth_quant_from_xp(const float *Xp, int64_t M, int K, int G, int unit_scales,
                             int8_t *codes, uint8_t *qX, float *s, float *scale_t)
{
    if (G <= 0 || K % G != 0 || K % 2 != 0) return -1;
    if (unit_scales) {
        for (int g = 0; g < K / G; ++g) s[g] = 1.0f;
    } else {
        orc_group_max(Xp, M, K, G, s);
    }
    float *z = (float *)malloc(sizeof(float) * (size_t)K);
    int8_t *q = (int8_t *)malloc((size_t)K);
    if (!z || !q) { free(z); free(q); return -2; }
    for (int64_t t = 0; t < M; ++t) {
        for (int j = 0; j < K; ++j) {
            float d = s[j / G];
            if (d == 0.0f) d = 1.0f;
            z[j] = Xp[t * (int64_t)K + j] / d;
        }
        scale_t[t] = quant_row(z, K, q);
        if (codes) memcpy(codes + t * (int64_t)K, q, (size_t)K);
        pack_row(q, K, qX + t * (int64_t)(K / 2));
    }
    free(z);
    free(q);
    return 0;
}

/* The whole online activation path: rotate (n), reorder (perm), smooth, quantise. */
int orc_smooth_quant(const float *X, int64_t M, int K, int G, int n, const int32_t *perm,
                     int unit_scales, int8_t *codes, uint8_t *qX, float *s, float *scale_t)
{
    float *rot = (float *)malloc(sizeof(float) * (size_t)M * (size_t)K);
    float *xp = (float *)malloc(sizeof(float) * (size_t)M * (size_t)K);
    int rc = -2;
    if (rot && xp) {
        rc = orc_rotate(X, M, K, n, rot);
        if (rc == 0) rc = orc_reorder(rot, M, K, perm, xp);
        if (rc == 0) rc = orc_smooth_quant_from_xp(xp, M, K, G, unit_scales, codes, qX, s, scale_t);
    }
    free(rot);
    free(xp);
    return rc;
}

/* Offline weight path: W' = reorder(rotate(W)) with the same n and perm as
 * the activations, then per-output-channel symmetric INT4 RTN ([RRS-summary]
 * "Approach": the scales are not folded into the weights; [L2Rot] Sec. 5:
 * per-output-channel symmetric weights; readings R6-R9). */
int orc_prepare_weights(const float *W, int64_t N, int K, int n, const int32_t *perm,
                        int8_t *codes, uint8_t *qW, float *scale_w)
{
    float *rot = (float *)malloc(sizeof(float) * (size_t)K);
    float *wp = (float *)malloc(sizeof(float) * (size_t)K);
    int8_t *q = (int8_t *)malloc((size_t)K);
    int rc = 0;
    if (!rot || !wp || !q) { rc = -2; goto done; }
    for (int64_t r = 0; r < N; ++r) {
        rc = orc_rotate(W + r * (int64_t)K, 1, K, n, rot);
        if (rc) goto done;
        rc = orc_reorder(rot, 1, K, perm, wp);
        if (rc) goto done;
        scale_w[r] = quant_row(wp, K, q);
        if (codes) memcpy(codes + r * (int64_t)K, q, (size_t)K);
        pack_row(q, K, qW + r * (int64_t)(K / 2));
    }
done:
    free(rot);
    free(wp);
    free(q);
    return rc;
}

static inline int nib(const uint8_t *row, int j)
{
    int v = (j & 1) ? (row[j >> 1] >> 4) : (row[j >> 1] & 0x0F);
    return v >= 8 ? v - 16 : v;
}

/* Exact per-group integer partial sums P[g][t][n] = sum_{j in g} qX[t][j] qW[n][j]
 * for the listed token rows (all rows when rows == NULL). */
int orc_group_partials(const uint8_t *qX, const uint8_t *qW, int64_t M, int64_t N, int K, int G,
                       const int64_t *rows, int64_t nrows, int32_t *P)
{
    if (G <= 0 || K % G != 0) return -1;
    int64_t R = rows ? nrows : M;
    for (int g = 0; g < K / G; ++g)
        for (int64_t i = 0; i < R; ++i) {
            int64_t t = rows ? rows[i] : i;
            const uint8_t *xr = qX + t * (int64_t)(K / 2);
            for (int64_t c = 0; c < N; ++c) {
                const uint8_t *wr = qW + c * (int64_t)(K / 2);
                int64_t acc = 0;
                for (int j = g * G; j < (g + 1) * G; ++j) acc += (int64_t)nib(xr, j) * nib(wr, j);
                P[((int64_t)g * R + i) * N + c] = (int32_t)acc;
            }
        }
    return 0;
}

/* Y[t][c] = (sum_g s_g * P_g[t][c]) * scale_t[t] * scale_w[c]  (the group-scaled
 * W4A4 product; [RRS-rebuttal] "Novelty": group-wise smoothing scale aligned
 * with the hardware GEMM).  Accumulation in double, one rounding to fp32.
 * bound[t][c] (optional) = sum_g |s_g * P_g| * scale_t * scale_w, the magnitude
 * that bounds fp32 summation error in any order. */
int orc_linear_rows(const uint8_t *qX, const float *s, const float *scale_t, const uint8_t *qW,
                    const float *scale_w, int64_t M, int64_t N, int K, int G,
                    const int64_t *rows, int64_t nrows, float *Y, double *bound)
{
    if (G <= 0 || K % G != 0) return -1;
    int NG = K / G;
    int64_t R = rows ? nrows : M;
    for (int64_t i = 0; i < R; ++i) {
        int64_t t = rows ? rows[i] : i;
        const uint8_t *xr = qX + t * (int64_t)(K / 2);
        for (int64_t c = 0; c < N; ++c) {
            const uint8_t *wr = qW + c * (int64_t)(K / 2);
            double acc = 0.0, mag = 0.0;
            for (int g = 0; g < NG; ++g) {
                int64_t p = 0;
                for (int j = g * G; j < (g + 1) * G; ++j) p += (int64_t)nib(xr, j) * nib(wr, j);
                double term = (double)s[g] * (double)p;
                acc += term;
                mag += fabs(term);
            }
            double sc = (double)scale_t[t] * (double)scale_w[c];
            Y[i * N + c] = (float)(acc * sc);
            if (bound) bound[i * N + c] = mag * sc;
        }
    }
    (void)M;
    return 0;
}

/* Calibration statistic for the reorder index: per-channel max over tokens of
 * |X_rot| (reading R3's plainest derivation of "collect outliers and normal
 * values", [RRS-rebuttal] "Novelty"). */
int orc_channel_absmax(const float *X, int64_t M, int K, int n, float *cmax)
{
    float *rot = (float *)malloc(sizeof(float) * (size_t)K);
    if (!rot) return -2;
    for (int j = 0; j < K; ++j) cmax[j] = 0.0f;
    for (int64_t t = 0; t < M; ++t) {
        int rc = orc_rotate(X + t * (int64_t)K, 1, K, n, rot);
        if (rc) { free(rot); return rc; }
        for (int j = 0; j < K; ++j) {
            float a = fabsf(rot[j]);
            if (a > cmax[j]) cmax[j] = a;
        }
    }
    free(rot);
    return 0;
}

/* KV-cache quantisation of the "4-4-4" setting ([RRS-summary] "Key results":
 * weights, activations and the KV cache held in 4 bits).  Reading R14: every
 * head vector of K or V (length D, one row here) is rotated by the normalised
 * Hadamard transform of size D (the rotation of R1-R2 with n = D) and then
 * quantised by the per-token symmetric INT4 quantiser (quant_row; readings
 * R4, R6-R9).  There is no runtime smoothing: the runtime group scales belong to
 * the linear layer's group-scaled GEMM, which the attention products lack.
 * KV fp32 [rows, D] -> codes int8 [rows, D] (optional, may be NULL), packed
 * q [rows, D/2], scale [rows]. */
int orc_kv_quant(const float *KV, int64_t rows, int D, int8_t *codes, uint8_t *q, float *scale)
{
    if (!is_pow2(D) || D < 2) return -1;
    float *rot = (float *)malloc(sizeof(float) * (size_t)D);
    int8_t *c = (int8_t *)malloc((size_t)D);
    int rc = 0;
    if (!rot || !c) { rc = -2; goto done; }
    for (int64_t r = 0; r < rows; ++r) {
        rc = orc_rotate(KV + r * (int64_t)D, 1, D, D, rot);
        if (rc) goto done;
        scale[r] = quant_row(rot, D, c);
        if (codes) memcpy(codes + r * (int64_t)D, c, (size_t)D);
        pack_row(c, D, q + r * (int64_t)(D / 2));
    }
done:
    free(rot);
    free(c);
    return rc;
}

/* The cached vector back in the rotated space: x_hat = code * scale in fp32
 * (the quantiser's own reconstruction, [L2Rot] Sec. 3.1: Delta * round(Z / Delta)). */
int orc_kv_dequant(const uint8_t *q, int64_t rows, int D, const float *scale, float *out)
{
    if (D < 2 || D % 2 != 0) return -1;
    for (int64_t r = 0; r < rows; ++r)
        for (int j = 0; j < D; ++j)
            out[r * (int64_t)D + j] = (float)nib(q + r * (int64_t)(D / 2), j) * scale[r];
    return 0;
}
