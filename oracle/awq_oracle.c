/*
 * AWQ per-layer scale search: CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, obviously-correct
 * restatement of what the hot path computes.  Only the test-suite, the smoke
 * check and the benchmark's CPU-baseline leg may load it.  The CUDA library
 * never links, includes or calls anything here, and nothing here includes or
 * calls the CUDA library.
 *
 * Sources (page title, then the part of the page):
 *   [AWQ-blog]  "AWQ: Activation-aware Weight Quantization ..." paper summary
 *               (bg51717 blog): the quantizer Q(w) = Delta*Round(w/Delta)
 *               (Method, first equation), the scaled product Q(w*s)*(x/s)
 *               (Method, second equation), the objective
 *               L(s) = ||Q(W*s)(s^-1*X) - W X|| and the grid search
 *               s = s_X^alpha, alpha* = argmin L (Method, the two optimisation
 *               equations), clipping of the enlarged weights (Method, the
 *               list of further optimisations).
 *   [AWQ-guide] "AWQ 量化方案：激活感知的权重量化与工程实现全解析" (qwbw.cn):
 *               section 三 (core algorithm): act_norm = mean |X| over tokens,
 *               scale = act_norm^alpha normalised by its maximum, per-group
 *               Delta = group max / (2^(w_bit-1) - 1), codes clamped to
 *               [-2^(w_bit-1), 2^(w_bit-1)-1], QuantLinear forward.
 *   [Q-tutorial] "量化方案详解" (luoboask): AWQ section, worked example of a
 *               16-level grid over [-3.2, 3.2].
 *
 * Readings where the pages are silent (each stated once, used everywhere):
 *   - precision: every sum is accumulated in fp64; the quantizer itself runs
 *     in IEEE fp32 (W*s, Delta = a/7, W'/Delta) with round-half-to-even;
 *   - mean |X| accumulates in fp64 over consecutive token chunks of
 *     ORC_STATS_CHUNK tokens (sequential inside a chunk, chunk partials added
 *     in ascending order), so that the statistic is one fixed function of X;
 *   - groups are (output row, group_size consecutive input columns);
 *   - asymmetric min-max: Delta = (max - min)/15, z = clamp(rint(-min/Delta),
 *     0, 15), q = clamp(rint(W'/Delta) + z, 0, 15), dequantised (q - z)*Delta;
 *   - w_bit b in {3, 4}: symmetric Delta = a/(2^(b-1) - 1) with codes in
 *     [-2^(b-1), 2^(b-1) - 1]; asymmetric Delta = range/(2^b - 1) with z and
 *     codes in [0, 2^b - 1] (the denominators of [AWQ-guide] section 三 at
 *     w_bit = b; [Q-tutorial] names INT3 as the lowest useful width);
 *   - clip ratio r scales the group bound(s) before Delta is formed; the
 *     clamp saturates the values beyond them.  Per-layer r: searched after
 *     alpha* on the layer loss.  Per-group r: each (row, group) takes the
 *     first r of the grid that minimises its own output error
 *     sum_n (sum_{i in group} X[n, i] dW[o, i])^2;
 *   - a group whose Delta is 0 gets code 0 (asymmetric: q = z = 0);
 *   - loss = sum of squared output errors / (N * out);
 *   - argmin = first index of the minimum.
 *
 * Built with -O2 -fno-fast-math -ffp-contract=off so that every float and
 * double operation is one IEEE operation in source order.  OpenMP splits work
 * only across output rows or columns; each row's arithmetic order is fixed, so
 * results do not depend on the thread count.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_STATS_CHUNK 128

#define ORC_SYM 0
#define ORC_ASYM 1

/* ---------------------------------------------------------------- helpers */

static float f32_max(float a, float b) { return a > b ? a : b; }
static float f32_min(float a, float b) { return a < b ? a : b; }

/* IEEE binary16 bits of x, round to nearest even (subnormals kept). */
static uint16_t f32_to_f16_bits(float x) {
    _Float16 h = (_Float16)x;
    uint16_t b;
    memcpy(&b, &h, 2);
    return b;
}

static float f16_bits_to_f32(uint16_t b) {
    _Float16 h;
    memcpy(&h, &b, 2);
    return (float)h;
}

int orc_stats_chunk(void) { return ORC_STATS_CHUNK; }

/* ------------------------------------------------------- activation stats */
/*
 * s_X[i] = mean over tokens n of |X[n, i]|, clamped from below by clamp_min.
 * [AWQ-guide] section 三 step 1 (act_norm = activation.abs().mean(dim=0));
 * [AWQ-blog] Method: s_X is the per-channel activation magnitude.
 * X is [N, I] row-major fp32 (bf16 inputs are widened exactly by the caller).
 */
void orc_act_stats(const float *X, int64_t N, int64_t I, float clamp_min,
                   float *sX) {
    double *total = (double *)calloc((size_t)I, sizeof(double));
    double *part = (double *)malloc((size_t)I * sizeof(double));
    for (int64_t c0 = 0; c0 < N; c0 += ORC_STATS_CHUNK) {
        int64_t c1 = c0 + ORC_STATS_CHUNK < N ? c0 + ORC_STATS_CHUNK : N;
        for (int64_t i = 0; i < I; ++i) part[i] = 0.0;
        for (int64_t n = c0; n < c1; ++n) {
            const float *row = X + n * I;
            for (int64_t i = 0; i < I; ++i) part[i] += fabs((double)row[i]);
        }
        for (int64_t i = 0; i < I; ++i) total[i] += part[i];
    }
    for (int64_t i = 0; i < I; ++i) {
        float m = (float)(total[i] / (double)N);
        sX[i] = m < clamp_min ? clamp_min : m;
    }
    free(part);
    free(total);
}

/* ----------------------------------------------------------- scale vector */
/*
 * s[i] = s_X[i]^alpha / max_j s_X[j]^alpha.
 * [AWQ-blog] Method: s = s_X^alpha; [AWQ-guide] section 三 step 2:
 * scale = act_norm.pow(alpha); scale = scale / scale.max().
 * pow and the division run in fp64, the result is rounded once to fp32.
 */
void orc_scale_vector(const float *sX, int64_t I, double alpha, float *s) {
    double *t = (double *)malloc((size_t)I * sizeof(double));
    double m = 0.0;
    for (int64_t i = 0; i < I; ++i) {
        t[i] = pow((double)sX[i], alpha);
        if (t[i] > m) m = t[i];
    }
    for (int64_t i = 0; i < I; ++i) s[i] = (float)(t[i] / m);
    free(t);
}

/* -------------------------------------------------------- group quantizer */
/*
 * Quantise one group of scaled weights wp[0..gs).
 * Symmetric ([AWQ-blog] Method, first equation, with the denominator
 * 2^(N-1)-1 = 7 and the clamp to [-8, 7] of [AWQ-guide] section 三 step 4):
 *     a = max |wp| (times clip),  Delta = a / 7,  q = clamp(rint(wp/Delta), -8, 7),
 *     dequantised value q*Delta;  *zero = 0.
 * Asymmetric min-max (16 levels, step = range/15 as in [Q-tutorial]'s example):
 *     mx = max wp, mn = min wp (each times clip),  Delta = (mx - mn)/15,
 *     z = clamp(rint(-mn/Delta), 0, 15),  q = clamp(rint(wp/Delta) + z, 0, 15),
 *     dequantised value (q - z)*Delta.
 * (The constants are those of wbit = 4; wbit = 3 uses 3, [-4, 3] and 7.)
 * A zero Delta gives q = 0 (and z = 0).
 */
void orc_quant_group(const float *wp, int gs, int qt, int wbit, double clip, int *q,
                     float *delta, int *zero) {
    /* symmetric: [-2^(b-1), 2^(b-1) - 1], Delta = a / (2^(b-1) - 1);
       asymmetric: [0, 2^b - 1], Delta = range / (2^b - 1) */
    const float shi = (float)((1 << (wbit - 1)) - 1), slo = -(float)(1 << (wbit - 1));
    const float ahi = (float)((1 << wbit) - 1);
    if (qt == ORC_SYM) {
        float a = 0.0f;
        for (int k = 0; k < gs; ++k) a = f32_max(a, fabsf(wp[k]));
        if (clip != 1.0) a = (float)((double)a * clip);
        float d = a / shi;
        *delta = d;
        *zero = 0;
        for (int k = 0; k < gs; ++k) {
            if (d == 0.0f) {
                q[k] = 0;
                continue;
            }
            float r = rintf(wp[k] / d);
            r = f32_min(f32_max(r, slo), shi);
            q[k] = (int)r;
        }
    } else {
        float mx = wp[0], mn = wp[0];
        for (int k = 1; k < gs; ++k) {
            mx = f32_max(mx, wp[k]);
            mn = f32_min(mn, wp[k]);
        }
        if (clip != 1.0) {
            mx = (float)((double)mx * clip);
            mn = (float)((double)mn * clip);
        }
        float d = (mx - mn) / ahi;
        *delta = d;
        if (d == 0.0f) {
            *zero = 0;
            for (int k = 0; k < gs; ++k) q[k] = 0;
            return;
        }
        float z = rintf(-mn / d);
        z = f32_min(f32_max(z, 0.0f), ahi);
        *zero = (int)z;
        for (int k = 0; k < gs; ++k) {
            float r = rintf(wp[k] / d) + z;
            r = f32_min(f32_max(r, 0.0f), ahi);
            q[k] = (int)r;
        }
    }
}

/*
 * Quantise a whole layer at scale s and clip ratio clip (or, when clip_g is
 * given, the ratio clip_g[o * I/gs + j] for group j of row o):
 *   W'[o, i] = W[o, i] * s[i]                      (one fp32 multiply)
 *   codes [O, I] (signed for SYM, 0..2^b-1 for ASYM), Delta [O, I/gs], z [O, I/gs].
 * [AWQ-blog] Method: Q(W*s) with the group-wise quantizer above.
 */
void orc_quant_layer(const float *W, int64_t O, int64_t I, const float *s,
                     int gs, int qt, int wbit, double clip, const double *clip_g,
                     int8_t *codes, float *delta, uint8_t *zeros) {
    int64_t nG = I / gs;
#pragma omp parallel for schedule(static)
    for (int64_t o = 0; o < O; ++o) {
        float wp[256];
        int q[256];
        for (int64_t j = 0; j < nG; ++j) {
            for (int k = 0; k < gs; ++k) {
                int64_t i = j * gs + k;
                wp[k] = W[o * I + i] * s[i];
            }
            float d;
            int z;
            orc_quant_group(wp, gs, qt, wbit, clip_g ? clip_g[o * nG + j] : clip, q, &d, &z);
            for (int k = 0; k < gs; ++k) codes[o * I + j * gs + k] = (int8_t)q[k];
            delta[o * nG + j] = d;
            zeros[o * nG + j] = (uint8_t)z;
        }
    }
}

/* ------------------------------------------------------------- the loss */
/*
 * For the listed output rows, the row loss
 *     loss_row[r] = sum_n ( sum_i X[n, i] * dW[o, i] )^2,
 *     dW[o, i] = (q[o, i] - z[o, g(i)]) * Delta[o, g(i)] / s[i] - W[o, i],
 * all in fp64.  This is the objective of [AWQ-blog] Method,
 * || Q(W*s)(s^-1 * X) - W X ||, written as X * (Q(W*s)/s - W)^T: the
 * rearrangement moves the 1/s from X's columns to the weights' columns, which
 * is exact in real arithmetic.
 * Returns the sum of the listed rows' losses (fp64, ascending row order).
 */
double orc_layer_loss_rows(const float *W, int64_t O, int64_t I, const float *X,
                           int64_t N, const float *s, int gs, const int8_t *codes,
                           const float *delta, const uint8_t *zeros,
                           const int64_t *rows, int64_t n_rows, double *loss_row) {
    int64_t nG = I / gs;
    double *lr = (double *)malloc((size_t)n_rows * sizeof(double));
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < n_rows; ++r) {
        int64_t o = rows[r];
        double *dw = (double *)malloc((size_t)I * sizeof(double));
        for (int64_t i = 0; i < I; ++i) {
            int64_t j = i / gs;
            double deq = (double)(codes[o * I + i] - (int)zeros[o * nG + j]) *
                         (double)delta[o * nG + j];
            dw[i] = deq / (double)s[i] - (double)W[o * I + i];
        }
        double acc = 0.0;
        for (int64_t n = 0; n < N; ++n) {
            const float *xr = X + n * I;
            double e = 0.0;
            for (int64_t i = 0; i < I; ++i) e += (double)xr[i] * dw[i];
            acc += e * e;
        }
        lr[r] = acc;
        free(dw);
    }
    double total = 0.0;
    for (int64_t r = 0; r < n_rows; ++r) {
        total += lr[r];
        if (loss_row) loss_row[r] = lr[r];
    }
    free(lr);
    return total;
}

/* ---------------------------------------------------------------- search */

static int first_argmin(const double *v, int n) {
    int best = 0;
    for (int k = 1; k < n; ++k)
        if (v[k] < v[best]) best = k;
    return best;
}

/*
 * The grid search of [AWQ-blog] Method: for every alpha on the grid,
 * s = s_X^alpha (normalised), quantise W*s, evaluate the loss; alpha* is the
 * first minimiser.  Then, with s fixed at alpha*, the same loss over the clip
 * ratios (the clipping of enlarged weights, [AWQ-blog] Method, further
 * optimisations); r* is the first minimiser.  The alpha points use clip 1.
 *   loss[k]      k < n_alpha : mean squared output error at alpha[k]
 *   loss[n_alpha + j]        : mean squared output error at (alpha*, clip[j])
 * rows == NULL evaluates every output row; otherwise only the listed rows and
 * the mean is taken over N * n_rows entries.
 * loss_row (optional) is [n_alpha + n_clip][n_rows] fp64 row sums.
 */
void orc_search_layer(const float *W, int64_t O, int64_t I, const float *X,
                      int64_t N, const float *sX, int gs, int qt, int wbit,
                      const double *alpha, int n_alpha, const double *clip,
                      int n_clip, const int64_t *rows, int64_t n_rows,
                      double *loss, double *loss_row, int *best_alpha,
                      int *best_clip) {
    int64_t nG = I / gs;
    int64_t *all_rows = NULL;
    if (rows == NULL) {
        all_rows = (int64_t *)malloc((size_t)O * sizeof(int64_t));
        for (int64_t o = 0; o < O; ++o) all_rows[o] = o;
        rows = all_rows;
        n_rows = O;
    }
    float *s = (float *)malloc((size_t)I * sizeof(float));
    int8_t *codes = (int8_t *)malloc((size_t)(O * I));
    float *delta = (float *)malloc((size_t)(O * nG) * sizeof(float));
    uint8_t *zeros = (uint8_t *)malloc((size_t)(O * nG));
    double denom = (double)N * (double)n_rows;

    for (int k = 0; k < n_alpha; ++k) {
        orc_scale_vector(sX, I, alpha[k], s);
        orc_quant_layer(W, O, I, s, gs, qt, wbit, 1.0, NULL, codes, delta, zeros);
        double tot = orc_layer_loss_rows(W, O, I, X, N, s, gs, codes, delta,
                                         zeros, rows, n_rows,
                                         loss_row ? loss_row + (int64_t)k * n_rows : NULL);
        loss[k] = tot / denom;
    }
    int ba = n_alpha > 0 ? first_argmin(loss, n_alpha) : 0;
    if (best_alpha) *best_alpha = ba;
    if (n_clip > 0) {
        orc_scale_vector(sX, I, alpha[ba], s);
        for (int j = 0; j < n_clip; ++j) {
            orc_quant_layer(W, O, I, s, gs, qt, wbit, clip[j], NULL, codes, delta, zeros);
            double tot = orc_layer_loss_rows(
                W, O, I, X, N, s, gs, codes, delta, zeros, rows, n_rows,
                loss_row ? loss_row + (int64_t)(n_alpha + j) * n_rows : NULL);
            loss[n_alpha + j] = tot / denom;
        }
        if (best_clip) *best_clip = first_argmin(loss + n_alpha, n_clip);
    } else if (best_clip) {
        *best_clip = -1;
    }
    free(zeros);
    free(delta);
    free(codes);
    free(s);
    free(all_rows);
}

/*
 * A joint grid: the same loss at each listed point (alpha[k], clip[k]),
 * k < n, e.g. every (alpha, r) pair of two grids ([AWQ-blog] Method: the
 * scale search and the clipping of the enlarged weights, searched together
 * instead of one after the other).  best = first minimiser.
 * rows / loss_row as for orc_search_layer.
 */
void orc_search_points(const float *W, int64_t O, int64_t I, const float *X,
                       int64_t N, const float *sX, int gs, int qt, int wbit,
                       const double *alpha, const double *clip, int n,
                       const int64_t *rows, int64_t n_rows, double *loss,
                       double *loss_row, int *best) {
    int64_t nG = I / gs;
    int64_t *all_rows = NULL;
    if (rows == NULL) {
        all_rows = (int64_t *)malloc((size_t)O * sizeof(int64_t));
        for (int64_t o = 0; o < O; ++o) all_rows[o] = o;
        rows = all_rows;
        n_rows = O;
    }
    float *s = (float *)malloc((size_t)I * sizeof(float));
    int8_t *codes = (int8_t *)malloc((size_t)(O * I));
    float *delta = (float *)malloc((size_t)(O * nG) * sizeof(float));
    uint8_t *zeros = (uint8_t *)malloc((size_t)(O * nG));
    double denom = (double)N * (double)n_rows;
    for (int k = 0; k < n; ++k) {
        orc_scale_vector(sX, I, alpha[k], s);
        orc_quant_layer(W, O, I, s, gs, qt, wbit, clip[k], NULL, codes, delta, zeros);
        double tot = orc_layer_loss_rows(W, O, I, X, N, s, gs, codes, delta, zeros, rows,
                                         n_rows, loss_row ? loss_row + (int64_t)k * n_rows : NULL);
        loss[k] = tot / denom;
    }
    if (best) *best = n > 0 ? first_argmin(loss, n) : 0;
    free(zeros);
    free(delta);
    free(codes);
    free(s);
    free(all_rows);
}

/*
 * Per-group clip ratio at scale s = s_X^alpha: for every output row o and
 * group j, and every ratio clip[r] of the grid, quantise the group with its
 * bound(s) times clip[r] and evaluate the group's own output error
 *     err[o][j][r] = sum_n ( sum_{i in group j} X[n, i] * dW_r[o, i] )^2
 * with dW_r = (q - z)*Delta/s - W (fp64).  best[o * I/gs + j] is the first r
 * with the smallest error.  This is the clipping of the enlarged weights
 * ([AWQ-blog] Method, further optimisations) with one ratio per quantisation
 * group instead of one per layer; the error is the layer objective restricted
 * to the group's columns.
 * err (optional) is [O][I/gs][n_clip] fp64.
 */
void orc_group_clip(const float *W, int64_t O, int64_t I, const float *X, int64_t N,
                    const float *sX, double alpha, int gs, int qt, int wbit,
                    const double *clip, int n_clip, int32_t *best, double *err) {
    int64_t nG = I / gs;
    float *s = (float *)malloc((size_t)I * sizeof(float));
    orc_scale_vector(sX, I, alpha, s);
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t o = 0; o < O; ++o) {
        float wp[256];
        int q[256];
        double dw[256];
        for (int64_t j = 0; j < nG; ++j) {
            double best_e = 0.0;
            int best_r = 0;
            for (int r = 0; r < n_clip; ++r) {
                for (int k = 0; k < gs; ++k) {
                    int64_t i = j * gs + k;
                    wp[k] = W[o * I + i] * s[i];
                }
                float d;
                int z;
                orc_quant_group(wp, gs, qt, wbit, clip[r], q, &d, &z);
                for (int k = 0; k < gs; ++k) {
                    int64_t i = j * gs + k;
                    dw[k] = (double)(q[k] - z) * (double)d / (double)s[i] - (double)W[o * I + i];
                }
                double acc = 0.0;
                for (int64_t n = 0; n < N; ++n) {
                    const float *xr = X + n * I + j * gs;
                    double e = 0.0;
                    for (int k = 0; k < gs; ++k) e += (double)xr[k] * dw[k];
                    acc += e * e;
                }
                if (err) err[(o * nG + j) * n_clip + r] = acc;
                if (r == 0 || acc < best_e) {
                    best_e = acc;
                    best_r = r;
                }
            }
            best[o * nG + j] = best_r;
        }
    }
    free(s);
}

/* ------------------------------------------------------------------ pack */
/*
 * Storage of the chosen quantisation at (alpha, clip), or at the per-group
 * ratios clip_g [O][I/gs] when given ([AWQ-guide] section 三: INT4-packed
 * qweight, per-group fp16 scales, per-channel awq scale):
 *   qweight [O][I/8] u32 : nibble k (bits 4k..4k+3) of word w holds column
 *                          8w + k; symmetric codes are stored as q + 8,
 *                          asymmetric codes as q (w_bit = 3 codes use the
 *                          same 4-bit container);
 *   scales  [O][I/gs]    : fp16 bits of Delta (round to nearest even);
 *   zeros   [O][ceil(I/gs/8)] u32 : nibble k of word w holds z of group 8w+k
 *                          (asymmetric only; unused nibbles are 0);
 *   s16     [I]          : fp16 bits of s;
 *   scales_f32 [O][I/gs] : Delta as computed (fp32).
 */
void orc_pack_int4(const float *W, int64_t O, int64_t I, const float *sX,
                   double alpha, double clip, const double *clip_g, int gs, int qt,
                   int wbit, uint32_t *qweight, uint16_t *scales, uint32_t *zeros,
                   uint16_t *s16, float *scales_f32) {
    int64_t nG = I / gs;
    int64_t nzw = (nG + 7) / 8;
    float *s = (float *)malloc((size_t)I * sizeof(float));
    int8_t *codes = (int8_t *)malloc((size_t)(O * I));
    float *delta = (float *)malloc((size_t)(O * nG) * sizeof(float));
    uint8_t *z = (uint8_t *)malloc((size_t)(O * nG));
    orc_scale_vector(sX, I, alpha, s);
    orc_quant_layer(W, O, I, s, gs, qt, wbit, clip, clip_g, codes, delta, z);
    for (int64_t o = 0; o < O; ++o) {
        for (int64_t w = 0; w < I / 8; ++w) {
            uint32_t word = 0;
            for (int k = 0; k < 8; ++k) {
                int c = codes[o * I + 8 * w + k];
                uint32_t nib = (uint32_t)(qt == ORC_SYM ? c + 8 : c) & 0xFu;
                word |= nib << (4 * k);
            }
            qweight[o * (I / 8) + w] = word;
        }
        for (int64_t j = 0; j < nG; ++j) {
            scales[o * nG + j] = f32_to_f16_bits(delta[o * nG + j]);
            if (scales_f32) scales_f32[o * nG + j] = delta[o * nG + j];
        }
        if (zeros) {
            for (int64_t w = 0; w < nzw; ++w) {
                uint32_t word = 0;
                for (int k = 0; k < 8 && 8 * w + k < nG; ++k)
                    word |= ((uint32_t)z[o * nG + 8 * w + k] & 0xFu) << (4 * k);
                zeros[o * nzw + w] = word;
            }
        }
    }
    for (int64_t i = 0; i < I; ++i) s16[i] = f32_to_f16_bits(s[i]);
    free(z);
    free(delta);
    free(codes);
    free(s);
}

/* ----------------------------------------------------------------- apply */
/*
 * W4A16 linear ([AWQ-guide] section 三, QuantLinear.forward: the activation
 * is rescaled by the per-channel awq scale, the weight is dequantised group by
 * group and a plain linear follows).  With the storage above:
 *     y[m, o] = sum_i (x[m, i] / s16[i]) * (code[o, i] - z[o, g(i)]) * Delta16[o, g(i)]
 * where z = 8 for symmetric storage.  x is [M, I] fp32 (bf16 widened exactly),
 * the result is fp64.  s16 == NULL means x has already been divided by s (the
 * 1/s folded into the previous operator, [AWQ-blog] Method) and is used as is.
 */
void orc_linear_w4a16(const float *x, int64_t M, int64_t I, int64_t O,
                      const uint32_t *qweight, const uint16_t *scales,
                      const uint32_t *zeros, const uint16_t *s16, int gs,
                      double *y) {
    int64_t nG = I / gs;
    int64_t nzw = (nG + 7) / 8;
#pragma omp parallel for schedule(static)
    for (int64_t o = 0; o < O; ++o) {
        for (int64_t m = 0; m < M; ++m) {
            double acc = 0.0;
            for (int64_t i = 0; i < I; ++i) {
                int64_t j = i / gs;
                int code = (int)((qweight[o * (I / 8) + i / 8] >> (4 * (i % 8))) & 0xFu);
                int zz = zeros ? (int)((zeros[o * nzw + j / 8] >> (4 * (j % 8))) & 0xFu) : 8;
                double d = (double)f16_bits_to_f32(scales[o * nG + j]);
                double xs = s16 ? (double)x[m * I + i] / (double)f16_bits_to_f32(s16[i])
                                : (double)x[m * I + i];
                acc += xs * (double)(code - zz) * d;
            }
            y[m * O + o] = acc;
        }
    }
}

/* ------------------------------------------------------------------ fold */
/*
 * Fold 1/s into the operator that produces this layer's input ([AWQ-blog]
 * Method: the division of X by s is merged into the preceding operator).  P
 * is [R, C] row-major, row c holding that operator's parameters for channel c
 * (an RMSNorm weight: C = 1; a previous linear's weight rows); every entry is
 * divided by the stored per-channel scale:
 *     out[c][k] = RN_fp32( P[c][k] / s16[c] )
 * one IEEE fp32 division; out_bf16 != 0 then rounds each value to bf16 (nearest
 * even) and stores the bit pattern, else stores the fp32 value.
 */
void orc_fold_scale(const float *P, int64_t R, int64_t C, const uint16_t *s16, int out_bf16,
                    void *out) {
    for (int64_t r = 0; r < R; ++r) {
        float sv = f16_bits_to_f32(s16[r]);
        for (int64_t k = 0; k < C; ++k) {
            float v = P[r * C + k] / sv;
            if (out_bf16) {
                uint32_t u;
                memcpy(&u, &v, 4);
                u += 0x7FFFu + ((u >> 16) & 1u);
                ((uint16_t *)out)[r * C + k] = (uint16_t)(u >> 16);
            } else {
                ((float *)out)[r * C + k] = v;
            }
        }
    }
}
