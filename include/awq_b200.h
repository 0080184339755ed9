/*
 * awq_b200.h — C ABI of the B200 (sm_100a) AWQ per-layer scale search.
 *
 * The operations follow the AWQ pages:
 *   [AWQ-blog]  "AWQ: Activation-aware Weight Quantization ..." paper summary
 *               (bg51717 blog), section Method: the quantizer
 *               Q(w) = Delta*Round(w/Delta), the objective
 *               L(s) = ||Q(W*s)(s^-1*X) - W X||, the grid s = s_X^alpha with
 *               alpha* = argmin L, clipping of the enlarged weights.
 *   [AWQ-guide] "AWQ 量化方案：激活感知的权重量化与工程实现全解析" (qwbw.cn),
 *               section 三: act_norm = mean |X| over calibration tokens,
 *               scale = act_norm^alpha / max, per-group Delta = max/7 with
 *               codes clamped to [-8, 7], QuantLinear (INT4-packed weight,
 *               per-group fp16 scales, per-channel scale applied to x).
 *
 * Conventions shared by every entry point
 *   - Tensors are row-major and live in device memory unless an argument says
 *     "host".  W is [out, in], X is [N, in] (tokens x input channels).
 *   - bf16 and fp16 values are passed as their 16-bit patterns (uint16_t).
 *   - Device pointers must be 16-byte aligned (AWQ_ERR_ALIGN otherwise).
 *   - The caller owns every buffer it passes.  The library allocates its own
 *     temporary device workspace with stream-ordered allocation on `stream`
 *     and frees it on the same stream before returning.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Work is
 *     enqueued on it; entry points return without synchronising unless noted.
 *   - Arguments are validated on the host before anything is enqueued; an
 *     invalid call returns AWQ_ERR_ARG / AWQ_ERR_ALIGN / AWQ_ERR_UNSUPPORTED
 *     and enqueues nothing.  A failing CUDA call returns AWQ_ERR_CUDA (see
 *     awq_last_error()).  In-kernel waits are bounded.  The search entry
 *     points synchronise and report a wait that gave up as AWQ_ERR_TIMEOUT;
 *     the W4A16 apply calls return before their kernels run, and a CTA whose
 *     wait gives up there exits without writing its part of y.
 *   - Each call is an NVTX range named after the function (visible under a
 *     profiler; free otherwise).
 *   - Supported: w_bit in {3, 4} (3-bit codes are stored in the same 4-bit
 *     container); group_size in {32, 64, 128}; in % 64 == 0;
 *     in % group_size == 0; any out >= 1 and N >= 1 (tails are masked).
 */
#ifndef AWQ_B200_H
#define AWQ_B200_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    AWQ_OK = 0,
    AWQ_ERR_ARG = 1,          /* null pointer, non-positive size, bad enum    */
    AWQ_ERR_ALIGN = 2,        /* device pointer not 16-byte aligned            */
    AWQ_ERR_UNSUPPORTED = 3,  /* valid request outside the supported set      */
    AWQ_ERR_CUDA = 4,         /* a CUDA runtime call failed                    */
    AWQ_ERR_TIMEOUT = 5       /* a bounded in-kernel wait gave up              */
} awq_status_t;

typedef enum { AWQ_F32 = 0, AWQ_BF16 = 1 } awq_dtype_t;

/* Most (alpha, clip) points one awq_search_points call evaluates. */
#define AWQ_MAX_POINTS 4096
typedef enum { AWQ_SYM = 0, AWQ_ASYM = 1 } awq_quant_t;

/* Library version, major*10000 + minor*100 + patch. */
int awq_version(void);

/* Static string for a status code. */
const char *awq_status_string(int status);

/* Text of the last error seen by the calling host thread ("" if none). */
const char *awq_last_error(void);

/*
 * awq_act_stats — per-input-channel activation statistic ([AWQ-guide] 三,
 * step 1; [AWQ-blog] Method, s_X).
 *     sX[i] = max(clamp_min, mean_n |X[n, i]|)
 * X        : [N, in] device, fp32 or bf16 (x_dtype).
 * sX       : [in] fp32 device, written.
 * The mean accumulates in fp64: tokens are summed sequentially within chunks
 * of 128 consecutive tokens and the chunk partials are added in ascending
 * chunk order, then the fp64 mean is rounded once to fp32.
 * Requires in % 8 == 0 and N <= 2^40.  Asynchronous.
 */
awq_status_t awq_act_stats(const void *X, int x_dtype, int64_t N, int64_t in,
                           float clamp_min, float *sX, void *stream);

/*
 * awq_search_layer — the AWQ grid search of one linear layer ([AWQ-blog]
 * Method: s = s_X^alpha, alpha* = argmin_alpha L(s); clipping of the enlarged
 * weights).  For every grid point k < n_alpha:
 *     s_k[i]   = s_X[i]^alpha[k] / max_j s_X[j]^alpha[k]   (fp64 pow, fp32 result)
 *     Q_k      = group-wise INT4 fake quantisation of W * s_k (quant, group_size)
 *     loss[k]  = mean over (n, o) of ( sum_i X[n, i] * (Q_k[o, i] / s_k[i] - W[o, i]) )^2
 * best_alpha = first k with the minimal loss.  Then, if n_clip > 0, with s fixed
 * at alpha[best_alpha], the same loss for each clip ratio clip[j] (the group
 * bounds are multiplied by clip[j] before Delta is formed; values beyond them
 * saturate), stored at loss[n_alpha + j]; best_clip = first minimiser.
 * Quantizers: AWQ_SYM  Delta = max|w|/7, q = clamp(rint(w/Delta), -8, 7);
 *             AWQ_ASYM Delta = (max w - min w)/15, z = clamp(rint(-min/Delta), 0, 15),
 *                      q = clamp(rint(w/Delta) + z, 0, 15), value (q - z)*Delta.
 *             At w_bit = 3: 3 and [-4, 3], 7 and [0, 7] ([AWQ-guide] 三's
 *             2^(w_bit-1) - 1 at w_bit = 3).
 * W         : [out, in] device, fp32 or bf16 (w_dtype).
 * X         : [N, in] device, fp32 or bf16 (x_dtype).  The tensor-core
 *             contraction reads an fp16 copy of X scaled by one power of two
 *             (largest magnitude in [2^14, 2^15)), so bf16 values down to 2^-28
 *             of the maximum are exact and fp32 values are rounded to fp16's
 *             11-bit significand; the losses are rescaled exactly.
 * sX        : [in] fp32 device (from awq_act_stats).
 * alpha     : [n_alpha] host, 1 <= n_alpha <= 64, each in [0, 1].
 * clip      : [n_clip] host or NULL, 0 <= n_clip <= 64, each in (0, 1].
 * loss      : [n_alpha + n_clip] host fp64, written.
 * loss_row  : optional [n_alpha + n_clip][out] fp32 device: per-row sums of
 *             squared output error (not divided by N).
 * best_alpha, best_clip : host, written (best_clip = -1 when n_clip == 0).
 * The error term dW = Q(W*s)/s - W enters the fp16 contraction multiplied by
 * one power of two per grid point (its bound over the layer lands in
 * [2^14, 2^15)), undone exactly in the loss, so small weights keep fp16's
 * full precision.
 * Synchronises `stream` (the losses are returned on the host).
 */
awq_status_t awq_search_layer(const void *W, int w_dtype, int64_t out, int64_t in,
                              const void *X, int x_dtype, int64_t N,
                              const float *sX, int group_size, int w_bit, int quant,
                              const double *alpha, int n_alpha,
                              const double *clip, int n_clip,
                              double *loss, float *loss_row,
                              int *best_alpha, int *best_clip, void *stream);

/*
 * awq_search_points — the same loss at an arbitrary list of grid points:
 * point k uses s = s_X^alpha[k] (normalised by its maximum) and clip ratio
 * clip[k] ([AWQ-blog] Method: the scale search and the clipping of the enlarged
 * weights, here searched jointly, e.g. every (alpha, r) pair of two grids,
 * instead of r after alpha*).
 * alpha, clip : [n_points] host, alpha in [0, 1], clip in (0, 1];
 *               1 <= n_points <= AWQ_MAX_POINTS (evaluated 64 at a time).
 * loss        : [n_points] host fp64, written.
 * loss_row    : optional [n_points][out] fp32 device per-row sums.
 * best        : host, the first k with the minimal loss.
 * Other arguments as for awq_search_layer.  Synchronises `stream`.
 */
awq_status_t awq_search_points(const void *W, int w_dtype, int64_t out, int64_t in,
                               const void *X, int x_dtype, int64_t N,
                               const float *sX, int group_size, int w_bit, int quant,
                               const double *alpha, const double *clip, int n_points,
                               double *loss, float *loss_row, int *best, void *stream);

/*
 * awq_pack_int4 — final quantisation at (alpha, clip) and INT4 packing
 * ([AWQ-guide] 三, step 4 and QuantLinear storage).  Bit-exact IEEE fp32:
 * W' = W*s (one multiply), Delta = bound/7 or range/15 (correctly rounded
 * divide), q from rint of the correctly rounded quotient W'/Delta.
 * qweight    : [out][in/8] u32 device: nibble k (bits 4k..4k+3) of word w holds
 *              column 8w+k; symmetric codes are stored as q+8, asymmetric as q.
 * scales     : [out][in/group_size] fp16 bits device: Delta rounded to nearest even.
 * zeros      : [out][ceil(in/group_size/8)] u32 device, nibble k of word w holds
 *              z of group 8w+k; required for AWQ_ASYM, must be NULL for AWQ_SYM.
 * s16        : [in] fp16 bits device: the per-channel scale s.
 * scales_f32 : optional [out][in/group_size] fp32 device: Delta as computed.
 * Asynchronous.
 */
awq_status_t awq_pack_int4(const void *W, int w_dtype, int64_t out, int64_t in,
                           const float *sX, double alpha, double clip,
                           int group_size, int quant,
                           uint32_t *qweight, uint16_t *scales, uint32_t *zeros,
                           uint16_t *s16, float *scales_f32, void *stream);

/*
 * awq_group_clip — one clip ratio per quantisation group ([AWQ-blog] Method,
 * clipping of the enlarged weights, chosen group by group): with
 * s = s_X^alpha (normalised by its maximum), for every output row o, group j
 * and ratio clip_grid[r]:
 *     err[o][j][r] = sum_n ( sum_{i in group j} X[n, i] * dW_r[o, i] )^2,
 *     dW_r = Q_r(W*s)/s - W, Q_r the group quantiser with its bound(s) times r;
 *     clip_idx[o][j] = the first r with the smallest err.
 * The kernels reduce the tokens once into each group's Gram matrix
 * H_j = X_j^T X_j (fp32 per 1024 tokens, fp64 across them) and evaluate
 * err = dW_r^T H_j dW_r in fp32: exact in real arithmetic, so near-equal
 * errors may order differently than a direct fp64 sum would.
 * clip_grid : [n_clip] host, 1 <= n_clip <= 64, each in (0, 1].
 * clip_idx  : [out][in/group_size] u8 device, written (for awq_pack_quant).
 * err       : optional [out][in/group_size][n_clip] fp32 device, written.
 * N <= 2^26.  Other arguments as for awq_search_layer.  Asynchronous.
 */
awq_status_t awq_group_clip(const void *W, int w_dtype, int64_t out, int64_t in,
                            const void *X, int x_dtype, int64_t N, const float *sX,
                            double alpha, int group_size, int w_bit, int quant,
                            const double *clip_grid, int n_clip,
                            uint8_t *clip_idx, float *err, void *stream);

/*
 * awq_pack_quant — awq_pack_int4 with the bit width and the clip choice open:
 * w_bit in {3, 4} (3-bit codes in the same nibble layout: symmetric q + 8,
 * asymmetric q), and either one ratio `clip` for the layer (clip_idx == NULL)
 * or one ratio per quantisation group: clip_idx [out][in/group_size] u8
 * device, each an index into clip_grid [n_clip] host (1 <= n_clip <= 64), as
 * written by awq_group_clip ([AWQ-blog] Method, clipping of the enlarged
 * weights, chosen per group).  Other arguments as for awq_pack_int4.
 * Asynchronous.
 */
awq_status_t awq_pack_quant(const void *W, int w_dtype, int64_t out, int64_t in,
                            const float *sX, double alpha, double clip,
                            const uint8_t *clip_idx, const double *clip_grid, int n_clip,
                            int group_size, int w_bit, int quant,
                            uint32_t *qweight, uint16_t *scales, uint32_t *zeros,
                            uint16_t *s16, float *scales_f32, void *stream);

/*
 * awq_linear_w4a16 — the W4A16 layer that applies the result ([AWQ-guide] 三,
 * QuantLinear.forward: x rescaled by the per-channel scale, weight dequantised
 * per group, linear):
 *     y[m, o] = sum_i (x[m, i] / s16[i]) * (code[o, i] - z[o, i/gs]) * scales[o, i/gs]
 * with z = 8 when zeros == NULL (symmetric storage).  fp32 accumulation.
 * s16 == NULL: x has already been divided by s (the division folded into the
 * operator that produces x, see awq_fold_scale) and is used as is.
 * x : [M, in] bf16 device;  y : [M, out] bf16 device, written.  in <= 49152.
 * Storage arguments as produced by awq_pack_int4.  Asynchronous.
 * Kernels by M: 1..4 a CUDA-core kernel streaming the packed weights (no
 * workspace), except 2..4 tokens on layers of at least 2^25 weights, which take
 * the persistent decode kernel of awq_linear_w4a16_batch; 5..16 warp-level
 * tensor-core MMA on the unpacked codes (an x / s workspace); 17 and more
 * tcgen05 tensor-core tiles.
 * Precision: x / s16 is rounded to fp16 after a power-of-two scale per
 * (token, group) for M <= 16, per token for M >= 17 (2^-11 relative); for
 * M >= 17 (code - z) * scale is also rounded to fp16 once, after a power-of-two
 * scale per output row.  Accumulation in fp32.
 * Ordering: the streaming (M <= 4), warp-MMA (5..16) and batched decode
 * kernels are launched with programmatic stream serialisation, so their
 * blocks may start while the preceding kernel on `stream` is still
 * running; until that kernel has completed they only ask L2 to prefetch
 * their weights (a hint that reads nothing into the SM), and every read of an
 * argument, and the write of y, happens after it.
 */
awq_status_t awq_linear_w4a16(const uint16_t *x, int64_t M, int64_t in, int64_t out,
                              const uint32_t *qweight, const uint16_t *scales,
                              const uint32_t *zeros, const uint16_t *s16,
                              int group_size, uint16_t *y, void *stream);

/*
 * awq_linear_w4a16_batch — awq_linear_w4a16 on up to AWQ_MAX_BATCH_LINEARS
 * independent linears at once (e.g. the projections of a decoder block that
 * read the same or different inputs): y_k = (x_k / s16_k) * dequant(W_k)^T for
 * every descriptor k, all at the same M and group_size, with zero points given
 * for every linear or for none ([AWQ-guide] 三, QuantLinear.forward).
 * For M <= 8, when the staged activations of the widest linear and a ring of
 * weight tiles fit one SM's shared memory (M <= 6 at in = 11008, M <= 8 at
 * in = 4096), this is one persistent launch, one block per SM: the 16-row
 * tiles of all linears are dealt out in contiguous, byte-balanced ranges, so
 * the layers share one ramp-up of the memory system; otherwise the linears run
 * one after the other through awq_linear_w4a16.  Each output is bit-identical
 * to the same call with that linear alone.  Precision as awq_linear_w4a16.
 * The outputs must not overlap each other or any input.  Asynchronous.
 */
#define AWQ_MAX_BATCH_LINEARS 8
typedef struct {
    const uint16_t *x;          /* [M, in] bf16 device */
    int64_t in, out;
    const uint32_t *qweight;    /* [out][in/8] u32 device (awq_pack_int4 layout) */
    const uint16_t *scales;     /* [out][in/group_size] fp16 bits device */
    const uint32_t *zeros;      /* [out][ceil(in/group_size/8)] u32 device, or NULL (symmetric) */
    const uint16_t *s16;        /* [in] fp16 bits device, or NULL (x already divided by s) */
    uint16_t *y;                /* [M, out] bf16 device, written */
} awq_linear_desc_t;

awq_status_t awq_linear_w4a16_batch(const awq_linear_desc_t *descs, int n, int64_t M,
                                    int group_size, void *stream);

/*
 * awq_fold_scale — fold the division by s into the operator that produces
 * this layer's input ([AWQ-blog] Method: X / s is merged into the preceding
 * operator, so the W4A16 layer runs with s16 == NULL):
 *     out[r][c] = P[r][c] / s16[r]    (one IEEE fp32 division; bf16: rounded
 *                                      to nearest even)
 * P    : [rows][cols] device, fp32 or bf16 (p_dtype): row r holds the producing
 *        operator's parameters for channel r, e.g. an RMSNorm weight
 *        (cols = 1) or a previous linear's weight rows (its output channels).
 * s16  : [rows] fp16 bits device (awq_pack_int4's s16); must be nonzero.
 * out  : [rows][cols] device, same dtype as P; may alias P (in place).
 * Asynchronous.
 */
awq_status_t awq_fold_scale(const void *P, int p_dtype, int64_t rows, int64_t cols,
                            const uint16_t *s16, void *out, void *stream);

/*
 * awq_wait_selftest — exercise the bounded in-kernel wait that guards every
 * mbarrier wait of the search and apply kernels.  One CTA waits on an
 * mbarrier that it arrives on only if `arrive` != 0, giving up after
 * limit_cycles SM clock cycles (1 <= limit_cycles <= 4e9, about 2 s); no copy
 * or MMA is in flight.  Returns AWQ_OK when the wait completed, AWQ_ERR_TIMEOUT
 * when it gave up (reported through the same device error word as the search
 * kernel).  Synchronises `stream`.
 */
awq_status_t awq_wait_selftest(int64_t limit_cycles, int arrive, void *stream);

/*
 * awq_act_stats_noalloc — awq_act_stats without any device allocation.  The
 * AWQ pages have no counterpart: this exists for callers that cannot allocate
 * device memory when they compute the statistic (processes that hand nearly
 * all device memory to their own pool allocator at start-up, or that must not
 * allocate inside a latency-critical section).  It computes the same values
 * with the same kernels, but keeps the fp64 chunk partials in a fixed 8 MiB
 * buffer compiled into the library instead of a temporary allocation, and
 * calls no allocating routine.
 * Limit: ceil(N / 128) * in <= 1,048,576; larger calls return
 * AWQ_ERR_UNSUPPORTED and enqueue nothing.  Timed as kind 0 when timing is on.
 * The first call on a device looks up the buffer's device address (a
 * cudaGetSymbolAddress call); make that first call before any stream capture.
 * Every call shares the one buffer per device, so calls whose work overlaps on
 * the GPU (different streams, or concurrent host threads) race; order them on
 * one stream.  Arguments and results as for awq_act_stats.  Asynchronous.
 */
awq_status_t awq_act_stats_noalloc(const void *X, int x_dtype, int64_t N, int64_t in,
                                   float clamp_min, float *sX, void *stream);

/*
 * Kernel timing (instrumentation, off by default).  When enabled, each entry
 * point brackets its main kernel launch(es) with CUDA events on `stream`;
 * awq_last_kernel_ms(kind) returns the device time of that kernel in the last
 * call of the calling host thread (summed over the two search phases), waiting
 * for the end event if needed.  Returns a negative value if nothing was timed.
 *   kind: 0 = activation statistics (both kernels), 1 = fused search kernel,
 *         2 = pack kernel, 3 = W4A16 apply kernel.
 */
void awq_set_kernel_timing(int enable);
double awq_last_kernel_ms(int kind);

#ifdef __cplusplus
}
#endif

#endif /* AWQ_B200_H */
