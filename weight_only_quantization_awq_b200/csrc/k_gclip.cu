// Per-group clip ratio (paper summary, Method, further optimisations: clip the
// enlarged weights), with one ratio per quantisation group: at s = s_X^alpha,
// every (row o, group j) takes the first ratio r of the grid that minimises the
// group's own output error
//     err(o, j, r) = sum_n ( sum_{i in j} X[n, i] * dW_r[o, i] )^2,
//     dW_r = Q_r(W*s)/s - W   (Q_r: the group quantiser with its bounds times r).
//
// The error is a quadratic form in the group's gs values of dW_r:
//     err = d^T H_j d,   H_j[i][k] = sum_n X[n, i] X[n, k]   (i, k in group j),
// so the tokens are reduced once, into one gs x gs Gram matrix per group
// (gram_kernel), and each (row, group, ratio) then costs gs^2 multiply-adds
// instead of 2 * N * gs (gclip_kernel).  The identity is exact in real
// arithmetic; here the Gram matrix is summed in fp32 per 1024-token chunk and
// in fp64 across chunks, the form in fp32.
//
// The quantiser decisions (Delta, z, codes) follow the same IEEE fp32 steps as
// the pack kernel (correctly rounded divisions), so the dW of each candidate
// is the one the final packing would produce.
#include <cuda_fp16.h>

#include "awq_internal.h"

namespace awq {

namespace {

constexpr int GRAM_THREADS = 256;
constexpr int GRAM_TOK = 32;          // tokens staged per step
constexpr int GRAM_CHUNK = 1024;      // tokens per block (fp32 partial sums)

// One block: group j = blockIdx.x, tokens [chunk * 1024, ...).  Thread (ty, tx)
// of a 16 x 16 layout owns an R x R tile of H_j, R = GS / 16.
template <int GS, bool XBF16>
__global__ void __launch_bounds__(GRAM_THREADS) gram_kernel(const void *__restrict__ X, int64_t N,
                                                            int64_t I, double *__restrict__ H) {
    constexpr int R = GS / 16;
    __shared__ float xs[GRAM_TOK][GS];
    const int j = blockIdx.x;
    const int64_t n0 = static_cast<int64_t>(blockIdx.y) * GRAM_CHUNK;
    const int64_t n1 = n0 + GRAM_CHUNK < N ? n0 + GRAM_CHUNK : N;
    const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
    float acc[R][R];
#pragma unroll
    for (int a = 0; a < R; ++a)
#pragma unroll
        for (int b = 0; b < R; ++b) acc[a][b] = 0.0f;
    for (int64_t t0 = n0; t0 < n1; t0 += GRAM_TOK) {
        __syncthreads();
        for (int k = threadIdx.x; k < GRAM_TOK * GS; k += GRAM_THREADS) {
            const int t = k / GS, c = k % GS;
            const int64_t n = t0 + t;
            float v = 0.0f;
            if (n < n1) {
                const int64_t idx = n * I + static_cast<int64_t>(j) * GS + c;
                v = XBF16 ? __uint_as_float(static_cast<uint32_t>(static_cast<const uint16_t *>(X)[idx]) << 16)
                          : static_cast<const float *>(X)[idx];
            }
            xs[t][c] = v;
        }
        __syncthreads();
#pragma unroll 4
        for (int t = 0; t < GRAM_TOK; ++t) {
            float av[R], bv[R];
#pragma unroll
            for (int a = 0; a < R; ++a) {
                av[a] = xs[t][ty + 16 * a];
                bv[a] = xs[t][tx + 16 * a];
            }
#pragma unroll
            for (int a = 0; a < R; ++a)
#pragma unroll
                for (int b = 0; b < R; ++b) acc[a][b] = __fmaf_rn(av[a], bv[b], acc[a][b]);
        }
    }
    double *Hj = H + static_cast<int64_t>(j) * GS * GS;
#pragma unroll
    for (int a = 0; a < R; ++a)
#pragma unroll
        for (int b = 0; b < R; ++b)
            atomicAdd(&Hj[(ty + 16 * a) * GS + (tx + 16 * b)], static_cast<double>(acc[a][b]));
}

constexpr int GC_WARPS = 8;
constexpr int GC_ROWS = 32;           // rows per block (4 per warp)
constexpr int GC_V = 4;               // ratios evaluated per pass over H

__device__ __forceinline__ float clip_b(float b, double r) {
    return r == 1.0 ? b : __double2float_rn(__dmul_rn(static_cast<double>(b), r));
}

// One block: group j = blockIdx.y, rows [32 * blockIdx.x, +32), one warp per
// row at a time.  H_j lives in shared memory (symmetric, so row k doubles as
// column k: lanes read consecutive entries).  Lane l holds columns l + 32 e.
template <int GS, bool WBF16>
__global__ void __launch_bounds__(GC_WARPS * 32) gclip_kernel(
    const void *__restrict__ W, int64_t O, int64_t I, const float *__restrict__ s,
    const double *__restrict__ H, bool asym, int wbit, GridParams grid, int n_clip,
    uint8_t *__restrict__ best, float *__restrict__ err_out) {
    constexpr int E = GS / 32;
    extern __shared__ float gsm[];
    float *Hs = gsm;                                     // [GS][GS]
    float *dsm = gsm + GS * GS;                          // [GC_WARPS][GC_V][GS]
    const int j = blockIdx.y;
    const int64_t nG = I / GS;
    for (int k = threadIdx.x; k < GS * GS; k += GC_WARPS * 32)
        Hs[k] = static_cast<float>(H[static_cast<int64_t>(j) * GS * GS + k]);
    __syncthreads();
    const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
    float *dw = dsm + warp * GC_V * GS;
    float sv[E];
#pragma unroll
    for (int e = 0; e < E; ++e) sv[e] = s[static_cast<int64_t>(j) * GS + lane + 32 * e];
    const float stop = static_cast<float>((1 << (wbit - 1)) - 1);
    const float atop = static_cast<float>((1 << wbit) - 1);
    for (int rr = warp; rr < GC_ROWS; rr += GC_WARPS) {
        const int64_t o = static_cast<int64_t>(blockIdx.x) * GC_ROWS + rr;
        if (o >= O) break;
        float w[E], wp[E];
        float mx = -3.4028234663852886e38f, mn = 3.4028234663852886e38f, am = 0.0f;
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const int64_t idx = o * I + static_cast<int64_t>(j) * GS + lane + 32 * e;
            w[e] = WBF16 ? __uint_as_float(static_cast<uint32_t>(static_cast<const uint16_t *>(W)[idx]) << 16)
                         : static_cast<const float *>(W)[idx];
            wp[e] = __fmul_rn(w[e], sv[e]);
            mx = fmaxf(mx, wp[e]);
            mn = fminf(mn, wp[e]);
            am = fmaxf(am, fabsf(wp[e]));
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
            mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
            am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, off));
        }
        float best_e = 0.0f;
        int best_r = 0;
        for (int r0 = 0; r0 < n_clip; r0 += GC_V) {
            // dW of up to GC_V candidate ratios, in this warp's shared slots
            float d[GC_V][E];
#pragma unroll
            for (int v = 0; v < GC_V; ++v) {
                const int ri = r0 + v < n_clip ? r0 + v : n_clip - 1;
                const double r = grid.value[ri];
                float D, z = 0.0f, lo, hi;
                if (!asym) {
                    D = __fdiv_rn(clip_b(am, r), stop);
                    lo = -stop - 1.0f;
                    hi = stop;
                } else {
                    const float bh = clip_b(mx, r), bl = clip_b(mn, r);
                    D = __fdiv_rn(__fsub_rn(bh, bl), atop);
                    if (D != 0.0f) z = fminf(fmaxf(rintf(__fdiv_rn(-bl, D)), 0.0f), atop);
                    lo = -z;
                    hi = atop - z;
                }
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    const float q = D != 0.0f ? fminf(fmaxf(rintf(__fdiv_rn(wp[e], D)), lo), hi) : 0.0f;
                    d[v][e] = __fsub_rn(__fdiv_rn(__fmul_rn(q, D), sv[e]), w[e]);
                    dw[v * GS + lane + 32 * e] = d[v][e];
                }
            }
            __syncwarp();
            float acc[GC_V][E];
#pragma unroll
            for (int v = 0; v < GC_V; ++v)
#pragma unroll
                for (int e = 0; e < E; ++e) acc[v][e] = 0.0f;
#pragma unroll 4
            for (int k = 0; k < GS; ++k) {
                float h[E];
#pragma unroll
                for (int e = 0; e < E; ++e) h[e] = Hs[k * GS + lane + 32 * e];
#pragma unroll
                for (int v = 0; v < GC_V; ++v) {
                    const float dk = dw[v * GS + k];
#pragma unroll
                    for (int e = 0; e < E; ++e) acc[v][e] = __fmaf_rn(h[e], dk, acc[v][e]);
                }
            }
            __syncwarp();
#pragma unroll
            for (int v = 0; v < GC_V; ++v) {
                float part = 0.0f;
#pragma unroll
                for (int e = 0; e < E; ++e) part = __fmaf_rn(acc[v][e], d[v][e], part);
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
                const int ri = r0 + v;
                if (ri < n_clip) {
                    if (err_out && lane == 0) err_out[(o * nG + j) * n_clip + ri] = part;
                    if (ri == 0 || part < best_e) {
                        best_e = part;
                        best_r = ri;
                    }
                }
            }
        }
        if (lane == 0) best[o * nG + j] = static_cast<uint8_t>(best_r);
    }
}

template <int GS>
cudaError_t launch_gclip_gs(const void *W, bool w_bf16, int64_t O, int64_t I, const void *X,
                            bool x_bf16, int64_t N, const float *s, bool asym, int wbit,
                            const GridParams &grid, int n_clip, double *H, uint8_t *best,
                            float *err, cudaStream_t st) {
    const int64_t nG = I / GS;
    cudaError_t e = cudaMemsetAsync(H, 0, sizeof(double) * nG * GS * GS, st);
    if (e != cudaSuccess) return e;
    const dim3 ggrid(static_cast<unsigned>(nG), static_cast<unsigned>((N + GRAM_CHUNK - 1) / GRAM_CHUNK));
    if (ggrid.y > 65535u) return cudaErrorInvalidConfiguration;
    if (x_bf16)
        gram_kernel<GS, true><<<ggrid, GRAM_THREADS, 0, st>>>(X, N, I, H);
    else
        gram_kernel<GS, false><<<ggrid, GRAM_THREADS, 0, st>>>(X, N, I, H);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const size_t smem = sizeof(float) * (GS * GS + GC_WARPS * GC_V * GS);
    auto kern = w_bf16 ? gclip_kernel<GS, true> : gclip_kernel<GS, false>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    const dim3 cgrid(static_cast<unsigned>((O + GC_ROWS - 1) / GC_ROWS), static_cast<unsigned>(nG));
    kern<<<cgrid, GC_WARPS * 32, smem, st>>>(W, O, I, s, H, asym, wbit, grid, n_clip, best, err);
    return cudaGetLastError();
}

}  // namespace

int64_t gclip_scratch_doubles(int64_t I, int gs) { return I * gs; }

cudaError_t launch_group_clip(const void *W, bool w_bf16, int64_t O, int64_t I, const void *X,
                              bool x_bf16, int64_t N, const float *s, int gs, bool asym, int wbit,
                              const GridParams &grid, int n_clip, double *H, uint8_t *best,
                              float *err, cudaStream_t st) {
    if (gs == 32)
        return launch_gclip_gs<32>(W, w_bf16, O, I, X, x_bf16, N, s, asym, wbit, grid, n_clip, H, best, err, st);
    if (gs == 64)
        return launch_gclip_gs<64>(W, w_bf16, O, I, X, x_bf16, N, s, asym, wbit, grid, n_clip, H, best, err, st);
    return launch_gclip_gs<128>(W, w_bf16, O, I, X, x_bf16, N, s, asym, wbit, grid, n_clip, H, best, err, st);
}

}  // namespace awq
