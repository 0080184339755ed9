// Scale vectors, group quantiser parameters and INT4 packing.
//
//   s[i]  = s_X[i]^alpha / max_j s_X[j]^alpha      (paper summary, Method:
//           s = s_X^alpha; AWQ guide, section 三, step 2: scale / scale.max())
//   Delta = max|W*s| / 7 over a (row, group) for the symmetric quantizer, or
//           (max - min) / 15 with zero point z = clamp(rint(-min/Delta), 0, 15)
//           for the asymmetric one (AWQ guide, section 三, step 4; paper
//           summary, Method, first equation); clip ratios scale the bounds.
//           At w_bit = 3 the constants are 3 (codes [-4, 3]) and 7 ([0, 7]).
//
// Everything that decides an integer (Delta, z, codes) uses IEEE fp32
// operations with explicit rounding intrinsics, so no FMA contraction or
// approximate divide can change a code.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "awq_internal.h"

namespace awq {

// ------------------------------------------------------------ scale table
// Pass 1: t[g][i] = pow(s_X[i], alpha_g) in fp64, and max_i t[g][i] through an
// atomic max on the bit patterns (t >= 0, so bit order is value order).
// Pass 2: s = fp32(t / max), -1/s.
__global__ void __launch_bounds__(256) scale_pow_kernel(const float *__restrict__ sX, int64_t I,
                                                        GridParams alpha,
                                                        const int *__restrict__ best_idx,
                                                        double *__restrict__ t,
                                                        unsigned long long *__restrict__ max_bits) {
    __shared__ double red[256];
    const int g = blockIdx.y;
    const double a = best_idx ? alpha.value[*best_idx] : alpha.value[g];
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    double v = 0.0;
    if (i < I) {
        v = pow(static_cast<double>(sX[i]), a);
        t[g * I + i] = v;
    }
    red[threadIdx.x] = v;
    __syncthreads();
    for (int off = 128; off > 0; off >>= 1) {
        if (threadIdx.x < off) red[threadIdx.x] = fmax(red[threadIdx.x], red[threadIdx.x + off]);
        __syncthreads();
    }
    if (threadIdx.x == 0)
        atomicMax(&max_bits[g], static_cast<unsigned long long>(__double_as_longlong(red[0])));
}

__global__ void __launch_bounds__(256) scale_div_kernel(const double *__restrict__ t, int64_t I,
                                                        const unsigned long long *__restrict__ max_bits,
                                                        float *__restrict__ sn) {
    const int g = blockIdx.y;
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= I) return;
    const double m = __longlong_as_double(static_cast<long long>(max_bits[g]));
    const float s = __double2float_rn(__ddiv_rn(t[g * I + i], m));
    sn[(2 * g) * I + i] = s;
    sn[(2 * g + 1) * I + i] = -__frcp_rn(s);
}

int64_t scale_scratch_bytes(int G, int64_t I) {
    return static_cast<int64_t>(G) * I * 8 + static_cast<int64_t>(G) * 8;
}

cudaError_t launch_scale_table(const float *sX, int64_t I, const GridParams &alpha, int G,
                               const int *best_idx, float *sn, void *scratch, cudaStream_t st) {
    double *t = static_cast<double *>(scratch);
    unsigned long long *mb = reinterpret_cast<unsigned long long *>(t + static_cast<int64_t>(G) * I);
    cudaError_t e = cudaMemsetAsync(mb, 0, sizeof(unsigned long long) * G, st);
    if (e != cudaSuccess) return e;
    const dim3 grid(static_cast<unsigned>((I + 255) / 256), static_cast<unsigned>(G));
    scale_pow_kernel<<<grid, 256, 0, st>>>(sX, I, alpha, best_idx, t, mb);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    scale_div_kernel<<<grid, 256, 0, st>>>(t, I, mb, sn);
    return cudaGetLastError();
}

// ------------------------------------------------- group quantiser params
__device__ __forceinline__ float clip_bound(float b, double r) {
    return r == 1.0 ? b : __double2float_rn(__dmul_rn(static_cast<double>(b), r));
}

__device__ __forceinline__ float safe_rcp(float d) {
    if (!(d > 0.0f)) return 0.0f;
    const float r = __frcp_rn(d);
    return isinf(r) ? 3.4028234663852886e38f : r;
}

// One thread per (row, group): the thread keeps its group's gs weights in
// registers and loops over the G grid points; each grid point's s values for
// the group are broadcast from shared memory.  Output layout qparam[g][j][o]
// (rows fastest) so the writes coalesce.
// It also bounds |dW| = |(q - z)*Delta/s - W| over the layer per grid point:
//     |dW[o, i]| <= max_group |W| + 2^w_bit * Delta / min_group s,
// folded into dw_bits[g] with an atomic max on the bit pattern (>= 0).
template <bool WBF16, int GS>
__global__ void __launch_bounds__(128) group_params_kernel(
    const void *__restrict__ W, int64_t O, int64_t I, bool asym, int wbit,
    const float *__restrict__ sn, GridParams clip, int G, float4 *__restrict__ qparam,
    unsigned *__restrict__ dw_bits) {
    __shared__ __align__(16) float s_sm[MAX_GRID][GS];
    const int64_t j = blockIdx.y;
    const int64_t nG = I / GS;
    for (int k = threadIdx.x; k < G * GS; k += blockDim.x)
        s_sm[k / GS][k % GS] = sn[static_cast<int64_t>(2 * (k / GS)) * I + j * GS + (k % GS)];
    __syncthreads();
    const int64_t o = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (o >= O) return;
    const unsigned live = __activemask();
    constexpr int NW = WBF16 ? GS / 2 : GS;      // 32-bit words of the group
    uint32_t wr[NW];
    const uint4 *src = WBF16 ? reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(W) + o * I + j * GS)
                             : reinterpret_cast<const uint4 *>(static_cast<const float *>(W) + o * I + j * GS);
#pragma unroll
    for (int k = 0; k < NW / 4; ++k) {
        const uint4 v = __ldg(src + k);
        wr[4 * k] = v.x; wr[4 * k + 1] = v.y; wr[4 * k + 2] = v.z; wr[4 * k + 3] = v.w;
    }
    float wabs = 0.0f;                           // max |W| of the group
#pragma unroll
    for (int e = 0; e < GS; ++e) {
        if constexpr (WBF16)
            wabs = fmaxf(wabs, fabsf(__uint_as_float((e & 1) ? (wr[e >> 1] & 0xFFFF0000u) : (wr[e >> 1] << 16))));
        else
            wabs = fmaxf(wabs, fabsf(__uint_as_float(wr[e])));
    }
    for (int g = 0; g < G; ++g) {
        // four independent max / min chains (max and min are exact, so the split
        // changes no result), merged at the end
        float mx4[4], mn4[4], am4[4], smin4[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            mx4[k] = -3.4028234663852886e38f;
            mn4[k] = 3.4028234663852886e38f;
            am4[k] = 0.0f;
            smin4[k] = 3.4028234663852886e38f;
        }
#pragma unroll
        for (int e4 = 0; e4 < GS / 4; ++e4) {
            const float4 s4 = *reinterpret_cast<const float4 *>(&s_sm[g][4 * e4]);
            const float sv[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int e = 4 * e4 + k;
                float w;
                if constexpr (WBF16)
                    w = (e & 1) ? __uint_as_float(wr[e >> 1] & 0xFFFF0000u) : __uint_as_float(wr[e >> 1] << 16);
                else
                    w = __uint_as_float(wr[e]);
                const float wp = __fmul_rn(w, sv[k]);
                smin4[k] = fminf(smin4[k], sv[k]);
                if (asym) {
                    mx4[k] = fmaxf(mx4[k], wp);
                    mn4[k] = fminf(mn4[k], wp);
                } else {
                    am4[k] = fmaxf(am4[k], fabsf(wp));
                }
            }
        }
        const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
        const float mn = fminf(fminf(mn4[0], mn4[1]), fminf(mn4[2], mn4[3]));
        const float amax = fmaxf(fmaxf(am4[0], am4[1]), fmaxf(am4[2], am4[3]));
        const double r = clip.value[g];
        float D, qlo, qhi;
        if (!asym) {
            const float top = static_cast<float>((1 << (wbit - 1)) - 1);   // 7 or 3
            D = __fdiv_rn(clip_bound(amax, r), top);
            qlo = -top - 1.0f;
            qhi = top;
        } else {
            const float top = static_cast<float>((1 << wbit) - 1);         // 15 or 7
            const float hi = clip_bound(mx, r), lo = clip_bound(mn, r);
            D = __fdiv_rn(__fsub_rn(hi, lo), top);
            float z = 0.0f;
            if (D != 0.0f) z = fminf(fmaxf(rintf(__fdiv_rn(-lo, D)), 0.0f), top);
            qlo = -z;
            qhi = top - z;
            if (D == 0.0f) qhi = 0.0f;
        }
        // {Delta, 1/Delta, -qhi, -qlo}: the search kernel works with -q.
        qparam[(static_cast<int64_t>(g) * nG + j) * O + o] = make_float4(D, safe_rcp(D), -qhi, -qlo);
        const float smin = fminf(fminf(smin4[0], smin4[1]), fminf(smin4[2], smin4[3]));
        const float bound = wabs + static_cast<float>(1 << wbit) * D / smin;
        const unsigned b = (bound >= 0.0f && bound < 3.0e38f) ? __float_as_uint(bound) : 0x7F000000u;
        const unsigned wmax = __reduce_max_sync(live, b);
        if ((threadIdx.x & 31) == __ffs(live) - 1) atomicMax(&dw_bits[g], wmax);
    }
}

// dW goes to fp16 for the tensor cores.  Grid point g's bound B on |dW| picks
// k with B * 2^k in [2^14, 2^15) (|k| <= 60); the -1/s row of the scale table
// is multiplied by 2^k (exact), so the search kernel forms 2^k * dW at no cost,
// and the loss reduction multiplies by 2^-2k.  Without it, a layer of small
// weights would put dW into fp16's subnormal range.
__global__ void __launch_bounds__(256) dw_scale_kernel(int64_t I, const unsigned *__restrict__ dw_bits,
                                                       float *__restrict__ sn, int *__restrict__ dw_exp) {
    const int g = blockIdx.y;
    const float b = __uint_as_float(dw_bits[g]);
    int k = 0;
    if (b > 0.0f) {
        int e;
        frexpf(b, &e);                            // b = f * 2^e, f in [0.5, 1)
        k = 15 - e;
        k = k < -60 ? -60 : (k > 60 ? 60 : k);
    }
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i < I) {
        float *row = sn + (2 * static_cast<int64_t>(g) + 1) * I;
        row[i] = ldexpf(row[i], k);
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) dw_exp[g] = k;
}

cudaError_t launch_group_params(const void *W, bool w_bf16, int64_t O, int64_t I, int gs,
                                bool asym, int wbit, float *sn, const GridParams &clip,
                                int G, float4 *qparam, unsigned *dw_bits, int *dw_exp,
                                cudaStream_t st) {
    cudaError_t e0 = cudaMemsetAsync(dw_bits, 0, sizeof(unsigned) * G, st);
    if (e0 != cudaSuccess) return e0;
    const dim3 grid(static_cast<unsigned>((O + 127) / 128), static_cast<unsigned>(I / gs));
#define AWQ_GP(WB, GSZ) \
    group_params_kernel<WB, GSZ><<<grid, 128, 0, st>>>(W, O, I, asym, wbit, sn, clip, G, qparam, dw_bits)
    if (w_bf16) {
        if (gs == 32) AWQ_GP(true, 32);
        else if (gs == 64) AWQ_GP(true, 64);
        else AWQ_GP(true, 128);
    } else {
        if (gs == 32) AWQ_GP(false, 32);
        else if (gs == 64) AWQ_GP(false, 64);
        else AWQ_GP(false, 128);
    }
#undef AWQ_GP
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    dw_scale_kernel<<<dim3(static_cast<unsigned>((I + 255) / 256), static_cast<unsigned>(G)), 256, 0, st>>>(
        I, dw_bits, sn, dw_exp);
    return cudaGetLastError();
}

// -------------------------------------------------------------------- pack
// 2-D grid: blockIdx.x = row, a thread packs PW consecutive words (8 columns
// each) of that row, issuing all of its loads (W and s) before any arithmetic.
// A group's gs/8 words belong to gs/(8*PW) consecutive lanes (or to part of
// one thread's words), which reduce with xor shuffles; the group's first
// thread writes its scale and zero point.
constexpr int PACK_PW = 4;                   // words per thread
constexpr int PACK_THREADS = 128;

template <bool WBF16>
__global__ void __launch_bounds__(PACK_THREADS) pack_kernel(const void *__restrict__ W, int O, int I,
                                                            int gs, bool asym, int wbit, double clip,
                                                            const uint8_t *__restrict__ clip_idx,
                                                            GridParams clip_grid,
                                                            const float *__restrict__ s,
                                                            uint32_t *__restrict__ qweight,
                                                            uint16_t *__restrict__ scales,
                                                            uint32_t *__restrict__ zeros,
                                                            uint16_t *__restrict__ s16,
                                                            float *__restrict__ scales_f32) {
    const int o = blockIdx.x;
    const int wpr = I / 8;                                  // words per row
    const int w0 = (blockIdx.y * PACK_THREADS + threadIdx.x) * PACK_PW;   // first word of this thread
    const int nG = I / gs, nzw = (nG + 7) / 8;
    const int wpg = gs / 8;                                 // words per group (4, 8 or 16)
    const bool active = w0 < wpr;                           // wpr is a multiple of PACK_PW (I % 64 == 0)
    // ---- loads: W (PW x 8 values) and s (PW x 8 values)
    float w[PACK_PW][8], sv[PACK_PW][8];
    if (active) {
        if constexpr (WBF16) {
            const uint4 *src = reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(W) +
                                                               static_cast<int64_t>(o) * I) + w0;
            uint4 v[PACK_PW];
#pragma unroll
            for (int k = 0; k < PACK_PW; ++k) v[k] = __ldg(src + k);
#pragma unroll
            for (int k = 0; k < PACK_PW; ++k) {
                const uint32_t u[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    w[k][2 * e] = __uint_as_float(u[e] << 16);
                    w[k][2 * e + 1] = __uint_as_float(u[e] & 0xFFFF0000u);
                }
            }
        } else {
            const float4 *src = reinterpret_cast<const float4 *>(static_cast<const float *>(W) +
                                                                 static_cast<int64_t>(o) * I) + 2 * w0;
            float4 v[2 * PACK_PW];
#pragma unroll
            for (int k = 0; k < 2 * PACK_PW; ++k) v[k] = __ldg(src + k);
#pragma unroll
            for (int k = 0; k < PACK_PW; ++k) {
                w[k][0] = v[2 * k].x; w[k][1] = v[2 * k].y; w[k][2] = v[2 * k].z; w[k][3] = v[2 * k].w;
                w[k][4] = v[2 * k + 1].x; w[k][5] = v[2 * k + 1].y; w[k][6] = v[2 * k + 1].z; w[k][7] = v[2 * k + 1].w;
            }
        }
        const float4 *sp = reinterpret_cast<const float4 *>(s) + 2 * w0;
        float4 sq[2 * PACK_PW];
#pragma unroll
        for (int k = 0; k < 2 * PACK_PW; ++k) sq[k] = __ldg(sp + k);
#pragma unroll
        for (int k = 0; k < PACK_PW; ++k) {
            sv[k][0] = sq[2 * k].x; sv[k][1] = sq[2 * k].y; sv[k][2] = sq[2 * k].z; sv[k][3] = sq[2 * k].w;
            sv[k][4] = sq[2 * k + 1].x; sv[k][5] = sq[2 * k + 1].y; sv[k][6] = sq[2 * k + 1].z; sv[k][7] = sq[2 * k + 1].w;
        }
    } else {
#pragma unroll
        for (int k = 0; k < PACK_PW; ++k)
#pragma unroll
            for (int e = 0; e < 8; ++e) { w[k][e] = 0.0f; sv[k][e] = 1.0f; }
    }
    // ---- per word: W' = W * s and its group bounds
    float wp[PACK_PW][8], mx[PACK_PW], mn[PACK_PW], am[PACK_PW];
#pragma unroll
    for (int k = 0; k < PACK_PW; ++k) {
        mx[k] = -3.4028234663852886e38f;
        mn[k] = 3.4028234663852886e38f;
        am[k] = 0.0f;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            wp[k][e] = __fmul_rn(w[k][e], sv[k][e]);
            mx[k] = fmaxf(mx[k], wp[k][e]);
            mn[k] = fminf(mn[k], wp[k][e]);
            am[k] = fmaxf(am[k], fabsf(wp[k][e]));
        }
    }
    // words of one thread that share a group (gs = 32: 4 words per group, the thread's
    // PW = 4 words are exactly one group; larger groups span 2 or 4 lanes)
    float gmx = mx[0], gmn = mn[0], gam = am[0];
#pragma unroll
    for (int k = 1; k < PACK_PW; ++k) {
        gmx = fmaxf(gmx, mx[k]);
        gmn = fminf(gmn, mn[k]);
        gam = fmaxf(gam, am[k]);
    }
    const int lpg = wpg / PACK_PW;                          // lanes per group: 1, 2 or 4
    for (int off = 1; off < lpg; off <<= 1) {
        gmx = fmaxf(gmx, __shfl_xor_sync(0xffffffffu, gmx, off));
        gmn = fminf(gmn, __shfl_xor_sync(0xffffffffu, gmn, off));
        gam = fmaxf(gam, __shfl_xor_sync(0xffffffffu, gam, off));
    }
    // the group's clip ratio: one per layer, or its own entry of the per-group choice
    const int jg = active ? w0 / wpg : 0;
    if (clip_idx && active) clip = clip_grid.value[clip_idx[static_cast<int64_t>(o) * nG + jg]];
    const float stop = static_cast<float>((1 << (wbit - 1)) - 1);   // symmetric top code: 7 or 3
    const float atop = static_cast<float>((1 << wbit) - 1);         // asymmetric top code: 15 or 7
    float D, z = 0.0f;
    if (!asym) {
        const float a = clip == 1.0 ? gam : __double2float_rn(__dmul_rn((double)gam, clip));
        D = __fdiv_rn(a, stop);
    } else {
        const float hi = clip == 1.0 ? gmx : __double2float_rn(__dmul_rn((double)gmx, clip));
        const float lo = clip == 1.0 ? gmn : __double2float_rn(__dmul_rn((double)gmn, clip));
        D = __fdiv_rn(__fsub_rn(hi, lo), atop);
        if (D != 0.0f) z = fminf(fmaxf(rintf(__fdiv_rn(-lo, D)), 0.0f), atop);
    }
    // q = rint(RN(W'/Delta)) from the reciprocal product W' * RN(1/Delta): every
    // decision that survives the clamp has |W'/Delta| <= 15.5, where the product
    // is within 2^-19 of RN(W'/Delta); products within 2^-16 of a half-integer
    // (exact ties included) are redone with the correctly rounded division.
    const float invD = D != 0.0f ? __frcp_rn(D) : 0.0f;
    uint32_t word[PACK_PW];
#pragma unroll
    for (int k = 0; k < PACK_PW; ++k) {
        float q[8];
        bool near_tie = false;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            q[e] = __fsub_rn(__fmaf_rn(wp[k][e], invD, 12582912.0f), 12582912.0f);
            near_tie |= fabsf(__fmaf_rn(wp[k][e], invD, -q[e])) > 0.5f - 1.0f / 65536.0f;
        }
        if (near_tie && D != 0.0f) {
#pragma unroll
            for (int e = 0; e < 8; ++e) q[e] = rintf(__fdiv_rn(wp[k][e], D));
        }
        uint32_t wd = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float c = asym ? fminf(fmaxf(q[e] + z, 0.0f), atop)
                                 : fminf(fmaxf(q[e], -stop - 1.0f), stop) + 8.0f;
            wd |= (static_cast<uint32_t>(static_cast<int>(c)) & 0xFu) << (4 * e);
        }
        word[k] = wd;
    }
    if (!active) return;
    *reinterpret_cast<uint4 *>(qweight + static_cast<int64_t>(o) * wpr + w0) =
        make_uint4(word[0], word[1], word[2], word[3]);
    if ((w0 % wpg) == 0) {                                  // the group's first thread
        const int j = w0 / wpg;
        scales[static_cast<int64_t>(o) * nG + j] = __half_as_ushort(__float2half_rn(D));
        if (scales_f32) scales_f32[static_cast<int64_t>(o) * nG + j] = D;
        if (zeros)
            atomicOr(&zeros[static_cast<int64_t>(o) * nzw + j / 8],
                     (static_cast<uint32_t>(z) & 0xFu) << (4 * (j % 8)));
    }
    if (o == 0) {
#pragma unroll
        for (int k = 0; k < PACK_PW; ++k)
#pragma unroll
            for (int e = 0; e < 8; ++e) s16[(w0 + k) * 8 + e] = __half_as_ushort(__float2half_rn(sv[k][e]));
    }
}

cudaError_t launch_pack(const void *W, bool w_bf16, int64_t O, int64_t I, int gs, bool asym,
                        int wbit, double clip, const uint8_t *clip_idx, const GridParams &clip_grid,
                        const float *s, uint32_t *qweight, uint16_t *scales, uint32_t *zeros,
                        uint16_t *s16, float *scales_f32, cudaStream_t st) {
    const int64_t wpr = I / 8;
    const dim3 grid(static_cast<unsigned>(O),
                    static_cast<unsigned>((wpr / PACK_PW + PACK_THREADS - 1) / PACK_THREADS));
    if (w_bf16)
        pack_kernel<true><<<grid, PACK_THREADS, 0, st>>>(W, static_cast<int>(O), static_cast<int>(I), gs, asym,
                                                         wbit, clip, clip_idx, clip_grid, s, qweight,
                                                         scales, zeros, s16, scales_f32);
    else
        pack_kernel<false><<<grid, PACK_THREADS, 0, st>>>(W, static_cast<int>(O), static_cast<int>(I), gs, asym,
                                                          wbit, clip, clip_idx, clip_grid, s, qweight,
                                                          scales, zeros, s16, scales_f32);
    return cudaGetLastError();
}

}  // namespace awq
