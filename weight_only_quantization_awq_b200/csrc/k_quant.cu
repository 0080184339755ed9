// Scale vectors, group quantiser parameters and INT4 packing.
//
//   s[i]  = s_X[i]^alpha / max_j s_X[j]^alpha      (paper summary, Method:
//           s = s_X^alpha; AWQ guide, section 三, step 2: scale / scale.max())
//   Delta = max|W*s| / 7 over a (row, group) for the symmetric quantizer, or
//           (max - min) / 15 with zero point z = clamp(rint(-min/Delta), 0, 15)
//           for the asymmetric one (AWQ guide, section 三, step 4; paper
//           summary, Method, first equation); clip ratios scale the bounds.
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
template <bool WBF16, int GS>
__global__ void __launch_bounds__(128) group_params_kernel(
    const void *__restrict__ W, int64_t O, int64_t I, bool asym, const float *__restrict__ sn,
    GridParams clip, int G, float4 *__restrict__ qparam) {
    __shared__ __align__(16) float s_sm[MAX_GRID][GS];
    const int64_t j = blockIdx.y;
    const int64_t nG = I / GS;
    for (int k = threadIdx.x; k < G * GS; k += blockDim.x)
        s_sm[k / GS][k % GS] = sn[static_cast<int64_t>(2 * (k / GS)) * I + j * GS + (k % GS)];
    __syncthreads();
    const int64_t o = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (o >= O) return;
    constexpr int NW = WBF16 ? GS / 2 : GS;      // 32-bit words of the group
    uint32_t wr[NW];
    const uint4 *src = WBF16 ? reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(W) + o * I + j * GS)
                             : reinterpret_cast<const uint4 *>(static_cast<const float *>(W) + o * I + j * GS);
#pragma unroll
    for (int k = 0; k < NW / 4; ++k) {
        const uint4 v = __ldg(src + k);
        wr[4 * k] = v.x; wr[4 * k + 1] = v.y; wr[4 * k + 2] = v.z; wr[4 * k + 3] = v.w;
    }
    for (int g = 0; g < G; ++g) {
        float mx = -3.4028234663852886e38f, mn = 3.4028234663852886e38f, amax = 0.0f;
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
                if (asym) {
                    mx = fmaxf(mx, wp);
                    mn = fminf(mn, wp);
                } else {
                    amax = fmaxf(amax, fabsf(wp));
                }
            }
        }
        const double r = clip.value[g];
        float D, qlo, qhi;
        if (!asym) {
            D = __fdiv_rn(clip_bound(amax, r), 7.0f);
            qlo = -8.0f;
            qhi = 7.0f;
        } else {
            const float hi = clip_bound(mx, r), lo = clip_bound(mn, r);
            D = __fdiv_rn(__fsub_rn(hi, lo), 15.0f);
            float z = 0.0f;
            if (D != 0.0f) z = fminf(fmaxf(rintf(__fdiv_rn(-lo, D)), 0.0f), 15.0f);
            qlo = -z;
            qhi = 15.0f - z;
            if (D == 0.0f) qhi = 0.0f;
        }
        // {Delta, 1/Delta, -qhi, -qlo}: the search kernel works with -q.
        qparam[(static_cast<int64_t>(g) * nG + j) * O + o] = make_float4(D, safe_rcp(D), -qhi, -qlo);
    }
}

cudaError_t launch_group_params(const void *W, bool w_bf16, int64_t O, int64_t I, int gs,
                                bool asym, const float *sn, const GridParams &clip, int G,
                                float4 *qparam, cudaStream_t st) {
    const dim3 grid(static_cast<unsigned>((O + 127) / 128), static_cast<unsigned>(I / gs));
#define AWQ_GP(WB, GSZ) \
    group_params_kernel<WB, GSZ><<<grid, 128, 0, st>>>(W, O, I, asym, sn, clip, G, qparam)
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
    return cudaGetLastError();
}

// -------------------------------------------------------------------- pack
// One thread per packed word (8 consecutive columns of a row).  The gs/8
// threads of a group are consecutive lanes of one warp and reduce with xor
// shuffles; the first of them writes the group's scale and zero point.
template <bool WBF16>
__global__ void __launch_bounds__(256) pack_kernel(const void *__restrict__ W, int64_t O, int64_t I,
                                                   int gs, bool asym, double clip,
                                                   const float *__restrict__ s,
                                                   uint32_t *__restrict__ qweight,
                                                   uint16_t *__restrict__ scales,
                                                   uint32_t *__restrict__ zeros,
                                                   uint16_t *__restrict__ s16,
                                                   float *__restrict__ scales_f32) {
    const int64_t wpr = I / 8;
    const int64_t total = O * wpr;
    const int seg = gs / 8;
    const int64_t nG = I / gs;
    const int64_t nzw = (nG + 7) / 8;
    const int64_t step = static_cast<int64_t>(gridDim.x) * blockDim.x;
    const int64_t iters = (total + step - 1) / step;
    for (int64_t it = 0; it < iters; ++it) {
        const int64_t idx = it * step + static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
        const bool active = idx < total;
        const int64_t o = active ? idx / wpr : 0;
        const int64_t wcol = active ? idx % wpr : 0;
        const int64_t c0 = wcol * 8;
        float w[8], sv[8], wp[8];
        if (active) {
            if constexpr (WBF16) {
                const uint4 v = *reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(W) +
                                                                o * I + c0);
                const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    w[2 * k] = __uint_as_float(u[k] << 16);
                    w[2 * k + 1] = __uint_as_float(u[k] & 0xFFFF0000u);
                }
            } else {
                const float4 *p = reinterpret_cast<const float4 *>(static_cast<const float *>(W) +
                                                                  o * I + c0);
                const float4 a = p[0], b = p[1];
                w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
                w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
            }
            const float4 sa = *reinterpret_cast<const float4 *>(s + c0);
            const float4 sb = *reinterpret_cast<const float4 *>(s + c0 + 4);
            sv[0] = sa.x; sv[1] = sa.y; sv[2] = sa.z; sv[3] = sa.w;
            sv[4] = sb.x; sv[5] = sb.y; sv[6] = sb.z; sv[7] = sb.w;
        } else {
#pragma unroll
            for (int k = 0; k < 8; ++k) { w[k] = 0.0f; sv[k] = 1.0f; }
        }
        float mx = -3.4028234663852886e38f, mn = 3.4028234663852886e38f, amax = 0.0f;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            wp[k] = __fmul_rn(w[k], sv[k]);
            mx = fmaxf(mx, wp[k]);
            mn = fminf(mn, wp[k]);
            amax = fmaxf(amax, fabsf(wp[k]));
        }
        for (int off = 1; off < seg; off <<= 1) {
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
            mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
        }
        float D, z = 0.0f;
        if (!asym) {
            const float a = clip == 1.0 ? amax : __double2float_rn(__dmul_rn((double)amax, clip));
            D = __fdiv_rn(a, 7.0f);
        } else {
            const float hi = clip == 1.0 ? mx : __double2float_rn(__dmul_rn((double)mx, clip));
            const float lo = clip == 1.0 ? mn : __double2float_rn(__dmul_rn((double)mn, clip));
            D = __fdiv_rn(__fsub_rn(hi, lo), 15.0f);
            if (D != 0.0f) z = fminf(fmaxf(rintf(__fdiv_rn(-lo, D)), 0.0f), 15.0f);
        }
        // q = rint(RN(W'/Delta)) from the reciprocal product W' * RN(1/Delta): every
        // decision that survives the clamp has |W'/Delta| <= 15.5, where the product
        // is within 2^-19 of RN(W'/Delta); products within 2^-16 of a half-integer
        // (exact ties included) are redone with the correctly rounded division.
        float q[8];
        const float invD = D != 0.0f ? __frcp_rn(D) : 0.0f;
        bool near_tie = false;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            q[k] = __fsub_rn(__fmaf_rn(wp[k], invD, 12582912.0f), 12582912.0f);
            near_tie |= fabsf(__fmaf_rn(wp[k], invD, -q[k])) > 0.5f - 1.0f / 65536.0f;
        }
        if (near_tie && D != 0.0f) {
#pragma unroll
            for (int k = 0; k < 8; ++k) q[k] = rintf(__fdiv_rn(wp[k], D));
        }
        uint32_t word = 0;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const float c = asym ? fminf(fmaxf(q[k] + z, 0.0f), 15.0f)
                                 : fminf(fmaxf(q[k], -8.0f), 7.0f) + 8.0f;
            word |= (static_cast<uint32_t>(static_cast<int>(c)) & 0xFu) << (4 * k);
        }
        if (!active) continue;
        qweight[idx] = word;
        if ((wcol % seg) == 0) {
            const int64_t j = c0 / gs;
            scales[o * nG + j] = __half_as_ushort(__float2half_rn(D));
            if (scales_f32) scales_f32[o * nG + j] = D;
            if (zeros)
                atomicOr(&zeros[o * nzw + j / 8],
                         (static_cast<uint32_t>(z) & 0xFu) << (4 * static_cast<int>(j % 8)));
        }
        if (o == 0) {
#pragma unroll
            for (int k = 0; k < 8; ++k) s16[c0 + k] = __half_as_ushort(__float2half_rn(sv[k]));
        }
    }
}

cudaError_t launch_pack(const void *W, bool w_bf16, int64_t O, int64_t I, int gs, bool asym,
                        double clip, const float *s, uint32_t *qweight, uint16_t *scales,
                        uint32_t *zeros, uint16_t *s16, float *scales_f32, cudaStream_t st) {
    const int64_t total = O * (I / 8);
    int64_t blocks = (total + 255) / 256;
    if (blocks > 148 * 8) blocks = 148 * 8;
    if (w_bf16)
        pack_kernel<true><<<static_cast<unsigned>(blocks), 256, 0, st>>>(
            W, O, I, gs, asym, clip, s, qweight, scales, zeros, s16, scales_f32);
    else
        pack_kernel<false><<<static_cast<unsigned>(blocks), 256, 0, st>>>(
            W, O, I, gs, asym, clip, s, qweight, scales, zeros, s16, scales_f32);
    return cudaGetLastError();
}

}  // namespace awq
