// Activation statistic s_X[i] = mean_n |X[n, i]| (AWQ guide, section 三, step 1;
// paper summary, Method: s_X is the per-channel activation magnitude).
//
// HBM-bound column reduction.  Phase 1: each thread owns 2 adjacent columns of
// one chunk of 128 tokens and sums |X| sequentially in fp64, with 32 loads in
// flight (a warp reads 128-256 contiguous bytes per token row).  Phase 2: one
// thread per column adds the chunk partials in ascending chunk order, divides
// by N in fp64 and rounds once to fp32.  The summation order is fixed, so the
// result is bitwise reproducible.
#include <cuda_bf16.h>

#include "awq_internal.h"
#include "awq_ptx.cuh"

namespace awq {

__device__ __forceinline__ double abs_bf16_lo(uint32_t v) {
    return fabs(static_cast<double>(__uint_as_float(v << 16)));
}
__device__ __forceinline__ double abs_bf16_hi(uint32_t v) {
    return fabs(static_cast<double>(__uint_as_float(v & 0xFFFF0000u)));
}

// Chunks are dealt over gridDim.y with a stride, so any number of tokens fits
// the grid's y limit; every chunk's partial is summed the same way whichever
// block computes it.
template <bool BF16>
__global__ void __launch_bounds__(128) stats_partial_kernel(const void *__restrict__ X, int64_t N,
                                                            int64_t I, double *__restrict__ part) {
    const int64_t q = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;  // column pair
    if (q * 2 >= I) return;
    const int64_t n_chunks = (N + STATS_CHUNK - 1) / STATS_CHUNK;
    const int64_t stride = I / 2;   // column pairs per row
    for (int64_t c = blockIdx.y; c < n_chunks; c += gridDim.y) {
        const int64_t n0 = c * STATS_CHUNK;
        const int64_t n1 = (n0 + STATS_CHUNK < N) ? n0 + STATS_CHUNK : N;
        double a0 = 0.0, a1 = 0.0;
        if constexpr (BF16) {
            const uint32_t *p = reinterpret_cast<const uint32_t *>(X) + n0 * stride + q;
#pragma unroll 32
            for (int64_t n = n0; n < n1; ++n) {
                const uint32_t v = __ldg(p);
                p += stride;
                a0 += abs_bf16_lo(v);
                a1 += abs_bf16_hi(v);
            }
        } else {
            const float2 *p = reinterpret_cast<const float2 *>(X) + n0 * stride + q;
#pragma unroll 32
            for (int64_t n = n0; n < n1; ++n) {
                const float2 v = __ldg(p);
                p += stride;
                a0 += fabs(static_cast<double>(v.x));
                a1 += fabs(static_cast<double>(v.y));
            }
        }
        reinterpret_cast<double2 *>(part + c * I)[q] = make_double2(a0, a1);
    }
}

__global__ void __launch_bounds__(256) stats_final_kernel(const double *__restrict__ part,
                                                          int64_t n_chunks, int64_t N, int64_t I,
                                                          float clamp_min, float *__restrict__ sX) {
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= I) return;
    double t = 0.0;
    for (int64_t c = 0; c < n_chunks; ++c) t = __dadd_rn(t, part[c * I + i]);
    const float m = __double2float_rn(__ddiv_rn(t, static_cast<double>(N)));
    sX[i] = m < clamp_min ? clamp_min : m;
}

// ------------------------------------------------- fp16 copy of X for the MMA
// The contraction runs on fp16 operands (11-bit significand: 8x finer rounding
// of dW than bf16 at the same tensor-core rate).  X is copied to fp16 with one
// power-of-two scale 2^-k chosen from max|X| so that the largest magnitude
// lands in [2^14, 2^15): every bf16 value down to 2^-28 of the maximum is then
// exact in fp16, and the losses are rescaled by 2^(2k) exactly afterwards.
__global__ void __launch_bounds__(256) absmax_kernel(const void *__restrict__ X, bool bf16,
                                                     int64_t n, unsigned *__restrict__ max_bits) {
    float m = 0.0f;
    const int64_t step = static_cast<int64_t>(gridDim.x) * blockDim.x;
    if (bf16) {
        const uint4 *p = reinterpret_cast<const uint4 *>(X);
        for (int64_t k = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; k < n / 8; k += step) {
            const uint4 v = __ldg(p + k);
            const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                m = fmaxf(m, fabsf(__uint_as_float(u[j] << 16)));
                m = fmaxf(m, fabsf(__uint_as_float(u[j] & 0xFFFF0000u)));
            }
        }
    } else {
        const float4 *p = reinterpret_cast<const float4 *>(X);
        for (int64_t k = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; k < n / 4; k += step) {
            const float4 v = __ldg(p + k);
            m = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fmaxf(fabsf(v.z), fabsf(v.w)), m));
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    if ((threadIdx.x & 31) == 0) atomicMax(max_bits, __float_as_uint(m));   // m >= 0: bits order as values
}

__device__ __forceinline__ int x_scale_exp(unsigned max_bits) {
    const float m = __uint_as_float(max_bits);
    if (!(m > 0.0f) || isinf(m)) return 0;
    int e;
    frexpf(m, &e);                               // m = f * 2^e, f in [0.5, 1)
    const int k = e - 15;                        // m * 2^-k in [2^14, 2^15)
    return k < -100 ? -100 : (k > 100 ? 100 : k);   // 2^-k stays a normal float
}

__global__ void __launch_bounds__(256) to_f16_kernel(const void *__restrict__ X, bool bf16, int64_t n,
                                                     const unsigned *__restrict__ max_bits,
                                                     int *__restrict__ k_out, uint4 *__restrict__ dst) {
    const int k = x_scale_exp(*max_bits);
    const float sc = ldexpf(1.0f, -k);           // exact power of two
    if (blockIdx.x == 0 && threadIdx.x == 0) *k_out = k;
    const int64_t step = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t q = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; q < n / 8; q += step) {
        float f[8];
        if (bf16) {
            const uint4 v = __ldg(reinterpret_cast<const uint4 *>(X) + q);
            const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                f[2 * j] = __uint_as_float(u[j] << 16);
                f[2 * j + 1] = __uint_as_float(u[j] & 0xFFFF0000u);
            }
        } else {
            const float4 a = __ldg(reinterpret_cast<const float4 *>(X) + 2 * q);
            const float4 b = __ldg(reinterpret_cast<const float4 *>(X) + 2 * q + 1);
            f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
            f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
        }
        uint4 o;
        o.x = f16x2_satfinite(f[0] * sc, f[1] * sc);
        o.y = f16x2_satfinite(f[2] * sc, f[3] * sc);
        o.z = f16x2_satfinite(f[4] * sc, f[5] * sc);
        o.w = f16x2_satfinite(f[6] * sc, f[7] * sc);
        dst[q] = o;
    }
}

cudaError_t launch_stats_partial(const void *X, bool x_bf16, int64_t N, int64_t I, double *part,
                                 cudaStream_t st) {
    const int64_t n_chunks = (N + STATS_CHUNK - 1) / STATS_CHUNK;
    const int64_t pairs = I / 2;
    const int64_t gy = n_chunks < STATS_MAX_GRID_Y ? n_chunks : STATS_MAX_GRID_Y;
    dim3 grid(static_cast<unsigned>((pairs + 127) / 128), static_cast<unsigned>(gy));
    if (x_bf16)
        stats_partial_kernel<true><<<grid, 128, 0, st>>>(X, N, I, part);
    else
        stats_partial_kernel<false><<<grid, 128, 0, st>>>(X, N, I, part);
    return cudaGetLastError();
}

cudaError_t launch_stats_final(const double *part, int64_t N, int64_t I, float clamp_min,
                               float *sX, cudaStream_t st) {
    const int64_t n_chunks = (N + STATS_CHUNK - 1) / STATS_CHUNK;
    stats_final_kernel<<<static_cast<unsigned>((I + 255) / 256), 256, 0, st>>>(
        part, n_chunks, N, I, clamp_min, sX);
    return cudaGetLastError();
}

cudaError_t launch_x_to_f16(const void *X, bool x_bf16, int64_t n, unsigned *max_bits, int *k_out,
                            uint16_t *dst, cudaStream_t st) {
    // n % 8 == 0 (in % 64 == 0); max_bits must be zeroed by the caller.
    int blocks = static_cast<int>((n / 8 + 255) / 256);
    if (blocks > 148 * 8) blocks = 148 * 8;
    if (blocks < 1) blocks = 1;
    absmax_kernel<<<blocks, 256, 0, st>>>(X, x_bf16, n, max_bits);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    to_f16_kernel<<<blocks, 256, 0, st>>>(X, x_bf16, n, max_bits, k_out, reinterpret_cast<uint4 *>(dst));
    return cudaGetLastError();
}

}  // namespace awq
