// W4A16 linear that applies the search result (AWQ guide, section 三,
// QuantLinear.forward: x is rescaled by the per-channel scale, the INT4 weight
// is dequantised group by group, then a plain linear):
//     y[m, o] = sum_g Delta[o, g] * ( sum_{i in g} xs[m, i] * code[o, i]  -  z[o, g] * sum_{i in g} xs[m, i] )
//     xs = x / s16
// Streaming kernel for small M (decode): one warp per output row at a time,
// lanes read consecutive packed words (coalesced 128-byte rows), xs for up to
// MT tokens is staged in shared memory as fp32 together with its per-group
// sums, so the zero point costs one multiply per group instead of one per
// element.  HBM-bound at M = 1.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "awq_internal.h"

namespace awq {

constexpr int W4_THREADS = 256;
constexpr int W4_MT = 4;                    // tokens per pass

template <int MT>
__global__ void __launch_bounds__(W4_THREADS) w4a16_rowwarp_kernel(
    const uint16_t *__restrict__ x, int64_t M, int64_t I, int64_t O,
    const uint32_t *__restrict__ qweight, const uint16_t *__restrict__ scales,
    const uint32_t *__restrict__ zeros, const uint16_t *__restrict__ s16, int gs,
    uint16_t *__restrict__ y) {
    extern __shared__ float xs_smem[];              // [MT][I] then [MT][nG] group sums
    const int64_t nG = I / gs;
    const int64_t nzw = (nG + 7) / 8;
    float *gsum = xs_smem + MT * I;
    const int64_t m0 = static_cast<int64_t>(blockIdx.y) * MT;
    const int mt = static_cast<int>(M - m0 < MT ? M - m0 : MT);

    for (int64_t k = threadIdx.x; k < static_cast<int64_t>(MT) * I; k += blockDim.x) {
        const int m = static_cast<int>(k / I);
        const int64_t i = k % I;
        float v = 0.0f;
        if (m < mt) {
            const float xv = __uint_as_float(static_cast<uint32_t>(x[(m0 + m) * I + i]) << 16);
            v = __fdiv_rn(xv, __half2float(__ushort_as_half(s16[i])));
        }
        xs_smem[k] = v;
    }
    __syncthreads();
    for (int64_t k = threadIdx.x; k < static_cast<int64_t>(MT) * nG; k += blockDim.x) {
        const int m = static_cast<int>(k / nG);
        const int64_t j = k % nG;
        float acc = 0.0f;
        for (int e = 0; e < gs; ++e) acc += xs_smem[m * I + j * gs + e];
        gsum[k] = acc;
    }
    __syncthreads();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t wpr = I / 8;
    const int64_t warps_total = static_cast<int64_t>(gridDim.x) * (W4_THREADS / 32);
    for (int64_t o = static_cast<int64_t>(blockIdx.x) * (W4_THREADS / 32) + warp; o < O;
         o += warps_total) {
        const uint32_t *qrow = qweight + o * wpr;
        float acc[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[m] = 0.0f;
        // Lanes walk the row in 32-word strides; each word is 8 columns of one group.
        for (int64_t w = lane; w < wpr; w += 32) {
            const uint32_t code = __ldg(qrow + w);
            const int64_t c0 = w * 8;
            const int64_t j = c0 / gs;
            const float d = __half2float(__ushort_as_half(__ldg(scales + o * nG + j)));
            float part[MT];
#pragma unroll
            for (int m = 0; m < MT; ++m) part[m] = 0.0f;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float c = static_cast<float>((code >> (4 * e)) & 0xFu);
#pragma unroll
                for (int m = 0; m < MT; ++m) part[m] = fmaf(xs_smem[m * I + c0 + e], c, part[m]);
            }
            // The zero-point term of a group is added once, by the lane holding its first word.
            float zc = 0.0f;
            if ((c0 % gs) == 0) {
                const float z = zeros ? static_cast<float>((__ldg(zeros + o * nzw + j / 8) >>
                                                            (4 * (j % 8))) & 0xFu)
                                      : 8.0f;
                zc = z;
            }
#pragma unroll
            for (int m = 0; m < MT; ++m) acc[m] = fmaf(d, part[m] - zc * gsum[m * nG + j], acc[m]);
        }
#pragma unroll
        for (int m = 0; m < MT; ++m) {
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) acc[m] += __shfl_xor_sync(0xffffffffu, acc[m], off);
        }
        if (lane == 0) {
            for (int m = 0; m < mt; ++m)
                y[(m0 + m) * O + o] = __bfloat16_as_ushort(__float2bfloat16_rn(acc[m]));
        }
    }
}

cudaError_t launch_w4a16(const uint16_t *x, int64_t M, int64_t I, int64_t O,
                         const uint32_t *qweight, const uint16_t *scales, const uint32_t *zeros,
                         const uint16_t *s16, int gs, uint16_t *y, cudaStream_t st) {
    const int64_t nG = I / gs;
    const size_t smem = sizeof(float) * static_cast<size_t>(W4_MT) * static_cast<size_t>(I + nG);
    static bool attr[64] = {};   // per device
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64 || !attr[dev]) {
        e = cudaFuncSetAttribute(w4a16_rowwarp_kernel<W4_MT>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attr[dev] = true;
    }
    int64_t bx = (O + 7) / 8;
    if (bx > 148 * 4) bx = 148 * 4;
    dim3 grid(static_cast<unsigned>(bx), static_cast<unsigned>((M + W4_MT - 1) / W4_MT));
    w4a16_rowwarp_kernel<W4_MT><<<grid, W4_THREADS, smem, st>>>(x, M, I, O, qweight, scales, zeros,
                                                                s16, gs, y);
    return cudaGetLastError();
}

}  // namespace awq
