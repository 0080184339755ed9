// Small kernels outside the search itself.
//
// fold_scale_kernel: the division of the layer input by the per-channel scale s
// merged into the operator that produces that input (paper summary, Method:
// X / s is fused into the previous operator).  Row c of P holds that operator's
// parameters for channel c (an RMSNorm weight, or a previous linear's weight
// row); every entry is divided by s16[c] with one IEEE fp32 division and, for
// bf16 tensors, rounded to bf16 (nearest even).  HBM-bound elementwise pass.
//
// wait_selftest_kernel: exercises the bounded mbarrier wait and the device
// error word that the search kernel uses, without any copy or MMA in flight.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "awq_internal.h"
#include "awq_ptx.cuh"

namespace awq {

template <bool BF16>
__global__ void __launch_bounds__(256) fold_scale_kernel(const void *__restrict__ P, int64_t R, int64_t C,
                                                         const uint16_t *__restrict__ s16,
                                                         void *__restrict__ out) {
    const int64_t total = R * C;
    const int64_t step = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t k = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; k < total; k += step) {
        const int64_t r = k / C;
        const float sv = __half2float(__ushort_as_half(__ldg(s16 + r)));
        if constexpr (BF16) {
            const float p = __uint_as_float(static_cast<uint32_t>(__ldg(static_cast<const uint16_t *>(P) + k)) << 16);
            static_cast<uint16_t *>(out)[k] = __bfloat16_as_ushort(__float2bfloat16_rn(__fdiv_rn(p, sv)));
        } else {
            static_cast<float *>(out)[k] = __fdiv_rn(__ldg(static_cast<const float *>(P) + k), sv);
        }
    }
}

cudaError_t launch_fold_scale(const void *P, bool bf16, int64_t R, int64_t C, const uint16_t *s16,
                              void *out, cudaStream_t st) {
    const int64_t total = R * C;
    int64_t blocks = (total + 255) / 256;
    if (blocks > 148 * 16) blocks = 148 * 16;
    if (blocks < 1) blocks = 1;
    if (bf16)
        fold_scale_kernel<true><<<static_cast<unsigned>(blocks), 256, 0, st>>>(P, R, C, s16, out);
    else
        fold_scale_kernel<false><<<static_cast<unsigned>(blocks), 256, 0, st>>>(P, R, C, s16, out);
    return cudaGetLastError();
}

__global__ void __launch_bounds__(32) wait_selftest_kernel(long long limit, int arrive, int *err) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncwarp();
    if (arrive && threadIdx.x == 0) mbar_arrive(&bar);
    __syncwarp();
    mbar_wait(&bar, 0, &abort_flag, limit);
    __syncwarp();
    if (threadIdx.x == 0 && abort_flag) atomicExch(err, DEV_ERR_TIMEOUT);
}

cudaError_t launch_wait_selftest(long long limit, bool arrive, int *err, cudaStream_t st) {
    wait_selftest_kernel<<<1, 32, 0, st>>>(limit, arrive ? 1 : 0, err);
    return cudaGetLastError();
}

}  // namespace awq
