// Loss reduction and grid-point selection (paper summary, Method:
// alpha* = argmin_alpha L(s_X^alpha)).
//
//   loss_row[g, o] = sum_tb part[g, tb, o]            (fp64, ascending tb)
//   loss[g]        = sum_o loss_row[g, o] / (N * O)   (fp64, fixed tree order)
//   best           = first g with the minimal loss
// All orders are fixed, so the losses are bitwise reproducible run to run.
#include "awq_internal.h"

namespace awq {

constexpr int RED_THREADS = 256;

__global__ void __launch_bounds__(RED_THREADS) reduce_rows_kernel(const float *__restrict__ part,
                                                                  int64_t TB, int64_t O,
                                                                  const int *__restrict__ x_exp,
                                                                  const int *__restrict__ dw_exp,
                                                                  float *__restrict__ loss_row,
                                                                  double *__restrict__ blocksum) {
    __shared__ double red[RED_THREADS];
    const int g = blockIdx.y;
    const int64_t o = static_cast<int64_t>(blockIdx.x) * RED_THREADS + threadIdx.x;
    double v = 0.0;
    if (o < O) {
        const float *p = part + static_cast<int64_t>(g) * TB * O + o;
        for (int64_t tb = 0; tb < TB; ++tb) v = __dadd_rn(v, static_cast<double>(p[tb * O]));
        v = ldexp(v, 2 * (*x_exp - dw_exp[g]));
        if (loss_row) loss_row[static_cast<int64_t>(g) * O + o] = __double2float_rn(v);
    }
    red[threadIdx.x] = v;
    __syncthreads();
    for (int off = RED_THREADS / 2; off > 0; off >>= 1) {
        if (threadIdx.x < off) red[threadIdx.x] = __dadd_rn(red[threadIdx.x], red[threadIdx.x + off]);
        __syncthreads();
    }
    if (threadIdx.x == 0) blocksum[static_cast<int64_t>(g) * gridDim.x + blockIdx.x] = red[0];
}

__global__ void __launch_bounds__(RED_THREADS) reduce_blocks_kernel(const double *__restrict__ blocksum,
                                                                    int nblk, double denom,
                                                                    double *__restrict__ loss) {
    __shared__ double red[RED_THREADS];
    const int g = blockIdx.x;
    double v = 0.0;
    for (int b = threadIdx.x; b < nblk; b += RED_THREADS)
        v = __dadd_rn(v, blocksum[static_cast<int64_t>(g) * nblk + b]);
    red[threadIdx.x] = v;
    __syncthreads();
    for (int off = RED_THREADS / 2; off > 0; off >>= 1) {
        if (threadIdx.x < off) red[threadIdx.x] = __dadd_rn(red[threadIdx.x], red[threadIdx.x + off]);
        __syncthreads();
    }
    if (threadIdx.x == 0) loss[g] = __ddiv_rn(red[0], denom);
}

__global__ void argmin_kernel(const double *__restrict__ loss, int G, int *__restrict__ best) {
    if (threadIdx.x != 0 || blockIdx.x != 0) return;
    int b = 0;
    for (int k = 1; k < G; ++k)
        if (loss[k] < loss[b]) b = k;
    *best = b;
}

int64_t reduce_scratch_doubles(int G, int64_t O) {
    return static_cast<int64_t>(G) * ((O + RED_THREADS - 1) / RED_THREADS);
}

cudaError_t launch_reduce_loss(const float *part, int G, int64_t TB, int64_t O, int64_t N,
                               const int *x_exp, const int *dw_exp, double *loss, float *loss_row,
                               double *blocksum, cudaStream_t st) {
    const int nblk = static_cast<int>((O + RED_THREADS - 1) / RED_THREADS);
    reduce_rows_kernel<<<dim3(nblk, G), RED_THREADS, 0, st>>>(part, TB, O, x_exp, dw_exp, loss_row,
                                                              blocksum);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    reduce_blocks_kernel<<<G, RED_THREADS, 0, st>>>(blocksum, nblk,
                                                    static_cast<double>(N) * static_cast<double>(O),
                                                    loss);
    return cudaGetLastError();
}

cudaError_t launch_argmin(const double *loss, int G, int *best, cudaStream_t st) {
    argmin_kernel<<<1, 32, 0, st>>>(loss, G, best);
    return cudaGetLastError();
}

}  // namespace awq
