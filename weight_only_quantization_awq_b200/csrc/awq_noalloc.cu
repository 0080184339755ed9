// awq_act_stats_noalloc: the activation statistic without any device
// allocation.
//
// Some callers cannot call cudaMalloc (or any allocating routine) when they
// compute the statistic: serving and calibration processes that hand nearly
// all device memory to their own pool allocator at start-up, and code that
// must not allocate inside a latency-critical section.  awq_act_stats needs
// a temporary buffer of fp64 chunk partials that it takes from the
// stream-ordered allocator; this entry point uses instead a fixed buffer
// compiled into the library as a file-scope __device__ array.  The caller
// still passes X and sX.
#include <cstdio>
#include <mutex>

#include "awq_b200.h"
#include "awq_internal.h"

namespace {

// Capacity of the fixed buffer: 1,048,576 fp64 chunk partials (8 MiB), i.e.
// ceil(N / 128) * in <= 1,048,576 (for example N = 16384 tokens with
// in <= 8192).  Every GPU that loads the library holds this array until the
// process exits.
constexpr int64_t kScratchPartials = int64_t(1) << 20;
__device__ __align__(256) double g_stats_scratch[kScratchPartials];

// In host code g_stats_scratch names a host-side stand-in, not device memory:
// the kernels get the device address, looked up once per device with that
// device current.
std::mutex g_scratch_mu;
double *g_scratch_dev[64] = {};

cudaError_t scratch_on_current_device(double **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (!g_scratch_dev[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_stats_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_dev[dev] = static_cast<double *>(p);
    }
    *out = g_scratch_dev[dev];
    return cudaSuccess;
}

awq_status_t reject(awq_status_t st, const char *msg) {
    awq::set_last_error(msg);
    return st;
}

}  // namespace

extern "C" awq_status_t awq_act_stats_noalloc(const void *X, int x_dtype, int64_t N, int64_t in,
                                              float clamp_min, float *sX, void *stream) {
    awq::NvtxRange nvtx_range("awq_act_stats_noalloc");
    awq::set_last_error("");
    if (!X || !sX) return reject(AWQ_ERR_ARG, "NULL pointer");
    if (x_dtype != AWQ_F32 && x_dtype != AWQ_BF16) return reject(AWQ_ERR_ARG, "bad x_dtype");
    if (N < 1 || in < 1) return reject(AWQ_ERR_ARG, "bad shape");
    if (in % 8 != 0) return reject(AWQ_ERR_UNSUPPORTED, "in is not a multiple of 8");
    if (!(clamp_min >= 0.0f)) return reject(AWQ_ERR_ARG, "clamp_min must be >= 0");
    if ((reinterpret_cast<uintptr_t>(X) & 15u) || (reinterpret_cast<uintptr_t>(sX) & 15u))
        return reject(AWQ_ERR_ALIGN, "X/sX not 16-byte aligned");
    const int64_t n_chunks = (N + awq::STATS_CHUNK - 1) / awq::STATS_CHUNK;
    if (n_chunks > kScratchPartials / in) {
        char buf[200];
        snprintf(buf, sizeof(buf),
                 "ceil(N/128)*in = %lld fp64 partials exceeds the fixed buffer of %lld "
                 "(use awq_act_stats)",
                 (long long)(n_chunks * in), (long long)kScratchPartials);
        return reject(AWQ_ERR_UNSUPPORTED, buf);
    }
    double *part = nullptr;
    cudaError_t e = scratch_on_current_device(&part);
    if (e != cudaSuccess) return reject(AWQ_ERR_CUDA, cudaGetErrorString(e));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // The partial kernel overwrites every partial it uses, so nothing needs clearing.
    // Timing (when enabled) is recorded as kind 0, like awq_act_stats.
    awq::kt_reset(0);
    awq::kt_begin(0, st);
    e = awq::launch_stats_partial(X, x_dtype == AWQ_BF16, N, in, part, st);
    if (e == cudaSuccess) e = awq::launch_stats_final(part, N, in, clamp_min, sX, st);
    if (e != cudaSuccess) return reject(AWQ_ERR_CUDA, cudaGetErrorString(e));
    awq::kt_end(0, st);
    return AWQ_OK;
}
