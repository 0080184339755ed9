// C ABI of the library (declared in include/awq_b200.h).  This layer checks
// arguments on the host, sizes and allocates the temporary device workspace
// with stream-ordered allocation, builds the TMA descriptor of the
// calibration activations, and enqueues the kernels.  No arithmetic of the
// method runs here: every step is a kernel.
#include <cudaTypedefs.h>

#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "awq_b200.h"
#include "awq_internal.h"

namespace {

thread_local std::string g_last_error;

awq_status_t fail(awq_status_t st, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return st;
}

awq_status_t cuda_fail(cudaError_t e, const char *what) {
    return fail(AWQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

#define AWQ_CUDA(call)                                          \
    do {                                                        \
        cudaError_t e_ = (call);                                \
        if (e_ != cudaSuccess) return cuda_fail(e_, #call);     \
    } while (0)

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Per-device facts and one-time set-up (SM count; the default memory pool keeps
// freed blocks cached so stream-ordered workspace allocation is cheap).
struct DeviceInfo {
    int sms = 0;
    bool ready = false;
};
std::mutex g_dev_mu;
DeviceInfo g_dev[64];

awq_status_t device_info(int *sms) {
    int dev = 0;
    AWQ_CUDA(cudaGetDevice(&dev));
    if (dev < 0 || dev >= 64) return fail(AWQ_ERR_UNSUPPORTED, "device index %d", dev);
    std::lock_guard<std::mutex> lk(g_dev_mu);
    DeviceInfo &d = g_dev[dev];
    if (!d.ready) {
        AWQ_CUDA(cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev));
        cudaMemPool_t pool;
        AWQ_CUDA(cudaDeviceGetDefaultMemPool(&pool, dev));
        uint64_t thr = UINT64_MAX;
        AWQ_CUDA(cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &thr));
        d.ready = true;
    }
    *sms = d.sms;
    return AWQ_OK;
}

// Temporary device workspace: one stream-ordered allocation per call, carved
// into 256-byte aligned pieces, freed on the same stream when the call ends.
struct Workspace {
    cudaStream_t st;
    char *base = nullptr;
    size_t size = 0, used = 0;
    explicit Workspace(cudaStream_t s) : st(s) {}
    ~Workspace() {
        if (base) cudaFreeAsync(base, st);
    }
    static size_t up(size_t b) { return (b + 255) & ~static_cast<size_t>(255); }
    awq_status_t reserve(size_t bytes) {
        size = bytes;
        cudaError_t e = cudaMallocAsync(reinterpret_cast<void **>(&base), bytes, st);
        if (e != cudaSuccess) {
            base = nullptr;
            return cuda_fail(e, "cudaMallocAsync(workspace)");
        }
        return AWQ_OK;
    }
    template <typename T>
    T *take(size_t count) {
        T *p = reinterpret_cast<T *>(base + used);
        used += up(count * sizeof(T));
        return p;
    }
};

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// A 2-D tiled tensor map over a row-major [dim1, dim0] array.
awq_status_t make_map_2d(CUtensorMap *map, CUtensorMapDataType dt, size_t elem, const void *ptr,
                         uint64_t dim0, uint64_t dim1, uint32_t box0, uint32_t box1,
                         CUtensorMapSwizzle swz) {
    auto enc = get_encode();
    if (!enc) return fail(AWQ_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(dim0), static_cast<cuuint64_t>(dim1)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(dim0 * elem)};
    cuuint32_t box[2] = {box0, box1};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, dt, 2, const_cast<void *>(ptr), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(AWQ_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return AWQ_OK;
}

// The search kernel's four tensor maps (out-of-bounds boxes read as zero, so
// ragged rows and token tails contribute nothing):
//   x  : fp16 copy of X [N, I], boxes of 64 channels x 128 tokens (one CTA's half of
//        a 256-token MMA tile), 128B swizzle;
//   w  : W [O, I], 128 rows x 128 bytes per box, 128B swizzle;
//   sn : scale table [2G, I] fp32, boxes of 64 channels x (s row, -1/s row);
//   qp : group parameters [G * I/gs][O][4] fp32 (3-D), boxes of 128 rows x the
//        groups one 64-column slab touches.
awq_status_t make_search_maps(awq::SearchMaps *m, const uint16_t *x16, int64_t N, const void *W,
                              bool w_bf16, int64_t O, int64_t I, const float *sn,
                              const float4 *qparam, int G, int gs) {
    if (awq_status_t s = make_map_2d(&m->x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, x16, I, N,
                                     awq::SLAB_K, awq::SUB_N / 2, CU_TENSOR_MAP_SWIZZLE_128B))
        return s;
    if (awq_status_t s = w_bf16 ? make_map_2d(&m->w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, W, I, O,
                                              64, awq::TILE_O, CU_TENSOR_MAP_SWIZZLE_128B)
                                : make_map_2d(&m->w, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, W, I, O,
                                              32, awq::TILE_O, CU_TENSOR_MAP_SWIZZLE_128B))
        return s;
    if (awq_status_t s = make_map_2d(&m->sn, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, sn, I, 2 * G,
                                     awq::SLAB_K, 2, CU_TENSOR_MAP_SWIZZLE_NONE))
        return s;
    auto enc = get_encode();
    if (!enc) return fail(AWQ_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
    const cuuint32_t gps = gs == 32 ? 2 : 1;
    cuuint64_t dims[3] = {4, static_cast<cuuint64_t>(O), static_cast<cuuint64_t>(G) * (I / gs)};
    cuuint64_t strides[2] = {16, static_cast<cuuint64_t>(O) * 16};
    cuuint32_t box[3] = {4, static_cast<cuuint32_t>(awq::TILE_O), gps};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(&m->qp, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float4 *>(qparam), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(AWQ_ERR_CUDA, "cuTensorMapEncodeTiled (qp) failed (%d)", (int)r);
    return AWQ_OK;
}

bool valid_dtype(int d) { return d == AWQ_F32 || d == AWQ_BF16; }

// Optional CUDA-event timing of the main kernels (see awq_set_kernel_timing).
constexpr int KT_KINDS = 4;
thread_local bool t_timing = false;
constexpr int KT_MAX = 64;          // launches one entry point may bracket
struct KTimer {
    cudaEvent_t beg[KT_MAX] = {}, end[KT_MAX] = {};
    int n = 0;
};
thread_local KTimer t_kt[KT_KINDS];

void kt_reset_impl(int kind) {
    KTimer &k = t_kt[kind];
    for (int i = 0; i < KT_MAX; ++i) {
        if (k.beg[i]) cudaEventDestroy(k.beg[i]);
        if (k.end[i]) cudaEventDestroy(k.end[i]);
        k.beg[i] = k.end[i] = nullptr;
    }
    k.n = 0;
}

void kt_begin_impl(int kind, cudaStream_t st) {
    if (!t_timing) return;
    KTimer &k = t_kt[kind];
    if (k.n >= KT_MAX) return;
    cudaEventCreate(&k.beg[k.n]);
    cudaEventCreate(&k.end[k.n]);
    cudaEventRecord(k.beg[k.n], st);
}

void kt_end_impl(int kind, cudaStream_t st) {
    if (!t_timing) return;
    KTimer &k = t_kt[kind];
    if (k.n >= KT_MAX || !k.end[k.n]) return;
    cudaEventRecord(k.end[k.n], st);
    ++k.n;
}

awq_status_t check_layer(const void *W, int w_dtype, int64_t out, int64_t in, int group_size,
                         int quant) {
    if (!W) return fail(AWQ_ERR_ARG, "W is NULL");
    if (!valid_dtype(w_dtype)) return fail(AWQ_ERR_ARG, "bad w_dtype %d", w_dtype);
    if (out < 1 || in < 1) return fail(AWQ_ERR_ARG, "bad shape out=%lld in=%lld", (long long)out, (long long)in);
    if (quant != AWQ_SYM && quant != AWQ_ASYM) return fail(AWQ_ERR_ARG, "bad quant %d", quant);
    if (group_size != 32 && group_size != 64 && group_size != 128)
        return fail(AWQ_ERR_UNSUPPORTED, "group_size %d not in {32, 64, 128}", group_size);
    if (in % 64 != 0) return fail(AWQ_ERR_UNSUPPORTED, "in=%lld is not a multiple of 64", (long long)in);
    if (in % group_size != 0)
        return fail(AWQ_ERR_UNSUPPORTED, "in=%lld is not a multiple of group_size %d", (long long)in, group_size);
    if (in > (1 << 20) || out > (1 << 24)) return fail(AWQ_ERR_UNSUPPORTED, "layer too large");
    if (!aligned16(W)) return fail(AWQ_ERR_ALIGN, "W not 16-byte aligned");
    return AWQ_OK;
}

}  // namespace

void awq::set_last_error(const char *msg) { g_last_error = msg ? msg : ""; }
void awq::kt_reset(int kind) { kt_reset_impl(kind); }
void awq::kt_begin(int kind, cudaStream_t st) { kt_begin_impl(kind, st); }
void awq::kt_end(int kind, cudaStream_t st) { kt_end_impl(kind, st); }

using awq::kt_begin;
using awq::kt_end;
using awq::kt_reset;

extern "C" {

int awq_version(void) { return 200; }

const char *awq_status_string(int status) {
    switch (status) {
        case AWQ_OK: return "AWQ_OK";
        case AWQ_ERR_ARG: return "AWQ_ERR_ARG";
        case AWQ_ERR_ALIGN: return "AWQ_ERR_ALIGN";
        case AWQ_ERR_UNSUPPORTED: return "AWQ_ERR_UNSUPPORTED";
        case AWQ_ERR_CUDA: return "AWQ_ERR_CUDA";
        case AWQ_ERR_TIMEOUT: return "AWQ_ERR_TIMEOUT";
        default: return "AWQ_ERR_UNKNOWN";
    }
}

const char *awq_last_error(void) { return g_last_error.c_str(); }

void awq_set_kernel_timing(int enable) {
    t_timing = enable != 0;
    for (int k = 0; k < KT_KINDS; ++k) kt_reset_impl(k);
}

double awq_last_kernel_ms(int kind) {
    if (kind < 0 || kind >= KT_KINDS) return -1.0;
    KTimer &k = t_kt[kind];
    if (k.n == 0) return -1.0;
    double total = 0.0;
    for (int i = 0; i < k.n; ++i) {
        float ms = 0.0f;
        if (cudaEventSynchronize(k.end[i]) != cudaSuccess) return -1.0;
        if (cudaEventElapsedTime(&ms, k.beg[i], k.end[i]) != cudaSuccess) return -1.0;
        total += ms;
    }
    return total;
}

awq_status_t awq_act_stats(const void *X, int x_dtype, int64_t N, int64_t in, float clamp_min,
                           float *sX, void *stream) {
    awq::NvtxRange nvtx_range("awq_act_stats");
    g_last_error.clear();
    if (!X || !sX) return fail(AWQ_ERR_ARG, "NULL pointer");
    if (!valid_dtype(x_dtype)) return fail(AWQ_ERR_ARG, "bad x_dtype %d", x_dtype);
    if (N < 1 || in < 1) return fail(AWQ_ERR_ARG, "bad shape N=%lld in=%lld", (long long)N, (long long)in);
    if (in % 8 != 0) return fail(AWQ_ERR_UNSUPPORTED, "in=%lld is not a multiple of 8", (long long)in);
    if (N > (int64_t(1) << 40)) return fail(AWQ_ERR_UNSUPPORTED, "N above 2^40");
    if (!(clamp_min >= 0.0f)) return fail(AWQ_ERR_ARG, "clamp_min must be >= 0");
    if (!aligned16(X) || !aligned16(sX)) return fail(AWQ_ERR_ALIGN, "X/sX not 16-byte aligned");
    int sms;
    if (awq_status_t s = device_info(&sms)) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int64_t n_chunks = (N + awq::STATS_CHUNK - 1) / awq::STATS_CHUNK;
    Workspace ws(st);
    if (awq_status_t s = ws.reserve(Workspace::up(sizeof(double) * n_chunks * in))) return s;
    double *part = ws.take<double>(n_chunks * in);
    kt_reset(0);
    kt_begin(0, st);
    AWQ_CUDA(awq::launch_stats_partial(X, x_dtype == AWQ_BF16, N, in, part, st));
    AWQ_CUDA(awq::launch_stats_final(part, N, in, clamp_min, sX, st));
    kt_end(0, st);
    return AWQ_OK;
}

}  // extern "C"

namespace {

// Device buffers of one search call, shared by its phases (each phase evaluates
// at most MAX_GRID grid points).
struct SearchBufs {
    uint16_t *x16;
    float *sn;
    char *sc_scratch;
    float4 *qparam;
    float *part;
    double *blocksum;
    int *flags;          // [0] best alpha, [1] best clip, [2] device error word, [3] max|X| bits, [4] X exponent
    unsigned *dw_bits;
    int *dw_exp;
};

awq_status_t reserve_search(Workspace &ws, SearchBufs *b, int64_t out, int64_t in, int64_t N,
                            int gs, int Gmax, int n_loss, double **loss_d) {
    const int64_t nG = in / gs;
    const int64_t TB = (N + awq::TILE_N - 1) / awq::TILE_N;
    size_t bytes = 0;
    bytes += Workspace::up(sizeof(uint16_t) * N * in);
    bytes += Workspace::up(sizeof(float) * 2 * Gmax * in);
    bytes += Workspace::up(awq::scale_scratch_bytes(Gmax, in));
    bytes += Workspace::up(sizeof(float4) * Gmax * out * nG);
    bytes += Workspace::up(sizeof(float) * Gmax * TB * out);
    bytes += Workspace::up(sizeof(double) * n_loss);
    bytes += Workspace::up(sizeof(double) * awq::reduce_scratch_doubles(Gmax, out));
    bytes += Workspace::up(sizeof(int) * 8);
    bytes += Workspace::up(sizeof(unsigned) * Gmax);
    bytes += Workspace::up(sizeof(int) * Gmax);
    if (awq_status_t s = ws.reserve(bytes)) return s;
    b->x16 = ws.take<uint16_t>(N * in);
    b->sn = ws.take<float>(2 * Gmax * in);
    b->sc_scratch = ws.take<char>(awq::scale_scratch_bytes(Gmax, in));
    b->qparam = ws.take<float4>(Gmax * out * nG);
    b->part = ws.take<float>(Gmax * TB * out);
    *loss_d = ws.take<double>(n_loss);
    b->blocksum = ws.take<double>(awq::reduce_scratch_doubles(Gmax, out));
    b->flags = ws.take<int>(8);
    b->dw_bits = ws.take<unsigned>(Gmax);
    b->dw_exp = ws.take<int>(Gmax);
    return AWQ_OK;
}

// One phase of the search: G <= MAX_GRID grid points, point g at
// alpha.value[g] (or alpha.value[*best_idx] for all g when best_idx is given)
// and clip ratio clip.value[g]; the losses go to loss_d[0..G) (device) and the
// optional per-row sums to loss_row[g][out].
awq_status_t search_phase(const SearchBufs &b, const void *W, bool w_bf16, int64_t out, int64_t in,
                          int64_t N, const float *sX, int gs, int wbit, bool asym,
                          const awq::GridParams &alpha, const int *best_idx,
                          const awq::GridParams &clip, int G, double *loss_d, float *loss_row,
                          int sms, cudaStream_t st) {
    const int64_t TB = (N + awq::TILE_N - 1) / awq::TILE_N;
    bool clipped = false;
    for (int g = 0; g < G; ++g) clipped |= clip.value[g] != 1.0;
    AWQ_CUDA(awq::launch_scale_table(sX, in, alpha, G, best_idx, b.sn, b.sc_scratch, st));
    AWQ_CUDA(awq::launch_group_params(W, w_bf16, out, in, gs, asym, wbit, b.sn, clip, G, b.qparam,
                                      b.dw_bits, b.dw_exp, st));
    awq::SearchArgs a{};
    a.w_bf16 = w_bf16;
    a.O = out;
    a.I = in;
    a.N = N;
    a.gs = gs;
    a.G = G;
    a.clamp = asym || clipped;
    a.part = b.part;
    a.err = b.flags + 2;
    a.wait = awq::AWQ_DEFAULT_WAIT_CYCLES;
    awq::SearchMaps maps;
    if (awq_status_t s = make_search_maps(&maps, b.x16, N, W, w_bf16, out, in, b.sn, b.qparam, G, gs))
        return s;
    kt_begin(1, st);
    AWQ_CUDA(awq::launch_search(a, maps, sms, st));
    kt_end(1, st);
    AWQ_CUDA(awq::launch_reduce_loss(b.part, G, TB, out, N, b.flags + 4, b.dw_exp, loss_d, loss_row,
                                     b.blocksum, st));
    return AWQ_OK;
}

awq_status_t device_error(int word, const char *what) {
    if (word != 0)
        return fail(AWQ_ERR_TIMEOUT, "%s: a bounded wait gave up (device error %d)", what, word);
    return AWQ_OK;
}

awq_status_t check_search_inputs(const void *W, int w_dtype, int64_t out, int64_t in, const void *X,
                                 int x_dtype, int64_t N, const float *sX, int group_size, int w_bit,
                                 int quant, const float *loss_row) {
    if (awq_status_t s = check_layer(W, w_dtype, out, in, group_size, quant)) return s;
    if (w_bit != 3 && w_bit != 4) return fail(AWQ_ERR_UNSUPPORTED, "w_bit %d (3 or 4)", w_bit);
    if (!X || !sX) return fail(AWQ_ERR_ARG, "NULL pointer");
    if (!valid_dtype(x_dtype)) return fail(AWQ_ERR_ARG, "bad x_dtype %d", x_dtype);
    if (N < 1 || N > (int64_t(1) << 30)) return fail(AWQ_ERR_ARG, "bad N=%lld", (long long)N);
    if (!aligned16(X) || !aligned16(sX) || (loss_row && !aligned16(loss_row)))
        return fail(AWQ_ERR_ALIGN, "device pointer not 16-byte aligned");
    return AWQ_OK;
}

}  // namespace

extern "C" {

awq_status_t awq_search_layer(const void *W, int w_dtype, int64_t out, int64_t in, const void *X,
                              int x_dtype, int64_t N, const float *sX, int group_size, int w_bit,
                              int quant, const double *alpha, int n_alpha, const double *clip,
                              int n_clip, double *loss, float *loss_row, int *best_alpha,
                              int *best_clip, void *stream) {
    awq::NvtxRange nvtx_range("awq_search_layer");
    g_last_error.clear();
    if (awq_status_t s = check_search_inputs(W, w_dtype, out, in, X, x_dtype, N, sX, group_size,
                                             w_bit, quant, loss_row))
        return s;
    if (!alpha || !loss || !best_alpha || !best_clip) return fail(AWQ_ERR_ARG, "NULL pointer");
    if (n_alpha < 1 || n_alpha > awq::MAX_GRID) return fail(AWQ_ERR_ARG, "n_alpha=%d", n_alpha);
    if (n_clip < 0 || n_clip > awq::MAX_GRID || (n_clip > 0 && !clip))
        return fail(AWQ_ERR_ARG, "n_clip=%d", n_clip);
    for (int k = 0; k < n_alpha; ++k)
        if (!(alpha[k] >= 0.0 && alpha[k] <= 1.0)) return fail(AWQ_ERR_ARG, "alpha[%d] out of [0,1]", k);
    for (int k = 0; k < n_clip; ++k)
        if (!(clip[k] > 0.0 && clip[k] <= 1.0)) return fail(AWQ_ERR_ARG, "clip[%d] out of (0,1]", k);
    int sms;
    if (awq_status_t s = device_info(&sms)) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);

    const int G = n_alpha > n_clip ? n_alpha : n_clip;
    const int Gtot = n_alpha + n_clip;
    const bool asym = quant == AWQ_ASYM, w_bf16 = w_dtype == AWQ_BF16;
    Workspace ws(st);
    SearchBufs b;
    double *loss_d;
    if (awq_status_t s = reserve_search(ws, &b, out, in, N, group_size, G, Gtot, &loss_d)) return s;
    AWQ_CUDA(cudaMemsetAsync(b.flags, 0, sizeof(int) * 8, st));
    AWQ_CUDA(awq::launch_x_to_f16(X, x_dtype == AWQ_BF16, N * in,
                                  reinterpret_cast<unsigned *>(b.flags + 3), b.flags + 4, b.x16, st));
    kt_reset(1);
    // Phase 1: the alpha grid (clip 1).
    awq::GridParams ap{}, cp{};
    for (int k = 0; k < n_alpha; ++k) {
        ap.value[k] = alpha[k];
        cp.value[k] = 1.0;
    }
    if (awq_status_t s = search_phase(b, W, w_bf16, out, in, N, sX, group_size, w_bit, asym, ap,
                                      nullptr, cp, n_alpha, loss_d, loss_row, sms, st))
        return s;
    AWQ_CUDA(awq::launch_argmin(loss_d, n_alpha, b.flags + 0, st));
    // Phase 2: the clip grid at alpha*.
    if (n_clip > 0) {
        awq::GridParams cp2{};
        for (int k = 0; k < n_clip; ++k) cp2.value[k] = clip[k];
        if (awq_status_t s = search_phase(
                b, W, w_bf16, out, in, N, sX, group_size, w_bit, asym, ap, b.flags + 0, cp2, n_clip,
                loss_d + n_alpha, loss_row ? loss_row + static_cast<int64_t>(n_alpha) * out : nullptr,
                sms, st))
            return s;
        AWQ_CUDA(awq::launch_argmin(loss_d + n_alpha, n_clip, b.flags + 1, st));
    }
    int hflags[4];
    AWQ_CUDA(cudaMemcpyAsync(loss, loss_d, sizeof(double) * Gtot, cudaMemcpyDeviceToHost, st));
    AWQ_CUDA(cudaMemcpyAsync(hflags, b.flags, sizeof(int) * 4, cudaMemcpyDeviceToHost, st));
    AWQ_CUDA(cudaStreamSynchronize(st));
    if (awq_status_t s = device_error(hflags[2], "search kernel")) return s;
    *best_alpha = hflags[0];
    *best_clip = n_clip > 0 ? hflags[1] : -1;
    return AWQ_OK;
}

awq_status_t awq_search_points(const void *W, int w_dtype, int64_t out, int64_t in, const void *X,
                               int x_dtype, int64_t N, const float *sX, int group_size, int w_bit,
                               int quant, const double *alpha, const double *clip, int n_points,
                               double *loss, float *loss_row, int *best, void *stream) {
    awq::NvtxRange nvtx_range("awq_search_points");
    g_last_error.clear();
    if (awq_status_t s = check_search_inputs(W, w_dtype, out, in, X, x_dtype, N, sX, group_size,
                                             w_bit, quant, loss_row))
        return s;
    if (!alpha || !clip || !loss || !best) return fail(AWQ_ERR_ARG, "NULL pointer");
    if (n_points < 1 || n_points > AWQ_MAX_POINTS) return fail(AWQ_ERR_ARG, "n_points=%d", n_points);
    for (int k = 0; k < n_points; ++k) {
        if (!(alpha[k] >= 0.0 && alpha[k] <= 1.0)) return fail(AWQ_ERR_ARG, "alpha[%d] out of [0,1]", k);
        if (!(clip[k] > 0.0 && clip[k] <= 1.0)) return fail(AWQ_ERR_ARG, "clip[%d] out of (0,1]", k);
    }
    int sms;
    if (awq_status_t s = device_info(&sms)) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int G = n_points < awq::MAX_GRID ? n_points : awq::MAX_GRID;
    const bool asym = quant == AWQ_ASYM, w_bf16 = w_dtype == AWQ_BF16;
    Workspace ws(st);
    SearchBufs b;
    double *loss_d;
    if (awq_status_t s = reserve_search(ws, &b, out, in, N, group_size, G, n_points, &loss_d)) return s;
    AWQ_CUDA(cudaMemsetAsync(b.flags, 0, sizeof(int) * 8, st));
    AWQ_CUDA(awq::launch_x_to_f16(X, x_dtype == AWQ_BF16, N * in,
                                  reinterpret_cast<unsigned *>(b.flags + 3), b.flags + 4, b.x16, st));
    kt_reset(1);
    for (int k0 = 0; k0 < n_points; k0 += awq::MAX_GRID) {
        const int g = n_points - k0 < awq::MAX_GRID ? n_points - k0 : awq::MAX_GRID;
        awq::GridParams ap{}, cp{};
        for (int k = 0; k < g; ++k) {
            ap.value[k] = alpha[k0 + k];
            cp.value[k] = clip[k0 + k];
        }
        if (awq_status_t s = search_phase(b, W, w_bf16, out, in, N, sX, group_size, w_bit, asym, ap,
                                          nullptr, cp, g, loss_d + k0,
                                          loss_row ? loss_row + static_cast<int64_t>(k0) * out : nullptr,
                                          sms, st))
            return s;
    }
    AWQ_CUDA(awq::launch_argmin(loss_d, n_points, b.flags + 0, st));
    int hflags[4];
    AWQ_CUDA(cudaMemcpyAsync(loss, loss_d, sizeof(double) * n_points, cudaMemcpyDeviceToHost, st));
    AWQ_CUDA(cudaMemcpyAsync(hflags, b.flags, sizeof(int) * 4, cudaMemcpyDeviceToHost, st));
    AWQ_CUDA(cudaStreamSynchronize(st));
    if (awq_status_t s = device_error(hflags[2], "search kernel")) return s;
    *best = hflags[0];
    return AWQ_OK;
}

awq_status_t awq_pack_quant(const void *W, int w_dtype, int64_t out, int64_t in, const float *sX,
                            double alpha, double clip, const uint8_t *clip_idx,
                            const double *clip_grid, int n_clip, int group_size, int w_bit,
                            int quant, uint32_t *qweight, uint16_t *scales, uint32_t *zeros,
                            uint16_t *s16, float *scales_f32, void *stream) {
    awq::NvtxRange nvtx_range("awq_pack_quant");
    g_last_error.clear();
    if (awq_status_t s = check_layer(W, w_dtype, out, in, group_size, quant)) return s;
    if (w_bit != 3 && w_bit != 4) return fail(AWQ_ERR_UNSUPPORTED, "w_bit %d (3 or 4)", w_bit);
    if (!sX || !qweight || !scales || !s16) return fail(AWQ_ERR_ARG, "NULL pointer");
    if (quant == AWQ_ASYM && !zeros) return fail(AWQ_ERR_ARG, "zeros required for AWQ_ASYM");
    if (quant == AWQ_SYM && zeros) return fail(AWQ_ERR_ARG, "zeros must be NULL for AWQ_SYM");
    if (!(alpha >= 0.0 && alpha <= 1.0)) return fail(AWQ_ERR_ARG, "alpha out of [0,1]");
    awq::GridParams cg{};
    if (clip_idx) {
        if (!clip_grid || n_clip < 1 || n_clip > awq::MAX_GRID)
            return fail(AWQ_ERR_ARG, "per-group clip needs a host grid of 1..%d ratios", awq::MAX_GRID);
        for (int k = 0; k < n_clip; ++k) {
            if (!(clip_grid[k] > 0.0 && clip_grid[k] <= 1.0))
                return fail(AWQ_ERR_ARG, "clip_grid[%d] out of (0,1]", k);
            cg.value[k] = clip_grid[k];
        }
    } else if (!(clip > 0.0 && clip <= 1.0)) {
        return fail(AWQ_ERR_ARG, "clip out of (0,1]");
    }
    if (!aligned16(sX) || !aligned16(qweight) || !aligned16(s16) ||
        (scales_f32 && (reinterpret_cast<uintptr_t>(scales_f32) & 3u)) ||
        (reinterpret_cast<uintptr_t>(scales) & 1u) || (zeros && (reinterpret_cast<uintptr_t>(zeros) & 3u)))
        return fail(AWQ_ERR_ALIGN, "misaligned pointer");
    int sms;
    if (awq_status_t s = device_info(&sms)) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    Workspace ws(st);
    if (awq_status_t s = ws.reserve(Workspace::up(sizeof(float) * 2 * in) +
                                    Workspace::up(awq::scale_scratch_bytes(1, in))))
        return s;
    float *sn = ws.take<float>(2 * in);   // row 0: s, row 1: -1/s
    char *sc_scratch = ws.take<char>(awq::scale_scratch_bytes(1, in));
    awq::GridParams ap{};
    ap.value[0] = alpha;
    AWQ_CUDA(awq::launch_scale_table(sX, in, ap, 1, nullptr, sn, sc_scratch, st));
    const int64_t nG = in / group_size;
    if (zeros) AWQ_CUDA(cudaMemsetAsync(zeros, 0, sizeof(uint32_t) * out * ((nG + 7) / 8), st));
    kt_reset(2);
    kt_begin(2, st);
    AWQ_CUDA(awq::launch_pack(W, w_dtype == AWQ_BF16, out, in, group_size, quant == AWQ_ASYM, w_bit,
                              clip_idx ? 1.0 : clip, clip_idx, cg, sn, qweight, scales, zeros, s16,
                              scales_f32, st));
    kt_end(2, st);
    return AWQ_OK;
}

awq_status_t awq_group_clip(const void *W, int w_dtype, int64_t out, int64_t in, const void *X,
                            int x_dtype, int64_t N, const float *sX, double alpha, int group_size,
                            int w_bit, int quant, const double *clip_grid, int n_clip,
                            uint8_t *clip_idx, float *err, void *stream) {
    awq::NvtxRange nvtx_range("awq_group_clip");
    g_last_error.clear();
    if (awq_status_t s = check_search_inputs(W, w_dtype, out, in, X, x_dtype, N, sX, group_size,
                                             w_bit, quant, err))
        return s;
    if (N > (int64_t(1) << 26)) return fail(AWQ_ERR_UNSUPPORTED, "N above 2^26 for the group clip");
    if (!clip_grid || !clip_idx) return fail(AWQ_ERR_ARG, "NULL pointer");
    if (!(alpha >= 0.0 && alpha <= 1.0)) return fail(AWQ_ERR_ARG, "alpha out of [0,1]");
    if (n_clip < 1 || n_clip > awq::MAX_GRID) return fail(AWQ_ERR_ARG, "n_clip=%d", n_clip);
    awq::GridParams cg{};
    for (int k = 0; k < n_clip; ++k) {
        if (!(clip_grid[k] > 0.0 && clip_grid[k] <= 1.0))
            return fail(AWQ_ERR_ARG, "clip_grid[%d] out of (0,1]", k);
        cg.value[k] = clip_grid[k];
    }
    int sms;
    if (awq_status_t s = device_info(&sms)) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    Workspace ws(st);
    if (awq_status_t s = ws.reserve(Workspace::up(sizeof(float) * 2 * in) +
                                    Workspace::up(awq::scale_scratch_bytes(1, in)) +
                                    Workspace::up(sizeof(double) * awq::gclip_scratch_doubles(in, group_size))))
        return s;
    float *sn = ws.take<float>(2 * in);
    char *sc_scratch = ws.take<char>(awq::scale_scratch_bytes(1, in));
    double *H = ws.take<double>(awq::gclip_scratch_doubles(in, group_size));
    awq::GridParams ap{};
    ap.value[0] = alpha;
    AWQ_CUDA(awq::launch_scale_table(sX, in, ap, 1, nullptr, sn, sc_scratch, st));
    AWQ_CUDA(awq::launch_group_clip(W, w_dtype == AWQ_BF16, out, in, X, x_dtype == AWQ_BF16, N, sn,
                                    group_size, quant == AWQ_ASYM, w_bit, cg, n_clip, H, clip_idx,
                                    err, st));
    return AWQ_OK;
}

awq_status_t awq_pack_int4(const void *W, int w_dtype, int64_t out, int64_t in, const float *sX,
                           double alpha, double clip, int group_size, int quant, uint32_t *qweight,
                           uint16_t *scales, uint32_t *zeros, uint16_t *s16, float *scales_f32,
                           void *stream) {
    awq::NvtxRange nvtx_range("awq_pack_int4");
    return awq_pack_quant(W, w_dtype, out, in, sX, alpha, clip, nullptr, nullptr, 0, group_size, 4,
                          quant, qweight, scales, zeros, s16, scales_f32, stream);
}

awq_status_t awq_linear_w4a16_batch(const awq_linear_desc_t *descs, int n, int64_t M,
                                    int group_size, void *stream) {
    awq::NvtxRange nvtx_range("awq_linear_w4a16_batch");
    g_last_error.clear();
    if (!descs) return fail(AWQ_ERR_ARG, "NULL descriptor list");
    if (n < 1 || n > AWQ_MAX_BATCH_LINEARS) return fail(AWQ_ERR_ARG, "n=%d not in [1, %d]", n, AWQ_MAX_BATCH_LINEARS);
    if (M < 1) return fail(AWQ_ERR_ARG, "bad M");
    if (group_size != 32 && group_size != 64 && group_size != 128)
        return fail(AWQ_ERR_UNSUPPORTED, "group_size %d not in {32, 64, 128}", group_size);
    const bool zeros = descs[0].zeros != nullptr;
    awq::DecBatch b{};
    b.n = n;
    for (int k = 0; k < n; ++k) {
        const awq_linear_desc_t &d = descs[k];
        if (!d.x || !d.qweight || !d.scales || !d.y) return fail(AWQ_ERR_ARG, "linear %d: NULL pointer", k);
        if (d.in < 1 || d.out < 1) return fail(AWQ_ERR_ARG, "linear %d: bad shape", k);
        if ((d.zeros != nullptr) != zeros)
            return fail(AWQ_ERR_ARG, "linear %d: zero points must be given for all linears or for none", k);
        if (d.in % 64 != 0 || d.in % group_size != 0 || d.in > 49152)
            return fail(AWQ_ERR_UNSUPPORTED, "linear %d: in=%lld", k, (long long)d.in);
        if (!aligned16(d.x) || !aligned16(d.qweight) || (reinterpret_cast<uintptr_t>(d.scales) & 1u) ||
            (d.zeros && (reinterpret_cast<uintptr_t>(d.zeros) & 3u)) || (d.s16 && !aligned16(d.s16)) ||
            (reinterpret_cast<uintptr_t>(d.y) & 1u))
            return fail(AWQ_ERR_ALIGN, "linear %d: misaligned pointer", k);
        b.lin[k] = awq::DecLinear{d.x, d.qweight, d.scales, d.zeros, d.s16, d.y, d.in, d.out};
    }
    int sms;
    if (awq_status_t s = device_info(&sms)) return s;
    if (!awq::w4a16_dec_config(b, M, group_size, zeros, sms)) {
        // outside the one-launch kernel's range (M > 8, or too wide to stage): one by one
        for (int k = 0; k < n; ++k) {
            const awq_linear_desc_t &d = descs[k];
            if (awq_status_t s = awq_linear_w4a16(d.x, M, d.in, d.out, d.qweight, d.scales, d.zeros,
                                                  d.s16, group_size, d.y, stream))
                return s;
        }
        return AWQ_OK;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    kt_reset(3);
    kt_begin(3, st);
    AWQ_CUDA(awq::launch_w4a16_dec(b, static_cast<int>(M), group_size, zeros, st));
    kt_end(3, st);
    return AWQ_OK;
}

awq_status_t awq_fold_scale(const void *P, int p_dtype, int64_t rows, int64_t cols,
                            const uint16_t *s16, void *out, void *stream) {
    awq::NvtxRange nvtx_range("awq_fold_scale");
    g_last_error.clear();
    if (!P || !s16 || !out) return fail(AWQ_ERR_ARG, "NULL pointer");
    if (!valid_dtype(p_dtype)) return fail(AWQ_ERR_ARG, "bad p_dtype %d", p_dtype);
    if (rows < 1 || cols < 1) return fail(AWQ_ERR_ARG, "bad shape rows=%lld cols=%lld", (long long)rows, (long long)cols);
    const uintptr_t am = p_dtype == AWQ_BF16 ? 1u : 3u;
    if ((reinterpret_cast<uintptr_t>(P) & am) || (reinterpret_cast<uintptr_t>(out) & am) ||
        (reinterpret_cast<uintptr_t>(s16) & 1u))
        return fail(AWQ_ERR_ALIGN, "misaligned pointer");
    int sms;
    if (awq_status_t s = device_info(&sms)) return s;
    AWQ_CUDA(awq::launch_fold_scale(P, p_dtype == AWQ_BF16, rows, cols, s16, out,
                                    static_cast<cudaStream_t>(stream)));
    return AWQ_OK;
}

awq_status_t awq_wait_selftest(int64_t limit_cycles, int arrive, void *stream) {
    awq::NvtxRange nvtx_range("awq_wait_selftest");
    g_last_error.clear();
    if (limit_cycles < 1 || limit_cycles > awq::AWQ_DEFAULT_WAIT_CYCLES)
        return fail(AWQ_ERR_ARG, "limit_cycles out of [1, %lld]", (long long)awq::AWQ_DEFAULT_WAIT_CYCLES);
    int sms;
    if (awq_status_t s = device_info(&sms)) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    Workspace ws(st);
    if (awq_status_t s = ws.reserve(Workspace::up(sizeof(int)))) return s;
    int *err = ws.take<int>(1);
    AWQ_CUDA(cudaMemsetAsync(err, 0, sizeof(int), st));
    AWQ_CUDA(awq::launch_wait_selftest(limit_cycles, arrive != 0, err, st));
    int h = 0;
    AWQ_CUDA(cudaMemcpyAsync(&h, err, sizeof(int), cudaMemcpyDeviceToHost, st));
    AWQ_CUDA(cudaStreamSynchronize(st));
    return device_error(h, "wait self-test");
}

awq_status_t awq_linear_w4a16(const uint16_t *x, int64_t M, int64_t in, int64_t out,
                              const uint32_t *qweight, const uint16_t *scales,
                              const uint32_t *zeros, const uint16_t *s16, int group_size,
                              uint16_t *y, void *stream) {
    awq::NvtxRange nvtx_range("awq_linear_w4a16");
    g_last_error.clear();
    if (!x || !qweight || !scales || !y) return fail(AWQ_ERR_ARG, "NULL pointer");
    if (M < 1 || in < 1 || out < 1) return fail(AWQ_ERR_ARG, "bad shape");
    if (group_size != 32 && group_size != 64 && group_size != 128)
        return fail(AWQ_ERR_UNSUPPORTED, "group_size %d not in {32, 64, 128}", group_size);
    if (in % 64 != 0) return fail(AWQ_ERR_UNSUPPORTED, "in=%lld is not a multiple of 64", (long long)in);
    if (in % group_size != 0)
        return fail(AWQ_ERR_UNSUPPORTED, "in=%lld is not a multiple of group_size %d", (long long)in, group_size);
    if (in > 49152) return fail(AWQ_ERR_UNSUPPORTED, "in=%lld above 49152", (long long)in);
    if (!aligned16(x) || !aligned16(qweight) || (reinterpret_cast<uintptr_t>(scales) & 1u) ||
        (zeros && (reinterpret_cast<uintptr_t>(zeros) & 3u)) || (s16 && !aligned16(s16)) ||
        (reinterpret_cast<uintptr_t>(y) & 1u))
        return fail(AWQ_ERR_ALIGN, "misaligned pointer");
    int sms;
    if (awq_status_t s = device_info(&sms)) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (M >= 2 && M <= 4 && out * in >= (int64_t(1) << 25)) {
        // 2-4 tokens on a large layer: the persistent tensor-core decode kernel
        // (measured faster there; on smaller layers, or one token, the CUDA-core
        // kernel below wins by its shorter ramp)
        awq::DecBatch b{};
        b.lin[0] = awq::DecLinear{x, qweight, scales, zeros, s16, y, in, out};
        b.n = 1;
        if (awq::w4a16_dec_config(b, M, group_size, zeros != nullptr, sms)) {
            kt_reset(3);
            kt_begin(3, st);
            AWQ_CUDA(awq::launch_w4a16_dec(b, static_cast<int>(M), group_size, zeros != nullptr, st));
            kt_end(3, st);
            return AWQ_OK;
        }
    }
    if (M <= 4) {
        // decode: CUDA-core kernels streaming the packed weights (one linear; several
        // linears at once go through awq_linear_w4a16_batch)
        kt_reset(3);
        kt_begin(3, st);
        AWQ_CUDA(awq::launch_w4a16(x, M, in, out, qweight, scales, zeros, s16, group_size, y, st));
        kt_end(3, st);
        return AWQ_OK;
    }
    if (M <= awq::W4A16_MMA_MAX_M) {
        // small batches: warp-level tensor-core kernel streaming the packed weights
        Workspace ws(st);
        const int64_t wb = awq::w4a16_mma_workspace_bytes(M, in, group_size);
        if (awq_status_t s = ws.reserve(wb)) return s;
        char *wsp = ws.take<char>(wb);
        kt_reset(3);
        kt_begin(3, st);
        AWQ_CUDA(awq::launch_w4a16_mma(x, M, in, out, qweight, scales, zeros, s16, group_size, y, wsp, st));
        kt_end(3, st);
        return AWQ_OK;
    }
    // prefill-sized M: tensor cores
    const awq::TcPlan plan = awq::w4a16_tc_plan(M, in, out, sms);
    Workspace ws(st);
    const int64_t wbytes = plan.xs_bytes + plan.part_bytes + plan.counter_bytes + plan.scale_bytes;
    if (awq_status_t s = ws.reserve(wbytes)) return s;
    char *wsp = ws.take<char>(wbytes);
    awq::TcMaps maps;
    if (awq_status_t s = make_map_2d(&maps.q, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, qweight, in / 8, out,
                                     32, 128, CU_TENSOR_MAP_SWIZZLE_128B))
        return s;
    if (awq_status_t s = make_map_2d(&maps.xs, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, wsp, in, M,
                                     awq::SLAB_K, static_cast<uint32_t>(plan.n_tile),
                                     CU_TENSOR_MAP_SWIZZLE_128B))
        return s;
    kt_reset(3);
    kt_begin(3, st);
    AWQ_CUDA(awq::launch_w4a16_tc(x, M, in, out, scales, zeros, s16, group_size, y, plan, wsp, maps,
                                  st));
    kt_end(3, st);
    return AWQ_OK;
}

}  // extern "C"
