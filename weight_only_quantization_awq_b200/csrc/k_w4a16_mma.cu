// W4A16 linear for decode-sized M (1..16 tokens) on warp-level tensor-core
// instructions (AWQ guide, section 三, QuantLinear.forward:
// y = (x / s) * dequant(W)^T).
//
// At these sizes the layer is bound by reading the packed weights from HBM;
// the instruction count per weight decides whether that bound is reached.
// Here a weight costs about one instruction: one LOP3 turns two nibbles into
// an fp16x2 pair (1024 + code) exactly, and one mma.sync.m16n8k16 consumes 256
// of them.  The zero point and the group scale are applied once per
// (row, group) after the MMA:
//     sum_i (code_i - z) * Delta * xs_i = Delta * (sum_i (1024 + code_i) * xs_i
//                                                  - (1024 + z) * sum_i xs_i).
//
//   xs_prep_kernel: xs = fp16((x / s16) * 2^-k) per (token, group), the power
//     of two putting the group's largest |x / s| in [2^14, 2^15), stored with the
//     8 columns of each packed word in the order (0,4,1,5,2,6,3,7) so a thread's
//     B fragments are consecutive words; beside it 2^k and the sum of the
//     rounded xs of the group.
//   w4a16_mma_kernel: one CTA per 16-row tile, 8 warps; warp w takes the groups
//     w, w + 8, ...  Per group a thread holds the B fragments of its token (or
//     two tokens, M > 8) for its quarter of the group's columns; per row tile it
//     loads its quarter of two rows' codes (one 16-byte load each at g = 128),
//     up to four groups ahead.  The fp32 accumulators of the 8 warps meet in
//     shared memory.  Launched with programmatic stream serialisation: the
//     first codes are requested before the dependency wait (they do not depend
//     on the preceding kernels), everything else after it.
//
// The m16n8k16 fragment layout (PTX ISA, mma.m16n8k16 with .f16 operands):
// lane = 4 g + j; A registers {row g, k 2j..2j+1}, {row g+8, k 2j..2j+1},
// {row g, k 2j+8..2j+9}, {row g+8, k 2j+8..2j+9}; B registers {k 2j..2j+1, n g},
// {k 2j+8..2j+9, n g}; D {row g, n 2j..2j+1}, {row g+8, n 2j..2j+1}.  Since the
// contraction over k is order-free, k-slot pairs are mapped to the column
// pairs (e, e+4) of a packed word, the pairs the LOP3 produces.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "awq_internal.h"
#include "awq_ptx.cuh"
#include "w4a16_frag.cuh"

namespace awq {

namespace {

constexpr int MMA_WARPS = 8;
constexpr int MMA_THREADS = MMA_WARPS * 32;
constexpr int MMA_AHEAD = 4;          // groups of codes in flight per warp

// One warp per (token, group) when gs = 128 (4 columns per lane); 2 or 4
// (token, group) pairs per warp for gs = 64 or 32, reduced over lane segments.
template <int GS>
__global__ void __launch_bounds__(256) xs_prep_kernel(const uint16_t *__restrict__ x,
                                                      const uint16_t *__restrict__ s16, int64_t M,
                                                      int64_t I, uint16_t *__restrict__ xsp,
                                                      float2 *__restrict__ xsm) {
    constexpr int LPG = GS / 4;                     // lanes per group: 32, 16 or 8
    // The main kernel may start (and read the packed codes) once every block here
    // has passed this wait, i.e. once whatever preceded this kernel on the stream
    // (possibly the kernel that wrote the codes) has completed.
    griddep_wait();
    griddep_launch_dependents();
    const int64_t nG = I / GS;
    const int64_t pair = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) / LPG;
    const int sub = threadIdx.x % LPG;
    const bool live = pair < M * nG;
    const int64_t m = live ? pair / nG : 0, g = live ? pair % nG : 0;
    float v[4];
    float mx = 0.0f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        v[e] = 0.0f;
        if (live) {
            // position p of the group -> column perm8 within its 8-column word
            const int p = sub * 4 + e;
            const int64_t c = g * GS + (p & ~7) + frag_perm8(p & 7);
            const float xv = __uint_as_float(static_cast<uint32_t>(x[m * I + c]) << 16);
            v[e] = s16 ? __fdividef(xv, __half2float(__ushort_as_half(s16[c]))) : xv;
        }
        mx = fmaxf(mx, fabsf(v[e]));
    }
#pragma unroll
    for (int off = LPG / 2; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    int k = 0;
    if (mx > 0.0f && !isinf(mx)) {
        int ex;
        frexpf(mx, &ex);
        k = ex - 15;
        k = k < -125 ? -125 : (k > 125 ? 125 : k);
    }
    const float sc = ldexpf(1.0f, -k);
    float sum = 0.0f;
    uint32_t h[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        const __half2 hv = __floats2half2_rn(v[2 * e] * sc, v[2 * e + 1] * sc);
        h[e] = *reinterpret_cast<const uint32_t *>(&hv);
        sum += __low2float(hv) + __high2float(hv);
    }
#pragma unroll
    for (int off = LPG / 2; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    if (live) {
        *reinterpret_cast<uint2 *>(xsp + m * I + g * GS + sub * 4) = make_uint2(h[0], h[1]);
        if (sub == 0) xsm[m * nG + g] = make_float2(ldexpf(1.0f, k), sum);
    }
}

template <int GS>
struct Codes {
    uint32_t r0[GS / 32], r1[GS / 32];   // rows g and g + 8: this lane's quarter of the group
};

template <int GS>
__device__ __forceinline__ void load_codes(Codes<GS> &c, const uint32_t *__restrict__ q, int64_t I,
                                           int64_t o0, int64_t O, int64_t grp, int j) {
    constexpr int NW = GS / 32;
    const int64_t col_word = (grp * GS + j * (GS / 4)) / 8;
    const int64_t wpr = I / 8;
#pragma unroll
    for (int w = 0; w < NW; ++w) c.r0[w] = c.r1[w] = 0u;
    if (o0 < O) {
        const uint32_t *p = q + o0 * wpr + col_word;
        if constexpr (NW == 4) {
            const uint4 v = __ldg(reinterpret_cast<const uint4 *>(p));
            c.r0[0] = v.x; c.r0[1] = v.y; c.r0[2] = v.z; c.r0[3] = v.w;
        } else if constexpr (NW == 2) {
            const uint2 v = __ldg(reinterpret_cast<const uint2 *>(p));
            c.r0[0] = v.x; c.r0[1] = v.y;
        } else {
            c.r0[0] = __ldg(p);
        }
    }
    if (o0 + 8 < O) {
        const uint32_t *p = q + (o0 + 8) * wpr + col_word;
        if constexpr (NW == 4) {
            const uint4 v = __ldg(reinterpret_cast<const uint4 *>(p));
            c.r1[0] = v.x; c.r1[1] = v.y; c.r1[2] = v.z; c.r1[3] = v.w;
        } else if constexpr (NW == 2) {
            const uint2 v = __ldg(reinterpret_cast<const uint2 *>(p));
            c.r1[0] = v.x; c.r1[1] = v.y;
        } else {
            c.r1[0] = __ldg(p);
        }
    }
}

template <int NT, int GS, bool ZEROS>
__global__ void __launch_bounds__(MMA_THREADS) w4a16_mma_kernel(
    const uint32_t *__restrict__ qweight, const uint16_t *__restrict__ scales,
    const uint32_t *__restrict__ zeros, const uint16_t *__restrict__ xsp,
    const float2 *__restrict__ xsm, int64_t M, int64_t I, int64_t O, uint16_t *__restrict__ y) {
    constexpr int NW = GS / 32;                  // words per lane per row per group
    __shared__ float red[MMA_WARPS][16][8 * NT];
    const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
    const int gi = lane >> 2, j = lane & 3;
    const int64_t o0 = static_cast<int64_t>(blockIdx.x) * 16 + gi;
    const int64_t nG = I / GS;
    const int64_t nzw = (nG + 7) / 8;
    const int my = nG > warp ? static_cast<int>((nG - warp + MMA_WARPS - 1) / MMA_WARPS) : 0;   // groups of this warp

    // ---- codes of the first groups: independent of the preceding kernels
    Codes<GS> ring[MMA_AHEAD];
#pragma unroll
    for (int s = 0; s < MMA_AHEAD; ++s)
        if (s < my) load_codes<GS>(ring[s], qweight, I, o0, O, warp + s * MMA_WARPS, j);
    griddep_launch_dependents();
    griddep_wait();

    float acc[NT][4];
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[t][e] = 0.0f;

    for (int it = 0; it < my; ++it) {
        const int grp = warp + it * MMA_WARPS;
        const int slot = it & (MMA_AHEAD - 1);
        Codes<GS> c;
#pragma unroll
        for (int s = 0; s < MMA_AHEAD; ++s)
            if (s == slot) c = ring[s];
        if (it + MMA_AHEAD < my) {
#pragma unroll
            for (int s = 0; s < MMA_AHEAD; ++s)
                if (s == slot) load_codes<GS>(ring[s], qweight, I, o0, O, grp + MMA_AHEAD * MMA_WARPS, j);
        }
        // Delta and (1024 + z) of rows g and g + 8 for this group
        float d0 = 0.0f, d1 = 0.0f, zb0 = 1032.0f, zb1 = 1032.0f;
        if (o0 < O) {
            d0 = __half2float(__ushort_as_half(__ldg(scales + o0 * nG + grp)));
            if (ZEROS) zb0 = 1024.0f + static_cast<float>((__ldg(zeros + o0 * nzw + (grp >> 3)) >> (4 * (grp & 7))) & 0xFu);
        }
        if (o0 + 8 < O) {
            d1 = __half2float(__ushort_as_half(__ldg(scales + (o0 + 8) * nG + grp)));
            if (ZEROS) zb1 = 1024.0f + static_cast<float>((__ldg(zeros + (o0 + 8) * nzw + (grp >> 3)) >> (4 * (grp & 7))) & 0xFu);
        }
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            // B fragments: token gi + 8 t, this lane's quarter of the group (zero past M)
            const int mb = gi + 8 * t;
            uint32_t b[GS / 8];
            if (mb < M) {
                const uint32_t *src = reinterpret_cast<const uint32_t *>(xsp + mb * I + grp * GS + j * (GS / 4));
#pragma unroll
                for (int k = 0; k < GS / 8; k += 4) {
                    const uint4 v = __ldg(reinterpret_cast<const uint4 *>(src + k));
                    b[k] = v.x; b[k + 1] = v.y; b[k + 2] = v.z; b[k + 3] = v.w;
                }
            } else {
#pragma unroll
                for (int k = 0; k < GS / 8; ++k) b[k] = 0u;
            }
            float dacc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
            for (int w = 0; w < NW; ++w) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint32_t a[4] = {frag_nib2(c.r0[w], 2 * h), frag_nib2(c.r1[w], 2 * h),
                                           frag_nib2(c.r0[w], 2 * h + 1), frag_nib2(c.r1[w], 2 * h + 1)};
                    frag_mma16816(dacc, a, b[4 * w + 2 * h], b[4 * w + 2 * h + 1]);
                }
            }
            // tokens 2j, 2j + 1 of this n8 tile: scale 2^k and the sum of xs
            float2 f0 = make_float2(0.0f, 0.0f), f1 = make_float2(0.0f, 0.0f);
            const int m0 = 8 * t + 2 * j;
            if (m0 < M) f0 = __ldg(xsm + m0 * nG + grp);
            if (m0 + 1 < M) f1 = __ldg(xsm + (m0 + 1) * nG + grp);
            acc[t][0] = __fmaf_rn(d0 * f0.x, __fmaf_rn(-zb0, f0.y, dacc[0]), acc[t][0]);
            acc[t][1] = __fmaf_rn(d0 * f1.x, __fmaf_rn(-zb0, f1.y, dacc[1]), acc[t][1]);
            acc[t][2] = __fmaf_rn(d1 * f0.x, __fmaf_rn(-zb1, f0.y, dacc[2]), acc[t][2]);
            acc[t][3] = __fmaf_rn(d1 * f1.x, __fmaf_rn(-zb1, f1.y, dacc[3]), acc[t][3]);
        }
    }
    // ---- the warps' partial sums meet in shared memory
#pragma unroll
    for (int t = 0; t < NT; ++t) {
        red[warp][gi][8 * t + 2 * j] = acc[t][0];
        red[warp][gi][8 * t + 2 * j + 1] = acc[t][1];
        red[warp][gi + 8][8 * t + 2 * j] = acc[t][2];
        red[warp][gi + 8][8 * t + 2 * j + 1] = acc[t][3];
    }
    __syncthreads();
    for (int k = threadIdx.x; k < 16 * 8 * NT; k += MMA_THREADS) {
        const int r = k % 16, m = k / 16;
        const int64_t o = static_cast<int64_t>(blockIdx.x) * 16 + r;
        if (o < O && m < M) {
            float s = 0.0f;
#pragma unroll
            for (int w = 0; w < MMA_WARPS; ++w) s += red[w][r][m];
            y[m * O + o] = __bfloat16_as_ushort(__float2bfloat16_rn(s));
        }
    }
}

template <int GS>
cudaError_t launch_prep(const uint16_t *x, const uint16_t *s16, int64_t M, int64_t I, uint16_t *xsp,
                        float2 *xsm, cudaStream_t st) {
    const int64_t pairs = M * (I / GS);
    const int64_t threads = pairs * (GS / 4);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>((threads + 255) / 256));
    cfg.blockDim = dim3(256);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, xs_prep_kernel<GS>, x, s16, M, I, xsp, xsm);
}

template <int NT, int GS, bool ZEROS>
cudaError_t launch_main(const uint32_t *qweight, const uint16_t *scales, const uint32_t *zeros,
                        const uint16_t *xsp, const float2 *xsm, int64_t M, int64_t I, int64_t O,
                        uint16_t *y, cudaStream_t st) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>((O + 15) / 16));
    cfg.blockDim = dim3(MMA_THREADS);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, w4a16_mma_kernel<NT, GS, ZEROS>, qweight, scales, zeros, xsp, xsm,
                              M, I, O, y);
}

template <int GS>
cudaError_t launch_gs(const uint16_t *x, int64_t M, int64_t I, int64_t O, const uint32_t *qweight,
                      const uint16_t *scales, const uint32_t *zeros, const uint16_t *s16,
                      uint16_t *y, uint16_t *xsp, float2 *xsm, cudaStream_t st) {
    cudaError_t e = launch_prep<GS>(x, s16, M, I, xsp, xsm, st);
    if (e != cudaSuccess) return e;
    if (M <= 8)
        return zeros ? launch_main<1, GS, true>(qweight, scales, zeros, xsp, xsm, M, I, O, y, st)
                     : launch_main<1, GS, false>(qweight, scales, zeros, xsp, xsm, M, I, O, y, st);
    return zeros ? launch_main<2, GS, true>(qweight, scales, zeros, xsp, xsm, M, I, O, y, st)
                 : launch_main<2, GS, false>(qweight, scales, zeros, xsp, xsm, M, I, O, y, st);
}

}  // namespace

int64_t w4a16_mma_workspace_bytes(int64_t M, int64_t I, int gs) {
    const int64_t xs = (M * I * 2 + 255) / 256 * 256;
    return xs + (M * (I / gs) * 8 + 255) / 256 * 256;
}

cudaError_t launch_w4a16_mma(const uint16_t *x, int64_t M, int64_t I, int64_t O,
                             const uint32_t *qweight, const uint16_t *scales, const uint32_t *zeros,
                             const uint16_t *s16, int gs, uint16_t *y, char *workspace,
                             cudaStream_t st) {
    uint16_t *xsp = reinterpret_cast<uint16_t *>(workspace);
    float2 *xsm = reinterpret_cast<float2 *>(workspace + (M * I * 2 + 255) / 256 * 256);
    if (gs == 32) return launch_gs<32>(x, M, I, O, qweight, scales, zeros, s16, y, xsp, xsm, st);
    if (gs == 64) return launch_gs<64>(x, M, I, O, qweight, scales, zeros, s16, y, xsp, xsm, st);
    return launch_gs<128>(x, M, I, O, qweight, scales, zeros, s16, y, xsp, xsm, st);
}

}  // namespace awq
