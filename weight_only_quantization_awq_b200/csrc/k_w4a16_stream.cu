// W4A16 linear for decode-sized M (1 to 4 tokens), bound by HBM (AWQ guide,
// section 三, QuantLinear.forward: y = (x / s) * dequant(W)^T with
// dequant(W)[o, i] = Delta[o, g(i)] * (code[o, i] - z[o, g(i)])).
//
// A CTA of 16 warps owns a contiguous range of output rows; warp w takes rows
// w, w + 16, ... of it, whole rows, so every output is finished by one warp and
// written without any cross-warp reduction.  Each lane streams the 16-byte
// groups of packed codes (32 columns) at columns lane * 32 + 1024 j of its rows
// through a ring of 8 loads in flight (with their Delta and z), so an SM keeps
// 64 KB of weight loads outstanding; the first 8 are issued before anything
// else, and the activations are prepared while they are in flight.
//
// Activations, staged once per CTA in shared memory: for every 32-column chunk
// and token, xs = (x / s) * 2^-k with k chosen so max |xs| over the chunk lies in
// [2^14, 2^15), as fp16 pairs (column e, column e + 4) of each packed word, the
// pairs e = 1, 3 divided by 16.
//
// One packed word (8 nibbles) costs one shift, four LOP3 and eight mixed
// fp16 x fp16 -> fp32 FMAs:
//   w & 0x000F000F | 0x6400_6400   -> fp16 pair (1024 + n0, 1024 + n4)
//   w & 0x00F000F0 | ...           -> (1024 + 16 n1, 1024 + 16 n5)
//   (w >> 8) & ...                 -> the same for nibbles 2, 6 and 3, 7;
// fma.rn.f32.f16 multiplies exactly and accumulates in fp32, so the chunk sum is
//   acc = sum n xs + B,  B = sum_{e = 0, 2} 1024 xs + sum_{e = 1, 3} 64 xs,
// and the chunk's contribution is Delta * 2^k * (acc - B - z * sum xs).
// The only rounding besides fp32 accumulation is xs to fp16 (relative 2^-11).
//
// Launched with programmatic stream serialisation: before griddepcontrol.wait a
// CTA only asks L2 to fetch its share of the weights (a hint that brings nothing
// into the SM, so it cannot observe data a preceding kernel is still writing)
// and lets the next kernel begin launching; every real read comes after the wait.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "awq_internal.h"
#include "awq_ptx.cuh"

namespace awq {

namespace {

constexpr int GV_WARPS = 16;
constexpr int GV_THREADS = GV_WARPS * 32;
constexpr int GV_RING = 8;                 // 16-byte code loads in flight per lane

struct GvArgs {
    const uint16_t *x;
    const uint32_t *qweight;
    const uint16_t *scales;
    const uint32_t *zeros;
    const uint16_t *s16;
    uint16_t *y;
    int64_t O;
    int M, I, gs;
    int rows_per_cta;
};

// (w & mask) | 0x64006400: an fp16 pair 1024 + (the masked nibble bits).
template <uint32_t MASK>
__device__ __forceinline__ uint32_t nib_pair(uint32_t w) {
    uint32_t r;
    asm("lop3.b32 %0, %1, %2, 0x64006400, 0xea;" : "=r"(r) : "r"(w), "n"(MASK));
    return r;
}

// a += lo(p) * lo(xv), b += hi(p) * hi(xv): fp16 operands, exact product, fp32 sum.
__device__ __forceinline__ void fma_pair(uint32_t p, uint32_t xv, float &a, float &b) {
    asm("{\n .reg .f16 p0, p1, x0, x1;\n mov.b32 {p0, p1}, %2;\n mov.b32 {x0, x1}, %3;\n"
        " fma.rn.f32.f16 %0, p0, x0, %0;\n fma.rn.f32.f16 %1, p1, x1, %1;\n}"
        : "+f"(a), "+f"(b)
        : "r"(p), "r"(xv));
}

template <int MT, bool ZEROS>
__global__ void __launch_bounds__(GV_THREADS, 1) w4a16_gemv_kernel(const GvArgs a) {
    extern __shared__ uint4 smem4[];
    const int I = a.I, nch = I / 32;                 // 32-column chunks
    const int NBL = (nch + 31) / 32;                 // chunks per lane per row
    uint4 *xh = smem4;                               // [MT][4 words][nch] fp16 pairs
    float4 *xb = reinterpret_cast<float4 *>(xh + MT * 4 * nch);   // [MT][nch] (B, sum xs, 2^k, 0)

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t row0 = static_cast<int64_t>(blockIdx.x) * a.rows_per_cta;
    const int nrows = static_cast<int>(a.O - row0 < a.rows_per_cta ? a.O - row0 : a.rows_per_cta);
    const int nG = I / a.gs;
    const int64_t nzw = (nG + 7) / 8;

    if (threadIdx.x == 0) {
        l2_prefetch_range(a.qweight + row0 * (I / 8), static_cast<uint64_t>(nrows) * (I / 2));
        l2_prefetch_range(a.scales + row0 * nG, static_cast<uint64_t>(nrows) * nG * 2);
        if (ZEROS) l2_prefetch_range(a.zeros + row0 * nzw, static_cast<uint64_t>(nrows) * nzw * 4);
    }
    griddep_launch_dependents();
    griddep_wait();

    // ---- this warp's chunk sequence: rows warp, warp + 16, ...; NBL chunks per row
    const int myrows = warp < nrows ? (nrows - warp + GV_WARPS - 1) / GV_WARPS : 0;
    const int ntot = myrows * NBL;
    uint4 q[GV_RING];
    uint32_t dz[GV_RING];                            // Delta bits | z << 16
    int ik = 0, ij = 0;                              // (row, chunk) of the next load to issue
    auto issue = [&](int s) {
        q[s] = make_uint4(0u, 0u, 0u, 0u);
        dz[s] = 0u;
        const int t = ij * 32 + lane;
        if (ik < myrows && t < nch) {
            const int64_t row = row0 + warp + static_cast<int64_t>(ik) * GV_WARPS;
            q[s] = __ldg(reinterpret_cast<const uint4 *>(a.qweight + row * (I / 8)) + t);
            const int g = t * 32 / a.gs;
            const uint32_t d = __ldg(a.scales + row * nG + g);
            const uint32_t z = ZEROS ? (__ldg(a.zeros + row * nzw + g / 8) >> (4 * (g % 8))) & 0xFu : 8u;
            dz[s] = d | (z << 16);
        }
        if (++ij == NBL) {
            ij = 0;
            ++ik;
        }
    };
#pragma unroll
    for (int s = 0; s < GV_RING; ++s) issue(s);

    // ---- activations: four threads per (token, chunk), one packed word's 8 columns each
    // (the loop bound is uniform per warp: the shuffles below need all 32 lanes)
    for (int tb = 0; tb < MT * nch * 4; tb += GV_THREADS) {
        const int task = tb + threadIdx.x;
        const bool live = task < MT * nch * 4;
        const int wd = task & 3, ch = task >> 2;
        const int m = live ? ch / nch : 0, t = live ? ch % nch : 0;
        const int c = t * 32 + wd * 8;
        uint4 xv = make_uint4(0u, 0u, 0u, 0u), sv = make_uint4(0u, 0u, 0u, 0u);
        if (live && m < a.M) {
            xv = __ldg(reinterpret_cast<const uint4 *>(a.x + static_cast<int64_t>(m) * I + c));
            sv = __ldg(reinterpret_cast<const uint4 *>(a.s16 + c));
        }
        const uint16_t *xe = reinterpret_cast<const uint16_t *>(&xv);
        const uint16_t *se = reinterpret_cast<const uint16_t *>(&sv);
        float v[8], mx = 0.0f;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            v[e] = (live && m < a.M) ? __fdividef(__uint_as_float(static_cast<uint32_t>(xe[e]) << 16),
                                        __half2float(__ushort_as_half(se[e])))
                           : 0.0f;
            mx = fmaxf(mx, fabsf(v[e]));
        }
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        int k = 0;
        if (mx > 0.0f && mx <= 3.0e38f) {
            int ex;
            frexpf(mx, &ex);
            k = ex - 15;
        }
        const float sc = ldexpf(1.0f, -k);
        uint32_t h[4];
        float L = 0.0f, B = 0.0f;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float f = (e & 1) ? 0.0625f : 1.0f;
            const __half2 p = __floats2half2_rn(v[e] * sc * f, v[e + 4] * sc * f);
            h[e] = *reinterpret_cast<const uint32_t *>(&p);
            const float s2 = __low2float(p) + __high2float(p);       // exact: two fp16 values
            L += s2 * ((e & 1) ? 16.0f : 1.0f);
            B += s2 * 1024.0f;
        }
        L += __shfl_xor_sync(0xffffffffu, L, 1);
        L += __shfl_xor_sync(0xffffffffu, L, 2);
        B += __shfl_xor_sync(0xffffffffu, B, 1);
        B += __shfl_xor_sync(0xffffffffu, B, 2);
        if (live) {
            xh[(m * 4 + wd) * nch + t] = make_uint4(h[0], h[1], h[2], h[3]);
            if (wd == 0) xb[m * nch + t] = make_float4(B, L, ldexpf(1.0f, k), 0.0f);
        }
    }
    __syncthreads();

    // ---- stream
    float acc[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[m] = 0.0f;
    int ck = 0, cj = 0;                              // (row, chunk) being consumed
    for (int base = 0; base < ntot; base += GV_RING) {
#pragma unroll
        for (int s = 0; s < GV_RING; ++s) {
            if (base + s >= ntot) break;
            const uint4 qq = q[s];
            const uint32_t dzs = dz[s];
            issue(s);                                // refill the slot 8 chunks ahead
            const int t = cj * 32 + lane;
            if (t < nch) {
                const uint32_t wv[4] = {qq.x, qq.y, qq.z, qq.w};
                float sa[MT][4];
#pragma unroll
                for (int m = 0; m < MT; ++m) sa[m][0] = sa[m][1] = sa[m][2] = sa[m][3] = 0.0f;
#pragma unroll
                for (int wd = 0; wd < 4; ++wd) {
                    const uint32_t w = wv[wd], w8 = wv[wd] >> 8;
                    const uint32_t p0 = nib_pair<0x000F000Fu>(w), p1 = nib_pair<0x00F000F0u>(w);
                    const uint32_t p2 = nib_pair<0x000F000Fu>(w8), p3 = nib_pair<0x00F000F0u>(w8);
#pragma unroll
                    for (int m = 0; m < MT; ++m) {
                        const uint4 xq = xh[(m * 4 + wd) * nch + t];
                        fma_pair(p0, xq.x, sa[m][0], sa[m][1]);
                        fma_pair(p1, xq.y, sa[m][2], sa[m][3]);
                        fma_pair(p2, xq.z, sa[m][0], sa[m][1]);
                        fma_pair(p3, xq.w, sa[m][2], sa[m][3]);
                    }
                }
                const float dv = __half2float(__ushort_as_half(static_cast<uint16_t>(dzs & 0xFFFFu)));
                const float zv = static_cast<float>(dzs >> 16);
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    const float4 bl = xb[m * nch + t];
                    const float sum = ((sa[m][0] + sa[m][1]) + (sa[m][2] + sa[m][3])) - bl.x;
                    acc[m] = fmaf(dv * bl.z, fmaf(-zv, bl.y, sum), acc[m]);
                }
            }
            if (++cj == NBL) {                       // row finished (warp-uniform)
                const int64_t row = row0 + warp + static_cast<int64_t>(ck) * GV_WARPS;
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    float v = acc[m];
#pragma unroll
                    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
                    if (lane == 0 && m < a.M)
                        a.y[static_cast<int64_t>(m) * a.O + row] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
                    acc[m] = 0.0f;
                }
                cj = 0;
                ++ck;
            }
        }
    }
}

template <int MT, bool ZEROS>
cudaError_t launch_t(const GvArgs &a, int grid, size_t smem, cudaStream_t st) {
    cudaError_t e = cudaFuncSetAttribute(w4a16_gemv_kernel<MT, ZEROS>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(GV_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, w4a16_gemv_kernel<MT, ZEROS>, a);
}

size_t gemv_smem(int64_t M, int64_t I) {
    const int MT = M == 1 ? 1 : (M == 2 ? 2 : 4);
    return static_cast<size_t>(MT) * (I / 32) * (64 + 16);
}

}  // namespace

bool w4a16_stream_supported(int64_t M, int64_t I) {
    return M >= 1 && M <= 4 && I % 64 == 0 && gemv_smem(M, I) <= 200 * 1024;
}

cudaError_t launch_w4a16_stream(const uint16_t *x, int64_t M, int64_t I, int64_t O,
                                const uint32_t *qweight, const uint16_t *scales, const uint32_t *zeros,
                                const uint16_t *s16, int gs, uint16_t *y, int num_sms, cudaStream_t st) {
    const int MT = M == 1 ? 1 : (M == 2 ? 2 : 4);
    GvArgs a;
    a.x = x;
    a.qweight = qweight;
    a.scales = scales;
    a.zeros = zeros;
    a.s16 = s16;
    a.y = y;
    a.O = O;
    a.M = static_cast<int>(M);
    a.I = static_cast<int>(I);
    a.gs = gs;
    // one CTA per SM, each a contiguous share of the rows
    int64_t rpc = (O + num_sms - 1) / num_sms;
    if (rpc < 1) rpc = 1;
    const int grid = static_cast<int>((O + rpc - 1) / rpc);
    a.rows_per_cta = static_cast<int>(rpc);
    const size_t smem = gemv_smem(M, I);
    const bool z = zeros != nullptr;
    if (MT == 1) return z ? launch_t<1, true>(a, grid, smem, st) : launch_t<1, false>(a, grid, smem, st);
    if (MT == 2) return z ? launch_t<2, true>(a, grid, smem, st) : launch_t<2, false>(a, grid, smem, st);
    return z ? launch_t<4, true>(a, grid, smem, st) : launch_t<4, false>(a, grid, smem, st);
}

}  // namespace awq
