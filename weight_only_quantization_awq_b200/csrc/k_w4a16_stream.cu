// W4A16 linear for decode-sized M (1 to 4 tokens), bound by HBM (AWQ guide,
// section 三, QuantLinear.forward: y = (x / s) * dequant(W)^T with
// dequant(W)[o, i] = Delta[o, g(i)] * (code[o, i] - z[o, g(i)])).
//
// A CTA of NW warps owns a contiguous range of output rows, one CTA per SM;
// warp w takes rows w, w + NW, ... of it, whole rows, so every output is
// finished by one warp and written without any cross-warp reduction.  Each lane
// streams the 16-byte groups of packed codes (32 columns, one "chunk") at
// columns lane * 32 + 1024 j of its rows through a register ring of RING loads
// in flight, each with its Delta and zero point: NW * RING = 96 or 128 loads of
// 16 bytes per lane slot, 48 to 64 KB per SM.  The load streams advance by fixed
// pointer steps (the lane's group index moves by 1024 / gs per chunk, its zero
// nibble never moves within the word), so a load costs no index arithmetic, and
// a refill past the warp's last chunk is skipped as a whole.  The activations
// of a thread's first staging task are requested first, then the first RING
// weight loads; the activations are staged while those are in flight.
//
// Activations, staged once per CTA in shared memory, per 32-column chunk t and
// token m: xs = (x / s) * 2^-k with k chosen per (t, m) from max |xs| over the
// chunk, as four 16-byte slots of fp16 pairs (column e, column e + 4) of each
// packed word (pairs e = 1, 3 divided by 16), then one float4 slot.  A chunk's
// slots of all tokens are contiguous with an odd slot count per chunk, so the
// lanes' 16-byte loads (32 consecutive chunks) are free of bank conflicts, and
// the chunk table is padded to a multiple of 32 chunks with zeros, so a ragged
// last chunk of a row contributes exactly zero without a test.
//
// One packed word (8 nibbles) costs one shift, four LOP3 and eight mixed
// fp16 x fp16 -> fp32 FMAs:
//   w & 0x000F000F | 0x6400_6400   -> fp16 pair (1024 + n0, 1024 + n4)
//   w & 0x00F000F0 | ...           -> (1024 + 16 n1, 1024 + 16 n5)
//   (w >> 8) & ...                 -> the same for nibbles 2, 6 and 3, 7;
// fma.rn.f32.f16 multiplies exactly and accumulates in fp32 (max |xs| in
// [2^14, 2^15)), so the chunk sum is
//   acc = sum n xs + B,  B = sum_{e = 0, 2} 1024 xs + sum_{e = 1, 3} 64 xs,
// and the chunk's contribution is Delta * 2^k * (acc - B - z * sum xs) (without
// zero points z = 8 and z * sum xs is folded into B when staging).  The only
// rounding besides fp32 accumulation is xs to fp16 (relative 2^-11).
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

// 16-byte shared-memory slots per chunk: 5 per token, rounded up to an odd count.
template <int MT>
struct ChunkSlots {
    static constexpr int value = (MT * 5) % 2 ? MT * 5 : MT * 5 + 1;
};

struct GvArgs {
    const uint16_t *x;
    const uint32_t *qweight;
    const uint16_t *scales;
    const uint32_t *zeros;
    const uint16_t *s16;
    uint16_t *y;
    int64_t O;
    int M, I, lgs;                                   // lgs = log2(group size), 5..7
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

// Warps per CTA and loads in flight per lane for MT tokens per pass: more warps
// hide the FMA latency better, but four tokens need the registers of 16.
template <int MT>
struct GvShape {
    static constexpr int NW = MT <= 2 ? 32 : 16;
    static constexpr int RING = MT <= 2 ? 3 : 8;
};

template <int MT, bool ZEROS>
__global__ void __launch_bounds__(GvShape<MT>::NW * 32, 1) w4a16_gemv_kernel(const GvArgs a) {
    constexpr int S = ChunkSlots<MT>::value;
    constexpr int GV_WARPS = GvShape<MT>::NW, GV_THREADS = GV_WARPS * 32;
    constexpr int RING = GvShape<MT>::RING;
    extern __shared__ uint4 xs4[];                   // [ncp chunks][S slots]
    const int I = a.I, nch = I / 32;                 // 32-column chunks per row
    const int NBL = (nch + 31) / 32;                 // chunks per lane per row
    const int ncp = NBL * 32;                        // chunk table, padded

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t row0 = static_cast<int64_t>(blockIdx.x) * a.rows_per_cta;
    const int nrows = static_cast<int>(a.O - row0 < a.rows_per_cta ? a.O - row0 : a.rows_per_cta);
    const int nG = I >> a.lgs;
    const int nzw = (nG + 7) >> 3;

    if (threadIdx.x == 0) {
        l2_prefetch_range(a.qweight + row0 * (I / 8), static_cast<uint64_t>(nrows) * (I / 2));
        l2_prefetch_range(a.scales + row0 * nG, static_cast<uint64_t>(nrows) * nG * 2);
        if (ZEROS) l2_prefetch_range(a.zeros + row0 * nzw, static_cast<uint64_t>(nrows) * nzw * 4);
        if (a.s16) l2_prefetch_range(a.s16, static_cast<uint64_t>(I) * 2);
        l2_prefetch_range(a.x, static_cast<uint64_t>(a.M) * I * 2);
    }
    griddep_launch_dependents();
    griddep_wait();

    // ---- this warp's chunk sequence: rows warp, warp + 16, ...; NBL chunks per row.
    const int myrows = warp < nrows ? (nrows - warp + GV_WARPS - 1) / GV_WARPS : 0;
    const int ntot = myrows * NBL;
    // Lane streams: codes at 16-byte group lane + 32 j of the row, the Delta of
    // group (lane * 32 + 1024 j) / gs, and the zero word holding it.
    const int g0 = (lane * 32) >> a.lgs;
    const int gstep = 1024 >> a.lgs;                 // groups per 1024 columns
    const int64_t r0 = row0 + warp;
    const uint4 *qp = reinterpret_cast<const uint4 *>(a.qweight) + r0 * (I / 32) + lane;
    const uint16_t *sp = a.scales + r0 * nG + g0;
    const uint32_t *zp = nullptr;
    if constexpr (ZEROS) zp = a.zeros + r0 * nzw + (g0 >> 3);
    // from past a row's last chunk to the warp's next row
    const int64_t qrow = static_cast<int64_t>(GV_WARPS) * (I / 32) - NBL * 32;
    const int64_t srow = static_cast<int64_t>(GV_WARPS) * nG - NBL * gstep;
    const int64_t zrow = static_cast<int64_t>(GV_WARPS) * nzw - NBL * (gstep >> 3);
    const bool tail_ok = lane < nch - 32 * (NBL - 1);  // lane's last chunk of a row exists
    const int zsh = 4 * (g0 & 7);

    // The activations of this thread's first staging task are requested before
    // the weight loads, so they do not queue behind them.
    const int ntask = MT * ncp * 4;                  // staging tasks: (chunk, token, packed word)
    auto stage_src = [&](int task, uint4 &xv, uint4 &sv) {
        const int wd = task & 3, ch = task >> 2, t = ch / MT, m = ch % MT;
        xv = sv = make_uint4(0u, 0u, 0u, 0u);
        if (task < ntask && m < a.M && t < nch) {
            xv = __ldg(reinterpret_cast<const uint4 *>(a.x + static_cast<int64_t>(m) * I + t * 32 + wd * 8));
            // no s16: x arrives already divided by s (fp16 ones leave it unchanged)
            sv = a.s16 ? __ldg(reinterpret_cast<const uint4 *>(a.s16 + t * 32 + wd * 8))
                       : make_uint4(0x3C003C00u, 0x3C003C00u, 0x3C003C00u, 0x3C003C00u);
        }
    };
    uint4 xv0, sv0;
    stage_src(threadIdx.x, xv0, sv0);

    uint4 q[RING];
    uint32_t sd[RING];                               // Delta bits | z << 16
    int ij = 0, nis = 0;                             // chunk of the next load, loads issued
    auto issue = [&](int s) {
        q[s] = make_uint4(0u, 0u, 0u, 0u);
        sd[s] = 0u;
        if (nis < ntot && (ij < NBL - 1 || tail_ok)) {
            q[s] = __ldg(qp);
            if constexpr (ZEROS)
                sd[s] = static_cast<uint32_t>(__ldg(sp)) | (((__ldg(zp) >> zsh) & 0xFu) << 16);
            else
                sd[s] = __ldg(sp);
        }
        ++nis;
        qp += 32;
        sp += gstep;
        if constexpr (ZEROS) zp += gstep >> 3;
        if (++ij == NBL) {
            ij = 0;
            qp += qrow;
            sp += srow;
            if constexpr (ZEROS) zp += zrow;
        }
    };
#pragma unroll
    for (int s = 0; s < RING; ++s) issue(s);

    // ---- activations: four threads per (token, chunk), one packed word's 8 columns each
    // (the loop bound is uniform per warp: the shuffles below need all 32 lanes)
    constexpr int KOFF = 15;                         // max |xs| lands in [2^(KOFF-1), 2^KOFF)
    for (int tb = 0; tb < ntask; tb += GV_THREADS) {
        if (tb + warp * 32 >= ntask) break;          // no task left for this warp (warp-uniform)
        const int task = tb + threadIdx.x;
        const bool live = task < ntask;
        const int wd = task & 3, ch = task >> 2;
        const int t = live ? ch / MT : 0, m = live ? ch % MT : 0;
        const bool has = live && m < a.M && t < nch;
        uint4 xv = xv0, sv = sv0;
        if (tb > 0) stage_src(task, xv, sv);
        const uint16_t *xe = reinterpret_cast<const uint16_t *>(&xv);
        const uint16_t *se = reinterpret_cast<const uint16_t *>(&sv);
        float v[8], mx = 0.0f;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            v[e] = has ? __fdividef(__uint_as_float(static_cast<uint32_t>(xe[e]) << 16),
                                    __half2float(__ushort_as_half(se[e])))
                       : 0.0f;
            mx = fmaxf(mx, fabsf(v[e]));
        }
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        // k from the biased exponent E of max |xs| (frexp's exponent is E - 126),
        // clamped so that 2^k and 2^-k stay normal floats; 0 for a zero or
        // non-finite maximum.
        const int E = static_cast<int>(__float_as_uint(mx) >> 23);
        int k = E - 126 - KOFF;
        k = (mx > 0.0f && E < 255) ? (k < -125 ? -125 : (k > 125 ? 125 : k)) : 0;
        const float sc = __uint_as_float(static_cast<uint32_t>(127 - k) << 23);
        const float sc16 = sc * 0.0625f;
        uint32_t h[4];
        float L = 0.0f, B = 0.0f;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float f = (e & 1) ? sc16 : sc;
            const __half2 p = __floats2half2_rn(v[e] * f, v[e + 4] * f);
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
            uint4 *slot = xs4 + t * S + m * 5;
            slot[wd] = make_uint4(h[0], h[1], h[2], h[3]);
            // without zero points z = 8: fold z * sum xs into the bias
            if (wd == 0)
                slot[4] = make_uint4(__float_as_uint(ZEROS ? B : B + 8.0f * L), __float_as_uint(L),
                                     has ? static_cast<uint32_t>(127 + k) << 23 : 0u, 0u);
        }
    }
    __syncthreads();

    // ---- stream
    float acc[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[m] = 0.0f;
    int ck = 0, cj = 0;                              // (row, chunk) being consumed
    int xo = lane * S;                               // this lane's chunk in the table
    for (int base = 0; base < ntot; base += RING) {
#pragma unroll
        for (int s = 0; s < RING; ++s) {
            if (base + s >= ntot) break;
            const uint4 qq = q[s];
            const uint32_t dd = sd[s];
            if (base + s + RING < ntot) issue(s);    // refill the slot RING chunks ahead
            const uint4 *xc = xs4 + xo;
            const uint32_t wv[4] = {qq.x, qq.y, qq.z, qq.w};
            const float dv = __half2float(__ushort_as_half(static_cast<uint16_t>(dd)));
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
                    const uint4 xq = xc[m * 5 + wd];
                    fma_pair(p0, xq.x, sa[m][0], sa[m][1]);
                    fma_pair(p1, xq.y, sa[m][2], sa[m][3]);
                    fma_pair(p2, xq.z, sa[m][0], sa[m][1]);
                    fma_pair(p3, xq.w, sa[m][2], sa[m][3]);
                }
            }
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                const uint4 bl = xc[m * 5 + 4];
                float sum = ((sa[m][0] + sa[m][1]) + (sa[m][2] + sa[m][3])) - __uint_as_float(bl.x);
                if constexpr (ZEROS)
                    sum = fmaf(-static_cast<float>(dd >> 16), __uint_as_float(bl.y), sum);
                acc[m] = fmaf(dv * __uint_as_float(bl.z), sum, acc[m]);
            }
            xo += 32 * S;
            if (++cj == NBL) {                       // row finished (warp-uniform)
                const int64_t row = r0 + static_cast<int64_t>(ck) * GV_WARPS;
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    float v = acc[m];
#pragma unroll
                    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
                    if (lane == m && m < a.M)
                        a.y[static_cast<int64_t>(m) * a.O + row] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
                    acc[m] = 0.0f;
                }
                cj = 0;
                ++ck;
                xo = lane * S;
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
    cfg.blockDim = dim3(GvShape<MT>::NW * 32);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, w4a16_gemv_kernel<MT, ZEROS>, a);
}

int tokens_per_pass(int64_t M) { return M == 1 ? 1 : (M == 2 ? 2 : 4); }

size_t gemv_smem(int64_t M, int64_t I) {
    const int MT = tokens_per_pass(M);
    const int64_t ncp = ((I / 32 + 31) / 32) * 32;
    const int S = MT == 1 ? ChunkSlots<1>::value : (MT == 2 ? ChunkSlots<2>::value : ChunkSlots<4>::value);
    return static_cast<size_t>(ncp) * S * 16;
}

}  // namespace

bool w4a16_stream_supported(int64_t M, int64_t I) {
    return M >= 1 && M <= 4 && I % 64 == 0 && gemv_smem(M, I) <= 200 * 1024;
}

cudaError_t launch_w4a16_stream(const uint16_t *x, int64_t M, int64_t I, int64_t O,
                                const uint32_t *qweight, const uint16_t *scales, const uint32_t *zeros,
                                const uint16_t *s16, int gs, uint16_t *y, int num_sms, cudaStream_t st) {
    const int MT = tokens_per_pass(M);
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
    a.lgs = gs == 32 ? 5 : (gs == 64 ? 6 : 7);
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
