// W4A16 linear on the tensor cores, for prefill-sized M (AWQ guide, section 三,
// QuantLinear.forward: y = (x / s) * dequant(W)^T).
//
//   xs_row_kernel:  one block per token m: xs[m] = fp16((x[m] / s16) * 2^-kx[m]),
//                   the power of two chosen from max_c |x[m, c] / s16[c]| so the
//                   token's largest magnitude lands in [2^14, 2^15), with the 8
//                   columns of each packed word stored in the order
//                   (0,4,1,5,2,6,3,7) (see below); row m of y is scaled back by
//                   sx[m] = 2^kx[m].  Further blocks give each weight row o its
//                   exponent kd[o] (below).  No reduction crosses blocks, so no
//                   memset or atomic precedes the main kernel.
//   w4a16_tc_kernel: one CTA per (128-row tile, token tile of 64, 128 or 256,
//                   K split); one K split whenever the tiles alone fill half the
//                   SMs, so most prefill shapes have no split-K partials.
//     warp 8 (TMA)  streams the packed codes, 4 slabs [128 rows x 32 words] per
//                   copy (128-byte swizzle), into a ring released by the
//                   dequantising warps;
//     warp 9 (TMA)  streams the xs tile [N tokens x 64 columns] of each 64-column
//                   slab into a ring released by the MMA;
//     warps 0-7     dequantise: warp w owns TMEM lane quadrant w % 4 (lane = row of
//                   the tile) and column half w / 4 of each slab (32 columns, 4
//                   packed words); each slab's Delta and zero word are loaded four
//                   slabs ahead; a word's nibbles e and e+4 become one fp16x2
//                   (1024 + code) with a shift and a LOP3 against the 0x6400 magic;
//                   an exact HSUB2 of (1024 + z) and an HMUL2 by Delta * 2^-kd[o]
//                   (kd[o] from the row's largest |Delta|, so the products stay
//                   normal fp16) give the pair's dequantised weights with one
//                   rounding, stored into the slab's A stage in TMEM (tcgen05.st,
//                   16 columns per thread).  Shared memory carries only the two
//                   streams: the A operand never passes through it.  The pair order
//                   (e, e+4) is why xs is permuted the same way: the contraction
//                   over K is order-independent.
//                   y[m][o] = accumulator * 2^kx[m] * 2^kd[o].
//     warp 10 (MMA) one thread issues tcgen05.mma M=128 N=tokens K=16 with A from
//                   TMEM and B (xs) from shared memory, fp16 in, fp32 accumulate in
//                   TMEM.
//     A pipeline step is two slabs: the dequantising warps unpack both, then hand
//     them over with one barrier arrival; the MMA releases both with one commit.
//     warps 0-7     epilogue: tcgen05.ld of the accumulator (two warps per lane
//                   quadrant, alternate 16-column chunks); with one K split
//                   y is written directly, otherwise each split adds its fp32
//                   partial, still unscaled (normal-range values, untouched by the
//                   atomic's flush of subnormals), into a zeroed fp32 tile with
//                   red.global.add (the order of those adds across splits is not
//                   fixed) and the last CTA of the tile (counter) applies the
//                   power-of-two scales and converts the tile to bf16.
//
// Every wait is an mbarrier wait bounded in time: on expiry the CTA raises its abort
// flag, every role stops waiting, the loaders wait (again bounded) for their copies in
// flight, the MMA thread for its MMAs, and the CTA frees its TMEM and exits without
// writing its tile.  A warp's waits have one outcome for the whole warp before its
// warp-wide TMEM instructions.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "awq_internal.h"
#include "awq_ptx.cuh"

namespace awq {

namespace {

constexpr int TC_DQ_WARPS = 8;                        // dequantisation warps: lane quadrant x column half
constexpr int TC_PF = 4;                              // group parameters fetched this many slabs ahead
constexpr int TC_WARP_QTMA = TC_DQ_WARPS;             // loads the packed codes
constexpr int TC_WARP_XTMA = TC_DQ_WARPS + 1;         // loads the activation tiles
constexpr int TC_WARP_MMA = TC_DQ_WARPS + 2;
constexpr int TC_THREADS = (TC_DQ_WARPS + 3) * 32;
constexpr int TC_TOKENS = 256;       // max tokens per tile (MMA N)
constexpr int TC_QC = 4;             // slabs per copy of packed codes (128 bytes of each row)
constexpr int QC_BYTES = 128 * TC_QC * 32;   // packed codes of a chunk: 128 rows x 32 words
constexpr int QS_MAX = 4;            // code ring stages
constexpr int XS_MAX = 8;            // activation ring stages
constexpr int AS_MAX = 8;            // A stages (TMEM)
constexpr int TC_SPS = 2;            // slabs per pipeline step (one handshake per step)
constexpr int A_COLS = TC_SPS * SLAB_K / 2;   // TMEM columns of one A stage: 128 fp16 per lane

// Power-of-two exponent k with max * 2^-k in [2^(top-1), 2^top) (0 for a zero or
// non-finite max), clamped to [-125, 125] so that 2^k and 2^-k stay normal floats.
__device__ __forceinline__ int pow2_exp(float mx, int top) {
    if (!(mx > 0.0f) || isinf(mx)) return 0;
    int e;
    frexpf(mx, &e);                                   // mx = f * 2^e, f in [0.5, 1)
    const int k = e - top;
    return k < -125 ? -125 : (k > 125 ? 125 : k);
}

// x / s16 of the 8 columns of packed word w of one token row (s16 may be null: 1).
__device__ __forceinline__ void xs_word(const uint4 *__restrict__ xr, const uint4 *__restrict__ sr, int w,
                                        float (&v)[8]) {
    const uint4 xv = __ldg(xr + w);
    const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
    uint32_t sw[4] = {0x3C003C00u, 0x3C003C00u, 0x3C003C00u, 0x3C003C00u};
    if (sr) {
        const uint4 sv = __ldg(sr + w);
        sw[0] = sv.x; sw[1] = sv.y; sw[2] = sv.z; sw[3] = sv.w;
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float x0 = __uint_as_float(xw[e] << 16), x1 = __uint_as_float(xw[e] & 0xFFFF0000u);
        const __half2 s2 = *reinterpret_cast<const __half2 *>(&sw[e]);
        v[2 * e] = sr ? __fdividef(x0, __low2float(s2)) : x0;
        v[2 * e + 1] = sr ? __fdividef(x1, __high2float(s2)) : x1;
    }
}

// Blocks [0, M): one token each (see the header), two passes over the row, the second
// from cache.  Blocks [M, gridDim.x): kd[o] for the rows of W, one warp per row at a
// time: from the row's largest |Delta| (fp16 bits of non-negative values order as
// the values), so that 15 * max |Delta| * 2^-kd < 2^15.
__global__ void __launch_bounds__(256) xs_row_kernel(const uint16_t *__restrict__ x,
                                                     const uint16_t *__restrict__ s16, int64_t M,
                                                     int64_t I, const uint16_t *__restrict__ scales,
                                                     int64_t O, int nG, uint16_t *__restrict__ xs,
                                                     float *__restrict__ sx, int *__restrict__ kd) {
    if (blockIdx.x >= M) {
        const int64_t nw = (static_cast<int64_t>(gridDim.x) - M) * (blockDim.x >> 5);
        const int lane = threadIdx.x & 31;
        for (int64_t o = (static_cast<int64_t>(blockIdx.x) - M) * (blockDim.x >> 5) + (threadIdx.x >> 5); o < O;
             o += nw) {
            uint32_t mb = 0u;
            for (int g = lane; g < nG; g += 32) {
                const uint32_t b = __ldg(scales + o * nG + g) & 0x7FFFu;
                mb = b > mb ? b : mb;
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                const uint32_t t = __shfl_xor_sync(0xffffffffu, mb, off);
                mb = t > mb ? t : mb;
            }
            if (lane == 0) kd[o] = pow2_exp(__half2float(__ushort_as_half(static_cast<unsigned short>(mb))), 11);
        }
        return;
    }
    __shared__ float wmax[8];
    const int64_t m = blockIdx.x;
    const int wpr = static_cast<int>(I / 8);
    const uint4 *xr = reinterpret_cast<const uint4 *>(x + m * I);
    const uint4 *sr = reinterpret_cast<const uint4 *>(s16);
    float mx = 0.0f;
    for (int w = threadIdx.x; w < wpr; w += blockDim.x) {
        float v[8];
        xs_word(xr, sr, w, v);
#pragma unroll
        for (int e = 0; e < 8; ++e) mx = fmaxf(mx, fabsf(v[e]));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = mx;
    __syncthreads();
    mx = wmax[0];
    for (int k = 1; k < static_cast<int>(blockDim.x >> 5); ++k) mx = fmaxf(mx, wmax[k]);
    const int k = pow2_exp(mx, 15);                   // the token's max |xs| -> [2^14, 2^15)
    const float sc = ldexpf(1.0f, -k);
    uint4 *out = reinterpret_cast<uint4 *>(xs + m * I);
    for (int w = threadIdx.x; w < wpr; w += blockDim.x) {
        float v[8];
        xs_word(xr, sr, w, v);
        uint32_t h[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {                 // position pair (2q, 2q + 1) holds columns (q, q + 4)
            const __half2 hv = __floats2half2_rn(v[q] * sc, v[q + 4] * sc);
            h[q] = *reinterpret_cast<const uint32_t *>(&hv);
        }
        out[w] = make_uint4(h[0], h[1], h[2], h[3]);
    }
    if (threadIdx.x == 0) sx[m] = ldexpf(1.0f, k);
}

struct TcArgs {
    int64_t M, I, O;
    int gs;
    int n_tile;            // tokens per tile (multiple of 16, <= 256)
    int splits;            // K splits
    int slabs_per_split;
    int as;                // A stages in TMEM (after the accumulator's columns)
    int tmem_cols;         // TMEM columns allocated
    int xs_stages;         // activation ring stages
    int q_stages;          // code ring stages
    const uint16_t *scales;
    const uint32_t *zeros;
    uint16_t *y;
    float *acc32;          // [M][O] fp32, zeroed (splits > 1)
    unsigned *counter;     // [row tiles * token tiles] (splits > 1), zeroed
    const float *sx;       // [M]: token m's xs carries 1 / sx[m] (sx[m] = 2^kx[m])
    const int *kd;         // [O]: row o's dequantised weights carry 2^-kd[o]
};

__device__ __forceinline__ uint32_t h2sub(uint32_t a, uint32_t b) {
    __half2 r = __hsub2(*reinterpret_cast<__half2 *>(&a), *reinterpret_cast<__half2 *>(&b));
    return *reinterpret_cast<uint32_t *>(&r);
}
__device__ __forceinline__ uint32_t h2mul(uint32_t a, uint32_t b) {
    __half2 r = __hmul2(*reinterpret_cast<__half2 *>(&a), *reinterpret_cast<__half2 *>(&b));
    return *reinterpret_cast<uint32_t *>(&r);
}
__device__ __forceinline__ uint32_t h2pack(float a) {
    const __half2 h = __floats2half2_rn(a, a);
    return *reinterpret_cast<const uint32_t *>(&h);
}

template <bool ZEROS>
__global__ void __launch_bounds__(TC_THREADS, 2)   // two CTAs per SM for narrow token tiles
    w4a16_tc_kernel(const __grid_constant__ TcMaps maps, const TcArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int xs_bytes = a.n_tile * 128;
    const int AS = a.as, XS = a.xs_stages, QS = a.q_stages;
    const int xstage = TC_SPS * xs_bytes;
    uint8_t *x_ring = base;                                  // XS x TC_SPS xs tiles (multiples of 2 KB)
    uint8_t *q_ring = x_ring + XS * xstage;                  // QS x codes of TC_QC slabs (1024-aligned)
    uint64_t *bars = reinterpret_cast<uint64_t *>(q_ring + QS * QC_BYTES);
    uint64_t *q_full = bars, *q_empty = bars + QS_MAX;
    uint64_t *x_full = q_empty + QS_MAX, *x_empty = x_full + XS_MAX;
    uint64_t *a_full = x_empty + XS_MAX, *a_empty = a_full + AS_MAX;
    uint64_t *acc_full = a_empty + AS_MAX, *drain = acc_full + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    volatile int *is_last = abort_flag + 1;

    const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
    const int64_t OT = (a.O + 127) / 128;
    const int64_t tile = blockIdx.x / a.splits;              // (token tile, row tile)
    const int split = static_cast<int>(blockIdx.x % a.splits);
    const int64_t ot = tile % OT, mt = tile / OT;
    const int64_t nK = a.I / SLAB_K;
    const int64_t kb0 = static_cast<int64_t>(split) * a.slabs_per_split;
    const int64_t kb1 = kb0 + a.slabs_per_split < nK ? kb0 + a.slabs_per_split : nK;
    const int nslab = static_cast<int>(kb1 > kb0 ? kb1 - kb0 : 0);
    const int nchunk = (nslab + TC_QC - 1) / TC_QC;
    const int nstep = (nslab + TC_SPS - 1) / TC_SPS;
    // accumulator: columns [0, tcols); A stage s: columns [tcols + 32 s, tcols + 32 s + 32)
    const uint32_t tcols = a.n_tile <= 32 ? 32 : (a.n_tile <= 64 ? 64 : (a.n_tile <= 128 ? 128 : 256));

    if (threadIdx.x == 0) {
        for (int s = 0; s < QS; ++s) {
            mbar_init(&q_full[s], 1);
            mbar_init(&q_empty[s], TC_DQ_WARPS);      // released once the dequantisers read the codes
        }
        for (int s = 0; s < XS; ++s) {
            mbar_init(&x_full[s], 1);
            mbar_init(&x_empty[s], 1);                // released by the MMA's commit
        }
        for (int s = 0; s < AS; ++s) {
            mbar_init(&a_full[s], TC_DQ_WARPS);
            mbar_init(&a_empty[s], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        *is_last = 0;
        fence_mbar_init();
    }
    if (warp == TC_WARP_MMA) {
        tmem_alloc(tmem_slot, static_cast<uint32_t>(a.tmem_cols));
        tmem_relinquish();
    }
    if (warp == TC_WARP_QTMA && lane == 0) tma_prefetch_desc(&maps.q);
    if (warp == TC_WARP_XTMA && lane == 0) tma_prefetch_desc(&maps.xs);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == TC_WARP_QTMA) {
        // ---- packed codes, TC_QC slabs (128 bytes of each row) per copy
        if (lane == 0) {
            int issued = 0;
            for (int c = 0; c < nchunk; ++c, ++issued) {
                const int st = c % QS;
                if (!mbar_wait(&q_empty[st], ((c / QS) & 1u) ^ 1u, abort_flag)) break;
                mbar_arrive_expect_tx(&q_full[st], QC_BYTES);
                tma_load_2d(q_ring + st * QC_BYTES, &maps.q, &q_full[st],
                            static_cast<int32_t>((kb0 + c * TC_QC) * 8), static_cast<int32_t>(ot * 128));
            }
            for (int st = 0; st < QS; ++st)          // wait (bounded) for the copies in flight
                if (issued > st) mbar_wait_drain(&q_full[st], static_cast<uint32_t>(((issued - 1 - st) / QS) & 1));
        }
        __syncwarp();
    } else if (warp == TC_WARP_XTMA) {
        // ---- the activation tiles of each step's TC_SPS slabs
        if (lane == 0) {
            int issued = 0;
            for (int t = 0; t < nstep; ++t, ++issued) {
                const int st = t % XS;
                if (!mbar_wait(&x_empty[st], ((t / XS) & 1u) ^ 1u, abort_flag)) break;
                const int cnt = nslab - t * TC_SPS < TC_SPS ? nslab - t * TC_SPS : TC_SPS;
                mbar_arrive_expect_tx(&x_full[st], static_cast<uint32_t>(cnt * xs_bytes));
                for (int u = 0; u < cnt; ++u)
                    tma_load_2d(x_ring + st * xstage + u * xs_bytes, &maps.xs, &x_full[st],
                                static_cast<int32_t>((kb0 + t * TC_SPS + u) * SLAB_K), static_cast<int32_t>(mt * a.n_tile));
            }
            for (int st = 0; st < XS; ++st)
                if (issued > st) mbar_wait_drain(&x_full[st], static_cast<uint32_t>(((issued - 1 - st) / XS) & 1));
        }
        __syncwarp();
    } else if (warp == TC_WARP_MMA) {
        if (lane == 0) {
            const uint32_t idesc = idesc_f16_f32(128, a.n_tile, false);
            const uint32_t a_base = tmem_base + tcols, x_base = smem_u32(x_ring);
            bool ok = true;
            uint32_t as = 0, as_ph = 0, xs = 0, xs_ph = 0;
            for (int t = 0; t < nstep && ok; ++t) {
                if (!mbar_wait(&a_full[as], as_ph, abort_flag) || !mbar_wait(&x_full[xs], xs_ph, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const int cnt = nslab - t * TC_SPS < TC_SPS ? nslab - t * TC_SPS : TC_SPS;
                for (int u = 0; u < cnt; ++u) {
                    const uint32_t a_addr = a_base + as * A_COLS + u * (SLAB_K / 2);
                    const uint32_t b_addr = x_base + xs * xstage + u * xs_bytes;
#pragma unroll
                    for (int k = 0; k < SLAB_K / 16; ++k)
                        umma_f16_ts(tmem_base, a_addr + k * 8, sdesc_kmajor_sw128(b_addr + k * 32), idesc,
                                    (t > 0 || u > 0 || k > 0) ? 1u : 0u);
                }
                umma_commit(&x_empty[xs]);
                umma_commit(&a_empty[as]);
                if (++as == static_cast<uint32_t>(AS)) {
                    as = 0;
                    as_ph ^= 1u;
                }
                if (++xs == static_cast<uint32_t>(XS)) {
                    xs = 0;
                    xs_ph ^= 1u;
                }
            }
            if (ok) umma_commit(acc_full);
            umma_commit(drain);
            mbar_wait_drain(drain, 0);
        }
        __syncwarp();
    } else {
        // ---- dequantisation: warp w writes TMEM lanes 32 (w % 4) .. + 31 (lane = row of
        // the tile), column half w / 4 of each slab (32 columns, 4 packed words).
        const int r = 32 * (warp & 3) + lane, hh = warp >> 2;
        const uint32_t a_lane = tmem_base + (static_cast<uint32_t>(32 * (warp & 3)) << 16) + tcols + hh * 16;
        const int64_t o = ot * 128 + r;
        const bool row_ok = o < a.O;
        const int nG = static_cast<int>(a.I / a.gs), nzw = (nG + 7) / 8;
        const int lg = a.gs == 32 ? 5 : (a.gs == 64 ? 6 : 7);          // group sizes are powers of two
        const uint16_t *srow = a.scales + (row_ok ? o : 0) * nG;
        const uint32_t *zrow = ZEROS ? a.zeros + (row_ok ? o : 0) * nzw : nullptr;
        const int col0 = static_cast<int>(kb0 * SLAB_K) + hh * 32;      // this thread's first column
        const float dscale = ldexpf(1.0f, -(row_ok ? __ldg(a.kd + o) : 0));
        // The raw scale and zero word of this thread's group in slab i, fetched TC_PF
        // slabs before use into a register ring (the slab loop is unrolled by TC_PF, so
        // each slot is a fixed register and no load result is touched early).
        auto fetch = [&](int i, uint32_t &sraw, uint32_t &zraw) {
            sraw = 0u;
            zraw = 0x88888888u;
            if (row_ok && i < nslab) {
                const int g = (col0 + i * SLAB_K) >> lg;
                sraw = __ldg(srow + g);
                if (ZEROS) zraw = __ldg(zrow + (g >> 3));
            }
        };
        uint32_t rs[TC_PF], rz[TC_PF];
#pragma unroll
        for (int u = 0; u < TC_PF; ++u) fetch(u, rs[u], rz[u]);
        static_assert(TC_PF % TC_QC == 0 && TC_QC % TC_SPS == 0, "unrolled block = whole code chunks = whole steps");
        bool ok = true;
        uint32_t as = 0, as_ph = 0;                      // A stage of the step and its phase
        uint32_t qs = 0, qs_ph = 0;                      // code ring slot of the step's chunk and its phase
        for (int i0 = 0; i0 < nslab && ok; i0 += TC_PF) {
#pragma unroll
        for (int s2 = 0; s2 < TC_PF / TC_SPS; ++s2) {
            const int ib = i0 + s2 * TC_SPS;             // the step's first slab
            if (ib >= nslab) break;
            const int cnt = nslab - ib < TC_SPS ? nslab - ib : TC_SPS;
            // (waits with one outcome per warp: the TMEM stores below are warp-wide)
            if ((s2 * TC_SPS) % TC_QC == 0 && !__all_sync(0xffffffffu, mbar_wait(&q_full[qs], qs_ph, abort_flag))) {
                ok = false;
                break;
            }
            // unpack all slabs of the step before the handshake, so their chains overlap
            uint32_t v[TC_SPS][16];
#pragma unroll
            for (int us = 0; us < TC_SPS; ++us) {
                const int u = s2 * TC_SPS + us, i = ib + us;
                // Delta * 2^-kd and (1024 + z) as fp16x2; the second is exact: OR-ing z
                // into the 0x6400 pattern of 1024 gives 1024 + z.
                const int g = (col0 + i * SLAB_K) >> lg;
                const uint32_t z = ZEROS ? (rz[u] >> (4 * (g & 7))) & 0xFu : 8u;
                const uint32_t d_cur =
                    h2pack(__half2float(__ushort_as_half(static_cast<unsigned short>(rs[u]))) * dscale);
                const uint32_t z_cur = (0x6400u | z) * 0x00010001u;
                fetch(i + TC_PF, rs[u], rz[u]);
                // the chunk holds 128-byte rows in the 128-byte swizzle: 16-byte unit w of row
                // r sits at unit w ^ (r % 8), so the 8 rows of a quarter warp hit distinct banks
                const int sub = u % TC_QC;               // slab within its code chunk
                const uint4 qw = *reinterpret_cast<const uint4 *>(
                    q_ring + qs * QC_BYTES + r * 128 + ((((sub * 2 + hh) ^ (r & 7)) & 7) << 4));
                const uint32_t wv[4] = {qw.x, qw.y, qw.z, qw.w};
#pragma unroll
                for (int wd = 0; wd < 4; ++wd) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        // nibbles e and e+4 -> fp16x2 (1024 + code) -> (code - z) * Delta * 2^-kd:
                        // TMEM column 4 wd + e of the half (K positions 2 e, 2 e + 1 of the word)
                        const uint32_t b = ((wv[wd] >> (4 * e)) & 0x000F000Fu) | 0x64006400u;
                        v[us][4 * wd + e] = h2mul(h2sub(b, z_cur), d_cur);
                    }
                }
            }
            if (((s2 + 1) * TC_SPS) % TC_QC == 0 || ib + cnt == nslab) {   // the chunk's codes are all read
                __syncwarp();
                if (lane == 0) mbar_arrive(&q_empty[qs]);
                if (++qs == static_cast<uint32_t>(QS)) {
                    qs = 0;
                    qs_ph ^= 1u;
                }
            }
            // the A stage may be overwritten once the MMAs that read it have completed
            if (!__all_sync(0xffffffffu, mbar_wait(&a_empty[as], as_ph ^ 1u, abort_flag))) {
                ok = false;
                break;
            }
            tc_fence_after();
#pragma unroll
            for (int us = 0; us < TC_SPS; ++us)
                if (us < cnt) tmem_st16(a_lane + as * A_COLS + us * (SLAB_K / 2), v[us]);
            tmem_wait_st();
            // one arrival per warp: the lanes' completed TMEM stores are ordered before
            // lane 0's arrive by the tcgen05 fence and the warp barrier
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&a_full[as]);
            if (++as == static_cast<uint32_t>(AS)) {
                as = 0;
                as_ph ^= 1u;
            }
        }
        }
        // ---- epilogue (the 8 dequantising warps): warp w reads TMEM lane quadrant w % 4
        // (lane = row of the tile) and the 16-column chunks j of the accumulator with
        // j % 2 = w / 4
        const int64_t eo = ot * 128 + 32 * (warp & 3) + lane;
        const bool erow_ok = eo < a.O;
        // y = accumulator * 2^kx[m] * 2^kd[o], two normal factors (their product can be subnormal)
        const float ysd = ldexpf(1.0f, erow_ok ? __ldg(a.kd + eo) : 0);
        named_bar_sync(1, TC_DQ_WARPS * 32);
        const bool got = ok && nslab > 0 && mbar_wait_sleep(acc_full, 0, abort_flag);
        tc_fence_after();
        const int64_t m0 = mt * a.n_tile;
        const int mcount = static_cast<int>(a.M - m0 < a.n_tile ? a.M - m0 : a.n_tile);
        const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(32 * (warp & 3)) << 16);
        if (__all_sync(0xffffffffu, got)) {
            for (int c = 16 * hh; c < a.n_tile; c += 32) {
                uint32_t rv[16];
                tmem_ld16_wait(lane_addr + static_cast<uint32_t>(c), rv);
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    const int n = c + k;
                    if (n < mcount && erow_ok) {
                        const float acc = __uint_as_float(rv[k]);
                        if (a.splits == 1) {
                            a.y[(m0 + n) * a.O + eo] =
                                __bfloat16_as_ushort(__float2bfloat16_rn((acc * __ldg(a.sx + m0 + n)) * ysd));
                        } else {
                            // split-K partials meet unscaled: they lie in the normal range,
                            // where the float atomic's flush of subnormals cannot bite
                            atomicAdd(a.acc32 + (m0 + n) * a.O + eo, acc);   // result unused: red.global.add
                        }
                    }
                }
            }
        }
        if (a.splits > 1) {
            __threadfence();
            named_bar_sync(1, TC_DQ_WARPS * 32);
            if (threadIdx.x == 0) {
                const unsigned prev = atomicAdd(&a.counter[tile], 1u);
                *is_last = prev == static_cast<unsigned>(a.splits - 1);
            }
            named_bar_sync(1, TC_DQ_WARPS * 32);
            if (*is_last) {
                __threadfence();
                if (erow_ok) {
#pragma unroll 4
                    for (int n = hh; n < mcount; n += 2)
                        a.y[(m0 + n) * a.O + eo] = __bfloat16_as_ushort(__float2bfloat16_rn(
                            (__ldcg(a.acc32 + (m0 + n) * a.O + eo) * __ldg(a.sx + m0 + n)) * ysd));
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == TC_WARP_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem_base, static_cast<uint32_t>(a.tmem_cols));
    }
}

}  // namespace

TcPlan w4a16_tc_plan(int64_t M, int64_t I, int64_t O, int num_sms) {
    TcPlan p;
    const int64_t OT = (O + 127) / 128;
    const int64_t nK = I / SLAB_K;
    // One K split when (128-row tile, token tile) pairs alone fill at least half
    // of the SMs: no split-K partial sums at all.  Among token tiles of 256, 128
    // and 64 pick the fewest waves x tile width (a 64-token tile runs the MMA at
    // about 2/3 of the wider tiles' rate: its A tile is re-read per 64 tokens).
    double best = 0.0;
    int best_n = 0;
    for (int n : {256, 128, 64}) {
        if (n > 64 && M <= n / 2) continue;                  // tile mostly empty
        const int64_t tiles = OT * ((M + n - 1) / n);
        if (tiles * 2 < num_sms) continue;
        const int64_t waves = (tiles + num_sms - 1) / num_sms;
        const double cost = static_cast<double>(waves) * n * (n == 64 ? 1.5 : 1.0);
        if (best_n == 0 || cost < best) {
            best = cost;
            best_n = n;
        }
    }
    if (best_n > 0) {
        p.n_tile = best_n < M ? best_n : static_cast<int>((M + 15) / 16 * 16);
        p.splits = 1;
        p.slabs_per_split = static_cast<int>(nK);
    } else {
        // Narrow or short layers: split K to fill the GPU; the partials meet in an
        // fp32 tile.  Wide token tiles: about one CTA per SM (the split-K adds grow
        // with the splits); narrow ones: about two per SM, for latency hiding.
        p.n_tile = static_cast<int>(M >= TC_TOKENS ? TC_TOKENS : (M + 15) / 16 * 16);
        const int64_t MT = (M + p.n_tile - 1) / p.n_tile;
        const int64_t target = M >= 128 ? num_sms : 2 * num_sms;
        int64_t splits = target / (OT * MT);          // at most one wave
        if (splits < 1) splits = 1;
        if (splits > nK) splits = nK;
        const int64_t spl = (nK + splits - 1) / splits;
        splits = (nK + spl - 1) / spl;
        p.splits = static_cast<int>(splits);
        p.slabs_per_split = static_cast<int>(spl);
    }
    const int64_t MT = (M + p.n_tile - 1) / p.n_tile;
    p.xs_bytes = (M * I * 2 + 255) / 256 * 256;
    p.part_bytes = p.splits > 1 ? (M * O * 4 + 255) / 256 * 256 : 0;
    p.counter_bytes = p.splits > 1 ? (OT * MT * 4 + 255) / 256 * 256 : 0;   // tile counters
    p.scale_bytes = ((M + O) * 4 + 255) / 256 * 256;                    // sx [M], kd [O]
    return p;
}

cudaError_t launch_w4a16_tc(const uint16_t *x, int64_t M, int64_t I, int64_t O,
                            const uint16_t *scales, const uint32_t *zeros, const uint16_t *s16,
                            int gs, uint16_t *y, const TcPlan &plan, char *workspace,
                            const TcMaps &maps, cudaStream_t st) {
    const int64_t OT = (O + 127) / 128, MT = (M + plan.n_tile - 1) / plan.n_tile;
    uint16_t *xs = reinterpret_cast<uint16_t *>(workspace);
    float *acc32 = plan.splits > 1 ? reinterpret_cast<float *>(workspace + plan.xs_bytes) : nullptr;
    unsigned *counter = reinterpret_cast<unsigned *>(workspace + plan.xs_bytes + plan.part_bytes);
    float *sx = reinterpret_cast<float *>(workspace + plan.xs_bytes + plan.part_bytes + plan.counter_bytes);
    int *kd = reinterpret_cast<int *>(sx + M);
    cudaError_t e = cudaSuccess;
    if (plan.splits > 1) {   // the fp32 accumulator tile and the tile counters start at zero
        e = cudaMemsetAsync(acc32, 0, plan.part_bytes + plan.counter_bytes, st);
        if (e != cudaSuccess) return e;
    }
    const int64_t row_blocks = (O + 7) / 8 < 148 ? (O + 7) / 8 : 148;
    xs_row_kernel<<<static_cast<unsigned>(M + row_blocks), 256, 0, st>>>(x, s16, M, I, scales, O,
                                                                          static_cast<int>(I / gs), xs, sx, kd);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    TcArgs a;
    a.M = M;
    a.I = I;
    a.O = O;
    a.gs = gs;
    a.n_tile = plan.n_tile;
    a.splits = plan.splits;
    a.slabs_per_split = plan.slabs_per_split;
    a.scales = scales;
    a.zeros = zeros;
    a.y = y;
    a.acc32 = acc32;
    a.counter = counter;
    a.sx = sx;
    a.kd = kd;
    // Token tiles of up to 64 keep two CTAs per SM (half the TMEM and 113 KB of shared
    // memory each); wider ones take the SM (all 512 TMEM columns, more than half the
    // shared memory, so no second CTA can be placed beside them).
    const int xs_b = plan.n_tile * 128;
    const int bar_bytes = (2 * QS_MAX + 2 * XS_MAX + 2 * AS_MAX + 2) * 8 + 16;
    const bool two = plan.n_tile <= 64;
    const int budget = (two ? 113 : 227) * 1024;
    const int qs = 3;
    int xsn = (budget - 1024 - bar_bytes - qs * QC_BYTES) / (TC_SPS * xs_b);
    xsn = xsn > XS_MAX ? XS_MAX : xsn;
    if (xsn < 2) return cudaErrorInvalidConfiguration;
    const int tmem_cols = two ? 256 : 512;
    const int tcols = plan.n_tile <= 32 ? 32 : (plan.n_tile <= 64 ? 64 : (plan.n_tile <= 128 ? 128 : 256));
    int as = (tmem_cols - tcols) / A_COLS;
    as = as > AS_MAX ? AS_MAX : as;
    a.as = as;
    a.tmem_cols = tmem_cols;
    a.xs_stages = xsn;
    a.q_stages = qs;
    int smem = 1024 + xsn * TC_SPS * xs_b + qs * QC_BYTES + bar_bytes;
    // (at least 80 KB: never three CTAs of 256 TMEM columns on one SM; at least
    // 120 KB: never two of 512)
    if (two && smem < 80 * 1024) smem = 80 * 1024;
    if (!two && smem < 120 * 1024) smem = 120 * 1024;
    const unsigned grid = static_cast<unsigned>(OT * MT * plan.splits);
    if (zeros) {
        e = cudaFuncSetAttribute(w4a16_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        w4a16_tc_kernel<true><<<grid, TC_THREADS, smem, st>>>(maps, a);
    } else {
        e = cudaFuncSetAttribute(w4a16_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        w4a16_tc_kernel<false><<<grid, TC_THREADS, smem, st>>>(maps, a);
    }
    return cudaGetLastError();
}

}  // namespace awq
