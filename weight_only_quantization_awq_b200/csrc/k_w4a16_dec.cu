// W4A16 decode (1..8 tokens) over one or several linear layers in one
// persistent launch (AWQ guide, section 三, QuantLinear.forward:
// y = (x / s) * dequant(W)^T).
//
// At decode sizes a layer is bound by reading its packed weights from HBM, and
// one layer of a few MB cannot keep HBM busy on its own: the ramp and tail of a
// launch cost about as much as the transfer.  So one launch takes a list of
// independent linears (e.g. the q, k, v, o, gate, up and down projections of a
// block) and streams all of them at once, one CTA per SM.
//
// Split: each CTA works on a single linear, so it stages that linear's
// activations once and never switches; the CTAs are shared out among the
// linears in proportion to their bytes, and a linear's tiles are cut into equal
// contiguous ranges among its CTAs (a few % of imbalance on a decoder block).
//
// Tiles: R = 8 k output rows, k = 45056 / (4 in) (at least 1), so a tile holds
// 32-44 KB of packed codes for the widths of a decoder block.  The R rows of
// codes are contiguous in memory and arrive with one bulk copy into a slot of a
// shared-memory ring (as many slots as fit, up to 8: 130-180 KB in flight per
// SM, what the HBM latency under full load asks for; the copy engine spends
// about a quarter of a microsecond per request whatever its size, so requests
// must be large).  The tile's fp16 scales and zero words, a few hundred bytes
// each, come through the load/store path instead: 16-byte cp.async by the
// producer's lanes, counted on the same barrier.
//
// Warp roles:
//   producer (1 warp): per tile, waits for a free slot and issues the copies
//     (the codes with an evict-first L2 hint: they are read once).
//   consumers (8 warps): warp w takes the groups w, w + 8, ... of each 16-row
//     sub-tile, so its pointers advance by constant steps and its zero point
//     always sits in nibble w of a zero word; one mma.sync.m16n8k16 covers 16
//     rows x 16 columns for the M <= 8 tokens (rows 8..15 zero when the tile has
//     only 8 rows).
//   epilogue (1 warp): sums the 8 warps' fp32 partials of a sub-tile (handed over
//     in one of 4 shared buffers) and writes each output once, in bf16, while the
//     consumers go on.
// The consumers and the epilogue warp stage the activations first, together.
//
// Unpacking (fragment layout of m16n8k16 in w4a16_frag.cuh): of a packed word w
// (8 nibbles n0..n7), with w8 = w >> 8 and P = 0x64006400,
//     (w  & 0x000F000F) | P = fp16 (1024 + n0, 1024 + n4)
//     (w  & 0x00F000F0) | P = fp16 (1024 + 16 n1, 1024 + 16 n5)
//     (w8 & 0x000F000F) | P = fp16 (1024 + n2, 1024 + n6)
//     (w8 & 0x00F000F0) | P = fp16 (1024 + 16 n3, 1024 + 16 n7),
// all exact: one shift and four LOP3 per 8 weights.  The activations of the
// pairs scaled by 16 are staged divided by 16 (a power of two: exact), so per
// (row, group) the MMA yields D = sum_i n_i xs_i + 1024 T1 with
// T1 = sum of the staged values and
//     sum_i (n_i - z) Delta xs_i = Delta (D - 1024 T1 - z T2),
// T2 = sum of the activations they stand for.  xs = fp16((x / s16) * 2^-k), k
// per (token, group) putting the group's largest |x / s| in [2^14, 2^15); the
// staging stores (2^k, 1024 T1, T2) beside it.
// Fragment order of xs: within a group, thread j (of the 4 sharing a row) owns
// the 8-column words NW j .. NW j + NW - 1 (NW = group / 32) of the codes; the
// activations of its word kk sit in the 16-byte slot 4 kk + j, so the 4 threads'
// reads of one token are one contiguous 64-byte span; within a slot the
// columns are in the order (0,4,1,5,2,6,3,7).
//
// Every wait is an mbarrier wait bounded in time: on expiry the CTA raises its
// abort flag, every role stops waiting and writing, and the producer waits (again
// bounded) for its copies in flight before the CTA exits.
//
// Launched with programmatic stream serialisation: before the dependency wait
// the producer only asks L2 for its first tile (a hint that reads nothing into
// the SM); every read of an argument, and every write, comes after the wait.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "awq_internal.h"
#include "awq_ptx.cuh"

namespace awq {

namespace {

constexpr int DEC_CWARPS = 8;                                   // consumers: warps 0..7
constexpr int DEC_EWARP = DEC_CWARPS;                           // epilogue: 8
constexpr int DEC_PWARP = DEC_EWARP + 1;                        // producer: 9
constexpr int DEC_THREADS = (DEC_PWARP + 1) * 32;
constexpr int DEC_STAGERS = (DEC_CWARPS + 1) * 32;              // threads that stage the activations
constexpr int DEC_MAX_STAGES = 8;
constexpr int DEC_RBUFS = 4;                                    // partial-sum hand-over buffers
constexpr int DEC_RED = DEC_CWARPS * 16 * 8;                    // floats per hand-over buffer
constexpr int DEC_XPAD = 32;                                    // fp16 of padding per staged token
constexpr int DEC_TILE_TARGET = 45056;                          // bytes of codes per tile, at most
// shared memory: barriers and the abort flag, the hand-over buffers, then the
// activations and the ring (offsets of both multiples of 128)
constexpr int DEC_BAR_BYTES = 256;
constexpr int DEC_ZERO_BYTES = 256;                             // zeros read by lanes past the tokens
constexpr int DEC_FIXED = DEC_BAR_BYTES + DEC_ZERO_BYTES + DEC_RBUFS * DEC_RED * 4;

// A wait taken by all 32 lanes of a warp (each observes the phase itself), with
// one outcome for the warp: if any lane gave up, all do.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
}

// Byte offsets of the arrays of a ring slot for a linear of width I (nG groups)
// and R-row tiles: codes [R][I / 2], scales [R][nG] fp16, zero words [R][nzw].
__host__ __device__ __forceinline__ int64_t dec_scales_off(int64_t I, int64_t R) { return R * (I / 2); }
__host__ __device__ __forceinline__ int64_t dec_zeros_off(int64_t I, int64_t nG, int64_t R) {
    return R * (I / 2) + R * nG * 2;
}

// ---- staging of one linear's activations by `nthreads` threads (a multiple of 32)
// into buf: xs [M][I + DEC_XPAD] fp16, then the factors [M][nG] float4.
template <int GS>
__device__ void dec_stage(const DecLinear &L, int M, uint8_t *buf, int tid, int nthreads) {
    constexpr int WPG = GS / 8;            // 8-column words per group: consecutive lanes
    constexpr int NW = GS / 32;            // words per fragment thread
    constexpr int U = 8;                   // words in flight per thread
    const int I = static_cast<int>(L.I), nG = I / GS, wpr = I / 8, IP = I + DEC_XPAD;
    uint16_t *xs = reinterpret_cast<uint16_t *>(buf);
    float4 *xf = reinterpret_cast<float4 *>(buf + M * IP * 2);
    const int total = M * wpr;             // (token, word) items; a group's items are consecutive
    const uint4 *xg = reinterpret_cast<const uint4 *>(L.x);
    const uint4 *sg = reinterpret_cast<const uint4 *>(L.s16);
    for (int base = 0; base < total; base += nthreads * U) {
        uint4 xv[U], sv[U];
#pragma unroll
        for (int k = 0; k < U; ++k) {
            const int it = base + k * nthreads + tid;
            xv[k] = make_uint4(0u, 0u, 0u, 0u);
            sv[k] = make_uint4(0x3C003C00u, 0x3C003C00u, 0x3C003C00u, 0x3C003C00u);   // fp16 1.0
            if (it < total) {
                xv[k] = __ldcg(xg + it);
                if (sg) sv[k] = __ldcg(sg + (it % wpr));
            }
        }
#pragma unroll
        for (int k = 0; k < U; ++k) {
            const int it = base + k * nthreads + tid;
            const uint32_t xw[4] = {xv[k].x, xv[k].y, xv[k].z, xv[k].w};
            const uint32_t sw[4] = {sv[k].x, sv[k].y, sv[k].z, sv[k].w};
            float v[8];
            float mx = 0.0f;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float x0 = __uint_as_float(xw[e] << 16), x1 = __uint_as_float(xw[e] & 0xFFFF0000u);
                const __half2 s2 = *reinterpret_cast<const __half2 *>(&sw[e]);
                v[2 * e] = sg ? __fdividef(x0, __low2float(s2)) : x0;
                v[2 * e + 1] = sg ? __fdividef(x1, __high2float(s2)) : x1;
                mx = fmaxf(mx, fmaxf(fabsf(v[2 * e]), fabsf(v[2 * e + 1])));
            }
#pragma unroll
            for (int off = WPG / 2; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
            int kx = 0;
            if (mx > 0.0f && !isinf(mx)) {
                int ex;
                frexpf(mx, &ex);
                kx = ex - 15;
                kx = kx < -125 ? -125 : (kx > 125 ? 125 : kx);
            }
            const float sc = ldexpf(1.0f, -kx);
            uint32_t h[4];
            float t1 = 0.0f, t2 = 0.0f;
#pragma unroll
            for (int q = 0; q < 4; ++q) {   // word q of the slot: columns (q, q + 4); odd q divided by 16
                const float f = (q & 1) ? sc * 0.0625f : sc;
                const __half2 hv = __floats2half2_rn(v[q] * f, v[q + 4] * f);
                h[q] = *reinterpret_cast<const uint32_t *>(&hv);
                const float p = __low2float(hv) + __high2float(hv);
                t1 += p;
                t2 += (q & 1) ? 16.0f * p : p;
            }
#pragma unroll
            for (int off = WPG / 2; off > 0; off >>= 1) {
                t1 += __shfl_xor_sync(0xffffffffu, t1, off);
                t2 += __shfl_xor_sync(0xffffffffu, t2, off);
            }
            if (it < total) {
                const int m = it / wpr, w = it - m * wpr;
                const int g = w / WPG, wg = w - g * WPG;
                const int slot = (wg % NW) * 4 + wg / NW;
                *reinterpret_cast<uint4 *>(xs + m * IP + g * GS + slot * 8) = make_uint4(h[0], h[1], h[2], h[3]);
                if (wg == 0) xf[m * nG + g] = make_float4(ldexpf(1.0f, kx), 1024.0f * t1, t2, 0.0f);
            }
        }
    }
}

// The two MMAs of one packed word per row: wl is row g's word, wh row g + 8's.
// The unpacked fp16 pairs (above; LOP3 table 0xEA is (a & b) | c) go straight
// into the A registers of mma.sync.m16n8k16 (rows g, g + 8; k-slot pairs
// (e0, e1) for the first MMA, (e2, e3) for the second), so no register has to
// be moved into place; (b0, b1) and (b2, b3) are the matching B registers.
__device__ __forceinline__ void dec_word_mma(float (&d)[4], uint32_t wl, uint32_t wh, uint32_t b0, uint32_t b1,
                                             uint32_t b2, uint32_t b3) {
    asm volatile(
        "{\n\t.reg .b32 a0, a1, a2, a3, s0, s1;\n\t"
        "shr.b32 s0, %4, 8;\n\t"
        "shr.b32 s1, %5, 8;\n\t"
        "lop3.b32 a0, %4, 0x000F000F, 0x64006400, 0xEA;\n\t"
        "lop3.b32 a1, %5, 0x000F000F, 0x64006400, 0xEA;\n\t"
        "lop3.b32 a2, %4, 0x00F000F0, 0x64006400, 0xEA;\n\t"
        "lop3.b32 a3, %5, 0x00F000F0, 0x64006400, 0xEA;\n\t"
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {a0, a1, a2, a3}, {%6, %7}, "
        "{%0, %1, %2, %3};\n\t"
        "lop3.b32 a0, s0, 0x000F000F, 0x64006400, 0xEA;\n\t"
        "lop3.b32 a1, s1, 0x000F000F, 0x64006400, 0xEA;\n\t"
        "lop3.b32 a2, s0, 0x00F000F0, 0x64006400, 0xEA;\n\t"
        "lop3.b32 a3, s1, 0x00F000F0, 0x64006400, 0xEA;\n\t"
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {a0, a1, a2, a3}, {%8, %9}, "
        "{%0, %1, %2, %3};\n\t"
        "}"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(wl), "r"(wh), "r"(b0), "r"(b1), "r"(b2), "r"(b3));
}

// One 16-row sub-tile (rows 8..15 present when HI) of one consumer warp: its
// groups w, w + 8, ...; every pointer advances by a constant step per group.
// Lanes past the tokens read zeros with a zero step (bstep, fstep0, fstep1), so
// the loop has no test besides its own.
template <int GS, bool ZEROS, bool HI>
__device__ __forceinline__ void dec_subtile(float (&acc)[4], const uint8_t *ap, int arow, const uint16_t *hs,
                                            int hrow, const uint32_t *hz, int zrow, const uint8_t *bp,
                                            int bstep, const float4 *f0p, int fstep0, const float4 *f1p,
                                            int fstep1, int nG, int warp) {
    constexpr int NW = GS / 32;
    const int sh = 4 * (warp & 7);
#pragma unroll 2
    for (int grp = warp; grp < nG; grp += DEC_CWARPS) {
        uint32_t c0[NW], c1[NW];
        if constexpr (NW == 4) {
            const uint4 v = *reinterpret_cast<const uint4 *>(ap);
            c0[0] = v.x; c0[1] = v.y; c0[2] = v.z; c0[3] = v.w;
            if constexpr (HI) {
                const uint4 u = *reinterpret_cast<const uint4 *>(ap + arow);
                c1[0] = u.x; c1[1] = u.y; c1[2] = u.z; c1[3] = u.w;
            }
        } else if constexpr (NW == 2) {
            const uint2 v = *reinterpret_cast<const uint2 *>(ap);
            c0[0] = v.x; c0[1] = v.y;
            if constexpr (HI) {
                const uint2 u = *reinterpret_cast<const uint2 *>(ap + arow);
                c1[0] = u.x; c1[1] = u.y;
            }
        } else {
            c0[0] = *reinterpret_cast<const uint32_t *>(ap);
            if constexpr (HI) c1[0] = *reinterpret_cast<const uint32_t *>(ap + arow);
        }
        uint32_t bw[4 * NW];
#pragma unroll
        for (int kk = 0; kk < NW; ++kk) {
            const uint4 v = *reinterpret_cast<const uint4 *>(bp + kk * 64);
            bw[4 * kk] = v.x; bw[4 * kk + 1] = v.y; bw[4 * kk + 2] = v.z; bw[4 * kk + 3] = v.w;
        }
        const float4 f0 = *f0p, f1 = *f1p;
        const float dlo = __half2float(__ushort_as_half(hs[0]));
        float zlo = 8.0f, zhi = 8.0f, dhi = 0.0f;
        if constexpr (HI) dhi = __half2float(__ushort_as_half(hs[hrow]));
        if constexpr (ZEROS) {
            zlo = static_cast<float>((hz[grp >> 3] >> sh) & 0xFu);
            if constexpr (HI) zhi = static_cast<float>((hz[zrow + (grp >> 3)] >> sh) & 0xFu);
        }
        // two independent MMA chains (first and second half of the group's k)
        float da[4] = {0.0f, 0.0f, 0.0f, 0.0f}, db[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int kk = 0; kk < NW; ++kk) {
            // (rows 8..15 of an 8-row tile: any code, their results are dropped)
            const uint32_t wh = HI ? c1[kk] : 0x88888888u;
            if (2 * kk < NW)
                dec_word_mma(da, c0[kk], wh, bw[4 * kk], bw[4 * kk + 1], bw[4 * kk + 2], bw[4 * kk + 3]);
            else
                dec_word_mma(db, c0[kk], wh, bw[4 * kk], bw[4 * kk + 1], bw[4 * kk + 2], bw[4 * kk + 3]);
        }
        acc[0] = __fmaf_rn(dlo * f0.x, __fmaf_rn(-zlo, f0.z, (da[0] + db[0]) - f0.y), acc[0]);
        acc[1] = __fmaf_rn(dlo * f1.x, __fmaf_rn(-zlo, f1.z, (da[1] + db[1]) - f1.y), acc[1]);
        if constexpr (HI) {
            acc[2] = __fmaf_rn(dhi * f0.x, __fmaf_rn(-zhi, f0.z, (da[2] + db[2]) - f0.y), acc[2]);
            acc[3] = __fmaf_rn(dhi * f1.x, __fmaf_rn(-zhi, f1.z, (da[3] + db[3]) - f1.y), acc[3]);
        }
        ap += DEC_CWARPS * (GS / 2);
        hs += DEC_CWARPS;
        bp += bstep;
        f0p += fstep0;
        f1p += fstep1;
    }
}

template <int GS, bool ZEROS>
__global__ void __launch_bounds__(DEC_THREADS, 1) w4a16_dec_kernel(const __grid_constant__ DecBatch b, int M) {
    constexpr int NW = GS / 32;
    extern __shared__ __align__(128) uint8_t dsm[];
    uint64_t *full = reinterpret_cast<uint64_t *>(dsm);
    uint64_t *empty = full + DEC_MAX_STAGES;
    uint64_t *rfull = empty + DEC_MAX_STAGES, *rempty = rfull + DEC_RBUFS;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(rempty + DEC_RBUFS);
    const uint8_t *zero = dsm + DEC_BAR_BYTES;                               // DEC_ZERO_BYTES of zeros
    float *red = reinterpret_cast<float *>(dsm + DEC_BAR_BYTES + DEC_ZERO_BYTES);   // [4][warps][16 rows][8]
    uint8_t *xbuf = dsm + DEC_FIXED;

    // ---- this CTA's linear and tile range
    int l = 0;
    while (l + 1 < b.n && static_cast<int>(blockIdx.x) >= b.cta0[l + 1]) ++l;
    const DecLinear &L = b.lin[l];
    const int R = b.rows[l], S = b.stages[l], SB = b.slot_bytes[l];
    uint8_t *ring = xbuf + b.xbuf_bytes[l];
    const int I = static_cast<int>(L.I), nG = I / GS, nzw = (nG + 7) >> 3, IP = I + DEC_XPAD;
    const int64_t O = L.O, T = (O + R - 1) / R;
    const int64_t cl = b.cta0[l + 1] - b.cta0[l], ci = static_cast<int64_t>(blockIdx.x) - b.cta0[l];
    const int64_t t0 = ci * T / cl, t1 = (ci + 1) * T / cl;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int k = 0; k < S; ++k) {
            mbar_init(&full[k], 1 + 32);   // the code copy's expect_tx and one per producer lane
            mbar_init(&empty[k], DEC_CWARPS);
        }
        for (int k = 0; k < DEC_RBUFS; ++k) {
            mbar_init(&rfull[k], DEC_CWARPS);
            mbar_init(&rempty[k], 1);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (threadIdx.x < DEC_ZERO_BYTES / 4) reinterpret_cast<uint32_t *>(dsm + DEC_BAR_BYTES)[threadIdx.x] = 0u;
    __syncthreads();

    if (warp == DEC_PWARP && lane == 0 && t0 < t1) {
        const int64_t o0 = t0 * R;
        const int64_t rows = O - o0 < R ? O - o0 : R;
        l2_prefetch_range(L.qweight + o0 * (I / 8), static_cast<uint64_t>(rows) * (I / 2));
    }
    griddep_launch_dependents();
    griddep_wait();
    if (t0 >= t1) return;

    if (warp == DEC_PWARP) {
        // ------------------------------------------------------------ producer
        const uint64_t pol = l2_policy_evict_first();
        int sc = 0;
        for (int64_t t = t0; t < t1; ++t, ++sc) {
            const int64_t o0 = t * R;
            const int rows = O - o0 < R ? static_cast<int>(O - o0) : R;
            const int slot = sc % S;
            if (!warp_wait(&empty[slot], ((sc / S) & 1) ^ 1, abort_flag)) break;
            uint8_t *sp = ring + slot * SB;
            const uint16_t *ssrc = L.scales + o0 * nG;
            const uint32_t *zsrc = ZEROS ? L.zeros + o0 * nzw : nullptr;
            const uint32_t cbytes = static_cast<uint32_t>(rows * (I / 2));
            const uint32_t sbytes = static_cast<uint32_t>(rows * nG * 2);
            const uint32_t zbytes = ZEROS ? static_cast<uint32_t>(rows * nzw * 4) : 0u;
            const bool vec = (sbytes % 16 == 0) && (reinterpret_cast<uintptr_t>(ssrc) % 16 == 0) &&
                             (!ZEROS || ((zbytes % 16 == 0) && (reinterpret_cast<uintptr_t>(zsrc) % 16 == 0)));
            if (lane == 0) {
                mbar_arrive_expect_tx(&full[slot], cbytes);
                bulk_load(sp, L.qweight + o0 * (I / 8), cbytes, &full[slot], pol);
            }
            // the header: one arrival per lane on the same barrier, after this lane's part
            if (vec) {
                const uint8_t *ss = reinterpret_cast<const uint8_t *>(ssrc);
                for (uint32_t i = 16u * lane; i < sbytes; i += 512u) cp_async16(sp + dec_scales_off(I, R) + i, ss + i);
                if (ZEROS) {
                    const uint8_t *zs = reinterpret_cast<const uint8_t *>(zsrc);
                    for (uint32_t i = 16u * lane; i < zbytes; i += 512u)
                        cp_async16(sp + dec_zeros_off(I, nG, R) + i, zs + i);
                }
                cp_async_arrive_noinc(&full[slot]);
            } else {
                // a ragged or unaligned header: plain loads, then a plain (releasing) arrival
                uint16_t *hs = reinterpret_cast<uint16_t *>(sp + dec_scales_off(I, R));
                for (int i = lane; i < rows * nG; i += 32) hs[i] = __ldcg(ssrc + i);
                if (ZEROS) {
                    uint32_t *hz = reinterpret_cast<uint32_t *>(sp + dec_zeros_off(I, nG, R));
                    for (int i = lane; i < rows * nzw; i += 32) hz[i] = __ldcg(zsrc + i);
                }
                mbar_arrive(&full[slot]);
            }
        }
        // wait (bounded) for every copy still in flight before the CTA may exit
        for (int k = 0; k < S; ++k)
            if (sc > k) mbar_wait_drain(&full[k], static_cast<uint32_t>(((sc - 1 - k) / S) & 1));
        return;
    }

    // ---- the activations, staged once by the consumers and the epilogue warp
    dec_stage<GS>(L, M, xbuf, threadIdx.x, DEC_STAGERS);
    named_bar_sync(1, DEC_STAGERS);

    if (warp == DEC_EWARP) {
        // ------------------------------------------------------------ epilogue
        int tc = 0;
        bool ok = true;
        for (int64_t t = t0; t < t1 && ok; ++t) {
            for (int64_t o0 = t * R; o0 < (t + 1) * R && o0 < O; o0 += 16, ++tc) {
                const int r = tc % DEC_RBUFS;
                if (!warp_wait(&rfull[r], (tc / DEC_RBUFS) & 1, abort_flag)) { ok = false; break; }
                const float *rd = red + r * DEC_RED;
                for (int idx = lane; idx < 16 * M; idx += 32) {
                    const int row = idx & 15, m = idx >> 4;
                    if (o0 + row < O && o0 + row < (t + 1) * R) {
                        float sum = 0.0f;
#pragma unroll
                        for (int w = 0; w < DEC_CWARPS; ++w) sum += rd[(w * 16 + row) * 8 + m];
                        L.y[m * O + o0 + row] = __bfloat16_as_ushort(__float2bfloat16_rn(sum));
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&rempty[r]);
            }
        }
        return;
    }

    // ------------------------------------------------------------------ consumers
    const int gi = lane >> 2, j = lane & 3;
    // per-lane activation and factor streams; lanes past the M tokens read zeros
    const float4 *fx = reinterpret_cast<const float4 *>(xbuf + M * IP * 2);
    const uint8_t *bbase = gi < M ? xbuf + (gi * IP + warp * GS) * 2 + j * 16 : zero;
    const int bstep = gi < M ? DEC_CWARPS * GS * 2 : 0;
    const float4 *f0base = 2 * j < M ? fx + 2 * j * nG + warp : reinterpret_cast<const float4 *>(zero);
    const float4 *f1base = 2 * j + 1 < M ? fx + (2 * j + 1) * nG + warp : reinterpret_cast<const float4 *>(zero);
    const int fstep0 = 2 * j < M ? DEC_CWARPS : 0, fstep1 = 2 * j + 1 < M ? DEC_CWARPS : 0;
    int sc = 0, tc = 0;
    bool ok = true;
    for (int64_t t = t0; t < t1; ++t, ++sc) {
        const int slot = sc % S;
        if (ok && !warp_wait(&full[slot], (sc / S) & 1, abort_flag)) ok = false;
        const uint8_t *sp = ring + slot * SB;
        for (int sub = 0; sub < R && t * R + sub < O; sub += 16, ++tc) {
            float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};   // rows gi, gi + 8; tokens 2j, 2j + 1
            if (ok) {
                // this warp's first group (w); the group loop steps by 8 groups
                const uint8_t *ap = sp + (sub + gi) * (I / 2) + warp * (GS / 2) + j * (NW * 4);
                const uint16_t *hs = reinterpret_cast<const uint16_t *>(sp + dec_scales_off(I, R)) + (sub + gi) * nG + warp;
                const uint32_t *hz = reinterpret_cast<const uint32_t *>(sp + dec_zeros_off(I, nG, R)) + (sub + gi) * nzw;
                if (sub + 8 < R)
                    dec_subtile<GS, ZEROS, true>(acc, ap, 8 * (I / 2), hs, 8 * nG, hz, 8 * nzw, bbase, bstep, f0base,
                                                 fstep0, f1base, fstep1, nG, warp);
                else
                    dec_subtile<GS, ZEROS, false>(acc, ap, 8 * (I / 2), hs, 8 * nG, hz, 8 * nzw, bbase, bstep, f0base,
                                                  fstep0, f1base, fstep1, nG, warp);
            }
            // hand the partial sums of the 16 rows to the epilogue warp
            const int r = tc % DEC_RBUFS;
            if (ok && !warp_wait(&rempty[r], ((tc / DEC_RBUFS) & 1) ^ 1, abort_flag)) ok = false;
            if (ok) {
                float *rd = red + r * DEC_RED + (warp * 16 + gi) * 8 + 2 * j;
                rd[0] = acc[0];
                rd[1] = acc[1];
                rd[64] = acc[2];
                rd[65] = acc[3];
            }
            __syncwarp();
            if (lane == 0 && ok) mbar_arrive(&rfull[r]);
        }
        __syncwarp();
        if (lane == 0 && ok) mbar_arrive(&empty[slot]);
    }
}

int64_t up128(int64_t v) { return (v + 127) & ~int64_t(127); }

}  // namespace

bool w4a16_dec_config(DecBatch &b, int64_t M, int gs, bool zeros, int num_sms) {
    if (M < 1 || M > DEC_MAX_M || b.n < 1 || b.n > DEC_MAX_LINEARS || num_sms < b.n) return false;
    int64_t smem = 0, weight[DEC_MAX_LINEARS], tiles[DEC_MAX_LINEARS], total = 0;
    for (int l = 0; l < b.n; ++l) {
        const int64_t I = b.lin[l].I, O = b.lin[l].O, nG = I / gs, nzw = (nG + 7) / 8;
        int64_t k = DEC_TILE_TARGET / (4 * I);
        k = k < 1 ? 1 : k;
        const int64_t R = 8 * k;
        const int64_t slot = up128(dec_zeros_off(I, nG, R) + (zeros ? R * nzw * 4 : 0));
        const int64_t xbuf = up128(M * (I + DEC_XPAD) * 2 + M * nG * 16);
        const int64_t room = DEC_MAX_SMEM - DEC_FIXED - xbuf;
        int64_t st = room > 0 ? room / slot : 0;
        st = st > DEC_MAX_STAGES ? DEC_MAX_STAGES : st;
        if (st < 2) return false;
        b.rows[l] = static_cast<int>(R);
        b.stages[l] = static_cast<int>(st);
        b.slot_bytes[l] = static_cast<int>(slot);
        b.xbuf_bytes[l] = static_cast<int>(xbuf);
        const int64_t need = DEC_FIXED + xbuf + st * slot;
        smem = need > smem ? need : smem;
        weight[l] = O * (I / 2 + nG * 2 + (zeros ? nzw * 4 : 0));
        tiles[l] = (O + R - 1) / R;
        total += weight[l];
    }
    // CTAs in proportion to the bytes, at least one and at most one per tile each;
    // the rest, one at a time, to the linear with the most bytes per CTA
    int cnt[DEC_MAX_LINEARS], used = 0;
    for (int l = 0; l < b.n; ++l) {
        int64_t c = static_cast<int64_t>(num_sms) * weight[l] / total;
        c = c < 1 ? 1 : (c > tiles[l] ? tiles[l] : c);
        cnt[l] = static_cast<int>(c);
        used += cnt[l];
    }
    while (used > num_sms) {   // (only when many linears were raised to one CTA)
        int w = -1;
        for (int l = 0; l < b.n; ++l)
            if (cnt[l] > 1 && (w < 0 || weight[l] * cnt[w] < weight[w] * cnt[l])) w = l;
        --cnt[w];
        --used;
    }
    while (used < num_sms) {
        int w = -1;
        for (int l = 0; l < b.n; ++l)
            if (cnt[l] < tiles[l] && (w < 0 || weight[l] * cnt[w] > weight[w] * cnt[l])) w = l;
        if (w < 0) break;
        ++cnt[w];
        ++used;
    }
    b.cta0[0] = 0;
    for (int l = 0; l < b.n; ++l) b.cta0[l + 1] = b.cta0[l] + cnt[l];
    b.ctas = used;
    b.smem = smem;
    return true;
}

cudaError_t launch_w4a16_dec(const DecBatch &b, int M, int gs, bool zeros, cudaStream_t st) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(b.ctas));
    cfg.blockDim = dim3(DEC_THREADS);
    cfg.dynamicSmemBytes = static_cast<size_t>(b.smem);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
#define AWQ_DEC(GSZ, Z)                                                                             \
    do {                                                                                            \
        cudaError_t e = cudaFuncSetAttribute(w4a16_dec_kernel<GSZ, Z>,                              \
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,           \
                                             static_cast<int>(b.smem));                             \
        if (e != cudaSuccess) return e;                                                             \
        return cudaLaunchKernelEx(&cfg, w4a16_dec_kernel<GSZ, Z>, b, M);                            \
    } while (0)
    if (gs == 32) {
        if (zeros) AWQ_DEC(32, true); else AWQ_DEC(32, false);
    } else if (gs == 64) {
        if (zeros) AWQ_DEC(64, true); else AWQ_DEC(64, false);
    } else {
        if (zeros) AWQ_DEC(128, true); else AWQ_DEC(128, false);
    }
#undef AWQ_DEC
}

}  // namespace awq
