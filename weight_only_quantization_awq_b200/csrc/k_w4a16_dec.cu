// W4A16 decode (1..8 tokens) over one or several linear layers in one
// persistent launch (AWQ guide, section 三, QuantLinear.forward:
// y = (x / s) * dequant(W)^T).
//
// At decode sizes a layer is bound by reading its packed weights from HBM, and
// one layer of a few MB cannot keep HBM busy on its own: the ramp and tail of a
// launch cost about as much as the transfer.  So one launch takes a list of
// independent linears (e.g. the q, k, v, o, gate, up and down projections of a
// block) and streams all of them through every SM.
//
// Work: units of 16 output rows x 4096 input columns (a "stage", 32 KB of codes).
// CTA c (one per SM) owns the 16-row tiles whose first unit falls in
// [c U / P, (c + 1) U / P), so every CTA streams about the same number of bytes,
// crossing from one linear to the next where its range does.  Warp roles:
//   producer (1 warp): per tile, one bulk copy of the tile's fp16 scales and one
//     of its zero words into a header buffer; per stage, 16 bulk copies (one per
//     row, 2 KB) into a ring slot whose rows are padded to 2112 bytes, so the
//     consumers' 16-byte reads of two rows are free of bank conflicts.  The copy
//     engine takes about a hundred cycles per request whatever its size, so the
//     requests are made as large as a row of the stage.  Codes and headers carry
//     an evict-first L2 hint: they are read once.
//   stagers (4 warps): per linear, xs = fp16((x / s16) * 2^-k) for all tokens,
//     k per (token, group) putting the group's largest |x / s| in [2^14, 2^15),
//     with 2^k and the group's sum of the rounded xs beside; written in the
//     fragment order below into one of two activation buffers, one linear ahead
//     of the consumers.  The CTA's first linear is staged by all 12 non-producer
//     warps together.
//   consumers (8 warps): a stage is walked as four sub-stages of 1024 columns;
//     warp w takes the 128 columns [128 w, 128 w + 128) of each sub-stage (1, 2
//     or 4 groups) of the tile's 16 rows.  One LOP3 turns two
//     nibbles into an fp16x2 (1024 + code) pair exactly, one mma.sync.m16n8k16
//     consumes 256 weights (fragment layout in w4a16_frag.cuh); per (row, group)
//         sum_i (code_i - z) Delta xs_i = Delta (sum_i (1024 + code_i) xs_i
//                                                 - (1024 + z) sum_i xs_i).
//     At the end of a tile the 8 warps' fp32 sums meet in shared memory and each
//     output is written once, in bf16.
// Fragment order of xs: within a group, thread j (of the 4 sharing a row) owns
// the 8-column words NW j .. NW j + NW - 1 (NW = group / 32) of the packed codes,
// one contiguous load per row; the activations of its word kk are stored in the
// 16-byte slot 4 kk + j, so the 4 threads' reads of one token are one contiguous
// 64-byte span.  Within a slot the columns are in the order (0,4,1,5,2,6,3,7).
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
#include "w4a16_frag.cuh"

namespace awq {

namespace {

constexpr int DEC_CWARPS = 8;                                  // consumers
constexpr int DEC_SWARPS = 4;                                  // stagers
constexpr int DEC_PWARP = DEC_CWARPS + DEC_SWARPS;             // producer
constexpr int DEC_THREADS = (DEC_CWARPS + DEC_SWARPS + 1) * 32;
constexpr int DEC_KC = 1024;                                   // columns per sub-stage
constexpr int DEC_SUB = 4;                                     // sub-stages per stage
constexpr int DEC_SC = DEC_KC * DEC_SUB;                       // columns per stage
constexpr int DEC_ROWB = DEC_SC / 2 + 64;                      // padded row of a stage, bytes
constexpr int DEC_STAGE = 16 * DEC_ROWB;
constexpr int DEC_RED = DEC_CWARPS * 16 * 8;                   // floats per reduction buffer
constexpr int DEC_XPAD = 32;                                   // fp16 of padding per staged token row

// ---- the CTA's tiles: those whose first unit lies in [u0, u1)
struct DecTile {
    int l;          // linear
    int t;          // 16-row tile within it
    int64_t a;      // first unit of the tile
};

__device__ __forceinline__ bool dec_first_tile(const DecBatch &b, int64_t u0, int64_t u1, DecTile &d) {
    int l = 0;
    while (l + 1 < b.n && u0 >= b.ucum[l + 1]) ++l;
    const int64_t t = (u0 - b.ucum[l] + b.spt[l] - 1) / b.spt[l];
    d.l = l;
    d.t = static_cast<int>(t);
    d.a = b.ucum[l] + t * b.spt[l];
    if (d.a >= b.ucum[l + 1]) {
        if (l + 1 >= b.n) return false;
        d.l = l + 1;
        d.t = 0;
        d.a = b.ucum[l + 1];
    }
    return d.a < u1;
}

__device__ __forceinline__ bool dec_next_tile(const DecBatch &b, int64_t u1, DecTile &d) {
    d.a += b.spt[d.l];
    ++d.t;
    if (d.a >= b.ucum[d.l + 1]) {
        if (d.l + 1 >= b.n) return false;
        ++d.l;
        d.t = 0;
        d.a = b.ucum[d.l];
    }
    return d.a < u1;
}

// A wait taken by all 32 lanes of a warp (each observes the phase itself), with
// one outcome for the warp: if any lane gave up, all do.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
}

// ---- staging of one linear's activations by `nthreads` threads (a multiple of 32)
template <int GS>
__device__ void dec_stage(const DecLinear &L, int M, uint8_t *buf, int tid, int nthreads) {
    constexpr int WPG = GS / 8;            // 8-column words per group: consecutive lanes
    constexpr int NW = GS / 32;            // words per fragment thread
    constexpr int U = 4;                   // words in flight per thread
    const int I = static_cast<int>(L.I), nG = I / GS, wpr = I / 8, IP = I + DEC_XPAD;
    uint16_t *xs = reinterpret_cast<uint16_t *>(buf);
    float2 *xf = reinterpret_cast<float2 *>(buf + M * IP * 2);
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
            float sum = 0.0f;
#pragma unroll
            for (int q = 0; q < 4; ++q) {   // word q of the slot: columns (q, q + 4)
                const __half2 hv = __floats2half2_rn(v[q] * sc, v[q + 4] * sc);
                h[q] = *reinterpret_cast<const uint32_t *>(&hv);
                sum += __low2float(hv) + __high2float(hv);
            }
#pragma unroll
            for (int off = WPG / 2; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
            if (it < total) {
                const int m = it / wpr, w = it - m * wpr;
                const int g = w / WPG, wg = w - g * WPG;
                const int slot = (wg % NW) * 4 + wg / NW;
                *reinterpret_cast<uint4 *>(xs + m * IP + g * GS + slot * 8) = make_uint4(h[0], h[1], h[2], h[3]);
                if (wg == 0) xf[m * nG + g] = make_float2(ldexpf(1.0f, kx), sum);
            }
        }
    }
}

// ---- one sub-stage (number s within the row, codes at stg) of one consumer warp:
// its GPW groups of the tile's 16 rows
template <int GS, bool ZEROS>
__device__ __forceinline__ void dec_consume(float (&acc)[4], const uint8_t *stg, const uint8_t *xsb,
                                            const float2 *xf, const uint16_t *hs, const uint32_t *hz,
                                            int s, int nG, int nzw, int IP, int M, int warp, int gi,
                                            int j) {
    constexpr int NW = GS / 32, GPW = 128 / GS;
#pragma unroll
    for (int q = 0; q < GPW; ++q) {
        const int gl = warp * GPW + q;                      // group within the stage
        const int grp = s * (DEC_KC / GS) + gl;             // group within the row
        if (grp >= nG) break;                               // ragged last stage (warp-uniform)
        uint32_t c0[NW], c1[NW];
        const uint8_t *ap = stg + gi * DEC_ROWB + gl * (GS / 2) + j * (NW * 4);
        if constexpr (NW == 4) {
            const uint4 v0 = *reinterpret_cast<const uint4 *>(ap);
            const uint4 v1 = *reinterpret_cast<const uint4 *>(ap + 8 * DEC_ROWB);
            c0[0] = v0.x; c0[1] = v0.y; c0[2] = v0.z; c0[3] = v0.w;
            c1[0] = v1.x; c1[1] = v1.y; c1[2] = v1.z; c1[3] = v1.w;
        } else if constexpr (NW == 2) {
            const uint2 v0 = *reinterpret_cast<const uint2 *>(ap);
            const uint2 v1 = *reinterpret_cast<const uint2 *>(ap + 8 * DEC_ROWB);
            c0[0] = v0.x; c0[1] = v0.y;
            c1[0] = v1.x; c1[1] = v1.y;
        } else {
            c0[0] = *reinterpret_cast<const uint32_t *>(ap);
            c1[0] = *reinterpret_cast<const uint32_t *>(ap + 8 * DEC_ROWB);
        }
        uint32_t bw[4 * NW];
        if (gi < M) {
            const uint8_t *bp = xsb + (gi * IP + grp * GS) * 2 + j * 16;
#pragma unroll
            for (int kk = 0; kk < NW; ++kk) {
                const uint4 v = *reinterpret_cast<const uint4 *>(bp + kk * 64);
                bw[4 * kk] = v.x; bw[4 * kk + 1] = v.y; bw[4 * kk + 2] = v.z; bw[4 * kk + 3] = v.w;
            }
        } else {
#pragma unroll
            for (int kk = 0; kk < 4 * NW; ++kk) bw[kk] = 0u;
        }
        const float2 f0 = 2 * j < M ? xf[2 * j * nG + grp] : make_float2(0.0f, 0.0f);
        const float2 f1 = 2 * j + 1 < M ? xf[(2 * j + 1) * nG + grp] : make_float2(0.0f, 0.0f);
        const float d0 = __half2float(__ushort_as_half(hs[gi * nG + grp]));
        const float d1 = __half2float(__ushort_as_half(hs[(gi + 8) * nG + grp]));
        float zb0 = 1032.0f, zb1 = 1032.0f;
        if constexpr (ZEROS) {
            zb0 = 1024.0f + static_cast<float>((hz[gi * nzw + (grp >> 3)] >> (4 * (grp & 7))) & 0xFu);
            zb1 = 1024.0f + static_cast<float>((hz[(gi + 8) * nzw + (grp >> 3)] >> (4 * (grp & 7))) & 0xFu);
        }
        // two independent MMA chains (first and second half of the group's k)
        float da[4] = {0.0f, 0.0f, 0.0f, 0.0f}, db[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int kk = 0; kk < NW; ++kk) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint32_t a[4] = {frag_nib2(c0[kk], 2 * h), frag_nib2(c1[kk], 2 * h),
                                       frag_nib2(c0[kk], 2 * h + 1), frag_nib2(c1[kk], 2 * h + 1)};
                if (2 * kk + h < NW)
                    frag_mma16816(da, a, bw[4 * kk + 2 * h], bw[4 * kk + 2 * h + 1]);
                else
                    frag_mma16816(db, a, bw[4 * kk + 2 * h], bw[4 * kk + 2 * h + 1]);
            }
        }
        acc[0] = __fmaf_rn(d0 * f0.x, __fmaf_rn(-zb0, f0.y, da[0] + db[0]), acc[0]);
        acc[1] = __fmaf_rn(d0 * f1.x, __fmaf_rn(-zb0, f1.y, da[1] + db[1]), acc[1]);
        acc[2] = __fmaf_rn(d1 * f0.x, __fmaf_rn(-zb1, f0.y, da[2] + db[2]), acc[2]);
        acc[3] = __fmaf_rn(d1 * f1.x, __fmaf_rn(-zb1, f1.y, da[3] + db[3]), acc[3]);
    }
}

template <int GS, bool ZEROS>
__global__ void __launch_bounds__(DEC_THREADS, 1) w4a16_dec_kernel(const __grid_constant__ DecBatch b, int M) {
    extern __shared__ __align__(128) uint8_t dsm[];
    uint8_t *ring = dsm;                                                  // [stages][16][576]
    uint8_t *hdr = ring + b.stages * DEC_STAGE;                           // [hbufs][hdr_bytes]
    uint8_t *xbuf = hdr + b.hbufs * b.hdr_bytes;                          // [xbufs][xbuf_bytes]
    float *red = reinterpret_cast<float *>(xbuf + b.xbufs * b.xbuf_bytes);   // [2][warps][16][8]
    uint64_t *full = reinterpret_cast<uint64_t *>(red + 2 * DEC_RED);
    uint64_t *empty = full + b.stages;
    uint64_t *hfull = empty + b.stages, *hempty = hfull + b.hbufs;
    uint64_t *xfull = hempty + b.hbufs, *xempty = xfull + b.xbufs;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(xempty + b.xbufs);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int k = 0; k < b.stages; ++k) {
            mbar_init(&full[k], 1);
            mbar_init(&empty[k], DEC_CWARPS);
        }
        for (int k = 0; k < b.hbufs; ++k) {
            mbar_init(&hfull[k], 1);
            mbar_init(&hempty[k], DEC_CWARPS);
        }
        for (int k = 0; k < b.xbufs; ++k) {
            mbar_init(&xfull[k], DEC_SWARPS);
            mbar_init(&xempty[k], DEC_CWARPS);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    const int64_t U = b.ucum[b.n];
    const int64_t u0 = static_cast<int64_t>(blockIdx.x) * U / b.ctas;
    const int64_t u1 = static_cast<int64_t>(blockIdx.x + 1) * U / b.ctas;
    DecTile d;
    const bool any = dec_first_tile(b, u0, u1, d);

    if (warp == DEC_PWARP && lane == 0 && any) {
        const DecLinear &L = b.lin[d.l];
        const int64_t o0 = static_cast<int64_t>(d.t) * 16;
        const int64_t rows = L.O - o0 < 16 ? L.O - o0 : 16;
        l2_prefetch_range(L.qweight + o0 * (L.I / 8), static_cast<uint64_t>(rows) * (L.I / 2));
    }
    griddep_launch_dependents();
    griddep_wait();
    if (!any) return;

    if (warp == DEC_PWARP) {
        // ------------------------------------------------------------ producer
        const uint64_t pol = l2_policy_evict_first();
        int sc = 0, hc = 0;
        bool ok = true, more = true;
        while (more && ok) {
            const DecLinear &L = b.lin[d.l];
            const int I = static_cast<int>(L.I), nG = I / GS, nzw = (nG + 7) >> 3;
            const int64_t o0 = static_cast<int64_t>(d.t) * 16;
            const int rows = L.O - o0 < 16 ? static_cast<int>(L.O - o0) : 16;
            // tile header: scales [rows][nG] fp16, then zero words [rows][nzw] at 32 nG bytes
            const int hb = hc % b.hbufs;
            if (!warp_wait(&hempty[hb], ((hc / b.hbufs) & 1) ^ 1, abort_flag)) { ok = false; break; }
            uint8_t *hd = hdr + hb * b.hdr_bytes;
            const uint16_t *ssrc = L.scales + o0 * nG;
            const uint32_t *zsrc = ZEROS ? L.zeros + o0 * nzw : nullptr;
            const uint32_t sbytes = static_cast<uint32_t>(rows * nG * 2);
            const uint32_t zbytes = ZEROS ? static_cast<uint32_t>(rows * nzw * 4) : 0u;
            const bool bulk = (sbytes % 16 == 0) && (reinterpret_cast<uintptr_t>(ssrc) % 16 == 0) &&
                              (!ZEROS || ((zbytes % 16 == 0) && (reinterpret_cast<uintptr_t>(zsrc) % 16 == 0)));
            if (bulk) {
                if (lane == 0) {
                    mbar_arrive_expect_tx(&hfull[hb], sbytes + zbytes);
                    bulk_load(hd, ssrc, sbytes, &hfull[hb], pol);
                    if (ZEROS) bulk_load(hd + 32 * nG, zsrc, zbytes, &hfull[hb], pol);
                }
            } else {
                // a ragged or unaligned tile: plain loads
                uint16_t *hs = reinterpret_cast<uint16_t *>(hd);
                for (int i = lane; i < rows * nG; i += 32) hs[i] = __ldcg(ssrc + i);
                if (ZEROS) {
                    uint32_t *hz = reinterpret_cast<uint32_t *>(hd + 32 * nG);
                    for (int i = lane; i < rows * nzw; i += 32) hz[i] = __ldcg(zsrc + i);
                }
                fence_proxy_async_smem();   // before later bulk copies into this buffer
                __syncwarp();
                if (lane == 0) mbar_arrive(&hfull[hb]);
            }
            ++hc;
            // codes, one stage of 16 rows x 4096 columns at a time
            const int64_t wpr = I / 8;
            for (int s = 0; s < b.spt[d.l]; ++s) {
                const int slot = sc % b.stages;
                if (!warp_wait(&empty[slot], ((sc / b.stages) & 1) ^ 1, abort_flag)) { ok = false; break; }
                const int c0 = s * DEC_SC;
                const uint32_t cb = static_cast<uint32_t>((I - c0 < DEC_SC ? I - c0 : DEC_SC) / 2);
                if (lane == 0) mbar_arrive_expect_tx(&full[slot], static_cast<uint32_t>(rows) * cb);
                __syncwarp();
                if (lane < rows)
                    bulk_load(ring + slot * DEC_STAGE + lane * DEC_ROWB, L.qweight + (o0 + lane) * wpr + c0 / 8, cb,
                              &full[slot], pol);
                ++sc;
            }
            if (ok) more = dec_next_tile(b, u1, d);
        }
        // wait (bounded) for every copy still in flight before the CTA may exit
        for (int k = 0; k < b.stages; ++k)
            if (sc > k) mbar_wait_drain(&full[k], static_cast<uint32_t>(((sc - 1 - k) / b.stages) & 1));
        for (int k = 0; k < b.hbufs; ++k)
            if (hc > k) mbar_wait_drain(&hfull[k], static_cast<uint32_t>(((hc - 1 - k) / b.hbufs) & 1));
        return;
    }

    // ---- the CTA's first linear: staged by consumers and stagers together
    {
        const int stagers = (DEC_CWARPS + DEC_SWARPS) * 32;
        dec_stage<GS>(b.lin[d.l], M, xbuf, threadIdx.x, stagers);
        named_bar_sync(2, stagers);
    }

    if (warp >= DEC_CWARPS) {
        // ------------------------------------------------------------- stagers
        __syncwarp();
        if (lane == 0) mbar_arrive(&xfull[0]);
        int xc = 1, cur = d.l;
        bool more = dec_next_tile(b, u1, d);
        while (more) {
            if (d.l != cur) {
                const int xb = xc % b.xbufs;
                if (!warp_wait(&xempty[xb], ((xc / b.xbufs) & 1) ^ 1, abort_flag)) break;
                dec_stage<GS>(b.lin[d.l], M, xbuf + xb * b.xbuf_bytes, threadIdx.x - DEC_CWARPS * 32,
                              DEC_SWARPS * 32);
                __syncwarp();
                if (lane == 0) mbar_arrive(&xfull[xb]);
                ++xc;
                cur = d.l;
            }
            more = dec_next_tile(b, u1, d);
        }
        return;
    }

    // ------------------------------------------------------------------ consumers
    const int gi = lane >> 2, j = lane & 3;
    int sc = 0, hc = 0, xc = 0, tc = 0, cur = -1;
    bool ok = true, more = true;
    const uint8_t *xsb = xbuf;
    const float2 *xf = nullptr;
    int I = 0, nG = 0, nzw = 0, IP = 0;
    while (more) {
        const DecLinear &L = b.lin[d.l];
        if (d.l != cur) {
            if (cur >= 0) {
                __syncwarp();
                if (lane == 0 && ok) mbar_arrive(&xempty[(xc - 1) % b.xbufs]);
            }
            const int xb = xc % b.xbufs;
            if (ok && !warp_wait(&xfull[xb], (xc / b.xbufs) & 1, abort_flag)) ok = false;
            ++xc;
            cur = d.l;
            I = static_cast<int>(L.I);
            nG = I / GS;
            nzw = (nG + 7) >> 3;
            IP = I + DEC_XPAD;
            xsb = xbuf + xb * b.xbuf_bytes;
            xf = reinterpret_cast<const float2 *>(xsb + M * IP * 2);
        }
        const int hb = hc % b.hbufs;
        if (ok && !warp_wait(&hfull[hb], (hc / b.hbufs) & 1, abort_flag)) ok = false;
        const uint16_t *hs = reinterpret_cast<const uint16_t *>(hdr + hb * b.hdr_bytes);
        const uint32_t *hz = reinterpret_cast<const uint32_t *>(hdr + hb * b.hdr_bytes + 32 * nG);
        float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        const int spt = b.spt[d.l];
        for (int s = 0; s < spt; ++s) {
            const int slot = sc % b.stages;
            if (ok && !warp_wait(&full[slot], (sc / b.stages) & 1, abort_flag)) ok = false;
            if (ok) {
#pragma unroll 1
                for (int k = 0; k < DEC_SUB && (s * DEC_SUB + k) * DEC_KC < I; ++k)
                    dec_consume<GS, ZEROS>(acc, ring + slot * DEC_STAGE + k * (DEC_KC / 2), xsb, xf, hs, hz,
                                           s * DEC_SUB + k, nG, nzw, IP, M, warp, gi, j);
            }
            __syncwarp();
            if (lane == 0 && ok) mbar_arrive(&empty[slot]);
            ++sc;
        }
        __syncwarp();
        if (lane == 0 && ok) mbar_arrive(&hempty[hb]);
        ++hc;
        // the 8 warps' partial sums meet in shared memory (double-buffered by tile)
        float *rd = red + (tc & 1) * DEC_RED;
        rd[(warp * 16 + gi) * 8 + 2 * j] = acc[0];
        rd[(warp * 16 + gi) * 8 + 2 * j + 1] = acc[1];
        rd[(warp * 16 + gi + 8) * 8 + 2 * j] = acc[2];
        rd[(warp * 16 + gi + 8) * 8 + 2 * j + 1] = acc[3];
        named_bar_sync(1, DEC_CWARPS * 32);
        if (static_cast<int>(threadIdx.x) < 16 * M && !*abort_flag) {
            const int r = threadIdx.x & 15, m = threadIdx.x >> 4;
            const int64_t o = static_cast<int64_t>(d.t) * 16 + r;
            if (o < L.O) {
                float sum = 0.0f;
#pragma unroll
                for (int w = 0; w < DEC_CWARPS; ++w) sum += rd[(w * 16 + r) * 8 + m];
                L.y[m * L.O + o] = __bfloat16_as_ushort(__float2bfloat16_rn(sum));
            }
        }
        ++tc;
        more = dec_next_tile(b, u1, d);
    }
}

int64_t up16(int64_t v) { return (v + 15) & ~int64_t(15); }
int64_t up128(int64_t v) { return (v + 127) & ~int64_t(127); }

}  // namespace

bool w4a16_dec_config(DecBatch &b, int64_t M, int gs, bool zeros, int num_sms) {
    if (M < 1 || M > DEC_MAX_M || b.n < 1 || b.n > DEC_MAX_LINEARS || num_sms < 1) return false;
    int64_t hdr = 0, xbuf = 0, tiles = 0;
    b.ucum[0] = 0;
    for (int l = 0; l < b.n; ++l) {
        const int64_t I = b.lin[l].I, O = b.lin[l].O, nG = I / gs, nzw = (nG + 7) / 8;
        const int64_t spt = (I + DEC_SC - 1) / DEC_SC, t = (O + 15) / 16;
        b.spt[l] = static_cast<int>(spt);
        b.ucum[l + 1] = b.ucum[l] + t * spt;
        tiles += t;
        const int64_t h = 32 * nG + (zeros ? 64 * nzw : 0);
        const int64_t x = M * (I + DEC_XPAD) * 2 + up16(M * nG * 8);
        hdr = h > hdr ? h : hdr;
        xbuf = x > xbuf ? x : xbuf;
    }
    hdr = up128(hdr);
    xbuf = up128(xbuf);
    // (stages, header buffers, activation buffers), most preferred first
    static const int opts[][3] = {{4, 3, 2}, {3, 3, 2}, {4, 3, 1}, {3, 2, 1}, {2, 2, 1}};
    for (const auto &o : opts) {
        const int64_t smem = int64_t(o[0]) * DEC_STAGE + o[1] * hdr + o[2] * xbuf + 2 * DEC_RED * 4 +
                             (2 * o[0] + 2 * o[1] + 2 * o[2]) * 8 + 16;
        if (smem <= DEC_MAX_SMEM) {
            b.stages = o[0];
            b.hbufs = o[1];
            b.xbufs = o[2];
            b.hdr_bytes = static_cast<int>(hdr);
            b.xbuf_bytes = static_cast<int>(xbuf);
            b.smem = smem;
            b.ctas = static_cast<int>(tiles < num_sms ? tiles : num_sms);
            return true;
        }
    }
    return false;
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
