// Fused AWQ grid-search kernel for sm_100a.
//
// For grid point g, output rows [128*ot, 128*ot + 128) and tokens
// [512*tb, 512*tb + 512), it accumulates
//     E[o, n] = sum_i dW_g[o, i] * X[n, i],   dW_g = Q(W * s_g) / s_g - W
// on the 5th-generation tensor cores (fp16 operands, fp32 accumulation) and
// reduces sum_n E[o, n]^2 per row.
// This is the objective L(s) = ||Q(W*s)(s^-1*X) - W X|| of the AWQ paper
// summary (Method), with the 1/s moved from X's columns onto the weight
// columns (exact in real arithmetic), evaluated for every s = s_X^alpha on the
// grid.  Neither dW nor E ever reaches global memory.
//
// Warp roles (448 threads, one CTA per SM, persistent over work units):
//   warps 0-7   dW producers: read W (bf16/fp32) and the per-group quantiser
//               parameters, form dW for a 128 x 64 slab in registers, write it
//               as fp16 into shared memory in the 128-byte-swizzled K-major
//               layout the MMA reads, then signal a_full.
//   warps 8-11  epilogue: tcgen05.ld of the 128 x 512 fp32 accumulator (lane =
//               output row), square-and-sum per row, one fp32 partial per
//               (grid point, token block, row).
//   warp 12     TMA: X tiles of 256 tokens x 64 channels (fp16 copy of X scaled
//               by a power of two, 128B swizzle) into a 5-stage ring.
//   warp 13     MMA: allocates 512 TMEM columns, one elected thread issues
//               tcgen05.mma M=128 N=256 K=16 (two N=256 halves per slab), and
//               tcgen05.commit releases ring stages and the accumulator.
// Work units are (g fastest, then output tile, then token block) and are dealt
// round-robin to the CTAs, so the CTAs running at one time share a few W tiles
// and X blocks in L2.
#include <cuda_bf16.h>

#include "awq_internal.h"
#include "awq_ptx.cuh"

namespace awq {

namespace {

constexpr int NUM_PRODUCER_WARPS = 8;
constexpr int WARP_TMA = 12;
constexpr int WARP_MMA = 13;
constexpr int NUM_THREADS = 14 * 32;
constexpr int XS = 5;                                  // X ring stages
constexpr int AS = 3;                                  // dW ring stages
constexpr int X_STAGE_BYTES = SUB_N * SLAB_K * 2;      // 32 KB
constexpr int A_STAGE_BYTES = TILE_O * SLAB_K * 2;     // 16 KB
constexpr int NUM_BARS = 2 * XS + 2 * AS + 3;
constexpr int SMEM_BYTES = 1024 + XS * X_STAGE_BYTES + AS * A_STAGE_BYTES + NUM_BARS * 8 + 16;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t IDESC = idesc_f16_f32(TILE_O, SUB_N, false);
constexpr float MAGIC = 12582912.0f;                   // 1.5 * 2^23: x + MAGIC - MAGIC = rint(x)

struct Unit {
    int g;
    int64_t ot, tb;
    int nsub;
};

__device__ __forceinline__ Unit decode(int64_t u, const SearchArgs &a, int64_t OT) {
    Unit r;
    r.g = static_cast<int>(u % a.G);
    const int64_t rest = u / a.G;
    r.ot = rest % OT;
    r.tb = rest / OT;
    const int64_t left = a.N - r.tb * TILE_N;
    r.nsub = left > SUB_N ? 2 : 1;
    return r;
}

// Distance from a half-integer below which the reciprocal product may round to
// a different code than the correctly rounded quotient: |W'/Delta| <= 32, so
// W' * RN(1/Delta) and RN(W'/Delta) differ by at most 32 * 2^-23 = 2^-18.
constexpr float TIE_BAND = 0.5f - 1.0f / 65536.0f;

// dW for 8 adjacent columns of one row (one group), packed as 4 x fp16x2.
// Codes follow the quantizer's definition q = rint(RN(W'/Delta)) exactly: the
// fast path rounds W' * (1/Delta), and any element whose product lies within
// 2^-16 of a half-integer (exact ties included) is redone with the correctly
// rounded division, so the result never depends on the reciprocal.
template <bool CLAMP>
__device__ __forceinline__ uint4 dw_chunk8(const float (&w)[8], const float (&s)[8],
                                           const float (&is)[8], const float4 &prm) {
    float wp[8], q[8];
    bool near_tie = false;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        wp[e] = __fmul_rn(w[e], s[e]);                                 // W * s
        q[e] = __fsub_rn(__fmaf_rn(wp[e], prm.y, MAGIC), MAGIC);        // rint(W*s * (1/Delta))
        near_tie |= fabsf(__fmaf_rn(wp[e], prm.y, -q[e])) > TIE_BAND;
    }
    if (near_tie) {
#pragma unroll
        for (int e = 0; e < 8; ++e)
            if (prm.x != 0.0f) q[e] = rintf(__fdiv_rn(wp[e], prm.x));
    }
    float r[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        float qe = q[e];
        if (CLAMP) qe = fminf(fmaxf(qe, prm.z), prm.w);                // code range
        r[e] = __fmul_rn(__fmaf_rn(qe, prm.x, -wp[e]), is[e]);         // (q*Delta - W*s) / s
    }
    uint4 pk;
    pk.x = f16x2_satfinite(r[0], r[1]);
    pk.y = f16x2_satfinite(r[2], r[3]);
    pk.z = f16x2_satfinite(r[4], r[5]);
    pk.w = f16x2_satfinite(r[6], r[7]);
    return pk;
}

template <bool WBF16, bool CLAMP>
__device__ __forceinline__ void producer_role(const SearchArgs &a, int64_t OT, int64_t U,
                                              uint8_t *a_ring, uint64_t *a_full, uint64_t *a_empty,
                                              volatile int *abort_flag) {
    const int t = threadIdx.x;          // 0..255
    const int r = t >> 1, hc = t & 1;   // row in tile, half of the 64-wide slab
    const int64_t nK = a.I / SLAB_K;
    const int64_t nG = a.I / a.gs;
    uint32_t it = 0;
    for (int64_t u = blockIdx.x; u < U; u += gridDim.x) {
        const Unit un = decode(u, a, OT);
        const int64_t row = un.ot * TILE_O + r;
        const bool valid = row < a.O;
        const float *srow = a.s_tab + static_cast<int64_t>(un.g) * a.I;
        const float *isrow = a.inv_s_tab + static_cast<int64_t>(un.g) * a.I;
        const float4 *qp = a.qparam + (static_cast<int64_t>(un.g) * a.O + (valid ? row : 0)) * nG;
        for (int64_t kb = 0; kb < nK; ++kb, ++it) {
            const int64_t col0 = kb * SLAB_K + hc * 32;
            uint32_t wraw[WBF16 ? 16 : 32];
            if (valid) {
                if constexpr (WBF16) {
                    const uint4 *src = reinterpret_cast<const uint4 *>(
                        static_cast<const uint16_t *>(a.W) + row * a.I + col0);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const uint4 v = __ldg(src + k);
                        wraw[4 * k] = v.x; wraw[4 * k + 1] = v.y;
                        wraw[4 * k + 2] = v.z; wraw[4 * k + 3] = v.w;
                    }
                } else {
                    const uint4 *src = reinterpret_cast<const uint4 *>(
                        static_cast<const float *>(a.W) + row * a.I + col0);
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const uint4 v = __ldg(src + k);
                        wraw[4 * k] = v.x; wraw[4 * k + 1] = v.y;
                        wraw[4 * k + 2] = v.z; wraw[4 * k + 3] = v.w;
                    }
                }
            } else {
#pragma unroll
                for (int k = 0; k < (WBF16 ? 16 : 32); ++k) wraw[k] = 0u;
            }
            const float4 prm = valid ? __ldg(qp + col0 / a.gs) : make_float4(0.f, 0.f, 0.f, 0.f);

            const uint32_t stage = it % AS, phase = (it / AS) & 1u;
            if (!mbar_wait(&a_empty[stage], phase ^ 1u, abort_flag)) return;
            uint8_t *dst = a_ring + stage * A_STAGE_BYTES;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float4 s0 = __ldg(reinterpret_cast<const float4 *>(srow + col0 + 8 * c));
                const float4 s1 = __ldg(reinterpret_cast<const float4 *>(srow + col0 + 8 * c + 4));
                const float4 i0 = __ldg(reinterpret_cast<const float4 *>(isrow + col0 + 8 * c));
                const float4 i1 = __ldg(reinterpret_cast<const float4 *>(isrow + col0 + 8 * c + 4));
                const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
                const float iv[8] = {i0.x, i0.y, i0.z, i0.w, i1.x, i1.y, i1.z, i1.w};
                float wv[8];
                if constexpr (WBF16) {
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const uint32_t u2 = wraw[4 * c + k];
                        wv[2 * k] = __uint_as_float(u2 << 16);
                        wv[2 * k + 1] = __uint_as_float(u2 & 0xFFFF0000u);
                    }
                } else {
#pragma unroll
                    for (int k = 0; k < 8; ++k) wv[k] = __uint_as_float(wraw[8 * c + k]);
                }
                *reinterpret_cast<uint4 *>(dst + sw128_offset(r, hc * 4 + c)) =
                    dw_chunk8<CLAMP>(wv, sv, iv, prm);
            }
            fence_proxy_async_smem();
            mbar_arrive(&a_full[stage]);
        }
    }
}

__device__ __forceinline__ void tma_role(const SearchArgs &a, const CUtensorMap *xmap, int64_t OT,
                                         int64_t U, uint8_t *x_ring, uint64_t *x_full,
                                         uint64_t *x_empty, volatile int *abort_flag) {
    const int64_t nK = a.I / SLAB_K;
    uint32_t it = 0;
    int64_t last[XS];
#pragma unroll
    for (int s = 0; s < XS; ++s) last[s] = -1;
    bool ok = true;
    for (int64_t u = blockIdx.x; u < U && ok; u += gridDim.x) {
        const Unit un = decode(u, a, OT);
        for (int64_t kb = 0; kb < nK && ok; ++kb) {
            for (int h = 0; h < un.nsub; ++h, ++it) {
                const uint32_t stage = it % XS, phase = (it / XS) & 1u;
                if (!mbar_wait(&x_empty[stage], phase ^ 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(&x_full[stage], X_STAGE_BYTES);
                tma_load_2d(x_ring + stage * X_STAGE_BYTES, xmap, &x_full[stage],
                            static_cast<int32_t>(kb * SLAB_K),
                            static_cast<int32_t>(un.tb * TILE_N + h * SUB_N));
#pragma unroll
                for (int s = 0; s < XS; ++s)
                    if (s == static_cast<int>(stage)) last[s] = it;
            }
        }
    }
    // Never leave the CTA with a copy still landing in its shared memory.
#pragma unroll
    for (int s = 0; s < XS; ++s)
        if (last[s] >= 0) mbar_wait_drain(&x_full[s], static_cast<uint32_t>((last[s] / XS) & 1));
}

__device__ __forceinline__ void mma_role(const SearchArgs &a, int64_t OT, int64_t U,
                                         uint32_t tmem_base, uint8_t *x_ring, uint8_t *a_ring,
                                         uint64_t *x_full, uint64_t *x_empty, uint64_t *a_full,
                                         uint64_t *a_empty, uint64_t *acc_full,
                                         uint64_t *acc_empty, uint64_t *drain,
                                         volatile int *abort_flag) {
    const int64_t nK = a.I / SLAB_K;
    uint32_t ait = 0, xit = 0, accit = 0;
    const uint32_t x_base = smem_u32(x_ring), a_base = smem_u32(a_ring);
    bool ok = true;
    for (int64_t u = blockIdx.x; u < U && ok; u += gridDim.x) {
        const Unit un = decode(u, a, OT);
        if (!mbar_wait(acc_empty, (accit & 1u) ^ 1u, abort_flag)) break;
        tc_fence_after();
        for (int64_t kb = 0; kb < nK && ok; ++kb, ++ait) {
            const uint32_t as = ait % AS;
            if (!mbar_wait(&a_full[as], (ait / AS) & 1u, abort_flag)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t a_addr = a_base + as * A_STAGE_BYTES;
            for (int h = 0; h < un.nsub; ++h, ++xit) {
                const uint32_t xs = xit % XS;
                if (!mbar_wait(&x_full[xs], (xit / XS) & 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t b_addr = x_base + xs * X_STAGE_BYTES;
#pragma unroll
                for (int k = 0; k < SLAB_K / 16; ++k) {
                    umma_f16(tmem_base + static_cast<uint32_t>(h * SUB_N),
                              sdesc_kmajor_sw128(a_addr + k * 32), sdesc_kmajor_sw128(b_addr + k * 32),
                              IDESC, (kb > 0 || k > 0) ? 1u : 0u);
                }
                umma_commit(&x_empty[xs]);
            }
            if (ok) umma_commit(&a_empty[as]);
        }
        if (!ok) break;
        umma_commit(acc_full);
        ++accit;
    }
    // Wait until every MMA this thread issued has finished before TMEM is freed.
    umma_commit(drain);
    mbar_wait_drain(drain, 0);
}

__device__ __forceinline__ void epilogue_role(const SearchArgs &a, int64_t OT, int64_t U, int64_t TB,
                                              uint32_t tmem_base, uint64_t *acc_full,
                                              uint64_t *acc_empty, volatile int *abort_flag) {
    const int quad = (threadIdx.x / 32) & 3;
    const int lane = threadIdx.x & 31;
    const int r = quad * 32 + lane;
    const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
    uint32_t accit = 0;
    for (int64_t u = blockIdx.x; u < U; u += gridDim.x, ++accit) {
        const Unit un = decode(u, a, OT);
        const bool ok = mbar_wait(acc_full, accit & 1u, abort_flag);
        if (!__all_sync(0xffffffffu, ok)) return;
        tc_fence_after();
        float sum = 0.0f;
        for (int h = 0; h < un.nsub; ++h) {
#pragma unroll 1
            for (int c = 0; c < SUB_N / 32; ++c) {
                float v[32];
                tmem_ld32_wait(lane_addr + static_cast<uint32_t>(h * SUB_N + c * 32), v);
#pragma unroll
                for (int k = 0; k < 32; ++k) sum = __fmaf_rn(v[k], v[k], sum);
            }
        }
        tc_fence_before();
        mbar_arrive(acc_empty);
        const int64_t row = un.ot * TILE_O + r;
        if (row < a.O) a.part[(static_cast<int64_t>(un.g) * TB + un.tb) * a.O + row] = sum;
    }
}

template <bool WBF16, bool CLAMP>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    search_kernel(const __grid_constant__ CUtensorMap xmap, const SearchArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t *x_ring = base;
    uint8_t *a_ring = base + XS * X_STAGE_BYTES;
    uint64_t *bars = reinterpret_cast<uint64_t *>(a_ring + AS * A_STAGE_BYTES);
    uint64_t *x_full = bars;
    uint64_t *x_empty = x_full + XS;
    uint64_t *a_full = x_empty + XS;
    uint64_t *a_empty = a_full + AS;
    uint64_t *acc_full = a_empty + AS;
    uint64_t *acc_empty = acc_full + 1;
    uint64_t *drain = acc_empty + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
    const int64_t OT = (a.O + TILE_O - 1) / TILE_O;
    const int64_t TB = (a.N + TILE_N - 1) / TILE_N;
    const int64_t U = OT * TB * a.G;

    if (threadIdx.x == 0) {
        for (int s = 0; s < XS; ++s) {
            mbar_init(&x_full[s], 1);
            mbar_init(&x_empty[s], 1);
        }
        for (int s = 0; s < AS; ++s) {
            mbar_init(&a_full[s], NUM_PRODUCER_WARPS * 32);
            mbar_init(&a_empty[s], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, 4 * 32);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == WARP_MMA) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == WARP_TMA && lane == 0) tma_prefetch_desc(&xmap);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp < NUM_PRODUCER_WARPS) {
        producer_role<WBF16, CLAMP>(a, OT, U, a_ring, a_full, a_empty, abort_flag);
    } else if (warp < WARP_TMA) {
        epilogue_role(a, OT, U, TB, tmem_base, acc_full, acc_empty, abort_flag);
    } else if (warp == WARP_TMA) {
        if (lane == 0) tma_role(a, &xmap, OT, U, x_ring, x_full, x_empty, abort_flag);
    } else {
        if (lane == 0)
            mma_role(a, OT, U, tmem_base, x_ring, a_ring, x_full, x_empty, a_full, a_empty,
                     acc_full, acc_empty, drain, abort_flag);
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0 && *abort_flag) atomicExch(a.err, DEV_ERR_TIMEOUT);
    if (warp == WARP_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

template <bool WBF16, bool CLAMP>
cudaError_t launch_search_t(const SearchArgs &a, const CUtensorMap &xmap, int num_sms,
                            cudaStream_t st) {
    static bool attr_set[64] = {};   // per device and template instance
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64 || !attr_set[dev]) {
        e = cudaFuncSetAttribute(search_kernel<WBF16, CLAMP>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attr_set[dev] = true;
    }
    const int64_t OT = (a.O + TILE_O - 1) / TILE_O;
    const int64_t TB = (a.N + TILE_N - 1) / TILE_N;
    const int64_t U = OT * TB * a.G;
    const int grid = static_cast<int>(U < num_sms ? U : num_sms);
    search_kernel<WBF16, CLAMP><<<grid, NUM_THREADS, SMEM_BYTES, st>>>(xmap, a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_search(const SearchArgs &a, const CUtensorMap &xmap, int num_sms,
                          cudaStream_t st) {
    if (a.w_bf16)
        return a.clamp ? launch_search_t<true, true>(a, xmap, num_sms, st)
                       : launch_search_t<true, false>(a, xmap, num_sms, st);
    return a.clamp ? launch_search_t<false, true>(a, xmap, num_sms, st)
                   : launch_search_t<false, false>(a, xmap, num_sms, st);
}

}  // namespace awq
