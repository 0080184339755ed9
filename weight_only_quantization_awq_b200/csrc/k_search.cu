// Fused AWQ grid-search kernel for sm_100a.
//
// For grid point g, output rows [256*ot, 256*ot + 256) and tokens
// [512*tb, 512*tb + 512), it accumulates
//     E[o, n] = sum_i dW_g[o, i] * X[n, i],   dW_g = Q(W * s_g) / s_g - W
// on the 5th-generation tensor cores (fp16 operands, fp32 accumulation) and
// reduces sum_n E[o, n]^2 per row.  This is the objective
// L(s) = ||Q(W*s)(s^-1*X) - W X|| of the AWQ paper summary (Method), with the
// 1/s moved from X's columns onto the weight columns (exact in real
// arithmetic), evaluated for every s = s_X^alpha on the grid.  Neither dW nor E
// ever reaches global memory.
//
// CTA pairs (clusters of two, one CTA per SM, persistent over work units) run
// the pair form of the 5th-generation MMA: M = 256 rows, of which each CTA
// forms and holds 128 (its own rows of dW), and N = 256 tokens per
// instruction, of which each CTA stages 128 (half of each X tile).  Each CTA's
// TMEM receives its 128 rows x all 512 tokens of the unit.  So each SM streams
// and stores half of the X tiles a single-CTA MMA of the same shape would need
// (the tensor cores of the pair read each other's halves).
//
// Warp roles (736 threads per CTA):
//   warps 0-15  dW producers (16 columns of one row per thread): read one slab's
//               inputs (W tile, s and -1/s, group parameters) from shared
//               memory, form dW for the CTA's 128 rows x 64 columns, write it
//               as fp16 into shared memory in the 128-byte-swizzled K-major
//               layout the MMA reads, arrive on the leader's a_full.
//   warps 16-19 epilogue: tcgen05.ld of the CTA's 128 x 512 fp32 accumulator
//               (lane = output row), square-and-sum per row, one fp32 partial
//               per (grid point, token block, row); each 256-column half is
//               handed back to the MMA as soon as it has been read.
//   warp 20     TMA, one lane: this CTA's half of the X tiles (128 tokens x 64
//               channels, fp16 copy of X scaled by a power of two) into the X
//               ring, counted on the leader's x_full.
//   warp 21     TMA, one lane: each slab's producer inputs into the (local) input
//               ring.  (The two loaders wait on different barriers, so each has a
//               warp of its own.)
//   warp 22     MMA: both CTAs allocate 512 TMEM columns as a pair; in the
//               leader (rank 0) one thread issues tcgen05.mma.cta_group::2
//               M=256 N=256 K=16 (two N=256 halves per slab), and
//               tcgen05.commit with a multicast arrive releases both CTAs' ring
//               stages and accumulators.
// Work units are (g fastest, then 256-row output tile, then token block) and
// are dealt round-robin to the pairs, so the pairs running at one time share a
// few W tiles and X blocks in L2.
#include <cuda_bf16.h>

#include "awq_internal.h"
#include "awq_ptx.cuh"

namespace awq {

namespace {

constexpr int NUM_PRODUCER_WARPS = 16;
constexpr int EPI_WARP0 = 16;                          // warps 16-19: TMEM lane quadrants 0-3
constexpr int WARP_TMA = 20;                           // X tiles
constexpr int WARP_IN = 21;                            // producer inputs
constexpr int WARP_MMA = 22;
constexpr int NUM_THREADS = 23 * 32;
constexpr int PAIR_O = 2 * TILE_O;                     // output rows per CTA pair
constexpr int X_HALF = SUB_N / 2;                      // tokens of an N = 256 tile per CTA
constexpr int X_STAGE_BYTES = X_HALF * SLAB_K * 2;     // 16 KB of fp16 X
constexpr int A_STAGE_BYTES = TILE_O * SLAB_K * 2;     // 16 KB of fp16 dW
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t IDESC = idesc_f16_f32(PAIR_O, SUB_N, false);   // M = 256 (pair), N = 256
constexpr uint16_t PAIR_MASK = 0x3;                    // multicast to both CTAs of the pair
constexpr float MAGIC = 12582912.0f;                   // 1.5 * 2^23: x + MAGIC - MAGIC = rint(x)

// Shared-memory plan, per weight type.  Input stage = W tile, then s / -1/s of
// the slab (2 x 64 fp32), then the group parameters [1 or 2 groups][128 rows] float4.
template <bool WBF16>
struct Plan {
    static constexpr int XS = 6;                        // X ring stages (two per slab)
    static constexpr int AS = 3;                        // dW ring stages
    static constexpr int IS = WBF16 ? 3 : 2;            // input ring stages
    static constexpr int W_BYTES = WBF16 ? 16384 : 32768;
    static constexpr int SN_OFF = W_BYTES;
    static constexpr int QP_OFF = SN_OFF + 512;
    static constexpr int IN_STAGE = ((QP_OFF + 4096) + 1023) / 1024 * 1024;
    static constexpr int NUM_BARS = 2 * XS + 2 * AS + 2 * IS + 5;
    static constexpr int SMEM_BYTES =
        1024 + XS * X_STAGE_BYTES + AS * A_STAGE_BYTES + IS * IN_STAGE + NUM_BARS * 8 + 16;
};
static_assert(Plan<true>::SMEM_BYTES <= 232448, "shared memory plan (bf16 W) too large");
static_assert(Plan<false>::SMEM_BYTES <= 232448, "shared memory plan (fp32 W) too large");

struct Unit {
    int g;
    int64_t ot, tb;
    int nsub;
};

// The pair (cluster) this CTA belongs to, and the number of pairs.
__device__ __forceinline__ int64_t pair_id() { return blockIdx.x >> 1; }
__device__ __forceinline__ int64_t pair_count() { return gridDim.x >> 1; }

// OT counts 256-row pair tiles.
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
// a different code than the correctly rounded quotient.  Every rounding
// decision that survives the code clamp has |W'/Delta| <= 15.5 (codes span at
// most 16 levels around 0), where W' * RN(1/Delta) and RN(W'/Delta) differ by at
// most 16 * 2^-23 = 2^-19; beyond that both sides saturate to the same code.
constexpr float TIE_BAND = 0.5f - 1.0f / 65536.0f;

__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }

// dW for 8 adjacent columns of one row (one group), packed as 4 x fp16x2, on
// packed f32x2 arithmetic.  With t = RN(W' * (1/Delta) + MAGIC):
//   nq = MAGIC - t = -q exactly,   frac = W' * (1/Delta) - q,
//   d  = W' - q*Delta,             dW = d * (-1/s) = (q*Delta - W') / s.
// Codes follow the quantizer's definition q = rint(RN(W'/Delta)): any element
// whose reciprocal product lies within 2^-16 of a half-integer (exact ties
// included) is redone with the correctly rounded division.
// prm = {Delta, 1/Delta, -qhi, -qlo}; ns = -1/s.
template <bool CLAMP>
__device__ __forceinline__ uint4 dw_chunk8(const float (&w)[8], const float4 &s0, const float4 &s1,
                                           const float4 &n0, const float4 &n1, const float4 &prm) {
    const float2 invD = f2(prm.y, prm.y), D = f2(prm.x, prm.x);
    const float2 M2 = f2(MAGIC, MAGIC), NEG1 = f2(-1.0f, -1.0f);
    const float2 sv[4] = {f2(s0.x, s0.y), f2(s0.z, s0.w), f2(s1.x, s1.y), f2(s1.z, s1.w)};
    const float2 nv[4] = {f2(n0.x, n0.y), f2(n0.z, n0.w), f2(n1.x, n1.y), f2(n1.z, n1.w)};
    float2 wp[4], nq[4];
    float worst = 0.0f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        wp[e] = __fmul2_rn(f2(w[2 * e], w[2 * e + 1]), sv[e]);
        const float2 t = __ffma2_rn(wp[e], invD, M2);
        nq[e] = __ffma2_rn(t, NEG1, M2);
        const float2 fr = __ffma2_rn(wp[e], invD, nq[e]);
        worst = fmaxf(worst, fmaxf(fabsf(fr.x), fabsf(fr.y)));
    }
    if (worst > TIE_BAND) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            if (prm.x != 0.0f) {
                nq[e].x = -rintf(__fdiv_rn(wp[e].x, prm.x));
                nq[e].y = -rintf(__fdiv_rn(wp[e].y, prm.x));
            }
        }
    }
    uint32_t out[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        float2 n = nq[e];
        if (CLAMP) {
            n.x = fminf(fmaxf(n.x, prm.z), prm.w);
            n.y = fminf(fmaxf(n.y, prm.z), prm.w);
        }
        const float2 d = __ffma2_rn(n, D, wp[e]);        // W' - q*Delta
        const float2 r = __fmul2_rn(d, nv[e]);           // (q*Delta - W') / s
        out[e] = f16x2_satfinite(r.x, r.y);
    }
    return make_uint4(out[0], out[1], out[2], out[3]);
}

template <bool WBF16, bool CLAMP>
__device__ __forceinline__ void producer_role(const SearchArgs &a, int64_t U,
                                              const uint8_t *in_ring, uint64_t *in_full,
                                              uint64_t *in_empty, uint8_t *a_ring,
                                              uint64_t *a_full, uint64_t *a_empty,
                                              volatile int *abort_flag) {
    // a_full lives in the leader CTA and counts the producer warps of both CTAs.
    using P = Plan<WBF16>;
    const int t = threadIdx.x;          // 0..511
    const int r = t >> 2, qc = t & 3;   // row in tile, 16-column quarter of the 64-wide slab
    const int lane = t & 31;
    const int jq = a.gs == 32 ? (qc >> 1) : 0;   // which of the slab's groups (stage holds [groups][128 rows])
    const int64_t nK = a.I / SLAB_K;
    uint32_t it = 0;
    for (int64_t u = pair_id(); u < U; u += pair_count()) {
        for (int64_t kb = 0; kb < nK; ++kb, ++it) {
            const uint32_t is = it % P::IS, as = it % P::AS;
            if (!mbar_wait(&in_full[is], (it / P::IS) & 1u, abort_flag, a.wait)) return;
            const uint8_t *in = in_ring + is * P::IN_STAGE;
            uint8_t *dst = a_ring + as * A_STAGE_BYTES;
            // Read all of this thread's inputs of the slab (16 weights, their s and
            // -1/s, the group parameters), then hand the input stage back at once so
            // the next slab's copy can land while this one is computed.
            const float4 prm = reinterpret_cast<const float4 *>(in + P::QP_OFF)[jq * TILE_O + r];
            float w[2][8];
            float4 sv[2][4];
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                // Quarters 2-3 take their two 8-column chunks in the opposite order, so
                // the s / -1/s loads of one warp instruction never share banks.
                const int c = cc ^ (qc >> 1);
                const int ch = qc * 2 + c;                 // 16-byte chunk within the 128-byte row
                const float *s_sm = reinterpret_cast<const float *>(in + P::SN_OFF) + ch * 8;
                if constexpr (WBF16) {
                    const uint4 v = *reinterpret_cast<const uint4 *>(in + sw128_offset(r, ch));
                    const uint32_t u4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        w[cc][2 * k] = __uint_as_float(u4[k] << 16);
                        w[cc][2 * k + 1] = __uint_as_float(u4[k] & 0xFFFF0000u);
                    }
                } else {
                    const uint8_t *sub = in + (ch >> 2) * 16384;   // 32-column fp32 sub-tile
                    const int sc = (ch & 3) * 2;                     // its 16-byte chunks
                    const float4 v0 = *reinterpret_cast<const float4 *>(sub + sw128_offset(r, sc));
                    const float4 v1 = *reinterpret_cast<const float4 *>(sub + sw128_offset(r, sc + 1));
                    w[cc][0] = v0.x; w[cc][1] = v0.y; w[cc][2] = v0.z; w[cc][3] = v0.w;
                    w[cc][4] = v1.x; w[cc][5] = v1.y; w[cc][6] = v1.z; w[cc][7] = v1.w;
                }
                sv[cc][0] = *reinterpret_cast<const float4 *>(s_sm);
                sv[cc][1] = *reinterpret_cast<const float4 *>(s_sm + 4);
                sv[cc][2] = *reinterpret_cast<const float4 *>(s_sm + 64);
                sv[cc][3] = *reinterpret_cast<const float4 *>(s_sm + 68);
            }
            // One arrival per warp: the warp barrier orders every lane's reads
            // before lane 0's arrive.
            __syncwarp();
            if (lane == 0) mbar_arrive(&in_empty[is]);
            if (!mbar_wait(&a_empty[as], ((it / P::AS) & 1u) ^ 1u, abort_flag, a.wait)) return;
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                const int ch = qc * 2 + (cc ^ (qc >> 1));
                *reinterpret_cast<uint4 *>(dst + sw128_offset(r, ch)) =
                    dw_chunk8<CLAMP>(w[cc], sv[cc][0], sv[cc][1], sv[cc][2], sv[cc][3], prm);
            }
            // One arrival per warp: every lane's fenced writes are ordered before
            // lane 0's arrive by the warp barrier.
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(cluster_addr(&a_full[as], 0));
        }
    }
}

// Lane 1 of the TMA warp: the producers' inputs, one stage per (unit, slab).
template <bool WBF16>
__device__ __forceinline__ void input_loader(const SearchArgs &a, const SearchMaps &m, int64_t OT,
                                             int64_t U, uint8_t *in_ring, uint64_t *in_full,
                                             uint64_t *in_empty, volatile int *abort_flag) {
    using P = Plan<WBF16>;
    const int64_t nK = a.I / SLAB_K;
    const int gps = a.gs == 32 ? 2 : 1;
    const uint32_t bytes = P::W_BYTES + 512 + 2048 * gps;
    uint32_t it = 0;
    int64_t last[P::IS];
#pragma unroll
    for (int s = 0; s < P::IS; ++s) last[s] = -1;
    bool ok = true;
    for (int64_t u = pair_id(); u < U && ok; u += pair_count()) {
        const Unit un = decode(u, a, OT);
        const int32_t y_w = static_cast<int32_t>(un.ot * PAIR_O + cluster_ctarank() * TILE_O);
        const int64_t nG = a.I / a.gs;
        for (int64_t kb = 0; kb < nK; ++kb, ++it) {
            const uint32_t st = it % P::IS;
            if (!mbar_wait(&in_empty[st], ((it / P::IS) & 1u) ^ 1u, abort_flag, a.wait)) {
                ok = false;
                break;
            }
            uint8_t *dst = in_ring + st * P::IN_STAGE;
            const int32_t x = static_cast<int32_t>(kb * SLAB_K);
            mbar_arrive_expect_tx(&in_full[st], bytes);
            if constexpr (WBF16) {
                tma_load_2d(dst, &m.w, &in_full[st], x, y_w);
            } else {
                tma_load_2d(dst, &m.w, &in_full[st], x, y_w);
                tma_load_2d(dst + 16384, &m.w, &in_full[st], x + 32, y_w);
            }
            tma_load_2d(dst + P::SN_OFF, &m.sn, &in_full[st], x, 2 * un.g);
            tma_load_3d(dst + P::QP_OFF, &m.qp, &in_full[st], 0, y_w,
                        static_cast<int32_t>(static_cast<int64_t>(un.g) * nG + (kb * SLAB_K) / a.gs));
#pragma unroll
            for (int s = 0; s < P::IS; ++s)
                if (s == static_cast<int>(st)) last[s] = it;
        }
    }
    // Never leave the CTA with a copy still landing in its shared memory.
#pragma unroll
    for (int s = 0; s < P::IS; ++s)
        if (last[s] >= 0) mbar_wait_drain(&in_full[s], static_cast<uint32_t>((last[s] / P::IS) & 1), a.wait);
}

// Lane 0 of the TMA warp: this CTA's half (128 tokens) of each X tile for the
// pair MMA.  The leader expects the bytes of both halves on its x_full; the
// peer's copy completes on the leader's barrier too.  Before refilling a stage
// each CTA waits for its own x_empty, which the leader's MMA commit signals in
// both CTAs.  (A copy still in flight when the loop stops was issued at least a
// full wait bound earlier, so it has landed before the CTA exits.)
template <int XS>
__device__ __forceinline__ void x_loader(const SearchArgs &a, const CUtensorMap *xmap, int64_t OT,
                                         int64_t U, uint8_t *x_ring, uint64_t *x_full,
                                         uint64_t *x_empty, volatile int *abort_flag) {
    const int64_t nK = a.I / SLAB_K;
    const uint32_t rank = cluster_ctarank();
    uint32_t it = 0;
    bool ok = true;
    for (int64_t u = pair_id(); u < U && ok; u += pair_count()) {
        const Unit un = decode(u, a, OT);
        for (int64_t kb = 0; kb < nK && ok; ++kb) {
            for (int h = 0; h < un.nsub; ++h, ++it) {
                const uint32_t stage = it % XS, phase = (it / XS) & 1u;
                if (!mbar_wait(&x_empty[stage], phase ^ 1u, abort_flag, a.wait)) {
                    ok = false;
                    break;
                }
                if (rank == 0) mbar_arrive_expect_tx(&x_full[stage], 2 * X_STAGE_BYTES);
                tma_load_2d_pair(x_ring + stage * X_STAGE_BYTES, xmap, cluster_addr(&x_full[stage], 0),
                                 static_cast<int32_t>(kb * SLAB_K),
                                 static_cast<int32_t>(un.tb * TILE_N + h * SUB_N + rank * X_HALF));
            }
        }
    }
}

template <int XS, int AS>
__device__ __forceinline__ void mma_role(const SearchArgs &a, int64_t OT, int64_t U,
                                         uint32_t tmem_base, uint8_t *x_ring, uint8_t *a_ring,
                                         uint64_t *x_full, uint64_t *x_empty, uint64_t *a_full,
                                         uint64_t *a_empty, uint64_t *acc_full,
                                         uint64_t *acc_empty, uint64_t *drain,
                                         volatile int *abort_flag) {
    const int64_t nK = a.I / SLAB_K;
    uint32_t ait = 0, xit = 0;
    uint32_t hit[2] = {0u, 0u};                    // units that have used each accumulator half
    const uint32_t x_base = smem_u32(x_ring), a_base = smem_u32(a_ring);
    bool ok = true;
    for (int64_t u = pair_id(); u < U && ok; u += pair_count()) {
        const Unit un = decode(u, a, OT);
        for (int64_t kb = 0; kb < nK && ok; ++kb, ++ait) {
            const uint32_t as = ait % AS;
            if (!mbar_wait(&a_full[as], (ait / AS) & 1u, abort_flag, a.wait)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t a_addr = a_base + as * A_STAGE_BYTES;
            for (int h = 0; h < un.nsub; ++h, ++xit) {
                // each 256-column half of the accumulator is waited for separately, so
                // this unit starts on half 0 while the epilogue still drains half 1
                if (kb == 0) {
                    if (!mbar_wait(&acc_empty[h], (hit[h] & 1u) ^ 1u, abort_flag, a.wait)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                }
                const uint32_t xs = xit % XS;
                if (!mbar_wait(&x_full[xs], (xit / XS) & 1u, abort_flag, a.wait)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t b_addr = x_base + xs * X_STAGE_BYTES;
#pragma unroll
                for (int k = 0; k < SLAB_K / 16; ++k) {
                    umma_f16_pair(tmem_base + static_cast<uint32_t>(h * SUB_N),
                                  sdesc_kmajor_sw128(a_addr + k * 32), sdesc_kmajor_sw128(b_addr + k * 32),
                                  IDESC, (kb > 0 || k > 0) ? 1u : 0u);
                }
                umma_commit_pair(&x_empty[xs], PAIR_MASK);
                if (kb == nK - 1) umma_commit_pair(&acc_full[h], PAIR_MASK);
            }
            if (ok) umma_commit_pair(&a_empty[as], PAIR_MASK);
        }
        if (!ok) break;
        for (int h = 0; h < un.nsub; ++h) ++hit[h];
    }
    // Both CTAs wait on their drain barrier until every MMA issued here has
    // finished, before TMEM is freed.
    umma_commit_pair(drain, PAIR_MASK);
}

__device__ __forceinline__ void epilogue_role(const SearchArgs &a, int64_t OT, int64_t U, int64_t TB,
                                              uint32_t tmem_base, uint64_t *acc_full,
                                              uint64_t *acc_empty, volatile int *abort_flag) {
    const int quad = (threadIdx.x / 32) & 3;
    const int lane = threadIdx.x & 31;
    const int r = quad * 32 + lane;
    const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
    uint32_t hit[2] = {0u, 0u};                    // units that have used each accumulator half
    for (int64_t u = pair_id(); u < U; u += pair_count()) {
        const Unit un = decode(u, a, OT);
        float sum = 0.0f;
        for (int h = 0; h < un.nsub; ++h) {
            const bool ok = mbar_wait_sleep(&acc_full[h], hit[h] & 1u, abort_flag, a.wait);
            if (!__all_sync(0xffffffffu, ok)) return;
            tc_fence_after();
#pragma unroll 1
            for (int c = 0; c < SUB_N / 32; ++c) {
                float v[32];
                tmem_ld32_wait(lane_addr + static_cast<uint32_t>(h * SUB_N + c * 32), v);
#pragma unroll
                for (int k = 0; k < 32; ++k) sum = __fmaf_rn(v[k], v[k], sum);
            }
            // this half may be overwritten by the next unit as soon as both CTAs' epilogues have read it
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(cluster_addr(&acc_empty[h], 0));
            ++hit[h];
        }
        const int64_t row = un.ot * PAIR_O + cluster_ctarank() * TILE_O + r;
        if (row < a.O) a.part[(static_cast<int64_t>(un.g) * TB + un.tb) * a.O + row] = sum;
    }
}

template <bool WBF16, bool CLAMP>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    search_kernel(const __grid_constant__ SearchMaps maps, const SearchArgs a) {
    using P = Plan<WBF16>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t *x_ring = base;
    uint8_t *a_ring = x_ring + P::XS * X_STAGE_BYTES;
    uint8_t *in_ring = a_ring + P::AS * A_STAGE_BYTES;
    uint64_t *bars = reinterpret_cast<uint64_t *>(in_ring + P::IS * P::IN_STAGE);
    uint64_t *x_full = bars;
    uint64_t *x_empty = x_full + P::XS;
    uint64_t *a_full = x_empty + P::XS;
    uint64_t *a_empty = a_full + P::AS;
    uint64_t *in_full = a_empty + P::AS;
    uint64_t *in_empty = in_full + P::IS;
    uint64_t *acc_full = in_empty + P::IS;         // [2]: one per 256-column accumulator half
    uint64_t *acc_empty = acc_full + 2;            // [2]
    uint64_t *drain = acc_empty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const int64_t OT = (a.O + PAIR_O - 1) / PAIR_O;
    const int64_t TB = (a.N + TILE_N - 1) / TILE_N;
    const int64_t U = OT * TB * a.G;

    // Barrier counts.  Leader-only barriers (x_full, a_full, acc_empty) count
    // arrivals from both CTAs; the peer initialises its copies but never waits
    // on them.
    if (threadIdx.x == 0) {
        for (int s = 0; s < P::XS; ++s) {
            mbar_init(&x_full[s], 1);                       // leader's expect_tx; bytes of both halves
            mbar_init(&x_empty[s], 1);                      // the leader's multicast commit
        }
        for (int s = 0; s < P::AS; ++s) {
            mbar_init(&a_full[s], 2 * NUM_PRODUCER_WARPS);  // producer warps of both CTAs
            mbar_init(&a_empty[s], 1);
        }
        for (int s = 0; s < P::IS; ++s) {
            mbar_init(&in_full[s], 1);
            mbar_init(&in_empty[s], NUM_PRODUCER_WARPS);
        }
        for (int h = 0; h < 2; ++h) {
            mbar_init(&acc_full[h], 1);
            mbar_init(&acc_empty[h], 2 * 4);                // epilogue warps of both CTAs
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == WARP_MMA) {
        tmem_alloc_pair(tmem_slot, TMEM_COLS);
        tmem_relinquish_pair();
    }
    if (warp == WARP_TMA && lane == 0) {
        tma_prefetch_desc(&maps.x);
        tma_prefetch_desc(&maps.w);
        tma_prefetch_desc(&maps.sn);
        tma_prefetch_desc(&maps.qp);
    }
    // Both CTAs' barriers are initialised, and TMEM allocated, before either
    // CTA signals the other.
    tc_fence_before();
    cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp < NUM_PRODUCER_WARPS) {
        producer_role<WBF16, CLAMP>(a, U, in_ring, in_full, in_empty, a_ring, a_full, a_empty,
                                    abort_flag);
    } else if (warp < EPI_WARP0 + 4) {
        epilogue_role(a, OT, U, TB, tmem_base, acc_full, acc_empty, abort_flag);
    } else if (warp == WARP_TMA) {
        if (lane == 0) x_loader<P::XS>(a, &maps.x, OT, U, x_ring, x_full, x_empty, abort_flag);
        __syncwarp();
    } else if (warp == WARP_IN) {
        if (lane == 0) input_loader<WBF16>(a, maps, OT, U, in_ring, in_full, in_empty, abort_flag);
        __syncwarp();
    } else {
        if (lane == 0 && rank == 0)
            mma_role<P::XS, P::AS>(a, OT, U, tmem_base, x_ring, a_ring, x_full, x_empty, a_full,
                                   a_empty, acc_full, acc_empty, drain, abort_flag);
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    // Every pair MMA has finished (the leader's last commit reaches both CTAs)
    // before TMEM is freed, and neither CTA leaves while the other may still
    // signal its barriers or read its shared memory.
    if (warp == WARP_MMA && lane == 0) mbar_wait_drain(drain, 0, a.wait);
    __syncwarp();
    cluster_sync_all();
    if (threadIdx.x == 0 && *abort_flag) atomicExch(a.err, DEV_ERR_TIMEOUT);
    if (warp == WARP_MMA) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, TMEM_COLS);
    }
}

template <bool WBF16, bool CLAMP>
cudaError_t launch_search_t(const SearchArgs &a, const SearchMaps &maps, int num_sms,
                            cudaStream_t st) {
    constexpr int smem = Plan<WBF16>::SMEM_BYTES;
    static bool attr_set[64] = {};   // per device and template instance
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64 || !attr_set[dev]) {
        e = cudaFuncSetAttribute(search_kernel<WBF16, CLAMP>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attr_set[dev] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(NUM_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // Persistent: as many pairs as can be resident at once (one CTA per SM).
    static int max_pairs[64] = {};
    int pairs_fit = (dev >= 0 && dev < 64) ? max_pairs[dev] : 0;
    if (pairs_fit == 0) {
        cfg.gridDim = dim3(static_cast<unsigned>(2 * (num_sms / 2)));
        e = cudaOccupancyMaxActiveClusters(&pairs_fit, search_kernel<WBF16, CLAMP>, &cfg);
        if (e != cudaSuccess) return e;
        if (pairs_fit < 1) return cudaErrorInvalidConfiguration;
        if (dev >= 0 && dev < 64) max_pairs[dev] = pairs_fit;
    }
    const int64_t OT = (a.O + PAIR_O - 1) / PAIR_O;
    const int64_t TB = (a.N + TILE_N - 1) / TILE_N;
    const int64_t U = OT * TB * a.G;
    const int64_t pairs = U < pairs_fit ? U : pairs_fit;
    cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs));
    return cudaLaunchKernelEx(&cfg, search_kernel<WBF16, CLAMP>, maps, a);
}

}  // namespace

cudaError_t launch_search(const SearchArgs &a, const SearchMaps &maps, int num_sms,
                          cudaStream_t st) {
    if (a.w_bf16)
        return a.clamp ? launch_search_t<true, true>(a, maps, num_sms, st)
                       : launch_search_t<true, false>(a, maps, num_sms, st);
    return a.clamp ? launch_search_t<false, true>(a, maps, num_sms, st)
                   : launch_search_t<false, false>(a, maps, num_sms, st);
}

}  // namespace awq
