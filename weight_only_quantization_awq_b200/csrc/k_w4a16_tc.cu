// W4A16 linear on the tensor cores, for prefill-sized M (AWQ guide, section 三,
// QuantLinear.forward: y = (x / s) * dequant(W)^T).
//
//   xs_absmax_kernel + xs_perm_kernel: xs = fp16((x / s16) * 2^-k), the power of
//                   two chosen from max |x / s16| so the largest magnitude lands in
//                   [2^14, 2^15), with the 8 columns of each packed word stored in
//                   the order (0,4,1,5,2,6,3,7) (see below); y is scaled back by 2^k.
//   w4a16_tc_kernel: one CTA per (128-row tile, token tile of 64, 128 or 256,
//                   K split); one K split whenever the tiles alone fill half the
//                   SMs, so most prefill shapes have no split-K partials.
//     warp 8 (TMA)  streams the packed codes [128 rows x 8 words] and the xs tile
//                   [N tokens x 64 columns] of each 64-column slab into a ring;
//     warps 0-7     dequantise: two threads per row (32 columns each); the next
//                   slab's Delta and z are loaded one slab ahead; a word's nibbles e and e+4 become one
//                   fp16x2 (1024 + code) with a shift and a LOP3 against the 0x6400
//                   magic; an exact HSUB2 of (1024 + z) and an HMUL2 by
//                   Delta * 2^-kd (kd from max Delta, so the products stay normal
//                   fp16) give the pair's dequantised weights with one rounding,
//                   written to the 128B-swizzled K-major A tile.  The pair order
//                   (e, e+4) is why xs is permuted the same way: the contraction
//                   over K is order-independent.  y = accumulator * 2^(kx + kd).
//     warp 9 (MMA)  one thread issues tcgen05.mma M=128 N=tokens K=16 (fp16 in,
//                   fp32 accumulate in TMEM).
//     warps 0-3     epilogue: tcgen05.ld of the accumulator; with one K split
//                   y is written directly, otherwise each split adds its fp32
//                   partial, still unscaled (normal-range values, untouched by the
//                   atomic's flush of subnormals), into a zeroed fp32 tile with
//                   red.global.add (the order of those adds across splits is not
//                   fixed) and the last CTA of the tile (counter) applies the
//                   power-of-two scales and converts the tile to bf16.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "awq_internal.h"
#include "awq_ptx.cuh"

namespace awq {

namespace {

constexpr int TC_DQ_WARPS = 8;       // dequantisation warps (2 threads per row)
constexpr int TC_WARP_TMA = 8;
constexpr int TC_WARP_MMA = 9;
constexpr int TC_THREADS = 10 * 32;
constexpr int TC_TOKENS = 256;       // max tokens per tile (MMA N)
constexpr int RS = 4;                // input ring stages
constexpr int AS_MAX = 8;            // A ring stages: as many as shared memory allows, up to 8
constexpr int Q_BYTES = 128 * 32;    // packed codes of a slab: 128 rows x 8 words
constexpr int A_BYTES = 128 * 128;   // bf16 A tile of a slab

__device__ __forceinline__ int perm8(int p) { return (p >> 1) + 4 * (p & 1); }   // position -> column

// max |x / s16| into max_bits[0] and max |Delta| into max_bits[2] (bit patterns of
// non-negative floats order as their values).
__global__ void __launch_bounds__(256) xs_absmax_kernel(const uint16_t *__restrict__ x,
                                                        const uint16_t *__restrict__ s16, int64_t M,
                                                        int64_t I, const uint16_t *__restrict__ scales,
                                                        int64_t n_scales, unsigned *__restrict__ max_bits) {
    float m = 0.0f, d = 0.0f;
    const int64_t step = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t k = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; k < M * I; k += step) {
        const int64_t c = k % I;
        const float xv = __uint_as_float(static_cast<uint32_t>(x[k]) << 16);
        m = fmaxf(m, fabsf(s16 ? __fdividef(xv, __half2float(__ushort_as_half(s16[c]))) : xv));
    }
    for (int64_t k = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; k < n_scales; k += step)
        d = fmaxf(d, fabsf(__half2float(__ushort_as_half(scales[k]))));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
        d = fmaxf(d, __shfl_xor_sync(0xffffffffu, d, off));
    }
    if ((threadIdx.x & 31) == 0) {
        atomicMax(max_bits, __float_as_uint(m));
        atomicMax(max_bits + 2, __float_as_uint(d));
    }
}

// Power-of-two exponent k with max * 2^-k in [2^(top-1), 2^top) (0 for a zero max),
// clamped to [-125, 125] so that 2^k and 2^-k stay normal floats.
__device__ __forceinline__ int pow2_exp(float mx, int top) {
    if (!(mx > 0.0f) || isinf(mx)) return 0;
    int e;
    frexpf(mx, &e);                                   // mx = f * 2^e, f in [0.5, 1)
    const int k = e - top;
    return k < -125 ? -125 : (k > 125 ? 125 : k);
}

// words: [0] max |xs| bits, [1] kx, [2] max |Delta| bits, [3] kd.
__global__ void xs_perm_kernel(const uint16_t *__restrict__ x, const uint16_t *__restrict__ s16,
                               int64_t M, int64_t I, unsigned *__restrict__ words,
                               uint16_t *__restrict__ xs) {
    const int k = pow2_exp(__uint_as_float(words[0]), 15);       // max |xs| -> [2^14, 2^15)
    const float sc = ldexpf(1.0f, -k);
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        words[1] = static_cast<unsigned>(k);
        words[3] = static_cast<unsigned>(pow2_exp(__uint_as_float(words[2]), 11));   // 15 * max Delta < 2^15
    }
    const int64_t total = M * I;
    for (int64_t q = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; q < total;
         q += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t m = q / I, c = q % I;
        const int64_t src = (c & ~int64_t(7)) + perm8(static_cast<int>(c & 7));
        const float xv = __uint_as_float(static_cast<uint32_t>(x[m * I + src]) << 16);
        const float v = s16 ? __fdividef(xv, __half2float(__ushort_as_half(s16[src]))) : xv;
        xs[q] = __half_as_ushort(__float2half_rn(v * sc));
    }
}

struct TcArgs {
    int64_t M, I, O;
    int gs;
    int n_tile;            // tokens per tile (multiple of 16, <= 256)
    int splits;            // K splits
    int slabs_per_split;
    int as;                // A ring stages
    const uint16_t *scales;
    const uint32_t *zeros;
    uint16_t *y;
    float *acc32;          // [M][O] fp32, zeroed (splits > 1)
    unsigned *counter;     // [row tiles * token tiles] (splits > 1), zeroed
    const unsigned *words; // [1] kx, [3] kd: the accumulator is y * 2^-(kx + kd)
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
__global__ void __launch_bounds__(TC_THREADS, 1)
    w4a16_tc_kernel(const __grid_constant__ TcMaps maps, const TcArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int xs_bytes = a.n_tile * 128;
    const int in_stage = (Q_BYTES + xs_bytes + 1023) / 1024 * 1024;
    const int AS = a.as;
    uint8_t *a_ring = base;                                  // AS x 16 KB (1024-aligned)
    uint8_t *in_ring = a_ring + AS * A_BYTES;                // RS x (xs tile | codes)
    uint64_t *bars = reinterpret_cast<uint64_t *>(in_ring + RS * in_stage);
    uint64_t *in_full = bars, *in_empty = bars + RS;
    uint64_t *a_full = in_empty + RS, *a_empty = a_full + AS_MAX;
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
    const uint32_t tcols = a.n_tile <= 32 ? 32 : (a.n_tile <= 64 ? 64 : (a.n_tile <= 128 ? 128 : 256));

    if (threadIdx.x == 0) {
        for (int s = 0; s < RS; ++s) {
            mbar_init(&in_full[s], 1);
            mbar_init(&in_empty[s], TC_DQ_WARPS + 1);   // dequant warps read the codes, the MMA reads xs
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
        tmem_alloc(tmem_slot, tcols);
        tmem_relinquish();
    }
    if (warp == TC_WARP_TMA && lane == 0) {
        tma_prefetch_desc(&maps.q);
        tma_prefetch_desc(&maps.xs);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == TC_WARP_TMA) {
        if (lane == 0) {
            int64_t last[RS];
#pragma unroll
            for (int s = 0; s < RS; ++s) last[s] = -1;
            for (int i = 0; i < nslab; ++i) {
                const uint32_t st = i % RS;
                if (!mbar_wait(&in_empty[st], ((i / RS) & 1u) ^ 1u, abort_flag)) break;
                uint8_t *dst = in_ring + st * in_stage;
                const int32_t kb = static_cast<int32_t>(kb0 + i);
                mbar_arrive_expect_tx(&in_full[st], Q_BYTES + xs_bytes);
                tma_load_2d(dst, &maps.xs, &in_full[st], kb * SLAB_K, static_cast<int32_t>(mt * a.n_tile));
                tma_load_2d(dst + xs_bytes, &maps.q, &in_full[st], kb * 8, static_cast<int32_t>(ot * 128));
#pragma unroll
                for (int s = 0; s < RS; ++s)
                    if (s == static_cast<int>(st)) last[s] = i;
            }
#pragma unroll
            for (int s = 0; s < RS; ++s)
                if (last[s] >= 0) mbar_wait_drain(&in_full[s], static_cast<uint32_t>((last[s] / RS) & 1));
        }
        __syncwarp();
    } else if (warp == TC_WARP_MMA) {
        if (lane == 0) {
            const uint32_t idesc = idesc_f16_f32(128, a.n_tile, false);
            const uint32_t a_base = smem_u32(a_ring), in_base = smem_u32(in_ring);
            bool ok = true;
            for (int i = 0; i < nslab && ok; ++i) {
                const uint32_t st = i % RS, as = i % AS;
                if (!mbar_wait(&a_full[as], (i / AS) & 1u, abort_flag) ||
                    !mbar_wait(&in_full[st], (i / RS) & 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t a_addr = a_base + as * A_BYTES;
                const uint32_t b_addr = in_base + st * in_stage;
#pragma unroll
                for (int k = 0; k < SLAB_K / 16; ++k)
                    umma_f16(tmem_base, sdesc_kmajor_sw128(a_addr + k * 32),
                             sdesc_kmajor_sw128(b_addr + k * 32), idesc, (i > 0 || k > 0) ? 1u : 0u);
                umma_commit(&in_empty[st]);
                umma_commit(&a_empty[as]);
            }
            if (ok) umma_commit(acc_full);
            umma_commit(drain);
            mbar_wait_drain(drain, 0);
        }
        __syncwarp();
    } else {
        // ---- dequantisation: two threads per row, 32 columns (4 packed words) each.
        const int r = threadIdx.x >> 1, hh = threadIdx.x & 1;
        const int64_t o = ot * 128 + r;
        const bool row_ok = o < a.O;
        const int64_t nG = a.I / a.gs, nzw = (nG + 7) / 8;
        const float dscale = ldexpf(1.0f, -static_cast<int>(a.words[3]));
        // Delta and (1024 + z) of this thread's group in slab i (fp16x2, exact).
        auto group_params = [&](int i, uint32_t &d2, uint32_t &z2) {
            float d = 0.0f, z = 8.0f;
            if (row_ok && i < nslab) {
                const int64_t g = ((kb0 + i) * SLAB_K + hh * 32) / a.gs;
                d = __half2float(__ushort_as_half(__ldg(a.scales + o * nG + g)));
                if (ZEROS) z = static_cast<float>((__ldg(a.zeros + o * nzw + g / 8) >> (4 * (g % 8))) & 0xFu);
            }
            d2 = h2pack(d * dscale);
            z2 = h2pack(1024.0f + z);
        };
        uint32_t d_cur, z_cur, d_nxt, z_nxt;
        group_params(0, d_cur, z_cur);
        bool ok = true;
        for (int i = 0; i < nslab; ++i) {
            const uint32_t st = i % RS, as = i % AS;
            group_params(i + 1, d_nxt, z_nxt);            // one slab ahead
            if (!mbar_wait(&in_full[st], (i / RS) & 1u, abort_flag)) { ok = false; break; }
            if (!mbar_wait(&a_empty[as], ((i / AS) & 1u) ^ 1u, abort_flag)) { ok = false; break; }
            const uint4 qw = *reinterpret_cast<const uint4 *>(in_ring + st * in_stage + xs_bytes + r * 32 + hh * 16);
            __syncwarp();
            if (lane == 0) mbar_arrive(&in_empty[st]);   // codes read (xs is released by the MMA)
            uint8_t *dst = a_ring + as * A_BYTES;
            const uint32_t wv[4] = {qw.x, qw.y, qw.z, qw.w};
#pragma unroll
            for (int wd = 0; wd < 4; ++wd) {
                uint32_t v[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    // nibbles e and e+4 -> fp16x2 (1024 + code) -> (code - z) * Delta * 2^-kd
                    const uint32_t b = ((wv[wd] >> (4 * e)) & 0x000F000Fu) | 0x64006400u;
                    v[e] = h2mul(h2sub(b, z_cur), d_cur);
                }
                *reinterpret_cast<uint4 *>(dst + sw128_offset(r, hh * 4 + wd)) = make_uint4(v[0], v[1], v[2], v[3]);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&a_full[as]);
            d_cur = d_nxt;
            z_cur = z_nxt;
        }
        if (warp < 4) {
        // ---- epilogue (warps 0-3): thread = TMEM lane = row of the tile
        const int64_t eo = ot * 128 + threadIdx.x;
        const bool erow_ok = eo < a.O;
        named_bar_sync(1, 128);
        const bool got = ok && nslab > 0 && mbar_wait_sleep(acc_full, 0, abort_flag);
        tc_fence_after();
        const int64_t m0 = mt * a.n_tile;
        const int mcount = static_cast<int>(a.M - m0 < a.n_tile ? a.M - m0 : a.n_tile);
        const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(warp * 32) << 16);
        // y = accumulator * 2^kx * 2^kd, two normal factors (their product can be subnormal)
        const float ysx = ldexpf(1.0f, static_cast<int>(a.words[1]));
        const float ysd = ldexpf(1.0f, static_cast<int>(a.words[3]));
        if (__all_sync(0xffffffffu, got)) {
            for (int c = 0; c < a.n_tile; c += 16) {
                uint32_t rv[16];
                tmem_ld16_wait(lane_addr + static_cast<uint32_t>(c), rv);
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    const int n = c + k;
                    if (n < mcount && erow_ok) {
                        const float acc = __uint_as_float(rv[k]);
                        if (a.splits == 1) {
                            a.y[(m0 + n) * a.O + eo] =
                                __bfloat16_as_ushort(__float2bfloat16_rn((acc * ysx) * ysd));
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
            named_bar_sync(1, 128);
            if (threadIdx.x == 0) {
                const unsigned prev = atomicAdd(&a.counter[tile], 1u);
                *is_last = prev == static_cast<unsigned>(a.splits - 1);
            }
            named_bar_sync(1, 128);
            if (*is_last) {
                __threadfence();
                if (erow_ok) {
#pragma unroll 8
                    for (int n = 0; n < mcount; ++n)
                        a.y[(m0 + n) * a.O + eo] = __bfloat16_as_ushort(
                            __float2bfloat16_rn((__ldcg(a.acc32 + (m0 + n) * a.O + eo) * ysx) * ysd));
                }
            }
        }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == TC_WARP_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem_base, tcols);
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
    p.counter_bytes = (OT * MT * 4 + 16 + 255) / 256 * 256;   // 4 scale words, tile counters
    return p;
}

cudaError_t launch_w4a16_tc(const uint16_t *x, int64_t M, int64_t I, int64_t O,
                            const uint16_t *scales, const uint32_t *zeros, const uint16_t *s16,
                            int gs, uint16_t *y, const TcPlan &plan, char *workspace,
                            const TcMaps &maps, cudaStream_t st) {
    const int64_t OT = (O + 127) / 128, MT = (M + plan.n_tile - 1) / plan.n_tile;
    uint16_t *xs = reinterpret_cast<uint16_t *>(workspace);
    float *acc32 = plan.splits > 1 ? reinterpret_cast<float *>(workspace + plan.xs_bytes) : nullptr;
    unsigned *words = reinterpret_cast<unsigned *>(workspace + plan.xs_bytes + plan.part_bytes);
    unsigned *xw = words;                                       // [4]: max|xs|, kx, max|Delta|, kd
    unsigned *counter = words + 4;                              // [OT * MT]
    // one memset zeroes the fp32 accumulator tile (if any), the scale words and the counters
    cudaError_t e = cudaMemsetAsync(workspace + plan.xs_bytes, 0, plan.part_bytes + plan.counter_bytes, st);
    if (e != cudaSuccess) return e;
    int blocks = static_cast<int>((M * I + 255) / 256);
    if (blocks > 148 * 8) blocks = 148 * 8;
    xs_absmax_kernel<<<blocks, 256, 0, st>>>(x, s16, M, I, scales, O * (I / gs), xw);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    xs_perm_kernel<<<blocks, 256, 0, st>>>(x, s16, M, I, xw, xs);
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
    a.words = xw;
    const int in_stage = (Q_BYTES + plan.n_tile * 128 + 1023) / 1024 * 1024;
    const int fixed = 1024 + RS * in_stage + (2 * RS + 2 * AS_MAX + 2) * 8 + 16;
    // Deep enough that dequantisation runs well ahead of the MMA completions, but
    // keep two CTAs per SM when the token tile is narrow.
    int as = (113 * 1024 - fixed) / A_BYTES;
    if (as < 3) as = (227 * 1024 - fixed) / A_BYTES;
    as = as > AS_MAX ? AS_MAX : (as < 2 ? 2 : as);
    a.as = as;
    const int smem = fixed + as * A_BYTES;
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
