// W4A16 linear that applies the search result (AWQ guide, section 三,
// QuantLinear.forward: x is rescaled by the per-channel scale, the INT4 weight
// is dequantised group by group, then a plain linear):
//     y[m, o] = sum_g Delta[o, g] * ( sum_{i in g} xs[m, i] * code[o, i]  -  z[o, g] * sum_{i in g} xs[m, i] )
//     xs = x / s16
//
// Fallback decode kernel for M <= 4 at input widths whose activations the
// streaming kernel (k_w4a16_stream.cu) cannot stage.  One warp streams one
// output row at a time: each lane owns 4 consecutive packed words (32 columns,
// inside one group) of every 1024-column block of the row and issues all of
// its 16-byte loads before using any.  A nibble becomes an exact float with a
// single LOP3 against a position-dependent magic (the nibble sits in the
// mantissa, value 2^23 + code * 16^j); one packed f32x2 add removes the magic
// and one packed f32x2 FMA multiplies by xs / 16^j, which the block staged in
// shared memory once, pre-scaled and laid out lane-interleaved so every warp
// load is conflict-free.  The sum of xs over each lane's 32 columns (which lie
// in one group) turns the zero point into one multiply per 32 columns.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "awq_internal.h"

namespace awq {

namespace {

constexpr int W4_THREADS = 256;
constexpr int W4_WARPS = W4_THREADS / 32;
constexpr int BLK_COLS = 1024;            // columns per lane-interleaved block (32 lanes x 32)
constexpr float MAGIC23 = 8388608.0f;     // 2^23

// Index (in float2 units) of pair (word wd in 0..3, position j in 0..3) of lane l
// in 1024-column block b: pairs hold the columns of nibble j and nibble j + 4.
// Lanes are XOR-swizzled by (wd, j): the compute loop's loads (fixed wd, j, all
// lanes) and the staging stores (fixed lane, all wd, j) are both conflict-free.
__device__ __forceinline__ int xs_pair_index(int b, int wd, int j, int l) {
    return ((b * 4 + wd) * 4 + j) * 32 + (l ^ (wd * 4 + j));
}

template <int MT, bool ZEROS>
__global__ void __launch_bounds__(W4_THREADS) w4a16_decode_kernel(
    const uint16_t *__restrict__ x, int64_t M, int I, int64_t O,
    const uint32_t *__restrict__ qweight, const uint16_t *__restrict__ scales,
    const uint32_t *__restrict__ zeros, const uint16_t *__restrict__ s16, int gs,
    uint16_t *__restrict__ y) {
    extern __shared__ float4 smem4[];
    const int NB = (I + BLK_COLS - 1) / BLK_COLS;           // column blocks (last may be partial)
    const int nG = I / gs;
    const int xs_floats = NB * BLK_COLS;                    // per token, padded
    float2 *xs = reinterpret_cast<float2 *>(smem4);         // [MT][xs_floats / 2]
    float *lsum = reinterpret_cast<float *>(smem4) + MT * xs_floats;   // [MT][NB * 32]
    const int64_t m0 = static_cast<int64_t>(blockIdx.y) * MT;
    const int mt = static_cast<int>(M - m0 < MT ? M - m0 : MT);

    // ---- stage xs = x / s, pre-scaled by 16^-j and lane-interleaved (coalesced reads).
    float *xsf = reinterpret_cast<float *>(smem4);
    for (int k = threadIdx.x; k < MT * xs_floats; k += W4_THREADS) {
        const int m = k / xs_floats, c = k % xs_floats;
        const int b = c >> 10, l = (c >> 5) & 31, e = c & 31;
        const int wd = e >> 3, j = e & 3, half = (e >> 2) & 1;
        float v = 0.0f;
        if (m < mt && c < I) {
            const float inv16 = j == 0 ? 1.0f : (j == 1 ? 0.0625f : (j == 2 ? 0.00390625f : 0.000244140625f));
            const float rs = s16 ? __frcp_rn(__half2float(__ushort_as_half(s16[c]))) : 1.0f;
            v = __uint_as_float(static_cast<uint32_t>(x[(m0 + m) * I + c]) << 16) * (rs * inv16);
        }
        xsf[m * xs_floats + 2 * xs_pair_index(b, wd, j, l) + half] = v;
    }
    __syncthreads();
    // ---- sum of xs over each lane's 32 columns, from the staged pairs.
    for (int k = threadIdx.x; k < MT * NB * 32; k += W4_THREADS) {
        const int m = k / (NB * 32), b = (k / 32) % NB, l = k & 31;
        float acc = 0.0f;
#pragma unroll
        for (int wd = 0; wd < 4; ++wd) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float2 v = xs[m * (xs_floats / 2) + xs_pair_index(b, wd, j, l)];
                acc = fmaf(v.x + v.y, static_cast<float>(1 << (4 * j)), acc);
            }
        }
        lsum[k] = acc;
    }
    __syncthreads();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int wpr = I / 8;
    const int64_t nzw = (nG + 7) / 8;
    const int64_t warps_total = static_cast<int64_t>(gridDim.x) * W4_WARPS;
    const float2 NEGM = make_float2(-MAGIC23, -MAGIC23);
    for (int64_t o = static_cast<int64_t>(blockIdx.x) * W4_WARPS + warp; o < O; o += warps_total) {
        const uint32_t *qrow = qweight + o * wpr;
        float acc[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[m] = 0.0f;
        for (int b0 = 0; b0 < NB; b0 += 8) {
            // Issue every load of up to 8 blocks before using any.
            uint4 qv[8];
            float dv[8], zv[8];
#pragma unroll
            for (int bb = 0; bb < 8; ++bb) {
                const int b = b0 + bb;
                const int c = b * BLK_COLS + lane * 32;
                qv[bb] = make_uint4(0u, 0u, 0u, 0u);
                dv[bb] = 0.0f;
                zv[bb] = 0.0f;
                if (b < NB && c < I) {
                    qv[bb] = __ldg(reinterpret_cast<const uint4 *>(qrow + c / 8));
                    const int g = c / gs;
                    dv[bb] = __half2float(__ushort_as_half(__ldg(scales + o * nG + g)));
                    if (ZEROS)
                        zv[bb] = static_cast<float>((__ldg(zeros + o * nzw + g / 8) >> (4 * (g % 8))) & 0xFu);
                    else
                        zv[bb] = 8.0f;
                }
            }
#pragma unroll
            for (int bb = 0; bb < 8; ++bb) {
                const int b = b0 + bb;
                const int c = b * BLK_COLS + lane * 32;
                if (b >= NB || c >= I) continue;
                const uint32_t wds[4] = {qv[bb].x, qv[bb].y, qv[bb].z, qv[bb].w};
                float2 part[MT];
#pragma unroll
                for (int m = 0; m < MT; ++m) part[m] = make_float2(0.0f, 0.0f);
#pragma unroll
                for (int wd = 0; wd < 4; ++wd) {
                    const uint32_t lo = wds[wd], hi = wds[wd] >> 16;
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint32_t mask = 0xFu << (4 * j);
                        const float2 f = make_float2(__uint_as_float((lo & mask) | 0x4B000000u),
                                                     __uint_as_float((hi & mask) | 0x4B000000u));
                        const float2 q = __fadd2_rn(f, NEGM);           // code * 16^j, exact
#pragma unroll
                        for (int m = 0; m < MT; ++m)
                            part[m] = __ffma2_rn(q, xs[m * (xs_floats / 2) + xs_pair_index(b, wd, j, lane)],
                                                 part[m]);
                    }
                }
#pragma unroll
                for (int m = 0; m < MT; ++m)
                    acc[m] = fmaf(dv[bb],
                                  part[m].x + part[m].y - zv[bb] * lsum[(m * NB + b) * 32 + lane],
                                  acc[m]);
            }
        }
#pragma unroll
        for (int m = 0; m < MT; ++m) {
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) acc[m] += __shfl_xor_sync(0xffffffffu, acc[m], off);
        }
        if (lane == 0) {
            for (int m = 0; m < mt; ++m)
                y[(m0 + m) * O + o] = __bfloat16_as_ushort(__float2bfloat16_rn(acc[m]));
        }
    }
}

template <int MT, bool ZEROS>
cudaError_t launch_decode(const uint16_t *x, int64_t M, int64_t I, int64_t O,
                          const uint32_t *qweight, const uint16_t *scales, const uint32_t *zeros,
                          const uint16_t *s16, int gs, uint16_t *y, cudaStream_t st) {
    const int NB = static_cast<int>((I + BLK_COLS - 1) / BLK_COLS);
    const size_t smem = sizeof(float) * static_cast<size_t>(MT) * (NB * BLK_COLS + NB * 32);
    static bool attr[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64 || !attr[dev]) {
        e = cudaFuncSetAttribute(w4a16_decode_kernel<MT, ZEROS>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attr[dev] = true;
    }
    int sms = 148;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    // One wave of resident blocks; each stages the activations once and then
    // streams rows grid-stride, so staging is amortised over many rows.
    int per_sm = 1;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, w4a16_decode_kernel<MT, ZEROS>,
                                                      W4_THREADS, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) per_sm = 1;
    int64_t bx = (O + W4_WARPS - 1) / W4_WARPS;
    if (bx > static_cast<int64_t>(sms) * per_sm) bx = static_cast<int64_t>(sms) * per_sm;
    dim3 grid(static_cast<unsigned>(bx), static_cast<unsigned>((M + MT - 1) / MT));
    w4a16_decode_kernel<MT, ZEROS><<<grid, W4_THREADS, smem, st>>>(
        x, M, static_cast<int>(I), O, qweight, scales, zeros, s16, gs, y);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_w4a16(const uint16_t *x, int64_t M, int64_t I, int64_t O,
                         const uint32_t *qweight, const uint16_t *scales, const uint32_t *zeros,
                         const uint16_t *s16, int gs, uint16_t *y, cudaStream_t st) {
    // Tokens per pass: as many as fit the block's staged activations (<= 227 KB).
    const int64_t per_token = 4 * (((I + BLK_COLS - 1) / BLK_COLS) * (BLK_COLS + 32));
    const bool z = zeros != nullptr;
    if (M <= 4 && w4a16_stream_supported(M, I)) {
        int dev = 0, sms = 148;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        return launch_w4a16_stream(x, M, I, O, qweight, scales, zeros, s16, gs, y, sms, st);
    }
#define AWQ_DEC(MT)                                                                      \
    return z ? launch_decode<MT, true>(x, M, I, O, qweight, scales, zeros, s16, gs, y, st) \
             : launch_decode<MT, false>(x, M, I, O, qweight, scales, zeros, s16, gs, y, st)
    if (2 * per_token > 227 * 1024) AWQ_DEC(1);      // wide inputs: one token's activations per pass
    if (M <= 2 || 4 * per_token > 227 * 1024) AWQ_DEC(2);
    if (M <= 4 || 8 * per_token > 227 * 1024) AWQ_DEC(4);
    AWQ_DEC(8);
#undef AWQ_DEC
}

}  // namespace awq
