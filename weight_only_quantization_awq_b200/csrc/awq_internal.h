// Internal launch interface between the C-ABI layer (awq_api.cu) and the
// kernels.  Every launcher enqueues on `st` and returns the launch status.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>
#include <stdint.h>

namespace awq {

// An NVTX range around one C-ABI call, so that each call shows on a profiler's
// timeline with its kernels under it.  Without a profiler's NVTX injection library
// the push and pop return at once.
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange &) = delete;
    NvtxRange &operator=(const NvtxRange &) = delete;
};

// Record the calling host thread's last-error text (read back by awq_last_error()).
void set_last_error(const char *msg);

constexpr int STATS_CHUNK = 128;   // tokens per fp64 partial sum of mean|X|
constexpr int64_t STATS_MAX_GRID_Y = 65535;   // chunks beyond this are strided over the grid

// Optional CUDA-event timing of an entry point's main kernels (awq_set_kernel_timing):
// kt_reset clears the record of `kind`, kt_begin / kt_end bracket launches on `st`.
void kt_reset(int kind);
void kt_begin(int kind, cudaStream_t st);
void kt_end(int kind, cudaStream_t st);
constexpr int MAX_GRID = 64;       // grid points per search phase

// Default bound of an in-kernel mbarrier wait: ~2 s of SM clock at 2 GHz, far
// above any legitimate wait in these kernels.
constexpr long long AWQ_DEFAULT_WAIT_CYCLES = 4000000000LL;

// Search tile shape: 128 output rows per CTA (256 per CTA pair) x 512 tokens per
// work unit (two MMA halves of 256), K slabs of 64.
constexpr int TILE_O = 128;
constexpr int TILE_N = 512;
constexpr int SUB_N = 256;
constexpr int SLAB_K = 64;

struct GridParams {
    double value[MAX_GRID];   // alpha per grid point (phase 1) or clip ratio (phase 2)
};

// ---- statistics
cudaError_t launch_stats_partial(const void *X, bool x_bf16, int64_t N, int64_t I, double *part,
                                 cudaStream_t st);
cudaError_t launch_stats_final(const double *part, int64_t N, int64_t I, float clamp_min,
                               float *sX, cudaStream_t st);
// fp16 copy of X scaled by 2^-k (k written to *k_out on the device); *max_bits zeroed by the caller.
cudaError_t launch_x_to_f16(const void *X, bool x_bf16, int64_t n, unsigned *max_bits, int *k_out,
                            uint16_t *dst, cudaStream_t st);

// ---- scale table sn[G][2][I]: row 2g holds s_g, row 2g+1 holds -1/s_g.
// alpha.value[g] is grid point g's alpha; if best_idx != nullptr every row uses
// alpha.value[*best_idx] instead (the second, clip phase).
// scratch: scale_scratch_bytes(G, I) bytes of device workspace.
int64_t scale_scratch_bytes(int G, int64_t I);
cudaError_t launch_scale_table(const float *sX, int64_t I, const GridParams &alpha, int G,
                               const int *best_idx, float *sn, void *scratch, cudaStream_t st);

// ---- per-(grid point, group, row) quantiser parameters {Delta, 1/Delta, -qhi, -qlo},
// layout qparam[g][group][row] (rows fastest).  Also picks each grid point's
// power-of-two range scale 2^k of dW (dw_exp[g] = k, device), multiplying the
// -1/s rows of sn by it; dw_bits: G words of device scratch.
cudaError_t launch_group_params(const void *W, bool w_bf16, int64_t O, int64_t I, int gs,
                                bool asym, int wbit, float *sn, const GridParams &clip,
                                int G, float4 *qparam, unsigned *dw_bits, int *dw_exp,
                                cudaStream_t st);

// ---- fused search
// Tensor maps of the kernel's four inputs:
//   x  : fp16 copy of X [N, I], box 64 x 128 (one CTA's half of a 256-token tile), 128B swizzle
//   w  : W [O, I] (bf16: box 64 x 128; fp32: box 32 x 128), 128B swizzle
//   sn : scale table [2G, I] fp32, box 64 x 2
//   qp : group parameters [G * I/gs][O][4] fp32 (3-D), box 4 x 128 rows x groups per slab
struct SearchMaps {
    CUtensorMap x, w, sn, qp;
};
struct SearchArgs {
    int64_t O, I, N;
    int gs;
    int G;
    bool w_bf16;
    bool clamp;                 // asymmetric or clipped: clamp codes to [qlo, qhi]
    float *part;                // [G][TB][O]
    int *err;
    long long wait;             // bound of every mbarrier wait, in SM clock cycles
};
cudaError_t launch_search(const SearchArgs &a, const SearchMaps &maps, int num_sms,
                          cudaStream_t st);

// ---- loss reduction and selection
// blocksum: scratch of reduce_scratch_doubles(G, O) doubles.
int64_t reduce_scratch_doubles(int G, int64_t O);
// Row sums of grid point g are multiplied by 2^(-2 * (*x_exp + dw_exp[g])) (the exact
// undo of the power-of-two scales of X and dW in the contraction).
cudaError_t launch_reduce_loss(const float *part, int G, int64_t TB, int64_t O, int64_t N,
                               const int *x_exp, const int *dw_exp, double *loss, float *loss_row,
                               double *blocksum, cudaStream_t st);
cudaError_t launch_argmin(const double *loss, int G, int *best, cudaStream_t st);

// ---- packing
// clip_idx (optional, [O][I/gs] device): each group's index into clip_grid, used
// instead of the layer ratio `clip`.
cudaError_t launch_pack(const void *W, bool w_bf16, int64_t O, int64_t I, int gs, bool asym,
                        int wbit, double clip, const uint8_t *clip_idx, const GridParams &clip_grid,
                        const float *s, uint32_t *qweight, uint16_t *scales, uint32_t *zeros,
                        uint16_t *s16, float *scales_f32, cudaStream_t st);

// ---- W4A16 apply on the tensor cores (M >= 17)
struct TcMaps {
    CUtensorMap q;    // qweight [O][I/8] u32, box 32 words (4 slabs) x 128 rows, 128B swizzle
    CUtensorMap xs;   // permuted, power-of-two scaled fp16 x/s [M][I], box 64 x n_tile, 128B swizzle
};
struct TcPlan {
    int n_tile;            // tokens per tile (multiple of 16, <= 256)
    int splits;            // K splits
    int slabs_per_split;
    int64_t xs_bytes, part_bytes, counter_bytes, scale_bytes;   // workspace pieces (256-byte rounded)
};
TcPlan w4a16_tc_plan(int64_t M, int64_t I, int64_t O, int num_sms);
// workspace: xs (plan.xs_bytes), the fp32 split-K accumulator (plan.part_bytes), the
// tile counters (plan.counter_bytes), then the token scales sx [M] fp32 and the row exponents
// kd [O] int32 (plan.scale_bytes).
cudaError_t launch_w4a16_tc(const uint16_t *x, int64_t M, int64_t I, int64_t O,
                            const uint16_t *scales, const uint32_t *zeros, const uint16_t *s16,
                            int gs, uint16_t *y, const TcPlan &plan, char *workspace,
                            const TcMaps &maps, cudaStream_t st);

// ---- W4A16 decode (M <= 8) over up to DEC_MAX_LINEARS independent linears in one
// persistent launch, one CTA per SM.  Each CTA works on one linear: linear l owns
// the CTAs [cta0[l], cta0[l + 1]) (their number in proportion to its bytes), and
// its tiles of rows[l] output rows (a multiple of 8; all input columns) are split
// into equal contiguous ranges among them.  A CTA's ring holds stages[l] slots of
// slot_bytes[l]; activations take xbuf_bytes[l].  All sizes come from
// w4a16_dec_config.
constexpr int DEC_MAX_LINEARS = 8;
constexpr int64_t DEC_MAX_M = 8;
constexpr int64_t DEC_MAX_SMEM = 227 * 1024;
struct DecLinear {
    const uint16_t *x;
    const uint32_t *qweight;
    const uint16_t *scales;
    const uint32_t *zeros;
    const uint16_t *s16;
    uint16_t *y;
    int64_t I, O;
};
struct DecBatch {
    DecLinear lin[DEC_MAX_LINEARS];
    int cta0[DEC_MAX_LINEARS + 1];
    int rows[DEC_MAX_LINEARS];
    int stages[DEC_MAX_LINEARS];
    int slot_bytes[DEC_MAX_LINEARS];
    int xbuf_bytes[DEC_MAX_LINEARS];
    int n, ctas;
    int64_t smem;                 // dynamic shared memory of the launch
};
// Fills the CTA split and the buffer plan of `b` (lin[] and n set by the caller);
// false when M or a linear does not fit the kernel's shared memory, or the
// linears outnumber the SMs.
bool w4a16_dec_config(DecBatch &b, int64_t M, int gs, bool zeros, int num_sms);
cudaError_t launch_w4a16_dec(const DecBatch &b, int M, int gs, bool zeros, cudaStream_t st);

// ---- W4A16 apply for decode-sized M (1..16): xs preparation + warp-level MMA kernel
constexpr int64_t W4A16_MMA_MAX_M = 16;
int64_t w4a16_mma_workspace_bytes(int64_t M, int64_t I, int gs);
cudaError_t launch_w4a16_mma(const uint16_t *x, int64_t M, int64_t I, int64_t O,
                             const uint32_t *qweight, const uint16_t *scales, const uint32_t *zeros,
                             const uint16_t *s16, int gs, uint16_t *y, char *workspace,
                             cudaStream_t st);

// ---- W4A16 apply
// Streaming GEMV for 1 <= M <= 4 (activations staged per CTA; see k_w4a16_stream.cu).
bool w4a16_stream_supported(int64_t M, int64_t I);
cudaError_t launch_w4a16_stream(const uint16_t *x, int64_t M, int64_t I, int64_t O,
                                const uint32_t *qweight, const uint16_t *scales, const uint32_t *zeros,
                                const uint16_t *s16, int gs, uint16_t *y, int num_sms, cudaStream_t st);
cudaError_t launch_w4a16(const uint16_t *x, int64_t M, int64_t I, int64_t O,
                         const uint32_t *qweight, const uint16_t *scales, const uint32_t *zeros,
                         const uint16_t *s16, int gs, uint16_t *y, cudaStream_t st);

// ---- per-group clip choice: Gram matrices of X per group (H: gclip_scratch_doubles
// device doubles), then for every (row, group) the first ratio of `grid` that
// minimises the group's output error; best [O][I/gs] u8, err (optional) [O][I/gs][n_clip].
int64_t gclip_scratch_doubles(int64_t I, int gs);
cudaError_t launch_group_clip(const void *W, bool w_bf16, int64_t O, int64_t I, const void *X,
                              bool x_bf16, int64_t N, const float *s, int gs, bool asym, int wbit,
                              const GridParams &grid, int n_clip, double *H, uint8_t *best,
                              float *err, cudaStream_t st);

// ---- bounded-wait self-test: one CTA waits on an mbarrier (arrived on only if
// `arrive`) with a limit of `limit` cycles; a wait that gives up writes the
// timeout code to *err.
cudaError_t launch_wait_selftest(long long limit, bool arrive, int *err, cudaStream_t st);

// ---- fold of 1/s into the previous operator: out[r][c] = P[r][c] / s16[r]
// (one IEEE fp32 division, then bf16 rounding when bf16).
cudaError_t launch_fold_scale(const void *P, bool bf16, int64_t R, int64_t C, const uint16_t *s16,
                              void *out, cudaStream_t st);

}  // namespace awq
