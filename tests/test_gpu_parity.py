"""GPU parity: every entry point of the CUDA library against the CPU oracle on
the same seeded inputs.

Bars (restating the target of the search path):
  * s_X, INT4 codes, fp16/fp32 group scales, zero points and s16: bit-exact;
  * losses at every grid point: relative 1e-3 (per-row sums: 2e-3);
  * selected alpha / clip index: equal, or a near-tie where the oracle's own
    losses at the two indices differ by at most 2e-3 relative (then both are
    correct minimisers within the contraction's bf16 rounding);
  * W4A16 output: |y - y_ref| <= 2^-7 |y_ref| + 1e-2 rms(y_ref) (bf16 output
    and bf16 operands of the dequantised product).
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from synthetic import ALPHA_GRID, CLIP_GRID, apply_activations, small_layer

pytestmark = pytest.mark.gpu

LOSS_RTOL = 1e-3
ROW_RTOL = 2e-3
TIE_RTOL = 2e-3


@pytest.fixture(scope="module")
def awq():
    import weight_only_quantization_awq_b200 as m
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return m


def dev(a: np.ndarray) -> torch.Tensor:
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def u32(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy().view(np.uint32)


def u16(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy().view(np.uint16)


def check_choice(idx_gpu, idx_ref, loss_ref):
    """The selected index equals the oracle's whenever the oracle's best loss is
    separated from every other by more than 2 x LOSS_RTOL (the most two losses
    each within LOSS_RTOL can swap by); otherwise any index of the oracle's
    near-tie set is a correct minimiser."""
    loss_ref = np.asarray(loss_ref, np.float64)
    near = np.abs(loss_ref - loss_ref[idx_ref]) <= TIE_RTOL * loss_ref[idx_ref]
    if near.sum() == 1:
        assert idx_gpu == idx_ref, (idx_gpu, idx_ref, loss_ref[idx_gpu], loss_ref[idx_ref])
    else:
        assert near[idx_gpu], (idx_gpu, idx_ref, loss_ref[idx_gpu], loss_ref[idx_ref])


# --------------------------------------------------------------------- stats
@pytest.mark.parametrize("N,I,dt", [(1, 64, "bf16"), (127, 72, "f32"), (300, 136, "bf16"),
                                    (1000, 520, "f32"), (4097, 1024, "bf16")])
def test_act_stats_bitexact(awq, N, I, dt):
    _, X = small_layer(8, I, N, xdtype=dt, seed=N + I)
    got = awq.awq_act_stats(dev(X)).cpu().numpy()
    assert np.array_equal(got, oracle.act_stats(X))


def test_act_stats_clamp_and_zero_column(awq):
    X = np.zeros((50, 64), np.float32)
    X[:, 1] = -3.0
    got = awq.awq_act_stats(dev(X), clamp_min=1e-4).cpu().numpy()
    assert got[0] == np.float32(1e-4) and got[1] == np.float32(3.0)
    assert np.array_equal(got, oracle.act_stats(X))


def test_act_stats_workload2_full(awq):
    X = synthetic.layer_activations(2, "attn_proj")
    got = awq.awq_act_stats(dev(X)).cpu().numpy()
    assert np.array_equal(got, oracle.act_stats(X))


# ---------------------------------------------------------------------- pack
PACK_CASES = [
    (200, 384, 128, 0, 1.0, "bf16"),
    (200, 384, 64, 1, 1.0, "bf16"),
    (130, 256, 32, 0, 0.85, "f32"),
    (77, 640, 128, 1, 0.7, "f32"),
    (64, 11008, 128, 1, 1.0, "bf16"),
]


@pytest.mark.parametrize("O,I,gs,qt,clip,wdt", PACK_CASES)
@pytest.mark.parametrize("alpha", [0.0, 0.45, 0.95])
def test_pack_bitexact(awq, O, I, gs, qt, clip, wdt, alpha):
    W, X = small_layer(O, I, 64, wdtype=wdt, seed=O * 7 + gs)
    sX = oracle.act_stats(X)
    ref = oracle.pack_int4(W, sX, alpha, clip, gs, qt)
    got = awq.awq_pack_int4(dev(W), dev(sX), alpha, clip, gs, qt, scales_f32=True)
    assert np.array_equal(u32(got["qweight"]), ref["qweight"])
    assert np.array_equal(u16(got["scales"]), ref["scales"])
    assert np.array_equal(got["scales_f32"].cpu().numpy(), ref["scales_f32"])
    assert np.array_equal(u16(got["s16"]), ref["s16"])
    if qt == 1:
        assert np.array_equal(u32(got["zeros"]), ref["zeros"])


def test_pack_workload2_full(awq):
    W = synthetic.layer_weights(2, "attn_proj")
    X = synthetic.layer_activations(2, "attn_proj")
    sX = oracle.act_stats(X)
    for alpha in (0.0, 0.5):
        ref = oracle.pack_int4(W, sX, alpha, 1.0, 128, 0)
        got = awq.awq_pack_int4(dev(W), dev(sX), alpha, 1.0, 128, 0, scales_f32=True)
        assert np.array_equal(u32(got["qweight"]), ref["qweight"])
        assert np.array_equal(u16(got["scales"]), ref["scales"])
        assert np.array_equal(u16(got["s16"]), ref["s16"])


# -------------------------------------------------------------------- search
SEARCH_CASES = [
    # O,  I,   N,    gs, qt, clip grid,     W,     X
    (200, 384, 700, 128, 0, None, "bf16", "bf16"),    # ragged rows and tokens
    (64, 256, 100, 64, 1, CLIP_GRID[:4], "f32", "f32"),  # one partial token block
    (128, 512, 1024, 32, 0, None, "bf16", "f32"),
    (300, 640, 513, 128, 1, CLIP_GRID, "bf16", "bf16"),  # 1-token tail block
    (16, 128, 2048, 128, 0, CLIP_GRID[:3], "bf16", "bf16"),
    (1, 64, 64, 32, 1, CLIP_GRID[:2], "bf16", "bf16"),  # one row, one slab
    (3, 64, 5, 64, 0, None, "f32", "bf16"),              # one slab: the first slab is the last
    (257, 192, 257, 64, 1, None, "bf16", "bf16"),       # one row into a second pair tile
]


@pytest.mark.parametrize("O,I,N,gs,qt,clip,wdt,xdt", SEARCH_CASES)
def test_search_parity(awq, O, I, N, gs, qt, clip, wdt, xdt):
    W, X = small_layer(O, I, N, wdtype=wdt, xdtype=xdt, seed=O + I + N, outlier=30.0)
    sX = oracle.act_stats(X)
    ref = oracle.search_layer(W, X, sX, gs, qt, ALPHA_GRID, clip=clip)
    got = awq.awq_search_layer(dev(W), dev(X), dev(sX), gs, 4, qt, ALPHA_GRID, clip=clip,
                               loss_row=True)
    G = len(ALPHA_GRID)
    check_choice(got["best_alpha"], ref["best_alpha"], ref["loss"][:G])
    if clip is None:
        np.testing.assert_allclose(got["loss"], ref["loss"], rtol=LOSS_RTOL, atol=0)
        np.testing.assert_allclose(got["loss_row"].cpu().numpy(), ref["loss_row"],
                                   rtol=ROW_RTOL, atol=1e-30)
        assert got["best_clip"] == -1
    else:
        np.testing.assert_allclose(got["loss"][:G], ref["loss"][:G], rtol=LOSS_RTOL, atol=0)
        # the clip phase runs at the GPU's alpha*: compare against the oracle at that alpha
        ref2 = oracle.search_layer(W, X, sX, gs, qt, ALPHA_GRID[[got["best_alpha"]]], clip=clip)
        np.testing.assert_allclose(got["loss"][G:], ref2["loss"][1:], rtol=LOSS_RTOL, atol=0)
        check_choice(got["best_clip"], ref2["best_clip"], ref2["loss"][1:])
        assert got["loss"][G] == pytest.approx(got["loss"][got["best_alpha"]], rel=1e-12)


def test_search_workload1_full(awq):
    W = synthetic.layer_weights(1, "linear")
    X = synthetic.layer_activations(1, "linear")
    sX = oracle.act_stats(X)
    ref = oracle.search_layer(W, X, sX, 128, 0, ALPHA_GRID)
    got = awq.awq_search_layer(dev(W), dev(X), dev(sX), 128, 4, 0, ALPHA_GRID, loss_row=True)
    np.testing.assert_allclose(got["loss"], ref["loss"], rtol=LOSS_RTOL, atol=0)
    np.testing.assert_allclose(got["loss_row"].cpu().numpy(), ref["loss_row"], rtol=ROW_RTOL)
    check_choice(got["best_alpha"], ref["best_alpha"], ref["loss"])


def test_search_workload2_sampled_rows(awq):
    """Full 4096x4096, N = 4096 search on the GPU; the oracle evaluates a
    seeded sample of output rows (first, last, and 30 random ones)."""
    W = synthetic.layer_weights(2, "attn_proj")
    X = synthetic.layer_activations(2, "attn_proj")
    Xd, Wd = dev(X), dev(W)
    sXd = awq.awq_act_stats(Xd)
    sX = sXd.cpu().numpy()
    assert np.array_equal(sX, oracle.act_stats(X))
    got = awq.awq_search_layer(Wd, Xd, sXd, 128, 4, 0, ALPHA_GRID, loss_row=True)
    rows = np.unique(np.concatenate([[0, 4095], np.random.default_rng(7).choice(4096, 30, False)]))
    ref = oracle.search_layer(W, X, sX, 128, 0, ALPHA_GRID, rows=rows)
    lr = got["loss_row"].cpu().numpy().astype(np.float64)
    np.testing.assert_allclose(lr[:, rows], ref["loss_row"], rtol=ROW_RTOL)
    # the reported losses are the row sums' mean, and the choice is their argmin
    np.testing.assert_allclose(got["loss"], lr.sum(axis=1) / (4096.0 * 4096.0), rtol=1e-6)
    assert got["best_alpha"] == int(np.argmin(got["loss"]))


def test_search_deterministic(awq):
    W, X = small_layer(256, 512, 1500, seed=99)
    Wd, Xd = dev(W), dev(X)
    sXd = awq.awq_act_stats(Xd)
    a = awq.awq_search_layer(Wd, Xd, sXd, 128, 4, 1, ALPHA_GRID, clip=CLIP_GRID, loss_row=True)
    b = awq.awq_search_layer(Wd, Xd, sXd, 128, 4, 1, ALPHA_GRID, clip=CLIP_GRID, loss_row=True)
    assert np.array_equal(a["loss"], b["loss"])
    assert torch.equal(a["loss_row"], b["loss_row"])


def test_search_then_pack_workload1(awq):
    """The end-to-end chain: stats -> search -> pack at the chosen alpha gives
    the oracle's codes at that alpha."""
    W = synthetic.layer_weights(1, "linear")
    X = synthetic.layer_activations(1, "linear")
    Wd, Xd = dev(W), dev(X)
    sXd = awq.awq_act_stats(Xd)
    res = awq.awq_search_layer(Wd, Xd, sXd, 128, 4, 0, ALPHA_GRID)
    a = float(ALPHA_GRID[res["best_alpha"]])
    got = awq.awq_pack_int4(Wd, sXd, a, 1.0, 128, 0)
    ref = oracle.pack_int4(W, sXd.cpu().numpy(), a, 1.0, 128, 0)
    assert np.array_equal(u32(got["qweight"]), ref["qweight"])
    assert np.array_equal(u16(got["scales"]), ref["scales"])


# --------------------------------------------------------------------- apply
def check_apply(y_gpu: torch.Tensor, y_ref: np.ndarray):
    y = y_gpu.float().cpu().numpy().astype(np.float64)
    rms = np.sqrt(np.mean(y_ref ** 2))
    err = np.abs(y - y_ref)
    bound = 2.0 ** -7 * np.abs(y_ref) + 1e-2 * rms
    assert np.all(err <= bound), (err.max(), np.argmax(err - bound))


@pytest.mark.parametrize("M", [1, 2, 3, 5, 16, 17, 32, 33, 300])
@pytest.mark.parametrize("O,I,gs,qt", [(200, 384, 128, 0), (96, 512, 64, 1), (130, 256, 32, 1)])
def test_linear_w4a16_parity(awq, M, O, I, gs, qt):
    W, X = small_layer(O, I, 64, seed=O + M)
    sX = oracle.act_stats(X)
    p = oracle.pack_int4(W, sX, 0.5, 1.0, gs, qt)
    x = apply_activations(M, I, seed=O)
    y_ref = oracle.linear_w4a16(x, p["qweight"], p["scales"], p["zeros"], p["s16"], gs)
    got = awq.awq_linear_w4a16(
        dev(x), dev(p["qweight"].view(np.int32)), dev(p["scales"].view(np.float16)),
        dev(p["zeros"].view(np.int32)) if p["zeros"] is not None else None,
        dev(p["s16"].view(np.float16)), gs)
    check_apply(got, y_ref)


@pytest.mark.parametrize("M", [1, 16, 256])
@pytest.mark.parametrize("layer", ["o", "gate", "down"])
def test_linear_w4a16_block_shape(awq, M, layer):
    """The decoder block's linear shapes (o 4096x4096, gate 11008x4096, down
    4096x11008), packed by the GPU itself."""
    src = {"o": "o", "gate": "gate_up", "down": "down"}[layer]
    W = synthetic.layer_weights(5, src)
    if layer == "gate":
        W = np.ascontiguousarray(W[:11008])
    X = synthetic.layer_activations(5, src, tokens=512)
    Wd = dev(W)
    sXd = awq.awq_act_stats(dev(X))
    p = awq.awq_pack_int4(Wd, sXd, 0.5, 1.0, 128, 1)
    x = apply_activations(M, W.shape[1])
    y = awq.awq_linear_w4a16(dev(x), p["qweight"], p["scales"], p["zeros"], p["s16"], 128)
    y_ref = oracle.linear_w4a16(x, u32(p["qweight"]), u16(p["scales"]), u32(p["zeros"]),
                                u16(p["s16"]), 128)
    check_apply(y, y_ref)


@pytest.mark.parametrize("M", [1, 2, 4, 5])
@pytest.mark.parametrize("pattern", ["tiny", "mixed", "zero"])
def test_linear_w4a16_activation_range(awq, M, pattern):
    """Activations far below 1 (whole rows near the bottom of the normal float
    range), rows mixing tiny, zero and ordinary 32-column chunks, and all-zero
    activations: every pass scales x / s by a power of two before rounding it to
    fp16, and that scale must stay finite.  in = 1088 leaves a ragged last block
    of 32-column chunks."""
    O, I, gs = 96, 1088, 64
    W, X = small_layer(O, I, 64, seed=M + 11)
    p = oracle.pack_int4(W, oracle.act_stats(X), 0.5, 1.0, gs, 1)
    xf = synthetic.bf16_to_f32(apply_activations(M, I, seed=M + 3)).astype(np.float64)
    if pattern == "tiny":
        xf *= 2.0 ** -118
    elif pattern == "mixed":
        xf[:, :256] *= 2.0 ** -118
        xf[:, 256:512] = 0.0
        xf[:, 1024:] *= 2.0 ** -60
    else:
        xf[:] = 0.0
    x = synthetic.bf16_bits(xf.astype(np.float32))
    y_ref = oracle.linear_w4a16(x, p["qweight"], p["scales"], p["zeros"], p["s16"], gs)
    got = awq.awq_linear_w4a16(
        dev(x), dev(p["qweight"].view(np.int32)), dev(p["scales"].view(np.float16)),
        dev(p["zeros"].view(np.int32)), dev(p["s16"].view(np.float16)), gs)
    y = got.float().cpu().numpy()
    assert np.all(np.isfinite(y))
    if pattern == "zero":
        assert np.all(y == 0.0)
    else:
        check_apply(got, y_ref)


@pytest.mark.parametrize("M,I", [(3, 24576), (4, 24576), (4, 40960), (2, 49152), (1, 49152)])
def test_linear_w4a16_widest_inputs(awq, M, I):
    """Input widths at the top of the supported range: 2-4 tokens this wide do
    not fit the streaming kernel's shared activation table and take the fallback
    decode kernel (two tokens per pass at 24576 columns, one per pass at 40960
    and 49152); in = 49152 is the largest width accepted."""
    O, gs = 96, 128
    W, X = small_layer(O, I, 16, seed=M + I)
    p = oracle.pack_int4(W, oracle.act_stats(X), 0.5, 1.0, gs, 1)
    x = apply_activations(M, I, seed=M + 7)
    y_ref = oracle.linear_w4a16(x, p["qweight"], p["scales"], p["zeros"], p["s16"], gs)
    got = awq.awq_linear_w4a16(
        dev(x), dev(p["qweight"].view(np.int32)), dev(p["scales"].view(np.float16)),
        dev(p["zeros"].view(np.int32)), dev(p["s16"].view(np.float16)), gs)
    check_apply(got, y_ref)
