"""GPU parity of the quantiser variants and auxiliary entry points against the
CPU oracle: 3-bit quantisation, the joint (alpha, clip) grid, per-group clip
packing, layers of very small weights (the power-of-two range scale of dW),
the fold of 1/s into the previous operator with the apply that skips the
division, the bounded-wait self-test, statistics over more token chunks
than one grid dimension holds, several linears per launch, and outputs written
in full (NaN-poisoned output buffers).

Bars as in test_gpu_parity: integer results bit-exact, losses within 1e-3
relative, selected indices equal or a near-tie of the oracle's own losses
(2e-3), the apply within 2^-7 |y| + 1e-2 rms(y).
"""
import numpy as np
import pytest
import torch

import oracle
from synthetic import ALPHA_GRID, CLIP_GRID, apply_activations, bf16_bits, small_layer

pytestmark = pytest.mark.gpu

LOSS_RTOL = 1e-3
TIE_RTOL = 2e-3
AWQ_ERR_TIMEOUT = 5


@pytest.fixture(scope="module")
def awq():
    import weight_only_quantization_awq_b200 as m
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return m


def dev(a: np.ndarray) -> torch.Tensor:
    """uint16 (bf16 bits) -> bfloat16, uint32 -> int32 bits, uint8 as is, else as is."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
    if a.dtype == np.uint32:
        return torch.from_numpy(a.view(np.int32)).cuda()
    return torch.from_numpy(a).cuda()


def u32(t):
    return t.cpu().numpy().view(np.uint32)


def u16(t):
    return t.cpu().view(torch.int16).numpy().view(np.uint16)


def check_choice(idx_gpu, idx_ref, loss_ref):
    """Exact unless the oracle's best loss has near-ties within 2 x LOSS_RTOL;
    then any index of that set (see test_gpu_parity.check_choice)."""
    loss_ref = np.asarray(loss_ref, np.float64)
    near = np.abs(loss_ref - loss_ref[idx_ref]) <= TIE_RTOL * loss_ref[idx_ref]
    if near.sum() == 1:
        assert idx_gpu == idx_ref, (idx_gpu, idx_ref, loss_ref[idx_gpu], loss_ref[idx_ref])
    else:
        assert near[idx_gpu], (idx_gpu, idx_ref, loss_ref[idx_gpu], loss_ref[idx_ref])


def check_pack(got, ref, qt):
    assert np.array_equal(u32(got["qweight"]), ref["qweight"])
    assert np.array_equal(u16(got["scales"]), ref["scales"])
    assert np.array_equal(u16(got["s16"]), ref["s16"])
    if got["scales_f32"] is not None:
        assert np.array_equal(got["scales_f32"].cpu().numpy(), ref["scales_f32"])
    if qt == 1:
        assert np.array_equal(u32(got["zeros"]), ref["zeros"])


def check_apply(y, y_ref):
    yd = y.float().cpu().numpy().astype(np.float64)
    rms = np.sqrt(np.mean(y_ref ** 2))
    err = np.abs(yd - y_ref)
    assert np.all(err <= 2.0 ** -7 * np.abs(y_ref) + 1e-2 * rms), float(err.max())


# ------------------------------------------------------------------ w_bit = 3
@pytest.mark.parametrize("O,I,N,gs,qt", [(200, 256, 300, 128, 0), (130, 384, 517, 64, 1),
                                         (257, 512, 700, 32, 1)])
def test_search_and_pack_w3(awq, O, I, N, gs, qt):
    W, X = small_layer(O, I, N, seed=O + I + gs, outlier=30.0)
    Wd, Xd = dev(W), dev(X)
    sXd = awq.awq_act_stats(Xd)
    sX = oracle.act_stats(X)
    clip = CLIP_GRID[::2] if qt == 1 else None
    got = awq.awq_search_layer(Wd, Xd, sXd, gs, 3, qt, ALPHA_GRID, clip=clip)
    ref = oracle.search_layer(W, X, sX, gs, qt, ALPHA_GRID, w_bit=3)
    G = len(ALPHA_GRID)
    np.testing.assert_allclose(got["loss"][:G], ref["loss"], rtol=LOSS_RTOL)
    check_choice(got["best_alpha"], ref["best_alpha"], ref["loss"])
    a = float(ALPHA_GRID[got["best_alpha"]])
    if clip is not None:
        ref2 = oracle.search_layer(W, X, sX, gs, qt, [a], clip=clip, w_bit=3)
        np.testing.assert_allclose(got["loss"][G:], ref2["loss"][1:], rtol=LOSS_RTOL)
        check_choice(got["best_clip"], ref2["best_clip"], ref2["loss"][1:])
    r = float(clip[got["best_clip"]]) if clip is not None else 1.0
    p = awq.awq_pack_quant(Wd, sXd, a, r, gs, qt, w_bit=3, scales_f32=True)
    check_pack(p, oracle.pack_int4(W, sX, a, r, gs, qt, w_bit=3), qt)
    codes = np.stack([(u32(p["qweight"]) >> np.uint32(4 * k)) & np.uint32(15) for k in range(8)], -1)
    assert codes.max() <= (11 if qt == 0 else 7) and codes.min() >= (4 if qt == 0 else 0)


# ------------------------------------------------------------------ joint grid
@pytest.mark.parametrize("qt", [0, 1])
def test_search_points_joint_grid(awq, qt):
    O, I, N, gs = 300, 512, 600, 128
    W, X = small_layer(O, I, N, seed=90 + qt, outlier=40.0)
    Wd, Xd = dev(W), dev(X)
    sXd = awq.awq_act_stats(Xd)
    sX = oracle.act_stats(X)
    A, C = np.meshgrid(ALPHA_GRID[::2], CLIP_GRID, indexing="ij")     # 10 x 11 = 110 points
    got = awq.awq_search_points(Wd, Xd, sXd, A.ravel(), C.ravel(), gs, 4, qt, loss_row=True)
    ref = oracle.search_points(W, X, sX, gs, qt, A.ravel(), C.ravel())
    np.testing.assert_allclose(got["loss"], ref["loss"], rtol=LOSS_RTOL)
    check_choice(got["best"], ref["best"], ref["loss"])
    lr = got["loss_row"].cpu().numpy().astype(np.float64)
    np.testing.assert_allclose(lr.sum(axis=1) / (N * O), got["loss"], rtol=1e-5)
    # the r = 1 column reproduces the alpha search
    plain = awq.awq_search_layer(Wd, Xd, sXd, gs, 4, qt, ALPHA_GRID[::2])
    np.testing.assert_allclose(got["loss"].reshape(A.shape)[:, 0], plain["loss"], rtol=1e-6)


# ------------------------------------------------------------------ small weights
@pytest.mark.parametrize("wdt,factor", [("bf16", 2.0 ** -10), ("f32", 2.0 ** -20), ("f32", 2.0 ** -30)])
def test_search_small_weights(awq, wdt, factor):
    """Weights far below the usual magnitude: dW would sit in fp16's subnormal
    range without its power-of-two range scale."""
    O, I, N, gs = 192, 256, 400, 64
    W, X = small_layer(O, I, N, wdtype="f32", seed=95, outlier=30.0)
    W = (W * np.float32(factor)).astype(np.float32)
    W = bf16_bits(W) if wdt == "bf16" else W
    Wd, Xd = dev(W), dev(X)
    sXd = awq.awq_act_stats(Xd)
    sX = oracle.act_stats(X)
    for qt in (0, 1):
        got = awq.awq_search_layer(Wd, Xd, sXd, gs, 4, qt, ALPHA_GRID, clip=CLIP_GRID[:4])
        ref = oracle.search_layer(W, X, sX, gs, qt, ALPHA_GRID)
        np.testing.assert_allclose(got["loss"][:len(ALPHA_GRID)], ref["loss"], rtol=LOSS_RTOL)
        check_choice(got["best_alpha"], ref["best_alpha"], ref["loss"])


# ------------------------------------------------------------------ per-group clip pack
@pytest.mark.parametrize("qt,wbit", [(0, 4), (1, 4), (1, 3)])
def test_pack_per_group_clip(awq, qt, wbit):
    O, I, gs = 133, 512, 128
    W, X = small_layer(O, I, 64, seed=96 + wbit)
    Wd = dev(W)
    sX = oracle.act_stats(X)
    idx = np.random.default_rng(97).integers(0, len(CLIP_GRID), size=(O, I // gs)).astype(np.uint8)
    got = awq.awq_pack_quant(Wd, dev(sX), 0.35, 1.0, gs, qt, w_bit=wbit,
                             clip_idx=dev(idx), clip_grid=CLIP_GRID, scales_f32=True)
    ref = oracle.pack_int4(W, sX, 0.35, 1.0, gs, qt, w_bit=wbit, clip_g=CLIP_GRID[idx])
    check_pack(got, ref, qt)


# ------------------------------------------------------------------ fold of 1/s
@pytest.mark.parametrize("dt", ["bf16", "f32"])
def test_fold_scale_bitexact(awq, dt):
    r = np.random.default_rng(98)
    R, C = 4096, 33
    P = r.standard_normal((R, C)).astype(np.float32)
    P = bf16_bits(P) if dt == "bf16" else P
    s16 = r.uniform(0.001, 1.0, size=R).astype(np.float16).view(np.uint16)
    got = awq.awq_fold_scale(dev(P), dev(s16).view(torch.float16))
    ref = oracle.fold_scale(P, s16, out_bf16=(dt == "bf16"))
    g = u16(got) if dt == "bf16" else got.cpu().numpy()
    assert np.array_equal(g.reshape(R, C), ref)
    # in place, and a 1-D RMSNorm weight
    gamma = dev(P[:, 0].copy())
    awq.awq_fold_scale(gamma, dev(s16).view(torch.float16), out=gamma)
    gg = u16(gamma) if dt == "bf16" else gamma.cpu().numpy()
    assert np.array_equal(gg, ref[:, 0])


@pytest.mark.parametrize("M", [1, 3, 16, 257])
def test_apply_with_folded_scale(awq, M):
    """x folded by 1/s (as the previous operator's output would be) through the
    apply without s16, against the oracle on the same folded x; and against the
    unfolded call within the apply tolerance."""
    O, I, gs = 520, 1024, 128
    W, X = small_layer(O, I, 256, seed=99)
    sX = oracle.act_stats(X)
    pk = oracle.pack_int4(W, sX, 0.5, 1.0, gs, oracle.ASYM)
    x = apply_activations(M, I, seed=3)
    xf = oracle.fold_scale(x.T.copy(), pk["s16"]).T.copy()          # channel = row of P
    q, z = dev(pk["qweight"]), dev(pk["zeros"])
    sc, s16 = dev(pk["scales"]).view(torch.float16), dev(pk["s16"]).view(torch.float16)
    xd = dev(x)
    xfd = awq.awq_fold_scale(xd.t().contiguous(), s16).t().contiguous()
    assert np.array_equal(u16(xfd), xf)
    y = awq.awq_linear_w4a16(xfd, q, sc, z, None, gs)
    check_apply(y, oracle.linear_w4a16(xf, pk["qweight"], pk["scales"], pk["zeros"], None, gs))
    check_apply(y, oracle.linear_w4a16(x, pk["qweight"], pk["scales"], pk["zeros"], pk["s16"], gs))


# ------------------------------------------------------------------ bounded wait
def test_wait_selftest_times_out_and_recovers(awq):
    """A wait whose barrier nobody arrives on gives up after its limit and is
    reported as AWQ_ERR_TIMEOUT; the context stays usable: the completed wait
    and a full search afterwards still match the oracle."""
    assert awq.awq_wait_selftest(2_000_000, arrive=True) == 0
    assert awq.awq_wait_selftest(2_000_000, arrive=False) == AWQ_ERR_TIMEOUT
    assert awq.awq_wait_selftest(20_000, arrive=False) == AWQ_ERR_TIMEOUT
    assert awq.awq_wait_selftest(2_000_000, arrive=True) == 0
    W, X = small_layer(128, 256, 200, seed=100)
    got = awq.awq_search_layer(dev(W), dev(X), awq.awq_act_stats(dev(X)), 128, 4, 0, ALPHA_GRID)
    ref = oracle.search_layer(W, X, oracle.act_stats(X), 128, 0, ALPHA_GRID)
    np.testing.assert_allclose(got["loss"], ref["loss"], rtol=LOSS_RTOL)


# ------------------------------------------------------------------ many token chunks
def test_act_stats_more_chunks_than_grid_rows(awq):
    """N = 128 * 65536 + 77 tokens: 65537 chunks of 128, more than one grid
    dimension holds; the chunks are strided over the grid.  The allocation-free
    entry takes exactly its capacity at in = 16 and N = 128 * 65536."""
    I = 16
    N = 128 * 65536 + 77
    r = np.random.default_rng(101)
    X = bf16_bits(r.standard_normal((N, I), dtype=np.float32))
    Xd = dev(X)
    got = awq.awq_act_stats(Xd).cpu().numpy()
    assert np.array_equal(got, oracle.act_stats(X))
    N2 = 128 * 65536
    got2 = awq.awq_act_stats_noalloc(Xd[:N2]).cpu().numpy()
    assert np.array_equal(got2, awq.awq_act_stats(Xd[:N2]).cpu().numpy())
    with pytest.raises(awq.AwqError) as e:
        awq.awq_act_stats_noalloc(Xd)
    assert e.value.status_name == "AWQ_ERR_UNSUPPORTED"


# ------------------------------------------------------------------ per-group clip search
@pytest.mark.parametrize("O,I,N,gs,qt,wbit", [(160, 512, 700, 128, 1, 4), (97, 256, 333, 64, 0, 4),
                                              (64, 256, 1500, 32, 1, 3)])
def test_group_clip_against_oracle(awq, O, I, N, gs, qt, wbit):
    """Each group's error at every ratio within 2e-3 of the oracle's direct fp64
    sum over tokens; the chosen ratio equal to the oracle's or a near-tie of its
    errors; packing at the chosen ratios bit-exact against the oracle."""
    W, X = small_layer(O, I, N, seed=110 + gs, outlier=40.0)
    Wd, Xd = dev(W), dev(X)
    sXd = awq.awq_act_stats(Xd)
    sX = oracle.act_stats(X)
    alpha = 0.45
    got = awq.awq_group_clip(Wd, Xd, sXd, alpha, CLIP_GRID, gs, wbit, qt, want_err=True)
    ref = oracle.group_clip(W, X, sX, alpha, gs, qt, CLIP_GRID, w_bit=wbit, want_err=True)
    eg = got["err"].cpu().numpy().astype(np.float64)
    er = ref["err"]
    scale = er.max(axis=2, keepdims=True)
    np.testing.assert_allclose(eg, er, rtol=2e-3, atol=0)
    ig = got["clip_idx"].cpu().numpy().astype(np.int64)
    ir = ref["best"].astype(np.int64)
    diff = ig != ir
    if diff.any():
        o, j = np.nonzero(diff)
        gap = np.abs(er[o, j, ig[o, j]] - er[o, j, ir[o, j]])
        assert np.all(gap <= TIE_RTOL * er[o, j, ir[o, j]] + 1e-12 * scale[o, j, 0]), gap.max()
    assert diff.mean() < 0.05
    p = awq.awq_pack_quant(Wd, sXd, alpha, 1.0, gs, qt, w_bit=wbit, clip_idx=got["clip_idx"],
                           clip_grid=CLIP_GRID, scales_f32=True)
    check_pack(p, oracle.pack_int4(W, sX, alpha, 1.0, gs, qt, w_bit=wbit, clip_g=CLIP_GRID[ig]), qt)


# ------------------------------------------------------------------ several linears per launch
@pytest.mark.parametrize("M", [1, 3, 8])
def test_linear_batch_block_shapes_against_oracle(awq, M):
    """The decoder block's seven linear shapes (q, k, v, o 4096x4096; gate, up
    11008x4096; down 4096x11008, scaled down 8x in their row counts) in one
    call: every output within the apply tolerance of the oracle, and each equal
    to what the same call gives for that linear alone (the tiles a linear
    contributes do not depend on the other linears of the launch)."""
    shapes = [(512, 512), (512, 512), (512, 512), (512, 512), (1376, 512), (1376, 512), (512, 1408)]
    gs = 128
    layers, refs = [], []
    for k, (o, i) in enumerate(shapes):
        W, X = small_layer(o, i, 64, seed=200 + k)
        pk = oracle.pack_int4(W, oracle.act_stats(X), 0.5, 1.0, gs, oracle.ASYM)
        x = apply_activations(M, i, seed=k)
        layers.append((dev(x), dev(pk["qweight"]), dev(pk["scales"]).view(torch.float16),
                       dev(pk["zeros"]), dev(pk["s16"]).view(torch.float16)))
        refs.append(oracle.linear_w4a16(x, pk["qweight"], pk["scales"], pk["zeros"], pk["s16"], gs))
    ys = awq.awq_linear_w4a16_batch(layers, gs)
    for layer, y, y_ref in zip(layers, ys, refs):
        check_apply(y, y_ref)
        (y1,) = awq.awq_linear_w4a16_batch([layer], gs)
        assert torch.equal(y, y1)


@pytest.mark.parametrize("M", [1, 2, 5, 8])
@pytest.mark.parametrize("gs,qt,with_s", [(64, oracle.ASYM, True), (128, oracle.SYM, False),
                                           (32, oracle.ASYM, True)])
def test_linear_batch_ragged_against_oracle(awq, M, gs, qt, with_s):
    """One launch over linears with ragged shapes, each output checked against
    the oracle: a last row tile of 5 or 8 rows whose scales are not 16-byte
    sized, an odd group count per row, an input width ending 64 columns into a
    1024-column stage, a single 16 x 64 tile, and more tiles in all than there
    are SMs, so CTAs cross from one linear into the next."""
    shapes = [(37, 1088), (512, 2112), (1000, 640), (16, 64), (3000, 1024), (200, 384)]
    shapes = [(o, i) for o, i in shapes if i % gs == 0]
    layers, refs = [], []
    for k, (o, i) in enumerate(shapes):
        W, X = small_layer(o, i, 32, seed=300 + k)
        pk = oracle.pack_int4(W, oracle.act_stats(X), 0.5, 1.0, gs, qt)
        x = apply_activations(M, i, seed=40 + k)
        s16 = pk["s16"] if with_s else None
        layers.append((dev(x), dev(pk["qweight"]), dev(pk["scales"]).view(torch.float16),
                       dev(pk["zeros"]) if pk["zeros"] is not None else None,
                       dev(s16).view(torch.float16) if s16 is not None else None))
        refs.append(oracle.linear_w4a16(x, pk["qweight"], pk["scales"], pk["zeros"], s16, gs))
    ys = awq.awq_linear_w4a16_batch(layers, gs)
    for y, y_ref in zip(ys, refs):
        check_apply(y, y_ref)


# ------------------------------------------------------------------ every output written
@pytest.mark.parametrize("M", [1, 3, 8, 16, 33, 256])
def test_apply_writes_every_output(awq, M):
    """The output buffer is filled with NaN before the call: every element must be
    overwritten (a tile that a kernel skipped would otherwise keep whatever the
    allocator handed back, possibly a previous call's correct values).  Ragged rows
    (300 = 2 x 128 + 44) over several slabs; every kernel by token count, and the
    batched call for M <= 8."""
    O, I, gs = 300, 1024, 128
    W, X = small_layer(O, I, 64, seed=77)
    pk = oracle.pack_int4(W, oracle.act_stats(X), 0.5, 1.0, gs, oracle.ASYM)
    x = apply_activations(M, I, seed=5)
    y_ref = oracle.linear_w4a16(x, pk["qweight"], pk["scales"], pk["zeros"], pk["s16"], gs)
    args = (dev(x), dev(pk["qweight"]), dev(pk["scales"]).view(torch.float16), dev(pk["zeros"]),
            dev(pk["s16"]).view(torch.float16))
    y = torch.full((M, O), float("nan"), dtype=torch.bfloat16, device="cuda")
    awq.awq_linear_w4a16(*args, gs, out=y)
    assert bool(torch.isfinite(y).all())
    check_apply(y, y_ref)
    if M <= 8:
        yb = torch.full((M, O), float("nan"), dtype=torch.bfloat16, device="cuda")
        awq.awq_linear_w4a16_batch([args], gs, outs=[yb])
        assert bool(torch.isfinite(yb).all())
        check_apply(yb, y_ref)
