"""Pins for the CPU oracle: each test ties one oracle function to something
other than itself — a value the pages print, a closed form, an invariant, or
brute force on a tiny input — chosen so that a dropped term, a wrong sign or
index, or a transposed operand fails at least one of them.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from synthetic import ALPHA_GRID, CLIP_GRID, bf16_bits, bf16_to_f32, small_layer

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rng(seed):
    return np.random.default_rng(seed)


# ----------------------------------------------------------------- worked example
def test_worked_example_16_levels():
    """The tutorial's 16-level example: step 0.427, 0.21 -> 0, output error 21."""
    g = json.load(open(os.path.join(GOLDEN, "worked_example_16level.json")))
    grp = np.array([g["range_min"], g["range_max"], g["weight"]] + [0.0] * 125, np.float32)
    q, d, z = oracle.quant_group(grp, oracle.ASYM)
    assert round(float(d), 3) == g["step_printed"]
    assert (q[0] - z) * d == pytest.approx(g["range_min"], abs=d / 2 * 1.0001)
    assert (q[1] - z) * d == pytest.approx(g["range_max"], abs=d / 2 * 1.0001)
    deq = (q[2] - z) * float(d)
    assert deq == g["dequantised"]
    err = abs(float(np.float32(g["weight"])) - deq)
    assert err == pytest.approx(g["weight_error"], rel=1e-6)
    assert err * g["activation"] == pytest.approx(g["output_error"], rel=1e-6)
    # the symmetric grid over the same range also sends 0.21 to 0
    qs, ds, zs = oracle.quant_group(grp, oracle.SYM)
    assert qs[2] == 0 and zs == 0


# ------------------------------------------------------------------ activation stats
def test_act_stats_integer_closed_form():
    """Integer-valued X: the fp64 sums are exact, so s_X = float32(S / N)."""
    r = rng(1)
    N, I = 300, 37                      # ragged: 3 chunks of 128 tokens, odd width
    Xi = r.integers(-9, 10, size=(N, I))
    Xi[:, 5] = 0                        # clamped column
    Xi[:, 6] = -2                       # sign: |X| not X
    got = oracle.act_stats(Xi.astype(np.float32), clamp_min=1e-4)
    S = np.abs(Xi).sum(axis=0)          # exact integer sums
    want = np.array([np.float32(float(Fraction(int(s), N))) for s in S])
    want[5] = np.float32(1e-4)
    assert np.array_equal(got, want)
    assert got[6] == np.float32(2.0)


def test_act_stats_fsum_within_one_ulp():
    """Random fp32 X: agrees with the exactly rounded mean (math.fsum) to 1 ulp."""
    r = rng(2)
    N, I = 517, 24
    X = (r.standard_normal((N, I)) * np.exp(r.uniform(-8, 8, size=(1, I)))).astype(np.float32)
    got = oracle.act_stats(X)
    for i in range(I):
        ref = np.float32(math.fsum(abs(float(v)) for v in X[:, i]) / N)
        assert abs(int(got[i].view(np.int32)) - int(ref.view(np.int32))) <= 1


def test_act_stats_axis_and_bf16():
    """Non-square bf16 input: reduced over tokens, one value per input channel."""
    W, X = small_layer(8, 64, 200, seed=3)
    s = oracle.act_stats(X)
    assert s.shape == (64,)
    Xf = bf16_to_f32(X).astype(np.float64)
    assert np.allclose(s, np.abs(Xf).mean(axis=0), rtol=1e-6)
    assert np.all(s >= np.float32(1e-4))


# ------------------------------------------------------------------ scale vector
def test_scale_vector_special_alphas():
    r = rng(4)
    sX = np.exp(r.uniform(-9, 4, size=257)).astype(np.float32)
    s0 = oracle.scale_vector(sX, 0.0)
    assert np.all(s0 == 1.0)                                   # alpha = 0: plain RTN
    s1 = oracle.scale_vector(sX, 1.0)
    assert s1.max() == 1.0 and s1[np.argmax(sX)] == 1.0
    assert np.allclose(s1, sX.astype(np.float64) / sX.max(), rtol=2 ** -24)
    sh = oracle.scale_vector(sX, 0.5)
    ref = np.sqrt(sX.astype(np.float64) / float(sX.max()))
    assert np.allclose(sh, ref, rtol=2 ** -23)


def test_scale_vector_power_law_and_order():
    r = rng(5)
    sX = np.exp(r.uniform(-9, 4, size=300)).astype(np.float32)
    for a in ALPHA_GRID[1:]:
        s = oracle.scale_vector(sX, a)
        assert s.max() == 1.0
        lhs = np.log(s.astype(np.float64)) / a
        rhs = np.log(sX.astype(np.float64)) - np.log(float(sX.max()))
        assert np.allclose(lhs, rhs, rtol=1e-5, atol=1e-5 / a)
        order = np.argsort(sX, kind="stable")
        assert np.all(np.diff(s[order]) >= 0)


# ------------------------------------------------------------------ quantizer
def _brute_nearest(t, lo, hi):
    """Nearest integer code to real t within [lo, hi], ties to the even code."""
    best, bd = None, None
    for c in range(lo, hi + 1):
        dd = abs(Fraction(t) - c)
        if bd is None or dd < bd or (dd == bd and c % 2 == 0):
            best, bd = c, dd
    return best


def test_quant_group_ties_to_even():
    g = np.array([7.0, 2.5, -1.5, 0.5, -0.5, 3.5, -6.5, 1.0], np.float32)
    q, d, z = oracle.quant_group(g, oracle.SYM)
    assert d == np.float32(1.0) and z == 0
    assert list(q) == [7, 2, -2, 0, 0, 4, -6, 1]


@pytest.mark.parametrize("gs", [32, 64, 128])
def test_quant_group_sym_brute_force(gs):
    r = rng(6 + gs)
    for trial in range(40):
        w = (r.standard_normal(gs) * 10.0 ** r.uniform(-4, 1)).astype(np.float32)
        q, d, z = oracle.quant_group(w, oracle.SYM)
        a = np.abs(w).max()
        assert d == np.float32(a) / np.float32(7.0)
        assert z == 0
        for k in range(gs):
            t = np.float32(w[k]) / d            # the fp32 quotient the pages' Round sees
            assert q[k] == _brute_nearest(float(t), -8, 7)
            assert abs(float(w[k]) - q[k] * float(d)) <= float(d) / 2 * (1 + 1e-6)
        assert abs(q[np.argmax(np.abs(w))]) == 7


@pytest.mark.parametrize("gs", [32, 128])
def test_quant_group_asym_brute_force(gs):
    r = rng(7 + gs)
    for trial in range(40):
        w = (r.standard_normal(gs) * 0.05 + r.uniform(-0.02, 0.02)).astype(np.float32)
        q, d, z = oracle.quant_group(w, oracle.ASYM)
        mx, mn = w.max(), w.min()
        assert d == (np.float32(mx) - np.float32(mn)) / np.float32(15.0)
        assert 0 <= z <= 15
        assert z == _brute_nearest(float(np.float32(-mn) / d), 0, 15)
        for k in range(gs):
            t = np.float32(w[k]) / d
            # one rule: the nearest representable offset q - z to the fp32 quotient,
            # ties to the even offset (rint(t) + z, then the clamp)
            assert q[k] == _brute_nearest(float(t), -z, 15 - z) + z
            assert abs(float(w[k]) - (q[k] - z) * float(d)) <= float(d) * (1 + 1e-6)
        assert q[np.argmin(w)] <= 1 and q[np.argmax(w)] >= 14


def test_quant_group_asym_tie_with_odd_zero_point():
    """Range [-3, 12]: Delta = 1 and z = 3 (odd).  Half-integer quotients round
    to the even offset q - z (2.5 -> 2 -> code 5; -0.5 -> 0 -> code 3), not to
    the even code (rounding t + z would give 6 and 2)."""
    g = np.array([12.0, -3.0, 2.5, -0.5, 0.5, 1.5, 4.5] + [1.0] * 121, np.float32)
    q, d, z = oracle.quant_group(g, oracle.ASYM)
    assert d == np.float32(1.0) and z == 3
    assert list(q[:7]) == [15, 0, 5, 3, 3, 5, 7]


def test_quant_group_asym_clip_hand_cases():
    """Clip r scales both bounds before Delta and z are formed; values beyond
    the clipped bounds saturate.  Range [-3, 12] at r = 0.5: bounds [-1.5, 6],
    Delta = 7.5 / 15 = 0.5, z = rint(1.5 / 0.5) = 3.  Clipping only the maximum
    would give Delta = 0.6, z = 5; a zero point from the unclipped minimum
    would give z = 6."""
    g = np.array([12.0, -3.0, 0.25, 0.75, 2.5, -0.5, 6.0, -1.5, 6.2, -1.8] + [1.0] * 118,
                 np.float32)
    q, d, z = oracle.quant_group(g, oracle.ASYM, clip=0.5)
    assert d == np.float32(0.5) and z == 3
    #            12  -3  .25 .75 2.5 -.5  6  -1.5 6.2 -1.8
    assert list(q[:10]) == [15, 0, 3, 5, 8, 2, 15, 0, 15, 0]
    # r = 0.25: bounds [-0.75, 3], Delta = 0.25, z = 3; 0.25 -> t = 1 -> code 4
    q, d, z = oracle.quant_group(g, oracle.ASYM, clip=0.25)
    assert d == np.float32(0.25) and z == 3
    assert list(q[:6]) == [15, 0, 4, 6, 13, 1]


@pytest.mark.parametrize("r", [0.9, 0.5])
def test_quant_group_asym_clip_fp32_and_enumeration(r):
    """Random groups at clip r: Delta and z bit-exact against the fp32 formulas
    (r applied to each bound in fp64 and rounded once, then one fp32 subtract and
    one fp32 divide); every code is the nearest representable offset after
    clipping, found by enumeration, ties to the even offset; elements beyond the
    clipped bounds saturate to 0 or 15."""
    g = rng(70 + int(r * 10))
    for trial in range(60):
        w = (g.standard_normal(128) * 0.05 + g.uniform(-0.03, 0.03)).astype(np.float32)
        q, d, z = oracle.quant_group(w, oracle.ASYM, clip=r)
        mxr = np.float32(np.float64(w.max()) * r)
        mnr = np.float32(np.float64(w.min()) * r)
        want_d = np.float32(mxr - mnr) / np.float32(15.0)
        assert d == want_d
        want_z = int(min(max(np.rint(np.float32(-mnr) / want_d), 0.0), 15.0))
        assert z == want_z
        for k in range(128):
            t = float(np.float32(w[k]) / d)
            assert q[k] == _brute_nearest(t, -z, 15 - z) + z
            if w[k] > mxr + d or w[k] < mnr - d:
                assert q[k] in (0, 15)
        assert q[np.argmax(w)] == 15 and q[np.argmin(w)] == 0


def test_quant_group_scale_invariance():
    """Codes are invariant under w -> w * 2^k, Delta scales by 2^k."""
    r = rng(8)
    w = (r.standard_normal(128) * 0.03).astype(np.float32)
    for qt in (oracle.SYM, oracle.ASYM):
        q0, d0, z0 = oracle.quant_group(w, qt)
        for k in (-7, -1, 3, 11):
            q1, d1, z1 = oracle.quant_group(w * np.float32(2.0 ** k), qt)
            assert np.array_equal(q0, q1) and z0 == z1
            assert d1 == d0 * np.float32(2.0 ** k)


def test_quant_group_degenerate_and_clip():
    q, d, z = oracle.quant_group(np.zeros(64, np.float32), oracle.SYM)
    assert d == 0 and np.all(q == 0)
    q, d, z = oracle.quant_group(np.full(64, 0.3, np.float32), oracle.ASYM)
    assert d == 0 and z == 0 and np.all(q == 0)
    r = rng(9)
    w = (r.standard_normal(128)).astype(np.float32)
    q, d, z = oracle.quant_group(w, oracle.SYM, clip=0.5)
    a = np.abs(w).max()
    assert d == np.float32(np.float64(a) * 0.5) / np.float32(7.0)
    big = np.abs(w) > 0.5 * a * 8.5 / 7
    assert np.all(np.abs(q[big]) >= 7) and q.min() >= -8 and q.max() <= 7
    assert np.any(q == -8) or np.any(q == 7)


def test_rounding_error_statistics():
    """Rounding error is ~U[0, 0.5] with mean 0.25 (paper summary, Method:
    the empirical observations on Round)."""
    r = rng(10)
    errs = []
    for _ in range(400):
        w = r.uniform(-1, 1, 128).astype(np.float32)
        w[0] = 1.0
        q, d, z = oracle.quant_group(w, oracle.SYM)
        errs.append(np.abs(w / d - q))
    e = np.concatenate(errs)
    assert e.max() <= 0.5 + 1e-6
    assert abs(e.mean() - 0.25) < 0.01


def test_salient_scaling_reduces_error():
    """Scaling one non-extreme weight by s = 2 leaves Delta unchanged and halves
    its expected error in original units (paper summary, Method: Err'/Err =
    (Delta'/Delta)(1/s))."""
    r = rng(11)
    e1, e2 = [], []
    for _ in range(3000):
        w = r.uniform(-1, 1, 128).astype(np.float32)
        w[0] = 1.0
        w[1] = np.float32(r.uniform(-0.45, 0.45))
        q, d, _ = oracle.quant_group(w, oracle.SYM)
        e1.append(abs(float(w[1]) - q[1] * float(d)))
        w2 = w.copy()
        w2[1] *= np.float32(2.0)
        q2, d2, _ = oracle.quant_group(w2, oracle.SYM)
        assert d2 == d
        e2.append(abs(q2[1] * float(d2) / 2.0 - float(w[1])))
    ratio = np.mean(e2) / np.mean(e1)
    assert 0.45 < ratio < 0.55


# ------------------------------------------------------------------ loss
def _lossless_layer(O, I, gs, seed):
    """W with W*s exactly on the quantisation grid (s powers of two)."""
    r = rng(seed)
    s = (2.0 ** r.integers(-3, 1, size=I)).astype(np.float32)
    s[0] = 1.0
    codes = r.integers(-7, 8, size=(O, I))
    codes[:, ::gs] = 7                               # every group reaches +-7
    delta = (2.0 ** r.integers(-9, -5, size=(O, I // gs))).astype(np.float32)
    W = (codes * np.repeat(delta, gs, axis=1) / s[None, :]).astype(np.float32)
    return W, s, codes, delta


def test_loss_zero_when_quantisation_is_exact():
    """W X = (W s)(X / s): with Q exact on W*s, the objective is exactly 0."""
    O, I, gs, N = 6, 256, 64, 40
    W, s, codes, delta = _lossless_layer(O, I, gs, 12)
    X = rng(13).integers(-3, 4, size=(N, I)).astype(np.float32)
    c, d, z = oracle.quant_layer(W, s, gs, oracle.SYM)
    assert np.array_equal(c, codes) and np.array_equal(d, delta)
    tot, lr = oracle.layer_loss_rows(W, X, s, gs, c, d, z)
    assert tot == 0.0 and np.all(lr == 0.0)


def test_loss_single_perturbation_closed_form():
    O, I, gs, N = 5, 128, 32, 33
    W, s, codes, delta = _lossless_layer(O, I, gs, 14)
    X = rng(15).integers(-5, 6, size=(N, I)).astype(np.float32)
    c, d, z = oracle.quant_layer(W, s, gs, oracle.SYM)
    o, k = 3, 77
    c = c.copy()
    c[o, k] += 1 if c[o, k] < 7 else -1
    tot, lr = oracle.layer_loss_rows(W, X, s, gs, c, d, z)
    e = float(d[o, k // gs]) / float(s[k])
    want = e * e * float((X[:, k].astype(np.float64) ** 2).sum())
    assert lr[o] == want and tot == want
    assert np.all(np.delete(lr, o) == 0.0)


def _brute_loss_rows(W, X, s, gs, c, d, z):
    O, I = W.shape
    out = []
    for o in range(O):
        acc = 0.0
        dw = [(int(c[o, i]) - int(z[o, i // gs])) * float(d[o, i // gs]) / float(s[i])
              - float(W[o, i]) for i in range(I)]
        for n in range(X.shape[0]):
            e = math.fsum(float(X[n, i]) * dw[i] for i in range(I))
            acc += e * e
        out.append(acc)
    return np.array(out)


@pytest.mark.parametrize("qt", [0, 1])
def test_loss_brute_force_tiny(qt):
    W, X = small_layer(3, 64, 7, wdtype="f32", xdtype="f32", seed=16, n_outliers=2)
    sX = oracle.act_stats(X)
    s = oracle.scale_vector(sX, 0.35)
    c, d, z = oracle.quant_layer(W, s, 32, qt)
    tot, lr = oracle.layer_loss_rows(W, X, s, 32, c, d, z)
    ref = _brute_loss_rows(W, X, s, 32, c, d, z)
    assert np.allclose(lr, ref, rtol=1e-12, atol=0)


def test_search_brute_force_argmin_and_invariants():
    """Non-square tiny layer: the search's losses equal the brute-force losses
    at each grid point, alpha* is their first minimiser, loss(alpha=0) is plain
    RTN, and loss(clip = 1.0) equals loss(alpha*)."""
    O, I, N, gs = 4, 96, 11, 32
    W, X = small_layer(O, I, N, wdtype="f32", xdtype="f32", seed=17, n_outliers=3, outlier=30.0)
    sX = oracle.act_stats(X)
    alpha = ALPHA_GRID[::4]
    res = oracle.search_layer(W, X, sX, gs, oracle.SYM, alpha, clip=CLIP_GRID[:4])
    ref = []
    for a in alpha:
        s = oracle.scale_vector(sX, a)
        c, d, z = oracle.quant_layer(W, s, gs, oracle.SYM)
        ref.append(_brute_loss_rows(W, X, s, gs, c, d, z).sum() / (N * O))
    assert np.allclose(res["loss"][:len(alpha)], ref, rtol=1e-12)
    assert res["best_alpha"] == int(np.argmin(ref))
    c, d, z = oracle.quant_layer(W, np.ones(I, np.float32), gs, oracle.SYM)
    rtn = _brute_loss_rows(W, X, np.ones(I, np.float32), gs, c, d, z).sum() / (N * O)
    assert res["loss"][0] == pytest.approx(rtn, rel=1e-12)
    assert res["loss"][len(alpha)] == res["loss"][res["best_alpha"]]
    assert res["best_clip"] == int(np.argmin(res["loss"][len(alpha):]))


def _enum_quant_layer(W, s, gs, qt, clip):
    """Codes of Q(W*s) found by enumeration: per group the bounds (times clip)
    give Delta (and z); each element takes the nearest representable offset to
    its fp32 quotient, ties to the even offset."""
    Wf = oracle.as_f32(W)
    O, I = Wf.shape
    c = np.zeros((O, I), np.int64)
    d = np.zeros((O, I // gs), np.float32)
    z = np.zeros((O, I // gs), np.int64)
    for o in range(O):
        for j in range(I // gs):
            wp = (Wf[o, j * gs:(j + 1) * gs] * s[j * gs:(j + 1) * gs]).astype(np.float32)
            if qt == oracle.SYM:
                a = np.float32(np.float64(np.abs(wp).max()) * clip)
                dd, zz, lo, hi = np.float32(a) / np.float32(7.0), 0, -8, 7
            else:
                mxr = np.float32(np.float64(wp.max()) * clip)
                mnr = np.float32(np.float64(wp.min()) * clip)
                dd = np.float32(mxr - mnr) / np.float32(15.0)
                zz = int(min(max(np.rint(np.float32(-mnr) / dd), 0.0), 15.0))
                lo, hi = -zz, 15 - zz
            d[o, j], z[o, j] = dd, zz
            for k in range(gs):
                c[o, j * gs + k] = _brute_nearest(float(np.float32(wp[k]) / dd), lo, hi) + zz
    return c, d, z


def test_search_asym_clip_grid_brute_force():
    """Asymmetric search with a clip grid on a tiny non-square layer: every
    alpha-phase and clip-phase loss equals the brute-force loss over codes found
    by enumeration; alpha* and r* are the first minimisers; loss(r = 1.0) equals
    loss(alpha*)."""
    O, I, N, gs = 3, 64, 9, 32
    W, X = small_layer(O, I, N, wdtype="f32", xdtype="f32", seed=71, n_outliers=2, outlier=25.0)
    sX = oracle.act_stats(X)
    alpha = ALPHA_GRID[::5]
    clip = CLIP_GRID[::2]
    res = oracle.search_layer(W, X, sX, gs, oracle.ASYM, alpha, clip=clip)
    ref = []
    for a in alpha:
        s = oracle.scale_vector(sX, a)
        c, d, z = _enum_quant_layer(W, s, gs, oracle.ASYM, 1.0)
        ref.append(_brute_loss_rows(W, X, s, gs, c, d, z).sum() / (N * O))
    assert np.allclose(res["loss"][:len(alpha)], ref, rtol=1e-12)
    ba = int(np.argmin(ref))
    assert res["best_alpha"] == ba
    s = oracle.scale_vector(sX, alpha[ba])
    ref_c = []
    for r in clip:
        c, d, z = _enum_quant_layer(W, s, gs, oracle.ASYM, float(r))
        ref_c.append(_brute_loss_rows(W, X, s, gs, c, d, z).sum() / (N * O))
    assert np.allclose(res["loss"][len(alpha):], ref_c, rtol=1e-12)
    assert res["best_clip"] == int(np.argmin(ref_c))
    assert res["loss"][len(alpha)] == res["loss"][ba]          # clip[0] = 1.0
    assert len(set(np.round(ref_c, 15))) > 2                   # the clip grid changes the loss


def test_search_first_minimum_on_ties():
    """With X = 0 every loss is 0: the first grid point wins."""
    W, _ = small_layer(4, 64, 8, seed=18)
    X = np.zeros((8, 64), np.float32)
    sX = oracle.act_stats(X)
    res = oracle.search_layer(W, X, sX, 32, oracle.SYM, ALPHA_GRID[:5], clip=CLIP_GRID[:3])
    assert np.all(res["loss"] == 0.0)
    assert res["best_alpha"] == 0 and res["best_clip"] == 0


def test_search_row_subset_matches_full():
    W, X = small_layer(12, 64, 20, seed=19)
    sX = oracle.act_stats(X)
    full = oracle.search_layer(W, X, sX, 32, oracle.ASYM, ALPHA_GRID[:3])
    rows = np.array([1, 5, 11])
    sub = oracle.search_layer(W, X, sX, 32, oracle.ASYM, ALPHA_GRID[:3], rows=rows)
    assert np.array_equal(sub["loss_row"], full["loss_row"][:, rows])


# ------------------------------------------------------------------ pack
@pytest.mark.parametrize("qt", [0, 1])
def test_pack_layout(qt):
    O, I, gs = 5, 640, 128               # 5 groups: a partly filled zero word
    W, X = small_layer(O, I, 16, seed=20)
    sX = oracle.act_stats(X)
    p = oracle.pack_int4(W, sX, 0.45, 0.9, gs, qt)
    s = oracle.scale_vector(sX, 0.45)
    c, d, z = oracle.quant_layer(W, s, gs, qt, clip=0.9)
    nib = np.stack([(p["qweight"] >> np.uint32(4 * k)) & np.uint32(15) for k in range(8)], axis=-1)
    codes = nib.reshape(O, I).astype(np.int64)
    assert np.array_equal(codes, c.astype(np.int64) + (8 if qt == 0 else 0))
    assert np.array_equal(p["scales"], d.astype(np.float16).view(np.uint16))
    assert np.array_equal(p["scales_f32"], d)
    assert np.array_equal(p["s16"], s.astype(np.float16).view(np.uint16))
    if qt == 1:
        zn = np.stack([(p["zeros"] >> np.uint32(4 * k)) & np.uint32(15) for k in range(8)], axis=-1)
        zn = zn.reshape(O, -1)
        assert np.array_equal(zn[:, :I // gs], z.astype(np.uint32))
        assert np.all(zn[:, I // gs:] == 0)
    else:
        assert p["zeros"] is None


# ------------------------------------------------------------------ apply
def test_apply_integer_closed_form():
    """s = 1, Delta = 1, symmetric: y = x (codes - 8)^T exactly."""
    r = rng(21)
    M, I, O, gs = 3, 256, 7, 64
    codes = r.integers(0, 16, size=(O, I)).astype(np.uint32)
    qw = np.zeros((O, I // 8), np.uint32)
    for k in range(8):
        qw |= codes[:, k::8] << np.uint32(4 * k)
    one16 = np.float16(1.0).view(np.uint16)
    scales = np.full((O, I // gs), one16, np.uint16)
    s16 = np.full(I, one16, np.uint16)
    x = r.integers(-4, 5, size=(M, I))
    y = oracle.linear_w4a16(x.astype(np.float32), qw, scales, None, s16, gs)
    assert np.array_equal(y, (x @ (codes.astype(np.int64) - 8).T).astype(np.float64))


def test_apply_matches_dense_dequant():
    O, I, gs, M = 9, 384, 128, 4
    W, X = small_layer(O, I, 32, seed=22)
    sX = oracle.act_stats(X)
    p = oracle.pack_int4(W, sX, 0.6, 1.0, gs, oracle.ASYM)
    x = bf16_bits(rng(23).standard_normal((M, I)).astype(np.float32))
    y = oracle.linear_w4a16(x, p["qweight"], p["scales"], p["zeros"], p["s16"], gs)
    s = oracle.scale_vector(sX, 0.6)
    c, d, z = oracle.quant_layer(W, s, gs, oracle.ASYM)
    d16 = d.astype(np.float16).astype(np.float64)
    deq = (c.astype(np.float64) - np.repeat(z.astype(np.float64), gs, axis=1)) * np.repeat(d16, gs, axis=1)
    xs = bf16_to_f32(x).astype(np.float64) / s.astype(np.float16).astype(np.float64)[None, :]
    assert np.allclose(y, xs @ deq.T, rtol=1e-12, atol=1e-12)
    # and it approximates the unquantised layer
    yf = bf16_to_f32(x).astype(np.float64) @ bf16_to_f32(W).astype(np.float64).T
    assert np.linalg.norm(y - yf) < 0.2 * np.linalg.norm(yf)


# ------------------------------------------------------------------ w_bit = 3
def test_quant_group_w3_hand_case():
    """3-bit symmetric: Delta = max / 3, codes in [-4, 3]; 3-bit asymmetric:
    Delta = range / 7, z and codes in [0, 7] ([AWQ-guide] 三's 2^(w_bit-1) - 1
    at w_bit = 3)."""
    g = np.array([3.0, -1.5, 1.5, 0.5, -0.5, 2.5, -3.0] + [0.0] * 57, np.float32)
    q, d, z = oracle.quant_group(g, oracle.SYM, w_bit=3)
    assert d == np.float32(1.0) and z == 0
    assert list(q[:7]) == [3, -2, 2, 0, 0, 2, -3]
    g = np.array([5.0, -2.0, 0.5, 1.5, 2.5] + [0.0] * 59, np.float32)
    q, d, z = oracle.quant_group(g, oracle.ASYM, w_bit=3)
    assert d == np.float32(1.0) and z == 2                  # range 7 over 7 steps
    assert list(q[:5]) == [7, 0, 2, 4, 4]                    # 0.5 -> 0, 1.5 -> 2, 2.5 -> 2 (+z)


@pytest.mark.parametrize("qt", [0, 1])
def test_quant_group_w3_enumeration(qt):
    g = rng(80 + qt)
    for trial in range(40):
        w = (g.standard_normal(64) * 0.04).astype(np.float32)
        for clip in (1.0, 0.8):
            q, d, z = oracle.quant_group(w, qt, clip=clip, w_bit=3)
            if qt == oracle.SYM:
                a = np.float32(np.float64(np.abs(w).max()) * clip)
                assert d == a / np.float32(3.0) and z == 0
                lo, hi = -4, 3
            else:
                mxr = np.float32(np.float64(w.max()) * clip)
                mnr = np.float32(np.float64(w.min()) * clip)
                assert d == np.float32(mxr - mnr) / np.float32(7.0)
                assert z == int(min(max(np.rint(np.float32(-mnr) / d), 0.0), 7.0))
                lo, hi = -z, 7 - z
            for k in range(64):
                assert q[k] == _brute_nearest(float(np.float32(w[k]) / d), lo, hi) + z
            if clip == 1.0:
                err = np.abs(w.astype(np.float64) - (q - z) * float(d))
                assert err.max() <= float(d) / 2 * (1 + 1e-6) + (float(d) if qt else 0.0)


def test_search_w3_brute_force():
    """The 3-bit search: losses equal brute-force losses over enumerated 3-bit
    codes, and every 3-bit loss exceeds the 4-bit loss at the same alpha."""
    O, I, N, gs = 3, 64, 8, 32
    W, X = small_layer(O, I, N, wdtype="f32", xdtype="f32", seed=81, n_outliers=2)
    sX = oracle.act_stats(X)
    alpha = ALPHA_GRID[::6]
    r3 = oracle.search_layer(W, X, sX, gs, oracle.SYM, alpha, w_bit=3)
    r4 = oracle.search_layer(W, X, sX, gs, oracle.SYM, alpha, w_bit=4)
    for k, a in enumerate(alpha):
        s = oracle.scale_vector(sX, a)
        Wf = oracle.as_f32(W)
        c = np.zeros((O, I), np.int64)
        d = np.zeros((O, I // gs), np.float32)
        for o in range(O):
            for j in range(I // gs):
                wp = (Wf[o, j * gs:(j + 1) * gs] * s[j * gs:(j + 1) * gs]).astype(np.float32)
                d[o, j] = np.float32(np.abs(wp).max()) / np.float32(3.0)
                for t in range(gs):
                    c[o, j * gs + t] = _brute_nearest(float(wp[t] / d[o, j]), -4, 3)
        ref = _brute_loss_rows(W, X, s, gs, c, d, np.zeros((O, I // gs), np.int64)).sum() / (N * O)
        assert r3["loss"][k] == pytest.approx(ref, rel=1e-12)
        assert r3["loss"][k] > r4["loss"][k]


# ------------------------------------------------------------------ joint grid
def test_search_points_joint_grid_brute_force():
    """Every (alpha, r) pair of a joint grid: the loss equals the brute-force
    loss over enumerated codes at that pair; the best pair is the first
    minimiser; pairs with r = 1 reproduce the alpha search."""
    O, I, N, gs = 3, 64, 9, 32
    W, X = small_layer(O, I, N, wdtype="f32", xdtype="f32", seed=82, n_outliers=2, outlier=25.0)
    sX = oracle.act_stats(X)
    al = ALPHA_GRID[::5]
    cl = CLIP_GRID[::3]
    A, C = np.meshgrid(al, cl, indexing="ij")
    res = oracle.search_points(W, X, sX, gs, oracle.ASYM, A.ravel(), C.ravel())
    ref = []
    for a, r in zip(A.ravel(), C.ravel()):
        s = oracle.scale_vector(sX, a)
        c, d, z = _enum_quant_layer(W, s, gs, oracle.ASYM, float(r))
        ref.append(_brute_loss_rows(W, X, s, gs, c, d, z).sum() / (N * O))
    assert np.allclose(res["loss"], ref, rtol=1e-12)
    assert res["best"] == int(np.argmin(ref))
    plain = oracle.search_layer(W, X, sX, gs, oracle.ASYM, al)
    assert np.array_equal(res["loss"].reshape(len(al), len(cl))[:, 0], plain["loss"])


# ------------------------------------------------------------------ per-group clip
def test_group_clip_brute_force():
    """Per-group clip: each group's error at each ratio equals the brute-force
    sum over tokens of its squared partial output error (codes by enumeration,
    fsum over the group's columns); the chosen ratio is the first minimiser."""
    O, I, N, gs = 2, 64, 6, 32
    W, X = small_layer(O, I, N, wdtype="f32", xdtype="f32", seed=83, n_outliers=2, outlier=25.0)
    sX = oracle.act_stats(X)
    clip = CLIP_GRID[::2]
    a = 0.4
    for qt in (oracle.SYM, oracle.ASYM):
        res = oracle.group_clip(W, X, sX, a, gs, qt, clip, want_err=True)
        s = oracle.scale_vector(sX, a)
        Wf, Xf = oracle.as_f32(W), oracle.as_f32(X)
        for ri, r in enumerate(clip):
            c, d, z = _enum_quant_layer(W, s, gs, qt, float(r))
            for o in range(O):
                for j in range(I // gs):
                    cols = range(j * gs, (j + 1) * gs)
                    dw = [(int(c[o, i]) - int(z[o, j])) * float(d[o, j]) / float(s[i]) - float(Wf[o, i])
                          for i in cols]
                    e = sum(math.fsum(float(Xf[n, i]) * dw[k] for k, i in enumerate(cols)) ** 2
                            for n in range(N))
                    assert res["err"][o, j, ri] == pytest.approx(e, rel=1e-12)
        assert np.array_equal(res["best"], np.argmin(res["err"], axis=2))
        assert np.all(np.min(res["err"], axis=2) <= res["err"][:, :, 0])


def test_group_clip_single_ratio_and_pack():
    """A one-point grid {1.0} selects index 0 everywhere; packing with per-group
    ratios all equal to r equals packing at the layer ratio r; per-group
    packing takes each group's codes at its own ratio."""
    O, I, N, gs = 4, 256, 10, 64
    W, X = small_layer(O, I, N, seed=84)
    sX = oracle.act_stats(X)
    res = oracle.group_clip(W, X, sX, 0.5, gs, oracle.ASYM, [1.0])
    assert np.all(res["best"] == 0)
    for qt in (oracle.SYM, oracle.ASYM):
        flat = oracle.pack_int4(W, sX, 0.5, 0.85, gs, qt)
        pg = oracle.pack_int4(W, sX, 0.5, 1.0, gs, qt, clip_g=np.full((O, I // gs), 0.85))
        for k in ("qweight", "scales", "s16", "scales_f32"):
            assert np.array_equal(flat[k], pg[k])
        ratios = CLIP_GRID[rng(85).integers(0, len(CLIP_GRID), size=(O, I // gs))]
        pg = oracle.pack_int4(W, sX, 0.5, 1.0, gs, qt, clip_g=ratios)
        s = oracle.scale_vector(sX, 0.5)
        nib = np.stack([(pg["qweight"] >> np.uint32(4 * k)) & np.uint32(15) for k in range(8)],
                       axis=-1).reshape(O, I).astype(np.int64)
        for o in range(O):
            for j in range(I // gs):
                c, d, z = _enum_quant_layer(W[o:o + 1], s, gs, qt, float(ratios[o, j]))
                sl = slice(j * gs, (j + 1) * gs)
                assert np.array_equal(nib[o, sl], c[0, sl] + (8 if qt == oracle.SYM else 0))
                assert pg["scales_f32"][o, j] == d[0, j]


# ------------------------------------------------------------------ fold of 1/s
def test_apply_without_scale_is_integer_closed_form():
    """s16 = None: x is used as is.  With Delta = 1 the result is x (codes - 8)^T
    exactly, and equals the call with s16 = 1."""
    r = rng(86)
    M, I, O, gs = 2, 128, 5, 64
    codes = r.integers(0, 16, size=(O, I)).astype(np.uint32)
    qw = np.zeros((O, I // 8), np.uint32)
    for k in range(8):
        qw |= codes[:, k::8] << np.uint32(4 * k)
    one16 = np.float16(1.0).view(np.uint16)
    scales = np.full((O, I // gs), one16, np.uint16)
    x = r.integers(-4, 5, size=(M, I)).astype(np.float32)
    y = oracle.linear_w4a16(x, qw, scales, None, None, gs)
    assert np.array_equal(y, (x.astype(np.int64) @ (codes.astype(np.int64) - 8).T).astype(np.float64))
    y1 = oracle.linear_w4a16(x, qw, scales, None, np.full(I, one16, np.uint16), gs)
    assert np.array_equal(y, y1)


def test_fold_scale_closed_forms():
    """Dividing by power-of-two scales is exact; s = 1 is the identity; random
    scales round once in fp32 then to bf16 (checked against torch's own
    float-to-bfloat16 conversion); a folded input through the apply without s
    equals the unfolded input through the apply with s when the division is
    exact."""
    import torch
    r = rng(87)
    R, C = 64, 24
    P = bf16_bits(r.standard_normal((R, C)).astype(np.float32))
    k = r.integers(-6, 1, size=R)
    s16 = (2.0 ** k).astype(np.float16).view(np.uint16)
    out = oracle.fold_scale(P, s16)
    assert np.array_equal(bf16_to_f32(out), bf16_to_f32(P) * (2.0 ** -k)[:, None].astype(np.float32))
    ones = np.full(R, np.float16(1.0).view(np.uint16), np.uint16)
    assert np.array_equal(oracle.fold_scale(P, ones), P)
    s_r = r.uniform(0.01, 1.0, size=R).astype(np.float16)
    got = oracle.fold_scale(P, s_r.view(np.uint16))
    q32 = bf16_to_f32(P) / s_r.astype(np.float32)[:, None]      # one fp32 division
    want = torch.from_numpy(q32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, want)
    got32 = oracle.fold_scale(P, s_r.view(np.uint16), out_bf16=False)
    assert np.array_equal(got32, q32)
    # fold then apply without s == apply with s, for exact (power-of-two) scales
    I, O, gs = 64, 6, 32
    W, X = small_layer(O, I, 12, seed=88)
    sX = (2.0 ** r.integers(-5, 1, size=I)).astype(np.float32)
    pk = oracle.pack_int4(W, sX, 1.0, 1.0, gs, oracle.ASYM)
    x = bf16_bits(r.standard_normal((3, I)).astype(np.float32))
    xf = oracle.fold_scale(x.T.copy(), pk["s16"]).T.copy()        # channel = row of P
    y_fold = oracle.linear_w4a16(xf, pk["qweight"], pk["scales"], pk["zeros"], None, gs)
    y = oracle.linear_w4a16(x, pk["qweight"], pk["scales"], pk["zeros"], pk["s16"], gs)
    assert np.array_equal(y_fold, y)
