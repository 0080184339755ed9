"""C-ABI boundary checks that need no GPU: the library loads, exports every
entry point the public header declares, and rejects invalid calls on the host
with the documented status before any CUDA work is enqueued."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "awq_b200.h")

awq = pytest.importorskip("weight_only_quantization_awq_b200")
lib = awq.lib

OK, ARG, ALIGN, UNSUP = 0, 1, 2, 3
FAKE = 0x10000          # a 16-byte aligned address that is never dereferenced
NULL = None


def header_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:awq_status_t|int|void|double|const char \*)\s*\*?(awq_\w+)\s*\(",
                                 text, re.M)))


def test_header_symbols_exported():
    syms = header_symbols()
    assert {"awq_act_stats", "awq_search_layer", "awq_pack_int4", "awq_linear_w4a16"} <= set(syms)
    for s in syms:
        assert hasattr(lib, s), s
    assert set(syms) <= set(awq.EXPORTS)


def test_version_and_status_strings():
    assert lib.awq_version() >= 100
    names = [lib.awq_status_string(k).decode() for k in range(6)]
    assert names == ["AWQ_OK", "AWQ_ERR_ARG", "AWQ_ERR_ALIGN", "AWQ_ERR_UNSUPPORTED",
                     "AWQ_ERR_CUDA", "AWQ_ERR_TIMEOUT"]


def _search(**kw):
    a = (ctypes.c_double * 20)(*[k / 20 for k in range(20)])
    c = (ctypes.c_double * 3)(1.0, 0.9, 0.8)
    loss = (ctypes.c_double * 23)()
    ba, bc = ctypes.c_int(), ctypes.c_int()
    args = dict(W=FAKE, wdt=1, out=256, inp=512, X=FAKE, xdt=1, N=1024, sX=FAKE, gs=128, wbit=4,
                quant=0, alpha=a, na=20, clip=c, nc=3, loss=loss, lrow=NULL,
                ba=ctypes.byref(ba), bc=ctypes.byref(bc), st=NULL)
    args.update(kw)
    return lib.awq_search_layer(*args.values())


@pytest.mark.parametrize("kw,status", [
    (dict(W=NULL), ARG), (dict(wdt=7), ARG), (dict(out=0), ARG), (dict(quant=2), ARG),
    (dict(gs=96), UNSUP), (dict(gs=256), UNSUP), (dict(inp=520), UNSUP), (dict(wbit=2), UNSUP), (dict(wbit=8), UNSUP),
    (dict(inp=576), UNSUP),          # a multiple of 64 that 128-column groups do not divide
    (dict(W=FAKE + 8), ALIGN), (dict(X=FAKE + 4), ALIGN), (dict(na=0), ARG), (dict(na=65), ARG),
    (dict(nc=-1), ARG), (dict(clip=NULL), ARG), (dict(N=0), ARG), (dict(loss=NULL), ARG),
    (dict(alpha=(ctypes.c_double * 20)(*([0.5] * 19 + [1.5]))), ARG),
    (dict(clip=(ctypes.c_double * 3)(1.0, 0.0, 0.5)), ARG),
])
def test_search_rejects_on_host(kw, status):
    assert _search(**kw) == status
    assert lib.awq_last_error().decode() != ""


def test_act_stats_rejects_on_host():
    f = lib.awq_act_stats
    assert f(NULL, 1, 16, 64, ctypes.c_float(1e-4), FAKE, NULL) == ARG
    assert f(FAKE, 3, 16, 64, ctypes.c_float(1e-4), FAKE, NULL) == ARG
    assert f(FAKE, 1, 0, 64, ctypes.c_float(1e-4), FAKE, NULL) == ARG
    assert f(FAKE, 1, 16, 12, ctypes.c_float(1e-4), FAKE, NULL) == UNSUP
    assert f(FAKE + 2, 1, 16, 64, ctypes.c_float(1e-4), FAKE, NULL) == ALIGN
    assert f(FAKE, 1, 16, 64, ctypes.c_float(-1.0), FAKE, NULL) == ARG


def test_pack_rejects_on_host():
    f = lib.awq_pack_int4
    base = [FAKE, 1, 128, 256, FAKE, ctypes.c_double(0.5), ctypes.c_double(1.0), 128, 0,
            FAKE, FAKE, NULL, FAKE, NULL, NULL]
    def call(kw):
        a = list(base)
        for k, v in kw.items():
            a[k] = v
        return f(*a)
    assert call({11: FAKE}) == ARG               # zeros given for symmetric storage
    assert call({8: 1}) == ARG                   # asymmetric without zeros
    assert call({5: ctypes.c_double(-0.1)}) == ARG
    assert call({6: ctypes.c_double(0.0)}) == ARG
    assert call({7: 48}) == UNSUP
    assert call({3: 320}) == UNSUP               # in = 320 is not a whole number of 128-column groups
    assert call({9: FAKE + 4}) == ALIGN
    assert call({4: NULL}) == ARG


def test_linear_rejects_on_host():
    f = lib.awq_linear_w4a16
    base = [FAKE, 1, 4096, 4096, FAKE, FAKE, NULL, FAKE, 128, FAKE, NULL]
    def call(kw):
        a = list(base)
        for k, v in kw.items():
            a[k] = v
        return f(*a)
    assert call({0: NULL}) == ARG
    assert call({1: 0}) == ARG
    assert call({2: 100}) == UNSUP
    assert call({2: 4160}) == UNSUP              # multiple of 64, not of the 128-column group
    assert call({8: 16}) == UNSUP
    assert call({0: FAKE + 2}) == ALIGN


def test_search_points_rejects_on_host():
    f = lib.awq_search_points
    n = 6
    a = (ctypes.c_double * n)(*([0.5] * n))
    c = (ctypes.c_double * n)(*([1.0, 0.9] * 3))
    loss = (ctypes.c_double * n)()
    best = ctypes.c_int()
    base = dict(W=FAKE, wdt=1, out=256, inp=512, X=FAKE, xdt=1, N=1024, sX=FAKE, gs=128, wbit=3,
                quant=1, alpha=a, clip=c, n=n, loss=loss, lrow=NULL, best=ctypes.byref(best),
                st=NULL)

    def call(**kw):
        args = dict(base)
        args.update(kw)
        return f(*args.values())
    assert call(n=0) == ARG
    assert call(n=4097) == ARG
    assert call(clip=NULL) == ARG
    assert call(alpha=(ctypes.c_double * n)(*([0.5] * 5 + [2.0]))) == ARG
    assert call(clip=(ctypes.c_double * n)(*([1.0] * 5 + [0.0]))) == ARG
    assert call(wbit=5) == UNSUP
    assert call(gs=96) == UNSUP
    assert call(best=NULL) == ARG
    assert call(lrow=FAKE + 4) == ALIGN


def test_pack_quant_rejects_on_host():
    f = lib.awq_pack_quant
    grid = (ctypes.c_double * 3)(1.0, 0.9, 0.8)
    base = [FAKE, 1, 128, 256, FAKE, ctypes.c_double(0.5), ctypes.c_double(1.0), NULL, NULL, 0,
            128, 3, 1, FAKE, FAKE, FAKE, FAKE, NULL, NULL]

    def call(kw):
        a = list(base)
        for k, v in kw.items():
            a[k] = v
        return f(*a)
    assert call({11: 2}) == UNSUP                # w_bit
    assert call({7: FAKE}) == ARG                # per-group indices without a grid
    assert call({7: FAKE, 8: grid, 9: 0}) == ARG
    assert call({7: FAKE, 8: grid, 9: 65}) == ARG
    assert call({7: FAKE, 8: (ctypes.c_double * 3)(1.0, 1.5, 0.8), 9: 3}) == ARG
    assert call({15: NULL}) == ARG               # asymmetric without zeros
    assert call({6: ctypes.c_double(0.0)}) == ARG


def test_fold_and_selftest_reject_on_host():
    f = lib.awq_fold_scale
    assert f(NULL, 1, 16, 4, FAKE, FAKE, NULL) == ARG
    assert f(FAKE, 2, 16, 4, FAKE, FAKE, NULL) == ARG
    assert f(FAKE, 1, 0, 4, FAKE, FAKE, NULL) == ARG
    assert f(FAKE, 1, 16, 4, NULL, FAKE, NULL) == ARG
    assert f(FAKE + 1, 1, 16, 4, FAKE, FAKE, NULL) == ALIGN
    assert f(FAKE + 2, 0, 16, 4, FAKE, FAKE, NULL) == ALIGN
    g = lib.awq_wait_selftest
    assert g(0, 0, NULL) == ARG
    assert g(5_000_000_000, 0, NULL) == ARG


def test_linear_accepts_missing_scale_vector_on_host():
    """s16 = NULL (x already divided by s) passes validation: the call only fails
    later, for want of a device, not as an argument error."""
    f = lib.awq_linear_w4a16
    st = f(FAKE, 1, 4096, 4096, FAKE, FAKE, NULL, NULL, 128, FAKE, NULL)
    assert st not in (ARG, ALIGN, UNSUP)


def test_linear_batch_rejects_on_host():
    from weight_only_quantization_awq_b200 import _LinearDesc
    f = lib.awq_linear_w4a16_batch

    def descs(*mods):
        d = (_LinearDesc * len(mods))()
        for k, m in enumerate(mods):
            v = dict(x=FAKE, in_=4096, out=4096, qweight=FAKE, scales=FAKE, zeros=FAKE, s16=FAKE, y=FAKE)
            v.update(m)
            d[k] = _LinearDesc(**v)
        return ctypes.cast(d, ctypes.c_void_p)
    assert f(NULL, 1, 1, 128, NULL) == ARG
    assert f(descs({}), 0, 1, 128, NULL) == ARG
    assert f(descs(*([{}] * 9)), 9, 1, 128, NULL) == ARG
    assert f(descs({}), 1, 0, 128, NULL) == ARG
    assert f(descs({}), 1, 1, 96, NULL) == UNSUP
    assert f(descs({}, {"zeros": None}), 2, 1, 128, NULL) == ARG      # zero points for some only
    assert f(descs({}, {"y": None}), 2, 1, 128, NULL) == ARG
    assert f(descs({}, {"in_": 100}), 2, 1, 128, NULL) == UNSUP
    assert f(descs({}, {"x": FAKE + 2}), 2, 1, 128, NULL) == ALIGN


def test_linear_binding_checks_operand_sizes_before_any_pointer():
    """The Python binding refuses operands that do not match the packed layout (a short
    tensor would be read past its end on the GPU), before the library sees a pointer."""
    import torch
    M, I, O, gs = 2, 256, 40, 64
    nG = I // gs
    x = torch.zeros((M, I), dtype=torch.bfloat16)
    q = torch.zeros((O, I // 8), dtype=torch.int32)
    sc = torch.zeros((O, nG), dtype=torch.float16)
    z = torch.zeros((O, (nG + 7) // 8), dtype=torch.int32)
    s16 = torch.ones(I, dtype=torch.float16)
    cases = [
        (dict(qweight=q[:, :-1]), "qweight"),
        (dict(qweight=q.to(torch.int16)), "qweight"),
        (dict(scales=sc[:-1]), "scales"),
        (dict(scales=sc.float()), "scales"),
        (dict(zeros=z[:-1]), "zeros"),
        (dict(s16=s16[:-8]), "s16"),
        (dict(x=x.float()), "x"),
        (dict(group_size=96), "group_size"),
    ]
    for change, word in cases:
        args = dict(x=x, qweight=q, scales=sc, zeros=z, s16=s16, group_size=gs)
        args.update(change)
        with pytest.raises(ValueError, match=word):
            awq.awq_linear_w4a16(**args)
        with pytest.raises(ValueError, match=word):
            awq.awq_linear_w4a16_batch([(args["x"], args["qweight"], args["scales"], args["zeros"],
                                         args["s16"])], args["group_size"])
    # every size right: refused only because the tensors are not on a GPU
    with pytest.raises(ValueError, match="CUDA"):
        awq.awq_linear_w4a16(x, q, sc, z, s16, gs)
    with pytest.raises(ValueError, match="CUDA"):
        awq.awq_linear_w4a16(x, q, sc, None, None, gs)


def test_search_and_pack_bindings_check_layer_inputs():
    """W [out, in], X [N, in] and s_X [in] float32 are checked before any pointer
    reaches the library (a narrower X, or a shorter or 16-bit s_X, would be read past
    its end on the GPU)."""
    import torch
    W = torch.zeros((32, 128), dtype=torch.bfloat16)
    X = torch.zeros((64, 128), dtype=torch.bfloat16)
    sX = torch.ones(128, dtype=torch.float32)
    calls = [
        lambda W, X, sX: awq.awq_search_layer(W, X, sX, 64),
        lambda W, X, sX: awq.awq_search_points(W, X, sX, [0.5], [1.0], 64),
        lambda W, X, sX: awq.awq_group_clip(W, X, sX, 0.5, [1.0, 0.9], 64),
        lambda W, X, sX: awq.awq_pack_int4(W, sX, 0.5, 1.0, 64),
        lambda W, X, sX: awq.awq_pack_quant(W, sX, 0.5, 1.0, 64),
    ]
    for call in calls:
        with pytest.raises(ValueError, match="sX"):
            call(W, X, sX.double())
        with pytest.raises(ValueError, match="sX"):
            call(W, X, sX.half())
        with pytest.raises(ValueError, match="sX"):
            call(W, X, sX[:-4])
        with pytest.raises(ValueError, match="2-D"):
            call(W.reshape(-1), X, sX)
        with pytest.raises(ValueError, match="CUDA"):
            call(W, X, sX)
    for call in calls[:3]:
        with pytest.raises(ValueError, match="input width"):
            call(W, X[:, :96], sX)
