"""B200 (sm_100a) AWQ per-layer scale search — Python binding.

Thin ctypes marshalling over libawq_b200.so (C ABI in include/awq_b200.h):
torch tensors supply device memory and the current CUDA stream, every step of
the computation runs in the library's kernels.  The functions carry the C
names:

    awq_act_stats(X)                         -> s_X = mean |X| per input channel
    awq_act_stats_noalloc(X)                 -> the same without any device allocation
    awq_search_layer(W, X, sX, ...)          -> losses over the alpha (and clip) grid, argmin
    awq_search_points(W, X, sX, alpha, clip) -> losses at listed (alpha, clip) points, argmin
    awq_pack_int4(W, sX, alpha, clip, ...)   -> packed INT4 codes, fp16 scales, zeros, s
    awq_pack_quant(W, sX, alpha, ...)        -> the same at w_bit 3 or 4, per-group clip ratios
    awq_linear_w4a16(x, packed...)           -> y = (x / s) @ dequant(W)^T (s16=None: x pre-divided)
    awq_fold_scale(P, s16)                   -> P / s per row (1/s folded into the previous op)
    awq_wait_selftest(limit, arrive)         -> status of one bounded in-kernel wait

Importing raises ImportError when the compiled library is missing; there is no
fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libawq_b200.so")

AWQ_F32, AWQ_BF16 = 0, 1
AWQ_SYM, AWQ_ASYM = 0, 1

ALPHA_GRID_20 = tuple(k / 20.0 for k in range(20))


class AwqError(RuntimeError):
    """A library call returned a non-OK status."""

    def __init__(self, fn: str, status: int, status_name: str, detail: str):
        super().__init__(f"{fn}: {status_name}: {detail}")
        self.status = status
        self.status_name = status_name


def _load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(
            f"{path} is not built; run `python weight_only_quantization_awq_b200/build.py`")
    lib = ctypes.CDLL(path)
    P, I, L, F, D = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float,
                     ctypes.c_double)
    lib.awq_version.restype = I
    lib.awq_status_string.restype = ctypes.c_char_p
    lib.awq_status_string.argtypes = [I]
    lib.awq_last_error.restype = ctypes.c_char_p
    lib.awq_act_stats.restype = I
    lib.awq_act_stats.argtypes = [P, I, L, L, F, P, P]
    lib.awq_search_layer.restype = I
    lib.awq_search_layer.argtypes = [P, I, L, L, P, I, L, P, I, I, I, P, I, P, I, P, P, P, P, P]
    lib.awq_pack_int4.restype = I
    lib.awq_pack_int4.argtypes = [P, I, L, L, P, D, D, I, I, P, P, P, P, P, P]
    lib.awq_linear_w4a16.restype = I
    lib.awq_linear_w4a16.argtypes = [P, L, L, L, P, P, P, P, I, P, P]
    lib.awq_act_stats_noalloc.restype = I
    lib.awq_act_stats_noalloc.argtypes = [P, I, L, L, F, P, P]
    lib.awq_search_points.restype = I
    lib.awq_search_points.argtypes = [P, I, L, L, P, I, L, P, I, I, I, P, P, I, P, P, P, P]
    lib.awq_pack_quant.restype = I
    lib.awq_pack_quant.argtypes = [P, I, L, L, P, D, D, P, P, I, I, I, I, P, P, P, P, P, P]
    lib.awq_linear_w4a16_batch.restype = I
    lib.awq_linear_w4a16_batch.argtypes = [P, I, L, I, P]
    lib.awq_group_clip.restype = I
    lib.awq_group_clip.argtypes = [P, I, L, L, P, I, L, P, D, I, I, I, P, I, P, P, P]
    lib.awq_fold_scale.restype = I
    lib.awq_fold_scale.argtypes = [P, I, L, L, P, P, P]
    lib.awq_wait_selftest.restype = I
    lib.awq_wait_selftest.argtypes = [L, I, P]
    lib.awq_set_kernel_timing.restype = None
    lib.awq_set_kernel_timing.argtypes = [I]
    lib.awq_last_kernel_ms.restype = D
    lib.awq_last_kernel_ms.argtypes = [I]
    return lib


lib = _load_library()

EXPORTS = ("awq_version", "awq_status_string", "awq_last_error", "awq_act_stats",
           "awq_search_layer", "awq_search_points", "awq_group_clip", "awq_pack_int4",
           "awq_pack_quant",
           "awq_linear_w4a16", "awq_linear_w4a16_batch", "awq_fold_scale", "awq_wait_selftest",
           "awq_set_kernel_timing",
           "awq_last_kernel_ms", "awq_act_stats_noalloc")

MAX_POINTS = 4096

KT_STATS, KT_SEARCH, KT_PACK, KT_APPLY = 0, 1, 2, 3


def set_kernel_timing(enable: bool) -> None:
    """Bracket each entry point's main kernel(s) with CUDA events (thread-local)."""
    lib.awq_set_kernel_timing(1 if enable else 0)


def last_kernel_ms(kind: int) -> float:
    """Device milliseconds of that kernel in the calling thread's last call (< 0: none)."""
    return float(lib.awq_last_kernel_ms(kind))


def _check(fn: str, status: int) -> None:
    if status != 0:
        raise AwqError(fn, status, lib.awq_status_string(status).decode(),
                       lib.awq_last_error().decode())


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return AWQ_F32
    if t.dtype == torch.bfloat16:
        return AWQ_BF16
    raise TypeError(f"unsupported dtype {t.dtype} (float32 or bfloat16)")


def _quant_code(quant) -> int:
    if quant in (AWQ_SYM, "sym", "symmetric"):
        return AWQ_SYM
    if quant in (AWQ_ASYM, "asym", "asymmetric"):
        return AWQ_ASYM
    raise ValueError(f"quant must be 'sym' or 'asym', got {quant!r}")


def _stream(t: torch.Tensor) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def _dev(t: torch.Tensor, name: str) -> torch.Tensor:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _out(t: torch.Tensor, name: str, like: torch.Tensor, dtype: torch.dtype, numel: int):
    """A caller-supplied result tensor: CUDA, contiguous, on `like`'s device, of
    `dtype` and `numel` elements (the library writes exactly that many)."""
    _dev(t, name)
    if t.device != like.device:
        raise ValueError(f"{name} is on {t.device}, the inputs on {like.device}")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if t.numel() != numel:
        raise ValueError(f"{name} must have {numel} elements, got {t.numel()}")
    return t


def _layer_inputs(W: torch.Tensor, sX: torch.Tensor, X: torch.Tensor | None = None):
    """W [out, in] and s_X [in] fp32 (and X [N, in]) on one device, before any pointer
    reaches the library: a narrower X or a shorter or 16-bit s_X would be read past its
    end.  Returns (out, in)."""
    if W.dim() != 2:
        raise ValueError("W must be 2-D [out, in]")
    out_f, inp = W.shape
    if sX.dtype != torch.float32 or sX.numel() != inp:
        raise ValueError(f"sX must be float32 with {inp} elements (one per input channel)")
    if X is not None and (X.dim() != 2 or X.shape[1] != inp):
        raise ValueError("W, X and sX disagree on the input width")
    for t, n in ((W, "W"), (sX, "sX"), (X, "X")):
        if t is not None:
            _dev(t, n)
            if t.device != W.device:
                raise ValueError(f"{n} is on {t.device}, W on {W.device}")
    return out_f, inp


def awq_act_stats(X: torch.Tensor, clamp_min: float = 1e-4, out: torch.Tensor | None = None):
    """s_X[i] = max(clamp_min, mean_n |X[n, i]|) for X [N, in] (fp32 or bf16)."""
    _dev(X, "X")
    N, inp = X.shape
    if out is None:
        out = torch.empty(inp, dtype=torch.float32, device=X.device)
    _out(out, "out", X, torch.float32, inp)
    _check("awq_act_stats", lib.awq_act_stats(X.data_ptr(), _dtype_code(X), N, inp,
                                              float(clamp_min), out.data_ptr(), _stream(X)))
    return out


def awq_act_stats_noalloc(X: torch.Tensor, clamp_min: float = 1e-4, out: torch.Tensor | None = None):
    """awq_act_stats through the library's allocation-free entry point (its fp64
    partials live in a fixed device buffer; ceil(N / 128) * in <= 1,048,576).
    Pass `out` ([in] fp32 device) to allocate nothing at all."""
    _dev(X, "X")
    N, inp = X.shape
    if out is None:
        out = torch.empty(inp, dtype=torch.float32, device=X.device)
    _out(out, "out", X, torch.float32, inp)
    _check("awq_act_stats_noalloc",
           lib.awq_act_stats_noalloc(X.data_ptr(), _dtype_code(X), N, inp, float(clamp_min),
                                     out.data_ptr(), _stream(X)))
    return out


def awq_search_layer(W: torch.Tensor, X: torch.Tensor, sX: torch.Tensor, group_size: int = 128,
                     w_bit: int = 4, quant="sym", alpha=ALPHA_GRID_20, clip=None,
                     loss_row: bool = False):
    """Grid search of one layer.  Returns dict(loss: np.ndarray [G + C] fp64,
    loss_row: tensor [G + C, out] fp32 or None, best_alpha, best_clip)."""
    out_f, inp = _layer_inputs(W, sX, X)
    N = X.shape[0]
    a = np.ascontiguousarray(np.asarray(alpha, dtype=np.float64))
    c = np.ascontiguousarray(np.asarray([] if clip is None else clip, dtype=np.float64))
    loss = np.empty(a.size + c.size, np.float64)
    lr = (torch.empty((a.size + c.size, out_f), dtype=torch.float32, device=W.device)
          if loss_row else None)
    ba, bc = ctypes.c_int(), ctypes.c_int()
    st = lib.awq_search_layer(
        W.data_ptr(), _dtype_code(W), out_f, inp, X.data_ptr(), _dtype_code(X), N, sX.data_ptr(),
        group_size, w_bit, _quant_code(quant), a.ctypes.data, a.size,
        c.ctypes.data if c.size else None, c.size, loss.ctypes.data,
        lr.data_ptr() if lr is not None else None, ctypes.byref(ba), ctypes.byref(bc), _stream(W))
    _check("awq_search_layer", st)
    return {"loss": loss, "loss_row": lr, "best_alpha": ba.value, "best_clip": bc.value}


def awq_search_points(W: torch.Tensor, X: torch.Tensor, sX: torch.Tensor, alpha, clip,
                      group_size: int = 128, w_bit: int = 4, quant="sym", loss_row: bool = False):
    """The loss at each listed (alpha[k], clip[k]) point (a joint grid).  Returns
    dict(loss: np.ndarray [n] fp64, loss_row: tensor [n, out] fp32 or None, best)."""
    out_f, inp = _layer_inputs(W, sX, X)
    N = X.shape[0]
    a = np.ascontiguousarray(np.asarray(alpha, dtype=np.float64).ravel())
    c = np.ascontiguousarray(np.asarray(clip, dtype=np.float64).ravel())
    if a.size != c.size:
        raise ValueError("alpha and clip must list the same number of points")
    loss = np.empty(a.size, np.float64)
    lr = (torch.empty((a.size, out_f), dtype=torch.float32, device=W.device)
          if loss_row else None)
    best = ctypes.c_int()
    st = lib.awq_search_points(
        W.data_ptr(), _dtype_code(W), out_f, inp, X.data_ptr(), _dtype_code(X), N, sX.data_ptr(),
        group_size, w_bit, _quant_code(quant), a.ctypes.data, c.ctypes.data, a.size,
        loss.ctypes.data, lr.data_ptr() if lr is not None else None, ctypes.byref(best), _stream(W))
    _check("awq_search_points", st)
    return {"loss": loss, "loss_row": lr, "best": best.value}


def awq_group_clip(W: torch.Tensor, X: torch.Tensor, sX: torch.Tensor, alpha: float, clip_grid,
                   group_size: int = 128, w_bit: int = 4, quant="asym", want_err: bool = False):
    """One clip ratio per (row, group) at s = s_X^alpha: the first ratio of
    clip_grid minimising the group's own output error.  Returns dict(clip_idx:
    uint8 [out, in/gs] device, err: fp32 [out, in/gs, n_clip] device or None)."""
    out_f, inp = _layer_inputs(W, sX, X)
    N = X.shape[0]
    g = np.ascontiguousarray(np.asarray(clip_grid, dtype=np.float64).ravel())
    nG = inp // group_size
    idx = torch.empty((out_f, nG), dtype=torch.uint8, device=W.device)
    err = (torch.empty((out_f, nG, g.size), dtype=torch.float32, device=W.device)
           if want_err else None)
    st = lib.awq_group_clip(
        W.data_ptr(), _dtype_code(W), out_f, inp, X.data_ptr(), _dtype_code(X), N, sX.data_ptr(),
        float(alpha), group_size, w_bit, _quant_code(quant), g.ctypes.data, g.size, idx.data_ptr(),
        err.data_ptr() if err is not None else None, _stream(W))
    _check("awq_group_clip", st)
    return {"clip_idx": idx, "err": err}


def awq_pack_quant(W: torch.Tensor, sX: torch.Tensor, alpha: float, clip: float = 1.0,
                   group_size: int = 128, quant="sym", w_bit: int = 4,
                   clip_idx: torch.Tensor | None = None, clip_grid=None,
                   scales_f32: bool = False):
    """Packed storage at w_bit 3 or 4, with one clip ratio for the layer or, given
    clip_idx (uint8 [out, in/gs] device) and clip_grid, one per group.  Same
    dict as awq_pack_int4."""
    out_f, inp = _layer_inputs(W, sX)
    q = _quant_code(quant)
    nG = inp // group_size
    dev = W.device
    grid = None
    if clip_idx is not None:
        _out(clip_idx, "clip_idx", W, torch.uint8, out_f * nG)
        grid = np.ascontiguousarray(np.asarray(clip_grid, dtype=np.float64).ravel())
    qweight = torch.empty((out_f, inp // 8), dtype=torch.int32, device=dev)
    scales = torch.empty((out_f, nG), dtype=torch.float16, device=dev)
    zeros = (torch.empty((out_f, (nG + 7) // 8), dtype=torch.int32, device=dev)
             if q == AWQ_ASYM else None)
    s16 = torch.empty(inp, dtype=torch.float16, device=dev)
    sf = torch.empty((out_f, nG), dtype=torch.float32, device=dev) if scales_f32 else None
    st = lib.awq_pack_quant(
        W.data_ptr(), _dtype_code(W), out_f, inp, sX.data_ptr(), float(alpha), float(clip),
        clip_idx.data_ptr() if clip_idx is not None else None,
        grid.ctypes.data if grid is not None else None, grid.size if grid is not None else 0,
        group_size, w_bit, q, qweight.data_ptr(), scales.data_ptr(),
        zeros.data_ptr() if zeros is not None else None, s16.data_ptr(),
        sf.data_ptr() if sf is not None else None, _stream(W))
    _check("awq_pack_quant", st)
    return {"qweight": qweight, "scales": scales, "zeros": zeros, "s16": s16, "scales_f32": sf,
            "group_size": group_size}


def awq_fold_scale(P: torch.Tensor, s16: torch.Tensor, out: torch.Tensor | None = None):
    """P [rows, cols] (or [rows]) fp32 / bf16 with row r divided by s16[r]: the
    division of the next layer's input by s folded into the operator that
    produces it (an RMSNorm weight, a previous linear's weight rows)."""
    _dev(P, "P"), _dev(s16, "s16")
    rows = P.shape[0]
    cols = P.numel() // rows if rows else 0
    if s16.numel() != rows or s16.dtype != torch.float16:
        raise ValueError("s16 must be fp16 with one entry per row of P")
    if out is None:
        out = torch.empty_like(P)
    _out(out, "out", P, P.dtype, P.numel())
    _check("awq_fold_scale", lib.awq_fold_scale(P.data_ptr(), _dtype_code(P), rows, cols,
                                                s16.data_ptr(), out.data_ptr(), _stream(P)))
    return out


def awq_wait_selftest(limit_cycles: int, arrive: bool, device=None) -> int:
    """Run the bounded-wait self-test on the current stream; returns the status
    code (0 = the wait completed, 5 = AWQ_ERR_TIMEOUT) instead of raising."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    st = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    return int(lib.awq_wait_selftest(int(limit_cycles), 1 if arrive else 0, st))


def awq_pack_int4(W: torch.Tensor, sX: torch.Tensor, alpha: float, clip: float = 1.0,
                  group_size: int = 128, quant="sym", scales_f32: bool = False):
    """Packed storage at (alpha, clip): dict(qweight int32 [out, in/8] (u32 bits),
    scales fp16 [out, in/gs], zeros int32 [out, ceil(in/gs/8)] or None,
    s16 fp16 [in], scales_f32 fp32 or None)."""
    out_f, inp = _layer_inputs(W, sX)
    q = _quant_code(quant)
    nG = inp // group_size
    dev = W.device
    qweight = torch.empty((out_f, inp // 8), dtype=torch.int32, device=dev)
    scales = torch.empty((out_f, nG), dtype=torch.float16, device=dev)
    zeros = (torch.empty((out_f, (nG + 7) // 8), dtype=torch.int32, device=dev)
             if q == AWQ_ASYM else None)
    s16 = torch.empty(inp, dtype=torch.float16, device=dev)
    sf = torch.empty((out_f, nG), dtype=torch.float32, device=dev) if scales_f32 else None
    st = lib.awq_pack_int4(
        W.data_ptr(), _dtype_code(W), out_f, inp, sX.data_ptr(), float(alpha), float(clip),
        group_size, q, qweight.data_ptr(), scales.data_ptr(),
        zeros.data_ptr() if zeros is not None else None, s16.data_ptr(),
        sf.data_ptr() if sf is not None else None, _stream(W))
    _check("awq_pack_int4", st)
    return {"qweight": qweight, "scales": scales, "zeros": zeros, "s16": s16, "scales_f32": sf,
            "group_size": group_size}


def _w4a16_operands(x, qweight, scales, zeros, s16, group_size: int, name: str = ""):
    """Check one linear's operands against the packed layout of awq_pack_int4 before any
    pointer reaches the library (a short tensor would be read past its end): x [M, in]
    bf16; qweight [out, in/8] of 4-byte words; scales [out, in/gs] of 2-byte values;
    zeros [out, ceil(in/gs/8)] of 4-byte words or None; s16 [in] of 2-byte values or
    None; every tensor contiguous, on CUDA and on x's device.  Returns out."""
    if x.dim() != 2 or x.dtype != torch.bfloat16:
        raise ValueError(f"{name}x must be a 2-D bfloat16 tensor")
    inp = x.shape[1]
    if group_size <= 0 or inp % 8 or inp % group_size:
        raise ValueError(f"{name}in={inp} must be a multiple of 8 and of group_size {group_size}")
    if qweight.element_size() != 4 or qweight.dim() != 2 or qweight.shape[1] != inp // 8:
        raise ValueError(f"{name}qweight must be [out, {inp // 8}] of 4-byte words")
    out_f = qweight.shape[0]
    nG = inp // group_size
    if scales.element_size() != 2 or scales.numel() != out_f * nG:
        raise ValueError(f"{name}scales must hold {out_f} x {nG} 2-byte values")
    if zeros is not None and (zeros.element_size() != 4 or zeros.numel() != out_f * ((nG + 7) // 8)):
        raise ValueError(f"{name}zeros must hold {out_f} x {(nG + 7) // 8} 4-byte words")
    if s16 is not None and (s16.element_size() != 2 or s16.numel() != inp):
        raise ValueError(f"{name}s16 must hold {inp} 2-byte values")
    for t, n in ((x, "x"), (qweight, "qweight"), (scales, "scales"), (zeros, "zeros"), (s16, "s16")):
        if t is not None:
            _dev(t, name + n)
            if t.device != x.device:
                raise ValueError(f"{name}{n} is on {t.device}, x on {x.device}")
    return out_f


def awq_linear_w4a16(x: torch.Tensor, qweight: torch.Tensor, scales: torch.Tensor,
                     zeros: torch.Tensor | None, s16: torch.Tensor | None, group_size: int = 128,
                     out: torch.Tensor | None = None):
    """y [M, out] bf16 = (x / s16) @ dequant(qweight, scales, zeros)^T for bf16 x [M, in];
    s16=None when x has already been divided by s (awq_fold_scale)."""
    out_f = _w4a16_operands(x, qweight, scales, zeros, s16, group_size)
    M, inp = x.shape
    if out is None:
        out = torch.empty((M, out_f), dtype=torch.bfloat16, device=x.device)
    _out(out, "out", x, torch.bfloat16, M * out_f)
    st = lib.awq_linear_w4a16(
        x.data_ptr(), M, inp, out_f, qweight.data_ptr(), scales.data_ptr(),
        zeros.data_ptr() if zeros is not None else None,
        s16.data_ptr() if s16 is not None else None, group_size, out.data_ptr(), _stream(x))
    _check("awq_linear_w4a16", st)
    return out


class _LinearDesc(ctypes.Structure):
    """awq_linear_desc_t of the C ABI."""
    _fields_ = [("x", ctypes.c_void_p), ("in_", ctypes.c_int64), ("out", ctypes.c_int64),
                ("qweight", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("zeros", ctypes.c_void_p), ("s16", ctypes.c_void_p), ("y", ctypes.c_void_p)]


MAX_BATCH_LINEARS = 8


def awq_linear_w4a16_batch(layers, group_size: int = 128, outs=None):
    """Several independent W4A16 linears at the same M in one call (one kernel
    launch for M <= 8).  `layers`: list of (x, qweight, scales, zeros, s16); returns
    the list of y [M, out] bf16 (or fills `outs`)."""
    if not 1 <= len(layers) <= MAX_BATCH_LINEARS:
        raise ValueError(f"1..{MAX_BATCH_LINEARS} linears per call")
    M = layers[0][0].shape[0]
    descs = (_LinearDesc * len(layers))()
    ys = []
    for k, (x, qweight, scales, zeros, s16) in enumerate(layers):
        out_f = _w4a16_operands(x, qweight, scales, zeros, s16, group_size, f"layer {k}: ")
        if x.shape[0] != M or x.device != layers[0][0].device:
            raise ValueError("every x must have the same number of tokens, on the same device")
        y = outs[k] if outs is not None else torch.empty((M, out_f), dtype=torch.bfloat16,
                                                          device=x.device)
        _out(y, "y", x, torch.bfloat16, M * out_f)
        ys.append(y)
        descs[k] = _LinearDesc(x.data_ptr(), x.shape[1], out_f, qweight.data_ptr(),
                               scales.data_ptr(), zeros.data_ptr() if zeros is not None else None,
                               s16.data_ptr() if s16 is not None else None, y.data_ptr())
    _check("awq_linear_w4a16_batch",
           lib.awq_linear_w4a16_batch(ctypes.cast(descs, ctypes.c_void_p), len(layers), M,
                                      group_size, _stream(layers[0][0])))
    return ys
