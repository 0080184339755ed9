"""CPU oracle for the AWQ per-layer scale search (test infrastructure only).

This package is the slow, plain reference the CUDA path is checked against.
Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg
may import it; the product library never does.  The arithmetic lives in
``awq_oracle.c`` (plain C, fp64 sums, IEEE fp32 quantizer); this module only
builds it with gcc, loads it with ctypes and moves numpy arrays in and out.

Which page each function follows is stated in ``awq_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "awq_oracle.c")
_LIB = os.path.join(_HERE, "liborc_awq.so")

SYM = 0
ASYM = 1


def build(force: bool = False) -> str:
    """Compile awq_oracle.c into liborc_awq.so next to it (gcc, OpenMP)."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp",
           "-std=gnu11", "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i64 = ctypes.c_int64
        I = ctypes.c_int
        D = ctypes.c_double
        F = ctypes.c_float
        lib.orc_stats_chunk.restype = I
        lib.orc_act_stats.argtypes = [P, i64, i64, F, P]
        lib.orc_scale_vector.argtypes = [P, i64, D, P]
        lib.orc_quant_group.argtypes = [P, I, I, I, D, P, P, P]
        lib.orc_quant_layer.argtypes = [P, i64, i64, P, I, I, I, D, P, P, P, P]
        lib.orc_layer_loss_rows.argtypes = [P, i64, i64, P, i64, P, I, P, P, P, P, i64, P]
        lib.orc_layer_loss_rows.restype = D
        lib.orc_search_layer.argtypes = [P, i64, i64, P, i64, P, I, I, I, P, I, P, I,
                                         P, i64, P, P, P, P]
        lib.orc_search_points.argtypes = [P, i64, i64, P, i64, P, I, I, I, P, P, I,
                                          P, i64, P, P, P]
        lib.orc_group_clip.argtypes = [P, i64, i64, P, i64, P, D, I, I, I, P, I, P, P]
        lib.orc_pack_int4.argtypes = [P, i64, i64, P, D, D, P, I, I, I, P, P, P, P, P]
        lib.orc_linear_w4a16.argtypes = [P, i64, i64, i64, P, P, P, P, I, P]
        lib.orc_fold_scale.argtypes = [P, i64, i64, P, I, P]
        _lib = lib
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def as_f32(a: np.ndarray) -> np.ndarray:
    """fp32 view of an input: fp32 as is, bf16 bit patterns (uint16) widened exactly."""
    if a.dtype == np.uint16:
        return np.ascontiguousarray((a.astype(np.uint32) << 16).view(np.float32))
    return np.ascontiguousarray(a, dtype=np.float32)


def stats_chunk() -> int:
    return int(_load().orc_stats_chunk())


def act_stats(X: np.ndarray, clamp_min: float = 1e-4) -> np.ndarray:
    X = as_f32(X)
    N, I = X.shape
    out = np.empty(I, np.float32)
    _load().orc_act_stats(_p(X), N, I, clamp_min, _p(out))
    return out


def scale_vector(sX: np.ndarray, alpha: float) -> np.ndarray:
    sX = np.ascontiguousarray(sX, np.float32)
    out = np.empty(sX.shape[0], np.float32)
    _load().orc_scale_vector(_p(sX), sX.shape[0], float(alpha), _p(out))
    return out


def _check_wbit(w_bit):
    if w_bit not in (3, 4):
        raise ValueError(f"w_bit {w_bit} not in (3, 4)")
    return int(w_bit)


def _clip_g(clip_g, O, nG):
    if clip_g is None:
        return None
    c = np.ascontiguousarray(clip_g, np.float64)
    if c.shape != (O, nG):
        raise ValueError(f"per-group clip must be [{O}, {nG}]")
    return c


def quant_group(wp: np.ndarray, qt: int = SYM, clip: float = 1.0, w_bit: int = 4):
    """Codes, Delta and zero of one group of already-scaled weights."""
    wp = np.ascontiguousarray(wp, np.float32)
    q = np.empty(wp.shape[0], np.int32)
    d = ctypes.c_float()
    z = ctypes.c_int()
    _load().orc_quant_group(_p(wp), wp.shape[0], qt, _check_wbit(w_bit), float(clip), _p(q),
                            ctypes.byref(d), ctypes.byref(z))
    return q, np.float32(d.value), int(z.value)


def quant_layer(W: np.ndarray, s: np.ndarray, gs: int, qt: int = SYM, clip: float = 1.0,
                w_bit: int = 4, clip_g=None):
    """codes [O, I] int8, Delta [O, I/gs] fp32, z [O, I/gs] uint8 of Q(W*s);
    clip_g [O, I/gs] (optional) gives each group its own clip ratio."""
    W = as_f32(W)
    O, I = W.shape
    s = np.ascontiguousarray(s, np.float32)
    codes = np.empty((O, I), np.int8)
    delta = np.empty((O, I // gs), np.float32)
    zeros = np.empty((O, I // gs), np.uint8)
    cg = _clip_g(clip_g, O, I // gs)
    _load().orc_quant_layer(_p(W), O, I, _p(s), gs, qt, _check_wbit(w_bit), float(clip),
                            _p(cg) if cg is not None else None, _p(codes), _p(delta), _p(zeros))
    return codes, delta, zeros


def layer_loss_rows(W, X, s, gs, codes, delta, zeros, rows=None):
    """(sum over listed rows of row losses, row losses) in fp64."""
    W = as_f32(W)
    X = as_f32(X)
    O, I = W.shape
    N = X.shape[0]
    rows = np.arange(O, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, np.int64)
    lr = np.empty(rows.shape[0], np.float64)
    tot = _load().orc_layer_loss_rows(
        _p(W), O, I, _p(X), N, _p(np.ascontiguousarray(s, np.float32)), gs,
        _p(np.ascontiguousarray(codes, np.int8)), _p(np.ascontiguousarray(delta, np.float32)),
        _p(np.ascontiguousarray(zeros, np.uint8)), _p(rows), rows.shape[0], _p(lr))
    return float(tot), lr


def search_layer(W, X, sX, gs, qt, alpha, clip=None, rows=None, w_bit=4):
    """Grid search.  Returns dict(loss [G+C] fp64, loss_row [G+C, R] fp64,
    best_alpha, best_clip)."""
    W = as_f32(W)
    X = as_f32(X)
    O, I = W.shape
    N = X.shape[0]
    alpha = np.ascontiguousarray(alpha, np.float64)
    clip = np.zeros(0, np.float64) if clip is None else np.ascontiguousarray(clip, np.float64)
    G, C = alpha.shape[0], clip.shape[0]
    if rows is None:
        rows_arr, R = None, O
    else:
        rows_arr = np.ascontiguousarray(rows, np.int64)
        R = rows_arr.shape[0]
    loss = np.empty(G + C, np.float64)
    loss_row = np.empty((G + C, R), np.float64)
    ba = ctypes.c_int()
    bc = ctypes.c_int()
    _load().orc_search_layer(
        _p(W), O, I, _p(X), N, _p(np.ascontiguousarray(sX, np.float32)), gs, qt,
        _check_wbit(w_bit), _p(alpha), G, _p(clip) if C else None, C,
        _p(rows_arr) if rows_arr is not None else None, R,
        _p(loss), _p(loss_row), ctypes.byref(ba), ctypes.byref(bc))
    return {"loss": loss, "loss_row": loss_row, "best_alpha": int(ba.value),
            "best_clip": int(bc.value)}


def search_points(W, X, sX, gs, qt, alpha, clip, rows=None, w_bit=4):
    """The loss at each listed (alpha[k], clip[k]) point.  Returns dict(loss [n],
    loss_row [n, R], best)."""
    W = as_f32(W)
    X = as_f32(X)
    O, I = W.shape
    N = X.shape[0]
    alpha = np.ascontiguousarray(alpha, np.float64)
    clip = np.ascontiguousarray(clip, np.float64)
    if alpha.shape != clip.shape:
        raise ValueError("alpha and clip must list the same number of points")
    n = alpha.shape[0]
    rows_arr = None if rows is None else np.ascontiguousarray(rows, np.int64)
    R = O if rows_arr is None else rows_arr.shape[0]
    loss = np.empty(n, np.float64)
    loss_row = np.empty((n, R), np.float64)
    best = ctypes.c_int()
    _load().orc_search_points(
        _p(W), O, I, _p(X), N, _p(np.ascontiguousarray(sX, np.float32)), gs, qt,
        _check_wbit(w_bit), _p(alpha), _p(clip), n,
        _p(rows_arr) if rows_arr is not None else None, R, _p(loss), _p(loss_row),
        ctypes.byref(best))
    return {"loss": loss, "loss_row": loss_row, "best": int(best.value)}


def group_clip(W, X, sX, alpha, gs, qt, clip, w_bit=4, want_err=False):
    """Per-group clip search at s = s_X^alpha.  Returns dict(best [O, I/gs]
    int32 indices into clip, err [O, I/gs, n_clip] fp64 or None)."""
    W = as_f32(W)
    X = as_f32(X)
    O, I = W.shape
    N = X.shape[0]
    clip = np.ascontiguousarray(clip, np.float64)
    best = np.empty((O, I // gs), np.int32)
    err = np.empty((O, I // gs, clip.shape[0]), np.float64) if want_err else None
    _load().orc_group_clip(_p(W), O, I, _p(X), N, _p(np.ascontiguousarray(sX, np.float32)),
                           float(alpha), gs, qt, _check_wbit(w_bit), _p(clip), clip.shape[0],
                           _p(best), _p(err) if err is not None else None)
    return {"best": best, "err": err}


def pack_int4(W, sX, alpha, clip, gs, qt, w_bit=4, clip_g=None):
    """Packed storage at (alpha, clip), or at the per-group ratios clip_g
    [O, I/gs]: dict(qweight u32 [O, I/8], scales f16 bits [O, I/gs] (uint16),
    zeros u32 [O, ceil(I/gs/8)] or None, s16 f16 bits [I], scales_f32 [O, I/gs])."""
    W = as_f32(W)
    O, I = W.shape
    nG = I // gs
    cg = _clip_g(clip_g, O, nG)
    qweight = np.empty((O, I // 8), np.uint32)
    scales = np.empty((O, nG), np.uint16)
    zeros = np.empty((O, (nG + 7) // 8), np.uint32) if qt == ASYM else None
    s16 = np.empty(I, np.uint16)
    sf = np.empty((O, nG), np.float32)
    _load().orc_pack_int4(_p(W), O, I, _p(np.ascontiguousarray(sX, np.float32)),
                          float(alpha), float(clip), _p(cg) if cg is not None else None,
                          gs, qt, _check_wbit(w_bit), _p(qweight), _p(scales),
                          _p(zeros) if zeros is not None else None, _p(s16), _p(sf))
    return {"qweight": qweight, "scales": scales, "zeros": zeros, "s16": s16,
            "scales_f32": sf}


def linear_w4a16(x, qweight, scales, zeros, s16, gs):
    """y [M, O] fp64 of the W4A16 linear on packed storage (s16 None: x is
    already divided by s)."""
    x = as_f32(x)
    M, I = x.shape
    O = qweight.shape[0]
    y = np.empty((M, O), np.float64)
    _load().orc_linear_w4a16(
        _p(x), M, I, O, _p(np.ascontiguousarray(qweight, np.uint32)),
        _p(np.ascontiguousarray(scales, np.uint16)),
        _p(np.ascontiguousarray(zeros, np.uint32)) if zeros is not None else None,
        _p(np.ascontiguousarray(s16, np.uint16)) if s16 is not None else None, gs, _p(y))
    return y


def fold_scale(P, s16, out_bf16=True):
    """P [R, C] (fp32, or bf16 bits as uint16) with row c divided by s16[c] in
    one fp32 division; bf16 bits (uint16) when out_bf16, else fp32."""
    P = as_f32(P)
    if P.ndim == 1:
        P = P.reshape(-1, 1)
    R, C = P.shape
    s16 = np.ascontiguousarray(s16, np.uint16)
    if s16.shape[0] != R:
        raise ValueError("s16 must have one entry per row of P")
    out = np.empty((R, C), np.uint16 if out_bf16 else np.float32)
    _load().orc_fold_scale(_p(P), R, C, _p(s16), 1 if out_bf16 else 0, _p(out))
    return out
