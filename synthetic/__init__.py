"""Seeded synthetic inputs for the AWQ per-layer scale search.

This module only draws numbers: weights W [out, in], calibration activations
X [tokens, in] and apply-path activations x [M, in], with the shapes and value
distributions of the workloads below.  It holds none of the method's
arithmetic, and both the CPU oracle and the CUDA path read exactly the bytes it
returns.  bf16 tensors are returned as uint16 bit patterns (rounded to nearest
even from an fp32 draw); fp32 tensors as float32.

No dataset ships with this code: the calibration activations stand in for the
128-sample x 512-token calibration set the AWQ pages describe, with a heavy
per-channel outlier structure (about 1% of input channels scaled up), which is
the property the method relies on.

Workloads (id: layers, tokens, distributions, quantizer):
  1  single 512x512 layer, fp32 W ~ N(0, 0.02^2), fp32 X [256, 512] ~ N(0, 1)
     with 5 outlier channels x20; symmetric INT4, group 128, 20-point alpha grid.
  2  Llama-7B attention projection 4096x4096, bf16 W ~ N(0, 0.02^2) times a
     per-row LogNormal(0, 0.3) factor; bf16 X [4096, 4096] ~ N(0, 1) with 41
     outlier channels x LogUniform(10, 100); symmetric INT4 group 128.
  3  Llama-7B MLP: gate and up (11008x4096 each, searched jointly as one
     22016x4096 matrix) and down (4096x11008); X [8192, in] ~ Student-t(4) with
     1% outlier channels x30; symmetric INT4 group 128.
  4  Llama-13B up_proj 13824x5120; X [65536, 5120] ~ N(0, 1) with 1% outlier
     channels x LogUniform(10, 100); asymmetric INT4 (uint4 zero point) group 128.
  5  Llama-7B decoder block: q,k,v (searched jointly as 12288x4096), o
     4096x4096, gate,up (jointly 22016x4096), down 4096x11008; X [16384, in]
     ~ N(0, 1) with 1% outlier channels x50, one independent draw per input;
     asymmetric INT4 group 128; 20-point alpha grid plus an 11-point clip grid;
     then the W4A16 apply at M in {1, 16, 256} with x ~ N(0, 1).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

SEED_BASE = 20261202

SYM = 0
ASYM = 1

ALPHA_GRID = np.array([k / 20.0 for k in range(20)], dtype=np.float64)
CLIP_GRID = np.array([(20 - j) / 20.0 for j in range(11)], dtype=np.float64)


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round an fp32 array to bf16 (nearest even) and return the uint16 bits."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    bias = ((u >> 16) & 1) + np.uint32(0x7FFF)
    return ((u + bias) >> 16).astype(np.uint16)


def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32."""
    return (b.astype(np.uint32) << 16).view(np.float32)


@dataclass
class Layer:
    name: str
    out: int
    inp: int
    x_key: str          # which calibration draw feeds this layer


@dataclass
class Workload:
    id: int
    name: str
    layers: list
    tokens: int
    wdtype: str         # "f32" or "bf16"
    xdtype: str
    qt: int
    group_size: int
    alpha: np.ndarray
    clip: np.ndarray
    w_dist: str
    x_dist: str
    outlier_scale: tuple  # ("const", c) or ("loguniform", lo, hi)
    n_outliers: dict = field(default_factory=dict)  # per input width
    apply_m: tuple = ()


def _k1(inp: int) -> int:
    return int(round(0.01 * inp))


WORKLOADS = {
    1: Workload(1, "single_linear_512x512_n256", [Layer("linear", 512, 512, "x")], 256,
                "f32", "f32", SYM, 128, ALPHA_GRID, np.zeros(0), "normal", "normal",
                ("const", 20.0), {512: 5}),
    2: Workload(2, "llama7b_attn_proj_4096x4096_n4096",
                [Layer("attn_proj", 4096, 4096, "x")], 4096, "bf16", "bf16", SYM, 128,
                ALPHA_GRID, np.zeros(0), "normal_rowlognormal", "normal",
                ("loguniform", 10.0, 100.0), {4096: 41}),
    3: Workload(3, "llama7b_mlp_n8192",
                [Layer("gate_up", 22016, 4096, "x_gate_up"), Layer("down", 4096, 11008, "x_down")],
                8192, "bf16", "bf16", SYM, 128, ALPHA_GRID, np.zeros(0), "normal", "student_t4",
                ("const", 30.0), {4096: _k1(4096), 11008: _k1(11008)}),
    4: Workload(4, "llama13b_up_proj_13824x5120_n65536",
                [Layer("up_proj", 13824, 5120, "x")], 65536, "bf16", "bf16", ASYM, 128,
                ALPHA_GRID, np.zeros(0), "normal", "normal", ("loguniform", 10.0, 100.0),
                {5120: _k1(5120)}),
    5: Workload(5, "llama7b_block_n16384",
                [Layer("qkv", 12288, 4096, "x_qkv"), Layer("o", 4096, 4096, "x_o"),
                 Layer("gate_up", 22016, 4096, "x_gate_up"), Layer("down", 4096, 11008, "x_down")],
                16384, "bf16", "bf16", ASYM, 128, ALPHA_GRID, CLIP_GRID, "normal", "normal",
                ("const", 50.0), {4096: _k1(4096), 11008: _k1(11008)}, apply_m=(1, 16, 256)),
}

# The seven linears of workload 5 as separate matrices (the apply path runs per linear).
BLOCK_LINEARS = [("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("o", 4096, 4096),
                 ("gate", 11008, 4096), ("up", 11008, 4096), ("down", 4096, 11008)]


def _rng(*key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64([SEED_BASE, *key]))


def _weights(rng, out: int, inp: int, dist: str) -> np.ndarray:
    w = rng.standard_normal((out, inp), dtype=np.float32) * np.float32(0.02)
    if dist == "normal_rowlognormal":
        row = rng.lognormal(0.0, 0.3, size=(out, 1)).astype(np.float32)
        w *= row
    return w


def _activations(rng, n: int, inp: int, dist: str, outlier_scale, k: int) -> np.ndarray:
    if dist == "normal":
        x = rng.standard_normal((n, inp), dtype=np.float32)
    elif dist == "student_t4":
        x = rng.standard_t(4.0, size=(n, inp)).astype(np.float32)
    else:
        raise ValueError(dist)
    cols = rng.choice(inp, size=k, replace=False)
    if outlier_scale[0] == "const":
        f = np.full(k, outlier_scale[1], np.float32)
    else:
        lo, hi = outlier_scale[1], outlier_scale[2]
        f = np.exp(rng.uniform(np.log(lo), np.log(hi), size=k)).astype(np.float32)
    x[:, cols] *= f[None, :]
    return x


def _cast(a: np.ndarray, dtype: str) -> np.ndarray:
    return bf16_bits(a) if dtype == "bf16" else np.ascontiguousarray(a, np.float32)


def workload(wid: int) -> Workload:
    return WORKLOADS[wid]


def layer_weights(wid: int, layer: str) -> np.ndarray:
    """W [out, in] of one (possibly joint) layer of a workload."""
    wl = WORKLOADS[wid]
    idx = [l.name for l in wl.layers].index(layer)
    L = wl.layers[idx]
    if wid == 3 and layer == "gate_up" or wid == 5 and layer in ("qkv", "gate_up"):
        parts = {"qkv": ["q", "k", "v"], "gate_up": ["gate", "up"]}[layer]
        ws = [_weights(_rng(wid, 100 + j, idx), L.out // len(parts), L.inp, wl.w_dist)
              for j, _ in enumerate(parts)]
        return _cast(np.concatenate(ws, axis=0), wl.wdtype)
    return _cast(_weights(_rng(wid, 100, idx), L.out, L.inp, wl.w_dist), wl.wdtype)


def layer_activations(wid: int, layer: str, tokens: int | None = None) -> np.ndarray:
    """Calibration X [tokens, in] feeding a layer of a workload."""
    wl = WORKLOADS[wid]
    L = next(l for l in wl.layers if l.name == layer)
    keys = sorted({l.x_key for l in wl.layers})
    n = wl.tokens if tokens is None else tokens
    rng = _rng(wid, 200 + keys.index(L.x_key))
    x = _activations(rng, n, L.inp, wl.x_dist, wl.outlier_scale, wl.n_outliers[L.inp])
    return _cast(x, wl.xdtype)


def apply_activations(m: int, inp: int, seed: int = 0) -> np.ndarray:
    """bf16 x [m, in] ~ N(0, 1) for the W4A16 apply path."""
    return bf16_bits(_rng(900, m, inp, seed).standard_normal((m, inp), dtype=np.float32))


def small_layer(out: int, inp: int, tokens: int, wdtype: str = "bf16", xdtype: str = "bf16",
                seed: int = 0, n_outliers: int | None = None, outlier: float = 20.0):
    """A small (W, X) pair with the same structure, for tests with ragged sizes."""
    rng = _rng(1000, out, inp, tokens, seed)
    w = _weights(rng, out, inp, "normal_rowlognormal")
    k = max(1, int(round(0.01 * inp))) if n_outliers is None else n_outliers
    x = _activations(rng, tokens, inp, "normal", ("const", outlier), k)
    return _cast(w, wdtype), _cast(x, xdtype)
