#!/usr/bin/env python
"""Benchmark of the AWQ per-layer scale search hot path on B200.

One step = the whole path over one layer: activation statistics -> fused grid
search (fake quantisation, output-error contraction, loss reduction, argmin)
-> INT4 packing at alpha* -> W4A16 apply at M = 1.  The default layer is the
Llama-13B up_proj at full calibration size: W 13824x5120 bf16, 65536
calibration tokens (128 samples x 512), asymmetric INT4 with a uint4 zero
point, group 128, 20-point alpha grid.  `--workload 2` runs the Llama-7B
attention projection instead (4096x4096, 4096 tokens, symmetric).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload 4|2]

Metric: search TFLOP/s = grid * 2 * N * in * out per step / device time per
step.  Inputs are resident in HBM when the timed region starts.  On the
default layer W (141.6 MB) and X (671.1 MB) are each larger than the 126 MB
L2, so every step reads them from HBM; the 4096x4096 layer rotates three
copies of (W, X) instead.  With N GPUs (torchrun, one process per GPU) every
rank quantises its own layer (independent units, no data-path collective):
weak scaling, time = max over ranks.  `--impl reference` times the CPU oracle
on a bounded row sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "AWQ search TFLOP/s (grid×2·N·in·out), ms/layer, % BF16 peak; W4A16 GB/s"
GROUP = 128
APPLY_M = 1
L2_BYTES = 126 * 1024 * 1024

# Per benchmarked workload: the layer, its quantiser, how many (W, X) copies rotate
# between steps, the default step count, and the rows of the oracle's timed sample.
BENCH_WORKLOADS = {
    4: {"layer": "up_proj", "quant": "asym", "rotate": 1, "steps": 10, "rows_per_core": 2},
    2: {"layer": "attn_proj", "quant": "sym", "rotate": 3, "steps": 100, "rows_per_core": 48},
}

# Kernels of one step: statistics 2 (partial, final); search 10 (absmax, fp16 copy,
# scale table 2, group parameters, dW range scale, search, row and block
# reductions, argmin); packing 3 (scale table 2, pack); apply 1.
LAUNCHES_PER_STEP = 16

# DRAM bytes (read + write) of one search-kernel launch per workload, from an ncu
# capture of that launch, valid only for the kernel source it was taken on
# (sha256 of csrc/k_search.cu, first 16 hex digits).
SEARCH_TRAFFIC = {
    2: {"source_sha": "44d2be88c075101e", "bytes": 440555008},
    # dram__bytes_read.sum 146.27 GB + dram__bytes_write.sum 153.65 MB, one launch at full size
    4: {"source_sha": "d8f32dc52ada6687", "bytes": 146423650000},
}


def _env_int(k, d):
    try:
        return int(os.environ.get(k, d))
    except ValueError:
        return d


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def source_sha(path):
    return hashlib.sha256(open(path, "rb").read()).hexdigest()[:16]


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""
    FIELDS = ("index,uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid):
        self.uuid = uuid
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 10:
                continue
            if self.uuid and self.uuid not in parts[1]:
                continue
            rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        smax = max(float(r[3]) for r in rows if r[3].replace(".", "").isdigit())
        loaded = [s for s in sm if s > 0.5 * smax] or sm
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for r in rows for k in range(4) if r[6 + k].lower() == "active"})
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": smax, "reasons": reasons,
                "samples": len(rows)}


# ----------------------------------------------------------------- our arm
def bench_config(wid, world):
    """The workload description both arms report (one layer per rank)."""
    import synthetic
    from synthetic import ALPHA_GRID
    bw = BENCH_WORKLOADS[wid]
    wl = synthetic.workload(wid)
    L = next(l for l in wl.layers if l.name == bw["layer"])
    O, I, N = L.out, L.inp, wl.tokens
    rot = bw["rotate"]
    per_copy = 2 * (O * I + N * I)
    if rot > 1:
        l2 = f"{rot} rotating (W, X) copies, {rot * per_copy / 1e6:.0f} MB > 126 MB L2"
    else:
        l2 = (f"inputs larger than L2: W {2 * O * I / 1e6:.1f} MB and X {2 * N * I / 1e6:.1f} MB "
              f"each > 126 MB, one copy")
    return {"workload": wl.name, "out": O, "in": I, "tokens": N, "grid": len(ALPHA_GRID),
            "quant": f"{bw['quant']}_int4", "group_size": GROUP, "apply_m": APPLY_M,
            "parallelism": f"replicas{world}" if world > 1 else "single", "l2": l2}


def max_over_ranks(value, world, device=None):
    """The largest `value` over all ranks (a job takes as long as its slowest
    rank); `value` itself when there is one rank."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tflops(flops_per_step, steps, world, ms):
    """Whole-job throughput: each of `world` ranks runs `steps` steps of its own
    layer, all within `ms` milliseconds (the max over ranks)."""
    return flops_per_step * steps * world / (ms * 1e-3) / 1e12


def _bf16_dev(a, dev):
    import numpy as np
    import torch
    return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)


def run_ours(args, rank, world, local_rank):
    import numpy as np
    import torch
    import torch.distributed as dist

    import synthetic
    import weight_only_quantization_awq_b200 as awq
    from synthetic import ALPHA_GRID

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    wid = args.workload
    bw = BENCH_WORKLOADS[wid]
    layer, quant, rot = bw["layer"], bw["quant"], bw["rotate"]
    wl = synthetic.workload(wid)
    L = next(l for l in wl.layers if l.name == layer)
    O, I, N, G = L.out, L.inp, wl.tokens, len(ALPHA_GRID)
    flops_step = G * 2.0 * N * I * O

    W_np = synthetic.layer_weights(wid, layer)
    X_np = synthetic.layer_activations(wid, layer)
    x_np = synthetic.apply_activations(APPLY_M, I)
    Ws = [_bf16_dev(W_np, dev) for _ in range(rot)]
    Xs = [_bf16_dev(X_np, dev) for _ in range(rot)]
    xd = _bf16_dev(x_np, dev)
    alphas = [float(a) for a in ALPHA_GRID]
    awq.set_kernel_timing(True)
    search_ms = []

    def step(k, record):
        Wd, Xd = Ws[k % rot], Xs[k % rot]
        sX = awq.awq_act_stats(Xd)
        res = awq.awq_search_layer(Wd, Xd, sX, GROUP, 4, quant, alphas)
        if record:
            search_ms.append(awq.last_kernel_ms(awq.KT_SEARCH))
        p = awq.awq_pack_int4(Wd, sX, alphas[res["best_alpha"]], 1.0, GROUP, quant)
        y = awq.awq_linear_w4a16(xd, p["qweight"], p["scales"], p["zeros"], p["s16"], GROUP)
        return res, p, y

    for k in range(args.warmup):
        step(k, False)
    torch.cuda.synchronize()

    uuid = None
    try:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    clocks = ClockSampler(uuid)
    clocks.start()
    if world > 1:
        dist.barrier(device_ids=[local_rank])
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record()
    for k in range(args.steps):
        res, p, y = step(k, True)
    ev1.record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier(device_ids=[local_rank])
    clk = clocks.stop()
    ms = max_over_ranks(ev0.elapsed_time(ev1), world, dev)
    ms_per_step = ms / args.steps
    value = job_tflops(flops_step, args.steps, world, ms)

    # ---- end to end through the public API: pinned host inputs in, results out.
    W_h = torch.from_numpy(W_np.view(np.int16)).view(torch.bfloat16).pin_memory()
    X_h = torch.from_numpy(X_np.view(np.int16)).view(torch.bfloat16).pin_memory()
    x_h = torch.from_numpy(x_np.view(np.int16)).view(torch.bfloat16).pin_memory()
    qh = torch.empty(p["qweight"].shape, dtype=torch.int32).pin_memory()
    sh = torch.empty(p["scales"].shape, dtype=torch.float16).pin_memory()
    zh = (torch.empty(p["zeros"].shape, dtype=torch.int32).pin_memory()
          if p["zeros"] is not None else None)
    s16h = torch.empty(p["s16"].shape, dtype=torch.float16).pin_memory()
    yh = torch.empty(y.shape, dtype=torch.bfloat16).pin_memory()
    # Two device input buffers: step k+1's host-to-device copies run on a copy
    # stream while step k computes (a layer-by-layer quantiser loads the next
    # layer during the current one).  Every step still copies its own inputs.
    del Ws, Xs
    torch.cuda.empty_cache()
    comp_st = torch.cuda.current_stream()
    copy_st = torch.cuda.Stream()
    bufs = [(torch.empty(W_h.shape, dtype=torch.bfloat16, device=dev),
             torch.empty(X_h.shape, dtype=torch.bfloat16, device=dev),
             torch.empty_like(xd)) for _ in range(2)]
    copied = [torch.cuda.Event() for _ in range(2)]
    done = [torch.cuda.Event() for _ in range(2)]

    def issue_copy(k):
        b = k % 2
        with torch.cuda.stream(copy_st):
            if k >= 2:
                copy_st.wait_event(done[b])          # step k-2 has finished with buffer b
            bufs[b][0].copy_(W_h, non_blocking=True)
            bufs[b][1].copy_(X_h, non_blocking=True)
            bufs[b][2].copy_(x_h, non_blocking=True)
            copied[b].record(copy_st)

    def e2e_step(k):
        b = k % 2
        comp_st.wait_event(copied[b])
        Wd_e, Xd_e, xd_e = bufs[b]
        sX = awq.awq_act_stats(Xd_e)
        r = awq.awq_search_layer(Wd_e, Xd_e, sX, GROUP, 4, quant, alphas)
        pk = awq.awq_pack_int4(Wd_e, sX, alphas[r["best_alpha"]], 1.0, GROUP, quant)
        yy = awq.awq_linear_w4a16(xd_e, pk["qweight"], pk["scales"], pk["zeros"], pk["s16"], GROUP)
        qh.copy_(pk["qweight"], non_blocking=True)
        sh.copy_(pk["scales"], non_blocking=True)
        if zh is not None:
            zh.copy_(pk["zeros"], non_blocking=True)
        s16h.copy_(pk["s16"], non_blocking=True)
        yh.copy_(yy, non_blocking=True)
        done[b].record(comp_st)

    def e2e_run(n, start=None):
        if start is not None:
            copy_st.wait_event(start)                # no copy begins before the timed region
        issue_copy(0)
        for k in range(n):
            if k + 1 < n:
                issue_copy(k + 1)
            e2e_step(k)

    e2e_run(2)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier(device_ids=[local_rank])
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_steps = max(1, min(args.steps, 50 if wid == 2 else 5))
    e0.record()
    e2e_run(e2e_steps, e0)
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    h2d = W_h.numel() * 2 + X_h.numel() * 2 + x_h.numel() * 2
    d2h = (qh.numel() * 4 + sh.numel() * 2 + (zh.numel() * 4 if zh is not None else 0) +
           s16h.numel() * 2 + yh.numel() * 2 + 8 * G + 4 * 8)
    e2e_value = job_tflops(flops_step, e2e_steps, world, e2e_ms)
    del bufs
    torch.cuda.empty_cache()

    # ---- W4A16 apply at M = 1 on this layer: rotating packed copies (> L2), one CUDA graph.
    Wd0 = _bf16_dev(W_np, dev)
    sX0 = awq.awq_act_stats(_bf16_dev(X_np[:4096], dev))
    one = awq.awq_pack_int4(Wd0, sX0, 0.5, 1.0, GROUP, quant)
    packed_bytes = sum(t.numel() * t.element_size() for t in
                       (one["qweight"], one["scales"], one["s16"]) + ((one["zeros"],) if one["zeros"] is not None else ()))
    n_copies = max(4, math.ceil(2 * L2_BYTES / packed_bytes))
    packs = [one] + [awq.awq_pack_int4(Wd0, sX0, 0.5, 1.0, GROUP, quant) for _ in range(n_copies - 1)]
    del Wd0
    ys = torch.empty((APPLY_M, O), dtype=torch.bfloat16, device=dev)
    reps = max(1, 128 // n_copies)
    awq.set_kernel_timing(False)

    def apply_all():
        for pk in packs:
            awq.awq_linear_w4a16(xd, pk["qweight"], pk["scales"], pk["zeros"], pk["s16"], GROUP,
                                 out=ys)

    apply_us = graph_time_us(apply_all, reps) / n_copies
    apply_bytes = packed_bytes + APPLY_M * I * 2 + APPLY_M * O * 2
    del packs
    torch.cuda.empty_cache()

    block_apply = measure_block_apply(dev)
    extra_search = measure_search_only(2, awq, dev) if wid != 2 else None
    block_search = measure_block_search(awq, dev) if args.block_search else None

    pk_ = peaks()
    # A kernel timed inside a timed region of a second or more runs under the
    # power cap: its roofline is the sustained GEMM figure; a short burst, the burst one.
    if ms >= 1000.0:
        peak, peak_kind = pk_["bf16_tflops_sustained"], "sustained"
        peak_why = f"the search kernel runs back to back for {ms / 1e3:.1f} s"
    else:
        peak, peak_kind = pk_["bf16_tflops"], "burst"
        peak_why = f"timed region {ms:.0f} ms"
    search_kernel_ms = statistics.mean(search_ms) if search_ms else None
    achieved = flops_step / (search_kernel_ms * 1e-3) / 1e12 if search_kernel_ms else None
    sha = source_sha(os.path.join(ROOT, "weight_only_quantization_awq_b200", "csrc", "k_search.cu"))
    tr = SEARCH_TRAFFIC.get(wid)
    traffic = tr["bytes"] if tr and tr["source_sha"] == sha else None
    out = {
        "metric": METRIC,
        "value": round(value, 3),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f16",
        "data": "synthetic",
        "config": bench_config(wid, world),
        "e2e": {"value": round(e2e_value, 3), "unit": "TFLOP/s",
                "ms_per_step": round(e2e_ms / e2e_steps, 4), "steps": e2e_steps,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": LAUNCHES_PER_STEP * args.steps,
        "clocks": clk,
        "roofline": {"bound": "tensor", "kernel": "search_kernel",
                     "achieved": round(achieved, 2) if achieved else None,
                     "peak": peak, "unit": "TFLOP/s",
                     "frac": round(achieved / peak, 4) if achieved else None,
                     "peak_source": f"{pk_['source']} {peak_kind} bf16 ({peak_why})",
                     "frac_burst": round(achieved / pk_["bf16_tflops"], 4) if achieved else None,
                     "frac_sustained": (round(achieved / pk_["bf16_tflops_sustained"], 4)
                                        if achieved else None),
                     "kernel_ms": round(search_kernel_ms, 4) if search_kernel_ms else None,
                     "algorithmic_flops": flops_step,
                     "traffic": traffic},
        "ms_per_layer": round(ms_per_step, 4),
        "pct_bf16_peak": round(100.0 * value / world / pk_["bf16_tflops"], 2),
        "w4a16": {"m": APPLY_M, "layer": f"{O}x{I}", "us_per_launch": round(apply_us, 3),
                  "gb_per_s": round(apply_bytes / (apply_us * 1e-6) / 1e9, 1),
                  "frac_hbm": round(apply_bytes / (apply_us * 1e-6) / 1e9 / pk_["hbm_gbs"], 4),
                  "bytes": apply_bytes,
                  "timing": f"CUDA graph of {reps * n_copies} launches over {n_copies} packed copies"},
        "w4a16_block": {str(m): {**v, "frac_hbm": round(v["gb_per_s"] / pk_["hbm_gbs"], 4),
                                 **({"batched": {**v["batched"], "frac_hbm": round(
                                     v["batched"]["gb_per_s"] / pk_["hbm_gbs"], 4)}}
                                    if "batched" in v else {})}
                        for m, v in block_apply.items()},
    }
    if block_search is not None:
        block_search["frac_sustained"] = round(block_search["tflops"] / pk_["bf16_tflops_sustained"], 4)
        out["search_block"] = block_search
    if extra_search is not None:
        extra_search["frac"] = round(extra_search["tflops"] / pk_["bf16_tflops"], 4)
        out["search_" + extra_search["workload"]] = extra_search
    if rank == 0 and world == 1:
        out["cpu_baseline"] = cpu_baseline(W_np, X_np, wid)
    if world > 1:
        dist.barrier(device_ids=[local_rank])
    return out


def graph_time_us(fn, reps):
    """Device microseconds of one call of `fn` (a sequence of launches on the
    current stream), from one CUDA graph that replays it `reps` times."""
    import torch
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(reps):
            fn()
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    g.replay()
    e1.record()
    torch.cuda.synchronize()
    del g
    return e0.elapsed_time(e1) * 1e3 / reps


def measure_block_search(awq, dev, reps=2):
    """The Llama-7B block's searches (workload 5: qkv 12288x4096, o 4096x4096,
    gate||up 22016x4096, down 4096x11008; 16384 tokens each, asymmetric INT4
    g128, 20 alphas then 11 clip ratios at alpha*): search-kernel device time
    per block (library CUDA events, both phases), mean of `reps` passes."""
    import torch
    import synthetic
    from synthetic import ALPHA_GRID, CLIP_GRID
    wl = synthetic.workload(5)
    alphas, clips = [float(a) for a in ALPHA_GRID], [float(c) for c in CLIP_GRID]
    awq.set_kernel_timing(True)
    per_layer, flops = {}, 0.0
    for L in wl.layers:
        Wd = _bf16_dev(synthetic.layer_weights(5, L.name), dev)
        Xd = _bf16_dev(synthetic.layer_activations(5, L.name), dev)
        sX = awq.awq_act_stats(Xd)
        awq.awq_search_layer(Wd, Xd, sX, GROUP, 4, "asym", alphas, clip=clips)   # warm-up
        ms = []
        for _ in range(reps):
            awq.awq_search_layer(Wd, Xd, sX, GROUP, 4, "asym", alphas, clip=clips)
            ms.append(awq.last_kernel_ms(awq.KT_SEARCH))
        per_layer[L.name] = round(statistics.mean(ms), 3)
        flops += (len(alphas) + len(clips)) * 2.0 * wl.tokens * L.inp * L.out
        del Wd, Xd
        torch.cuda.empty_cache()
    awq.set_kernel_timing(False)
    total = sum(per_layer.values())
    return {"workload": wl.name, "kernel_ms": round(total, 3), "per_layer_ms": per_layer,
            "tflops": round(flops / (total * 1e-3) / 1e12, 2), "algorithmic_flops": flops,
            "timing": f"library CUDA events around the search kernel (alpha and clip phases), mean of {reps}"}


def measure_search_only(wid, awq, dev, reps=6):
    """Search-kernel device time (library CUDA events) on another workload's
    layer, rotating three input copies; reported beside the headline."""
    import torch
    import synthetic
    from synthetic import ALPHA_GRID
    bw = BENCH_WORKLOADS[wid]
    wl = synthetic.workload(wid)
    L = next(l for l in wl.layers if l.name == bw["layer"])
    W_np = synthetic.layer_weights(wid, bw["layer"])
    X_np = synthetic.layer_activations(wid, bw["layer"])
    Ws = [_bf16_dev(W_np, dev) for _ in range(3)]
    Xs = [_bf16_dev(X_np, dev) for _ in range(3)]
    awq.set_kernel_timing(True)
    alphas = [float(a) for a in ALPHA_GRID]
    sXs = [awq.awq_act_stats(X) for X in Xs]
    ms = []
    for k in range(reps + 2):
        awq.awq_search_layer(Ws[k % 3], Xs[k % 3], sXs[k % 3], GROUP, 4, bw["quant"], alphas)
        if k >= 2:
            ms.append(awq.last_kernel_ms(awq.KT_SEARCH))
    awq.set_kernel_timing(False)
    del Ws, Xs
    torch.cuda.empty_cache()
    flops = len(ALPHA_GRID) * 2.0 * wl.tokens * L.inp * L.out
    kms = statistics.mean(ms)
    return {"workload": wl.name, "kernel_ms": round(kms, 4),
            "tflops": round(flops / (kms * 1e-3) / 1e12, 2), "algorithmic_flops": flops,
            "timing": f"library CUDA events around the search kernel, mean of {reps} calls over 3 rotating input copies"}


def measure_block_apply(dev, ms=(1, 16, 256), copies=2, reps=4):
    """W4A16 apply over the seven linears of the Llama-7B decoder block (q, k, v, o
    4096x4096; gate, up 11008x4096; down 4096x11008), asymmetric INT4 g128, for
    each M: one CUDA graph replays `reps` passes over `copies` packed copies of
    the block (2 x 105 MB > L2).  Weights are seeded bf16 draws packed on the GPU."""
    import torch
    import weight_only_quantization_awq_b200 as awq
    from synthetic import BLOCK_LINEARS
    gen = torch.Generator(device=dev).manual_seed(20261202)
    packs = []
    for c in range(copies):
        layer = []
        for name, o, i in BLOCK_LINEARS:
            W = (torch.randn((o, i), generator=gen, device=dev) * 0.02).to(torch.bfloat16)
            sX = torch.rand(i, generator=gen, device=dev) + 0.5
            layer.append((awq.awq_pack_int4(W, sX, 0.5, 1.0, GROUP, "asym"), o, i))
            del W
        packs.append(layer)
    torch.cuda.synchronize()
    out = {}
    for m in ms:
        xs = {i: (torch.randn((m, i), generator=gen, device=dev)).to(torch.bfloat16)
              for i in {i for _, _, i in BLOCK_LINEARS}}
        ys = [torch.empty((m, o), dtype=torch.bfloat16, device=dev) for _, o, _ in BLOCK_LINEARS]

        def run_all():
            for layer in packs:
                for k, (p, o, i) in enumerate(layer):
                    awq.awq_linear_w4a16(xs[i], p["qweight"], p["scales"], p["zeros"], p["s16"],
                                         GROUP, out=ys[k])

        def run_batched():
            for layer in packs:
                awq.awq_linear_w4a16_batch(
                    [(xs[i], p["qweight"], p["scales"], p["zeros"], p["s16"]) for p, o, i in layer],
                    GROUP, outs=ys)

        us = graph_time_us(run_all, reps) / copies
        byts = sum(p["qweight"].numel() * 4 + p["scales"].numel() * 2 + p["zeros"].numel() * 4 +
                   p["s16"].numel() * 2 + m * i * 2 + m * o * 2 for p, o, i in packs[0])
        flops = sum(2.0 * m * o * i for _, o, i in BLOCK_LINEARS)
        out[m] = {"us_per_block": round(us, 2), "gb_per_s": round(byts / (us * 1e-6) / 1e9, 1),
                  "tflops": round(flops / (us * 1e-6) / 1e12, 2), "bytes": byts,
                  "timing": f"one launch per linear, CUDA graph of {reps} passes over {copies} packed copies"}
        if m <= 8:
            ub = graph_time_us(run_batched, reps) / copies
            out[m]["batched"] = {"us_per_block": round(ub, 2),
                                 "gb_per_s": round(byts / (ub * 1e-6) / 1e9, 1),
                                 "timing": "awq_linear_w4a16_batch: the seven linears in one launch"}
    return out


# --------------------------------------------------------------- the oracle
def _oracle_threads():
    n = len(os.sched_getaffinity(0))
    os.environ.setdefault("OMP_NUM_THREADS", str(n))
    return int(os.environ["OMP_NUM_THREADS"])


def oracle_step(W_np, X32, rows, qt):
    """The oracle's pass of the path on a row sample: statistics over all of X,
    the 20-point search evaluated on `rows`, packing of the whole layer."""
    import oracle
    from synthetic import ALPHA_GRID
    sX = oracle.act_stats(X32)
    res = oracle.search_layer(W_np, X32, sX, GROUP, qt, ALPHA_GRID, rows=rows)
    oracle.pack_int4(W_np, sX, float(ALPHA_GRID[res["best_alpha"]]), 1.0, GROUP, qt)
    return res


def _oracle_sample(wid, W_np, rows_scale=1.0):
    import numpy as np
    cores = _oracle_threads()
    O = W_np.shape[0]
    R = min(O, max(1, int(BENCH_WORKLOADS[wid]["rows_per_core"] * cores * rows_scale)))
    return cores, np.arange(R, dtype=np.int64)


def cpu_baseline(W_np, X_np, wid):
    import oracle
    from synthetic import ALPHA_GRID
    cores, rows = _oracle_sample(wid, W_np)
    qt = 1 if BENCH_WORKLOADS[wid]["quant"] == "asym" else 0
    X32 = oracle.as_f32(X_np)
    O = W_np.shape[0]
    N, I = X32.shape
    R = rows.shape[0]
    t0 = time.perf_counter()
    oracle_step(W_np, X32, rows, qt)
    dt = time.perf_counter() - t0
    flops = len(ALPHA_GRID) * 2.0 * N * I * R
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": cores,
            "kind": "oracle", "seconds": round(dt, 2),
            "sample": f"full statistics and packing, 20-point search on the first {R} of {O} rows "
                      f"(grid*2*N*in*rows = {flops:.3e} flop)"}


def run_reference(args):
    import oracle
    import synthetic
    from synthetic import ALPHA_GRID
    wid = args.workload
    bw = BENCH_WORKLOADS[wid]
    qt = 1 if bw["quant"] == "asym" else 0
    wl = synthetic.workload(wid)
    L = next(l for l in wl.layers if l.name == bw["layer"])
    W_np = synthetic.layer_weights(wid, bw["layer"])
    X32 = oracle.as_f32(synthetic.layer_activations(wid, bw["layer"]))
    cores, rows = _oracle_sample(wid, W_np, rows_scale=0.5)
    R = rows.shape[0]
    flops = len(ALPHA_GRID) * 2.0 * wl.tokens * L.inp * R
    for _ in range(args.warmup):
        oracle_step(W_np, X32, rows, qt)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(W_np, X32, rows, qt)
    dt = time.perf_counter() - t0
    value = flops * args.steps / dt / 1e12
    sample = (f"per step: full statistics and packing, 20-point search on the first {R} of "
              f"{L.out} rows")
    return {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(dt * 1e3 / args.steps, 2), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": bench_config(wid, 1),
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", type=int, choices=sorted(BENCH_WORKLOADS), default=4)
    ap.add_argument("--block-search", dest="block_search", action=argparse.BooleanOptionalAction,
                    default=True, help="also time the Llama-7B block's four joint layers' searches")
    ap.add_argument("--apply-only", dest="apply_only", type=int, nargs="+", default=None, metavar="M",
                    help="only time the W4A16 apply over the Llama-7B block at these token counts "
                         "(a short program to profile the apply kernels under ncu; prints one JSON line)")
    args = ap.parse_args()
    if args.apply_only:
        import torch
        torch.cuda.set_device(0)
        res = measure_block_apply(torch.device("cuda", 0), ms=tuple(args.apply_only), copies=2, reps=1)
        print(json.dumps({"w4a16_block": {str(m): v for m, v in res.items()}}), flush=True)
        return 0
    if args.steps is None:
        args.steps = BENCH_WORKLOADS[args.workload]["steps"]
    if args.warmup < 3:
        args.warmup = 3
    world = _env_int("WORLD_SIZE", 1)
    rank = _env_int("RANK", 0)
    local_rank = _env_int("LOCAL_RANK", 0)

    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args)), flush=True)
        return 0

    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        out = run_ours(args, rank, world, local_rank)
        if rank == 0:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
