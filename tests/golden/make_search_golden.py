"""Write the oracle's full-layer search results for the large workloads.

    OMP_NUM_THREADS=8 python tests/golden/make_search_golden.py [wid:layer ...]

For each listed layer (default: every layer of workloads 2, 3 and 5) this
draws the seeded inputs from `synthetic`, runs the CPU oracle's statistics and
its full grid search over every output row (the 20-point alpha grid, plus the
11-point clip grid at alpha* for workload 5), and writes
`search_w<wid>_<layer>.json` beside this script: the loss at every grid point,
alpha* and r*, and sha256 digests of the inputs so a test can tell that it
reads the same bytes.  Only `synthetic` and `oracle` are called: no value here
comes from the CUDA path.  The oracle's rate is about 0.02-0.05 TFLOP/s on a
host's cores, so workload 5 alone takes hours.
"""
from __future__ import annotations

import hashlib
import json
import os
import sys
import time

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import oracle  # noqa: E402
import synthetic  # noqa: E402
from synthetic import ALPHA_GRID, CLIP_GRID  # noqa: E402

LAYERS = [(2, "attn_proj"), (3, "down"), (3, "gate_up"), (5, "o"), (5, "down"), (5, "qkv"),
          (5, "gate_up")]


def digest(a: np.ndarray) -> str:
    return hashlib.sha256(np.ascontiguousarray(a).tobytes()).hexdigest()


def path_for(wid: int, layer: str) -> str:
    return os.path.join(HERE, f"search_w{wid}_{layer}.json")


def make(wid: int, layer: str) -> dict:
    wl = synthetic.workload(wid)
    W = synthetic.layer_weights(wid, layer)
    X = synthetic.layer_activations(wid, layer)
    clip = wl.clip if wl.clip.size else None
    t0 = time.time()
    X32 = oracle.as_f32(X)
    sX = oracle.act_stats(X32)
    res = oracle.search_layer(W, X32, sX, wl.group_size, wl.qt, wl.alpha, clip=clip)
    dt = time.time() - t0
    return {
        "workload": wid, "name": wl.name, "layer": layer,
        "out": int(W.shape[0]), "in": int(W.shape[1]), "tokens": int(X.shape[0]),
        "quant": "asym" if wl.qt == synthetic.ASYM else "sym", "group_size": wl.group_size,
        "alpha": [float(a) for a in wl.alpha],
        "clip": [float(c) for c in clip] if clip is not None else [],
        "loss": [float(v) for v in res["loss"]],
        "best_alpha": res["best_alpha"], "best_clip": res["best_clip"],
        "sha256": {"W": digest(W), "X": digest(X), "sX": digest(sX)},
        "oracle_seconds": round(dt, 1),
        "threads": int(os.environ.get("OMP_NUM_THREADS", "0") or 0),
        "command": "python tests/golden/make_search_golden.py " + f"{wid}:{layer}",
    }


def main(argv):
    todo = LAYERS
    if argv:
        todo = [(int(a.split(":")[0]), a.split(":")[1]) for a in argv]
    for wid, layer in todo:
        d = make(wid, layer)
        tmp = path_for(wid, layer) + ".tmp"
        with open(tmp, "w") as f:
            json.dump(d, f, indent=1)
        os.replace(tmp, path_for(wid, layer))
        print(f"w{wid}:{layer} alpha*={d['best_alpha']} clip*={d['best_clip']} "
              f"{d['oracle_seconds']} s", flush=True)


if __name__ == "__main__":
    main(sys.argv[1:])
