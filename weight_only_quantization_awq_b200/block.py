"""Layer-parallel quantisation of a block of linear layers over ranks.

The per-layer scale search of the AWQ pages runs one (joint) linear layer at a
time; its layers are independent units of work.  A decoder block's layers
(q/k/v searched jointly, o, gate/up jointly, down) are therefore spread over the
ranks of a process group, one GPU per rank, each rank running the whole search
and packing of its own layers on its own GPU with no communication; only the
packed results are exchanged at the end, so that every rank holds the whole
quantised block.

    assign_layers(costs, world)  -> owner rank of each layer (longest first)
    quantize_layer(layer)        -> the search, the packing and the choice of one layer
    quantize_block(layers, ...)  -> every layer's result on every rank

The exchange is one broadcast per result tensor from the layer's owner, in
layer order, so every rank issues the same collectives in the same order.  With
NCCL the tensors stay on the GPU; with gloo (tests) they live on the CPU.
"""
from __future__ import annotations

import math
from dataclasses import dataclass


@dataclass
class BlockLayer:
    """One (joint) linear layer of a block: W [out, in], calibration X [N, in]."""
    name: str
    W: object                     # torch tensor
    X: object                     # torch tensor
    quant: str = "asym"
    group_size: int = 128
    w_bit: int = 4
    alpha: tuple = tuple(k / 20.0 for k in range(20))
    clip: tuple = ()

    @property
    def out(self) -> int:
        return int(self.W.shape[0])

    @property
    def inp(self) -> int:
        return int(self.W.shape[1])

    @property
    def tokens(self) -> int:
        return int(self.X.shape[0])

    def cost(self) -> float:
        """Search work in flops: grid points x 2 * N * in * out."""
        return (len(self.alpha) + len(self.clip)) * 2.0 * self.tokens * self.inp * self.out


def assign_layers(costs, world: int) -> list:
    """Owner rank of each layer: layers in decreasing cost (ties: lower index
    first) each go to the rank with the least work so far (ties: lower rank).
    Deterministic, so every rank computes the same plan."""
    if world < 1:
        raise ValueError("world must be >= 1")
    order = sorted(range(len(costs)), key=lambda k: (-float(costs[k]), k))
    load = [0.0] * world
    owner = [0] * len(costs)
    for k in order:
        r = min(range(world), key=lambda q: (load[q], q))
        owner[k] = r
        load[r] += float(costs[k])
    return owner


def result_spec(layer: BlockLayer) -> dict:
    """Names, shapes and dtypes of one layer's result tensors (known on every
    rank before the exchange)."""
    import torch
    nG = layer.inp // layer.group_size
    spec = {"qweight": ((layer.out, layer.inp // 8), torch.int32),
            "scales": ((layer.out, nG), torch.float16),
            "s16": ((layer.inp,), torch.float16),
            "meta": ((4 + len(layer.alpha) + len(layer.clip),), torch.float64)}
    if layer.quant == "asym":
        spec["zeros"] = ((layer.out, (nG + 7) // 8), torch.int32)
    return spec


def quantize_layer(layer: BlockLayer) -> dict:
    """The whole path for one layer on the current GPU: statistics, the grid
    search (alpha, then the clip grid if any), packing at the choice.  `meta`
    holds [best_alpha, best_clip, alpha*, clip*, losses...]."""
    import torch

    import weight_only_quantization_awq_b200 as awq
    sX = awq.awq_act_stats(layer.X)
    res = awq.awq_search_layer(layer.W, layer.X, sX, layer.group_size, layer.w_bit, layer.quant,
                               list(layer.alpha), clip=list(layer.clip) or None)
    a = float(layer.alpha[res["best_alpha"]])
    c = float(layer.clip[res["best_clip"]]) if layer.clip else 1.0
    p = awq.awq_pack_quant(layer.W, sX, a, c, layer.group_size, layer.quant, w_bit=layer.w_bit)
    meta = torch.tensor([res["best_alpha"], res["best_clip"], a, c, *res["loss"]],
                        dtype=torch.float64, device=layer.W.device)
    out = {"qweight": p["qweight"], "scales": p["scales"], "s16": p["s16"], "meta": meta}
    if p["zeros"] is not None:
        out["zeros"] = p["zeros"]
    return out


def quantize_block(layers: list, rank: int = 0, world: int = 1, device=None, quantize=quantize_layer,
                   group=None) -> dict:
    """Quantise `layers` over `world` ranks; returns {name: result} on every rank.

    Each rank runs `quantize` on the layers it owns (assign_layers on their
    search cost); then, for each layer in order, its owner broadcasts the result
    tensors to the other ranks (torch.distributed on `group`).  With world == 1
    this is a plain loop over the layers."""
    import torch
    owner = assign_layers([l.cost() for l in layers], world)
    results = {}
    for k, layer in enumerate(layers):
        if owner[k] == rank:
            results[layer.name] = quantize(layer)
    if world == 1:
        return results
    import torch.distributed as dist
    dev = torch.device("cpu") if device is None else torch.device(device)
    for k, layer in enumerate(layers):
        spec = result_spec(layer)
        if owner[k] == rank:
            mine = results[layer.name]
            for key in sorted(spec):
                t = mine[key].contiguous()
                if t.device != dev:
                    t = t.to(dev)
                dist.broadcast(t, src=owner[k], group=group)
                mine[key] = t
        else:
            got = {}
            for key in sorted(spec):
                shape, dtype = spec[key]
                t = torch.empty(shape, dtype=dtype, device=dev)
                dist.broadcast(t, src=owner[k], group=group)
                got[key] = t
            results[layer.name] = got
    return results


def block_plan_summary(layers: list, world: int) -> dict:
    """The assignment and each rank's share of the block's search work."""
    costs = [l.cost() for l in layers]
    owner = assign_layers(costs, world)
    load = [0.0] * world
    for c, r in zip(costs, owner):
        load[r] += c
    total = sum(costs)
    return {"owner": {l.name: r for l, r in zip(layers, owner)},
            "load": load, "max_share": max(load) / total if total else 0.0,
            "ideal_speedup": total / max(load) if max(load) else math.inf}
