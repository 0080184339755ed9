"""Layer-parallel block quantisation: the assignment of layers to ranks and
the exchange of results, on CPU ranks over gloo (world size 2) with a stand-in
for the per-layer GPU work.  The GPU path of each layer is the one the other
tests check; here what is checked is that every rank ends with every layer's
result, identical to a single-rank run, and that the plan balances the work."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from weight_only_quantization_awq_b200.block import (BlockLayer, assign_layers,  # noqa: E402
                                                     block_plan_summary, quantize_block,
                                                     result_spec)


def test_assign_longest_first_balances():
    assert assign_layers([5, 3, 2], 1) == [0, 0, 0]
    owner = assign_layers([9, 8, 2, 1], 2)
    load = [sum(c for c, r in zip([9, 8, 2, 1], owner) if r == q) for q in range(2)]
    assert sorted(load) == [10, 10]
    assert assign_layers([1, 1, 1, 1], 4) == [0, 1, 2, 3]
    assert assign_layers([3, 3], 2) == [0, 1]                  # ties: lower rank, lower index
    costs = list(np.random.default_rng(0).uniform(1, 10, size=13))
    for world in (2, 3, 5):
        owner = assign_layers(costs, world)
        load = [sum(c for c, r in zip(costs, owner) if r == q) for q in range(world)]
        assert max(load) <= sum(costs) / world + max(costs)   # the greedy bound
        assert owner == assign_layers(costs, world)           # deterministic
    with pytest.raises(ValueError):
        assign_layers([1.0], 0)


def _layers(shapes):
    g = torch.Generator().manual_seed(7)
    out = []
    for name, o, i, n, quant, clip in shapes:
        out.append(BlockLayer(name, torch.randn(o, i, generator=g), torch.randn(n, i, generator=g),
                              quant=quant, group_size=64, clip=clip))
    return out


SHAPES = [("qkv", 96, 128, 40, "asym", (1.0, 0.9)), ("o", 32, 128, 40, "asym", (1.0, 0.9)),
          ("gate_up", 160, 128, 40, "sym", ()), ("down", 32, 320, 40, "asym", (1.0,))]


def fake_quantize(layer):
    """Deterministic stand-in with the shapes and dtypes of a real result."""
    spec = result_spec(layer)
    W = layer.W
    res = {}
    for key, (shape, dtype) in spec.items():
        n = int(np.prod(shape))
        base = torch.arange(n, dtype=torch.float64) * float(W.abs().sum()) % 1000.0
        res[key] = (base.reshape(shape) - 500.0).to(dtype)
    return res


def _rank_main(rank, world, port, out):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        res = quantize_block(_layers(SHAPES), rank=rank, world=world, quantize=fake_quantize)
        out[rank] = {k: {kk: v.numpy().tobytes() for kk, v in d.items()} for k, d in res.items()}
    finally:
        dist.destroy_process_group()


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_quantize_block_gloo_world2():
    single = quantize_block(_layers(SHAPES), rank=0, world=1, quantize=fake_quantize)
    want = {k: {kk: v.numpy().tobytes() for kk, v in d.items()} for k, d in single.items()}
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world,
                           start_method="spawn", join=True)
        res = dict(out)
    for rank in range(world):
        assert set(res[rank]) == {name for name, *_ in SHAPES}
        assert res[rank] == want


def test_block_plan_of_the_llama7b_block():
    """The workload-5 block: qkv 12288x4096, o 4096x4096, gate||up 22016x4096,
    down 4096x11008, 16384 tokens, 20 + 11 grid points.  gate||up alone is 45%
    of the work, which bounds the speed-up of whole-layer parallelism."""
    class L:
        def __init__(self, name, o, i):
            self.name, self.o, self.i = name, o, i

        def cost(self):
            return 31 * 2.0 * 16384 * self.i * self.o
    layers = [L("qkv", 12288, 4096), L("o", 4096, 4096), L("gate_up", 22016, 4096),
              L("down", 4096, 11008)]
    s1 = block_plan_summary(layers, 1)
    assert s1["ideal_speedup"] == pytest.approx(1.0)
    s2 = block_plan_summary(layers, 2)
    assert s2["owner"]["gate_up"] != s2["owner"]["qkv"]
    assert 1.5 < s2["ideal_speedup"] <= 2.0
    s4 = block_plan_summary(layers, 4)
    assert len(set(s4["owner"].values())) == 4
    assert s4["max_share"] == pytest.approx(22016 / (12288 + 4096 + 22016 + 11008 * 4096 / 4096), rel=1e-9)
