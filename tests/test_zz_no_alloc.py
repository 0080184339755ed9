"""The allocation-free activation statistic (awq_act_stats_noalloc).

Some callers cannot allocate device memory when they compute the statistic:
processes that give nearly all device memory to their own pool allocator at
start-up, or code that must not allocate inside a latency-critical section.
For them the library keeps the fp64 chunk partials in a fixed buffer compiled
into the library instead of a temporary allocation.  This file checks, through
the C ABI, that two calls in a row give exactly what the allocating entry point
gives (the statistic is bit-exact by construction, as everywhere in the tests),
and that calls beyond the buffer's capacity are refused before any work.
"""
import ctypes

import numpy as np
import pytest
import torch

from synthetic import small_layer

pytestmark = pytest.mark.gpu

AWQ_BF16, AWQ_F32 = 1, 0
AWQ_ERR_UNSUPPORTED = 3


def _dev(a: np.ndarray) -> torch.Tensor:
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def test_act_stats_noalloc_matches_allocating_entry_point():
    import weight_only_quantization_awq_b200 as awq
    assert torch.cuda.is_available()
    lib = awq.lib
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    cases = [small_layer(8, 1024, 4099, xdtype="bf16", seed=41)[1],
             small_layer(8, 520, 777, xdtype="f32", seed=42)[1]]
    for X in cases:                      # two calls in a row, different shapes and dtypes
        Xd = _dev(X)
        N, inp = X.shape
        dt = AWQ_BF16 if X.dtype == np.uint16 else AWQ_F32
        out = torch.full((inp,), float("nan"), dtype=torch.float32, device="cuda")
        st = lib.awq_act_stats_noalloc(Xd.data_ptr(), dt, N, inp, ctypes.c_float(1e-4),
                                       out.data_ptr(), stream)
        assert st == 0, lib.awq_last_error().decode()
        ref = awq.awq_act_stats(Xd)
        via_binding = awq.awq_act_stats_noalloc(Xd)
        torch.cuda.synchronize()
        assert torch.equal(out, ref)
        assert torch.equal(via_binding, ref)

    # beyond the fixed buffer (ceil(N/128) * in > 2^20): refused, nothing enqueued
    big = torch.empty((128 * 129, 8192), dtype=torch.bfloat16, device="cuda")
    out = torch.empty(8192, dtype=torch.float32, device="cuda")
    st = lib.awq_act_stats_noalloc(big.data_ptr(), AWQ_BF16, big.shape[0], big.shape[1],
                                   ctypes.c_float(1e-4), out.data_ptr(), stream)
    assert st == AWQ_ERR_UNSUPPORTED
    assert "fixed buffer" in lib.awq_last_error().decode()
