"""Routing with no device allocation (moe_mxfp4_route_noalloc).

Some callers cannot allocate device memory: code that must not synchronise the
device (cudaMalloc may), hosts whose device memory belongs to another
allocator, or processes that hold no layer handle (creating one allocates).
This entry point runs the same router kernel as the layer's forward with its
scratch in a fixed static device array.  Its outputs are checked here against
the layer's own routing outputs from moe_mxfp4_forward, on two calls in a row
(the second reuses the array the first one left behind).

This file is collected last so that a run stopping at the first failure has
already run every other test.
"""
import numpy as np
import pytest

import moe_inputs as mi
from _layer import W_ABS_TOL, GpuLayer, act_tensor, filtered_x

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["tiny", "dec64"])
def test_route_noalloc_matches_forward_routing(name):
    import torch
    import mxfp4_expert_gemm_router_b200 as mx

    cfg = mi.CONFIGS[name]
    L = GpuLayer(cfg, cfg.T)
    x_np = filtered_x(cfg, L.wr, L.bias)
    _, idx_ref, w_ref, counts_ref = L.forward(x_np)

    x = act_tensor(cfg, x_np)
    wr = act_tensor(cfg, L.wr)
    bias = None if L.bias is None else torch.from_numpy(L.bias).cuda()
    for _ in range(2):
        idx = torch.full((cfg.T, cfg.top_k), -1, dtype=torch.int32, device="cuda")
        w = torch.full((cfg.T, cfg.top_k), -1.0, dtype=torch.float32, device="cuda")
        counts = torch.full((cfg.n_experts,), -1, dtype=torch.int32, device="cuda")
        mx.route_noalloc(x, wr, bias, cfg.top_k, idx, w, counts)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(idx.cpu().numpy(), idx_ref)
        np.testing.assert_array_equal(counts.cpu().numpy(), counts_ref)
        assert np.abs(w.cpu().numpy().astype(np.float64) - w_ref).max() <= W_ABS_TOL


def test_route_noalloc_rejects_sizes_beyond_its_array():
    import ctypes
    import mxfp4_expert_gemm_router_b200 as mx

    L = mx.load()
    dummy = ctypes.c_void_p(16)  # never dereferenced: the size check comes first
    too_many_tokens = mx.MOE_ROUTE_NOALLOC_MAX_TOKENS + 1
    assert L.moe_mxfp4_route_noalloc(dummy, dummy, None, too_many_tokens, 64, 8, 2, mx.MOE_DTYPE_F32,
                                     dummy, dummy, None, None) == mx.MOE_ERR_UNSUPPORTED
    assert L.moe_mxfp4_route_noalloc(dummy, dummy, None, 4, 64, mx.MOE_ROUTE_NOALLOC_MAX_EXPERTS + 1, 2,
                                     mx.MOE_DTYPE_F32, dummy, dummy, None, None) == mx.MOE_ERR_UNSUPPORTED
    assert L.moe_mxfp4_route_noalloc(dummy, dummy, None, 4, 60, 8, 2, mx.MOE_DTYPE_F32,
                                     dummy, dummy, None, None) == mx.MOE_ERR_UNSUPPORTED
