"""Routing with no device allocation (moe_mxfp4_route_noalloc).

Some callers cannot allocate device memory: code that must not synchronise the
device (cudaMalloc may), hosts whose device memory belongs to another
allocator, or processes that hold no layer handle (creating one allocates).
This entry point runs the same router kernel as the layer's forward with its
scratch in a fixed static device array.  Its outputs are checked here against
the layer's own routing outputs from moe_mxfp4_forward and against the CPU
oracle's router, on two calls in a row (the second reuses the array the first
one left behind), including a case that fills the array to its documented
limits (T = 256 tokens, E = 128 experts).

This file is collected last so that a run stopping at the first failure has
already run every other test.
"""
import numpy as np
import pytest

import moe_inputs as mi
import oracle
from _layer import W_ABS_TOL, GpuLayer, OracleExperts, act_tensor, check_layer, filtered_x

pytestmark = pytest.mark.gpu


def _route_twice(cfg, x_np, wr_np, bias_np):
    """Two back-to-back calls through the C ABI; returns the outputs of each."""
    import torch
    import mxfp4_expert_gemm_router_b200 as mx

    x = act_tensor(cfg, x_np)
    wr = act_tensor(cfg, wr_np)
    bias = None if bias_np is None else torch.from_numpy(bias_np.astype(np.float32)).cuda()
    outs = []
    for _ in range(2):
        idx = torch.full((cfg.T, cfg.top_k), -1, dtype=torch.int32, device="cuda")
        w = torch.full((cfg.T, cfg.top_k), -1.0, dtype=torch.float32, device="cuda")
        counts = torch.full((cfg.n_experts,), -1, dtype=torch.int32, device="cuda")
        mx.route_noalloc(x, wr, bias, cfg.top_k, idx, w, counts)
        torch.cuda.synchronize()
        outs.append((idx.cpu().numpy(), w.cpu().numpy().astype(np.float64), counts.cpu().numpy()))
    return outs


@pytest.mark.parametrize("name", ["tiny", "dec64"])
def test_route_noalloc_matches_forward_routing(name):
    cfg = mi.CONFIGS[name]
    L = GpuLayer(cfg, cfg.T)
    x_np = filtered_x(cfg, L.wr, L.bias)
    _, idx_fwd, w_fwd, counts_fwd = L.forward(x_np)
    _, idx_ref, w_ref, counts_ref = oracle.router(x_np, L.wr, L.bias, cfg.top_k)
    for idx, w, counts in _route_twice(cfg, x_np, L.wr, L.bias):
        # the layer's own forward
        np.testing.assert_array_equal(idx, idx_fwd)
        np.testing.assert_array_equal(counts, counts_fwd)
        assert np.abs(w - w_fwd).max() <= W_ABS_TOL
        # and the oracle's router, independently
        np.testing.assert_array_equal(idx, idx_ref)
        np.testing.assert_array_equal(counts, counts_ref)
        assert np.abs(w - w_ref).max() <= W_ABS_TOL


def test_route_noalloc_at_its_array_limits():
    """T = 256 and E = 128 (four experts per lane): the partial-score and
    histogram regions of the static array at their documented maximum."""
    import mxfp4_expert_gemm_router_b200 as mx
    cfg = mi.MoeConfig("noalloc_max", mx.MOE_ROUTE_NOALLOC_MAX_TOKENS, 2880, 2880,
                       mx.MOE_ROUTE_NOALLOC_MAX_EXPERTS, 4, "bf16")
    wr = mi.draw_router(cfg)
    x_np = filtered_x(cfg, wr, None)
    _, idx_ref, w_ref, counts_ref = oracle.router(x_np, wr, None, cfg.top_k)
    for idx, w, counts in _route_twice(cfg, x_np, wr, None):
        np.testing.assert_array_equal(idx, idx_ref)
        np.testing.assert_array_equal(counts, counts_ref)
        assert np.abs(w - w_ref).max() <= W_ABS_TOL


def test_route_noalloc_leaves_a_256_expert_layer_working():
    """A layer may have up to 256 experts; the no-allocation router must not
    lower the router kernel's shared-memory limit below what such a layer's
    forward needs (create, then route_noalloc, then the layer's forward)."""
    cfg = mi.MoeConfig("e256", 48, 64, 64, 256, 4, "f32")
    L = GpuLayer(cfg, cfg.T)
    ox = OracleExperts(cfg)
    x_np = filtered_x(cfg, L.wr, L.bias)
    small = mi.MoeConfig("e8", 16, 64, 64, 8, 2, "f32")
    wr_small = mi.draw_router(small)
    _route_twice(small, filtered_x(small, wr_small, None), wr_small, None)
    y, idx, w, counts = L.forward(x_np)
    check_layer(cfg, x_np, L.wr, L.bias, y, idx, w, counts, ox, n_sample=cfg.T)
