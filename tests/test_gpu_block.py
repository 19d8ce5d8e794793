"""The MoE block with its adjacent steps fused (RMSNorm pre-norm in the router
and the gather, the residual as the output accumulator's initial value),
through the C ABI, against the oracle's block (page "GPT-OSS vs Qwen3 :
comparaison détaillée", Adoption de RMSNorm).

Bars as for the layer: top-k indices and per-expert counts bit-exact (inputs
margin-filtered on the normalised scores), routing weights within 1e-6, and
max|y - y_ref| <= 2e-2 * max|MoE part of y_ref| (the residual itself is exact).
"""
import numpy as np
import pytest

import moe_inputs as mi
from _layer import GpuLayer, OracleExperts, check_block, filtered_x_norm

pytestmark = pytest.mark.gpu


def _set_block(L, cfg, gamma, residual):
    import torch
    g = None if gamma is None else torch.from_numpy(gamma).cuda()
    L.layer.set_norm_residual(g, mi.NORM_EPS, residual)
    L._gamma_t = g   # keep the source alive until the copy ran
    torch.cuda.synchronize()


@pytest.mark.parametrize("norm,residual", [(True, True), (True, False), (False, True)])
def test_tiny_block_every_token(norm, residual):
    cfg = mi.CONFIGS["tiny"]
    L = GpuLayer(cfg, cfg.T)
    gamma = mi.draw_gamma(cfg) if norm else None
    _set_block(L, cfg, gamma, residual)
    x = filtered_x_norm(cfg, L.wr, L.bias, gamma, mi.NORM_EPS)
    y, idx, w, counts = L.forward(x)
    check_block(cfg, x, L.wr, L.bias, gamma, mi.NORM_EPS, residual, y, idx, w, counts, OracleExperts(cfg),
                n_sample=cfg.T)


@pytest.fixture(scope="module")
def block20b():
    cfg = mi.CONFIGS["dec64"]
    L = GpuLayer(cfg, mi.CONFIGS["zipf"].T)
    return L, OracleExperts(cfg)


@pytest.mark.parametrize("name", ["dec1", "dec8", "dec64", "pre4096", "zipf"])
def test_20b_shaped_block(block20b, name):
    L, ox = block20b
    cfg = mi.CONFIGS[name]
    wr, bias = mi.draw_router(cfg), mi.draw_bias(cfg)
    L.set_router(wr, bias)
    gamma = mi.draw_gamma(cfg)
    _set_block(L, cfg, gamma, True)
    x = filtered_x_norm(cfg, wr, bias, gamma, mi.NORM_EPS)
    y, idx, w, counts = L.forward(x)
    check_block(cfg, x, wr, bias, gamma, mi.NORM_EPS, True, y, idx, w, counts, ox, n_sample=16)
    # back to the plain layer for whoever uses the handle next
    _set_block(L, cfg, None, False)


def test_e128_block():
    cfg = mi.CONFIGS["e128"]
    L = GpuLayer(cfg, cfg.T)
    gamma = mi.draw_gamma(cfg)
    _set_block(L, cfg, gamma, True)
    x = filtered_x_norm(cfg, L.wr, L.bias, gamma, mi.NORM_EPS)
    y, idx, w, counts = L.forward(x)
    check_block(cfg, x, L.wr, L.bias, gamma, mi.NORM_EPS, True, y, idx, w, counts, OracleExperts(cfg),
                n_sample=12)


def test_set_norm_residual_rejects_bad_arguments():
    import ctypes
    import mxfp4_expert_gemm_router_b200 as mx
    cfg = mi.CONFIGS["tiny"]
    L = GpuLayer(cfg, cfg.T, quantize=False)
    lib = mx.load()
    assert lib.moe_mxfp4_set_norm_residual(L.layer.h, None, -1.0, 0, None) == mx.MOE_ERR_INVALID_ARG
    assert lib.moe_mxfp4_set_norm_residual(L.layer.h, None, float("nan"), 0, None) == mx.MOE_ERR_INVALID_ARG
    assert lib.moe_mxfp4_set_norm_residual(L.layer.h, ctypes.c_void_p(4098), 1e-5, 0, None) == \
        mx.MOE_ERR_INVALID_ARG
    assert lib.moe_mxfp4_set_norm_residual(None, None, 1e-5, 0, None) == mx.MOE_ERR_INVALID_ARG
