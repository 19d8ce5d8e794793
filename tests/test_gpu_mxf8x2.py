"""The two-MXFP8-term operand format (MOE_FLAG_ACT_MXF8X2): the same layer,
with every activation block fed to the expert MMAs as two E4M3 terms
(kind::mxf8f6f4 against the unchanged MXFP4 weights), held to the same bars as
the default format: codes and scales bit-exact through the export, top-k and
counts bit-exact, routing weights within 1e-6, output within 2e-2 of max|ref|.
"""
import numpy as np
import pytest

import moe_inputs as mi
from _layer import (GpuLayer, OracleExperts, check_layer, filtered_x, library_token_tile, tile_boundary_tokens)

pytestmark = pytest.mark.gpu

CFG20 = mi.CONFIGS["dec64"]
MAX_T20 = mi.CONFIGS["pre4096"].T


def _flag():
    import mxfp4_expert_gemm_router_b200 as mx
    return mx.MOE_FLAG_ACT_MXF8X2


def _export(layer, cfg, which):
    import torch
    K, N = (cfg.d_model, cfg.d_ff) if which < 2 else (cfg.d_ff, cfg.d_model)
    codes = torch.empty((cfg.n_experts, N, K // 2), dtype=torch.uint8, device="cuda")
    scales = torch.empty((cfg.n_experts, N, K // 32), dtype=torch.uint8, device="cuda")
    layer.export_weights(which, codes, scales)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), scales.cpu().numpy()


@pytest.fixture(scope="module")
def layer8():
    return GpuLayer(CFG20, MAX_T20, flags=_flag())


@pytest.fixture(scope="module")
def ox20b():
    return OracleExperts(CFG20)


@pytest.mark.parametrize("d,f_", [(192, 320), (96, 160)])
def test_padded_weight_layout_exports_bit_exact(d, f_):
    """Quantised into the padded layout (short last feature tile and K chunk),
    exported back to the canonical layout: identical to the oracle's codes."""
    cfg = mi.MoeConfig("ragged8", 8, d, f_, 4, 2, "f32")
    L = GpuLayer(cfg, cfg.T, flags=_flag())
    q = OracleExperts(cfg).ensure(range(cfg.n_experts))
    for which, (rc, rs) in enumerate([(q.g_codes, q.g_scales), (q.u_codes, q.u_scales), (q.d_codes, q.d_scales)]):
        c, s = _export(L.layer, cfg, which)
        np.testing.assert_array_equal(c, rc)
        np.testing.assert_array_equal(s, rs)


def test_padded_weight_layout_full_size(layer8, ox20b):
    experts = [0, 31]
    q = ox20b.ensure(experts)
    for which, (rc, rs) in enumerate([(q.g_codes, q.g_scales), (q.u_codes, q.u_scales), (q.d_codes, q.d_scales)]):
        c, s = _export(layer8.layer, CFG20, which)
        for e in experts:
            np.testing.assert_array_equal(c[e], rc[e])
            np.testing.assert_array_equal(s[e], rs[e])


@pytest.mark.parametrize("d,f_", [(192, 320), (96, 160)])
@pytest.mark.parametrize("bn", [16, 48, 64, 96, 112, 128])
def test_every_token_tile_on_ragged_shapes(d, f_, bn):
    """Stacked (2 BN <= 192: one MMA per K step over both terms) and per-term
    tiles, on shapes with a short last feature tile and a short last K chunk."""
    import mxfp4_expert_gemm_router_b200 as mx
    cfg = mi.MoeConfig("ragged", 40, d, f_, 4, 2, "f32")
    L = GpuLayer(cfg, cfg.T, flags=_flag() | mx.token_tile_flag(bn))
    ox = OracleExperts(cfg)
    x = filtered_x(cfg, L.wr, L.bias)
    y, idx, w, counts = L.forward(x)
    check_layer(cfg, x, L.wr, L.bias, y, idx, w, counts, ox, n_sample=cfg.T)


@pytest.mark.parametrize("name", ["dec1", "dec8", "dec64", "pre4096"])
def test_20b_shaped_layer_parity(layer8, ox20b, name):
    """dec1 and dec8 split K in both GEMMs (the split-K H encode and the
    scatter-add); dec64 and pre4096 do not."""
    cfg = mi.CONFIGS[name]
    wr, bias = mi.draw_router(cfg), mi.draw_bias(cfg)
    layer8.set_router(wr, bias)
    x = filtered_x(cfg, wr, bias)
    y, idx, w, counts = layer8.forward(x)
    extra = None
    if cfg.T >= 1024:
        extra = tile_boundary_tokens(idx, counts, library_token_tile(cfg.T, cfg.top_k, cfg.n_experts))
    check_layer(cfg, x, wr, bias, y, idx, w, counts, ox20b, n_sample=16, extra_tokens=extra)


def test_two_mxfp8_terms_are_at_least_as_accurate(layer8, ox20b):
    """Two E4M3 terms keep about 8 significant bits per element, three E2M1
    terms about 6: on the same tokens the two-MXFP8 output is no further from
    the oracle than the three-MXFP4 output (with a 10 % allowance), and both
    are well inside the bar."""
    cfg = mi.CONFIGS["dec64"]
    wr, bias = mi.draw_router(cfg), mi.draw_bias(cfg)
    x = filtered_x(cfg, wr, bias)
    layer8.set_router(wr, bias)
    y8, idx8, w8, c8 = layer8.forward(x)
    r8 = check_layer(cfg, x, wr, bias, y8, idx8, w8, c8, ox20b, n_sample=cfg.T)
    L4 = GpuLayer(CFG20, cfg.T)
    L4.set_router(wr, bias)
    y4, idx4, w4, c4 = L4.forward(x)
    r4 = check_layer(cfg, x, wr, bias, y4, idx4, w4, c4, ox20b, n_sample=cfg.T)
    assert r8 <= 1.1 * r4, (r8, r4)
    assert r8 < 1e-2, r8
