"""Parity of the CUDA layer (through the C ABI) against the CPU oracle.

Bars: quantised codes and scales bit-exact; top-k
indices and per-expert counts bit-exact (inputs redrawn so no selection margin
is below 1e-4); routing weights within 1e-6; layer output within
max|gpu - ref| <= 2e-2 * max|ref|.
"""
import numpy as np
import pytest

import moe_inputs as mi
import oracle
from _layer import (GpuLayer, OracleExperts, W_ABS_TOL, Y_REL_TOL, act_tensor, check_layer, filtered_x,
                    library_token_tile, tile_boundary_tokens, to_f64)

pytestmark = pytest.mark.gpu

CFG20 = mi.CONFIGS["dec64"]       # all E=32, 2880-wide configs share these weights
MAX_T20 = mi.CONFIGS["zipf"].T


@pytest.fixture(scope="module")
def layer20b():
    return GpuLayer(CFG20, MAX_T20)


@pytest.fixture(scope="module")
def ox20b():
    return OracleExperts(CFG20)


@pytest.fixture(scope="module")
def layer20b_unfused():
    """The same layer with every forward on the multi-launch path."""
    import mxfp4_expert_gemm_router_b200 as mx
    return GpuLayer(CFG20, 256, flags=mx.MOE_FLAG_UNFUSED_DECODE)


def _export(layer, cfg, which):
    import torch
    K, N = (cfg.d_model, cfg.d_ff) if which < 2 else (cfg.d_ff, cfg.d_model)
    codes = torch.empty((cfg.n_experts, N, K // 2), dtype=torch.uint8, device="cuda")
    scales = torch.empty((cfg.n_experts, N, K // 32), dtype=torch.uint8, device="cuda")
    layer.export_weights(which, codes, scales)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), scales.cpu().numpy()


# ------------------------------------------------------------------ quantiser

def test_quantize_bit_exact_tiny():
    cfg = mi.CONFIGS["tiny"]
    L = GpuLayer(cfg, cfg.T)
    ox = OracleExperts(cfg)
    q = ox.ensure(range(cfg.n_experts))
    for which, (rc, rs) in enumerate([(q.g_codes, q.g_scales), (q.u_codes, q.u_scales), (q.d_codes, q.d_scales)]):
        c, s = _export(L.layer, cfg, which)
        np.testing.assert_array_equal(c, rc)
        np.testing.assert_array_equal(s, rs)


def test_quantize_bit_exact_full_size(layer20b, ox20b):
    experts = [0, 13, 31]
    q = ox20b.ensure(experts)
    for which, (rc, rs) in enumerate([(q.g_codes, q.g_scales), (q.u_codes, q.u_scales), (q.d_codes, q.d_scales)]):
        c, s = _export(layer20b.layer, CFG20, which)
        for e in experts:
            np.testing.assert_array_equal(c[e], rc[e])
            np.testing.assert_array_equal(s[e], rs[e])


def test_quantize_hand_worked_blocks():
    """GPU quantiser against the hand-worked blocks of tests/golden/mxfp4_blocks.txt."""
    import os
    import torch
    import mxfp4_expert_gemm_router_b200 as mx
    rows = []
    with open(os.path.join(os.path.dirname(__file__), "golden", "mxfp4_blocks.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                rows.append([p.strip() for p in line.split("|")])
    d, f_ = 32, 32
    W = np.zeros((d, f_), np.float32)          # y = x . W: column n is one 32-block
    for n, (_, vals, _, _) in enumerate(rows):
        W[:, n] = np.array([float(v) for v in vals.split()], np.float32)
    layer = mx.MoeMxfp4(d, f_, 1, 1, 1, "f32")
    wt = torch.from_numpy(W).cuda()
    layer.quantize_expert(0, wt, wt, torch.zeros((f_, d), device="cuda"))
    cfg = mi.MoeConfig("blocks", 1, d, f_, 1, 1, "f32")
    c, s = _export(layer, cfg, 0)
    for n, (name, _, scale, codes) in enumerate(rows):
        got = []
        for b in c[0, n]:
            got += [int(b) & 15, int(b) >> 4]
        assert int(s[0, n, 0]) == int(scale), name
        assert got == [int(v) for v in codes.split()], name
    # all-zero columns beyond the listed blocks
    assert (c[0, len(rows):] == 0).all() and (s[0, len(rows):] == 127).all()


# ------------------------------------------------------------------ layer parity

def test_tiny_layer_full_parity():
    cfg = mi.CONFIGS["tiny"]
    L = GpuLayer(cfg, cfg.T)
    ox = OracleExperts(cfg)
    x = filtered_x(cfg, L.wr, L.bias)
    y, idx, w, counts = L.forward(x)
    rel = check_layer(cfg, x, L.wr, L.bias, y, idx, w, counts, ox, n_sample=cfg.T)
    assert rel < Y_REL_TOL


@pytest.mark.parametrize("name", ["dec1", "dec8", "dec64", "pre4096", "zipf"])
def test_20b_shaped_layer_parity(layer20b, ox20b, name):
    cfg = mi.CONFIGS[name]
    wr, bias = mi.draw_router(cfg), mi.draw_bias(cfg)
    layer20b.set_router(wr, bias)
    x = filtered_x(cfg, wr, bias)
    y, idx, w, counts = layer20b.forward(x)
    extra = None
    if cfg.T >= 1024:
        # every row of the most-loaded expert's first and last token tiles and of
        # every expert's last (ragged) tile
        extra = tile_boundary_tokens(idx, counts, library_token_tile(cfg.T, cfg.top_k, cfg.n_experts))
    check_layer(cfg, x, wr, bias, y, idx, w, counts, ox20b, n_sample=16, extra_tokens=extra)
    if name == "zipf":
        # skewed routing: the most popular expert takes far more than the mean share
        assert counts.max() > 3 * counts.mean()


def test_e128_layer_parity():
    cfg = mi.CONFIGS["e128"]
    L = GpuLayer(cfg, cfg.T)
    ox = OracleExperts(cfg)
    x = filtered_x(cfg, L.wr, L.bias)
    y, idx, w, counts = L.forward(x)
    # 128 experts: the whole last tile of 16 seeded experts (and of the most and
    # least loaded), the first and last rows of every other expert's last tile
    extra = tile_boundary_tokens(idx, counts, library_token_tile(cfg.T, cfg.top_k, cfg.n_experts),
                                 max_full_experts=16)
    check_layer(cfg, x, L.wr, L.bias, y, idx, w, counts, ox, n_sample=12, extra_tokens=extra)


@pytest.mark.parametrize("d,f_", [(192, 320), (96, 160)])
@pytest.mark.parametrize("bn", [16, 48, 64, 112, 128])
def test_every_token_tile_on_ragged_shapes(d, f_, bn):
    """Token tiles from 16 to 128 rows (one or two accumulator buffers) on
    shapes with a short last feature tile (64 or 32 rows), a short last K
    chunk, and K a multiple of 32 but not of 64."""
    import mxfp4_expert_gemm_router_b200 as mx
    cfg = mi.MoeConfig("ragged", 40, d, f_, 4, 2, "f32")
    L = GpuLayer(cfg, cfg.T, flags=mx.token_tile_flag(bn))
    ox = OracleExperts(cfg)
    x = filtered_x(cfg, L.wr, L.bias)
    y, idx, w, counts = L.forward(x)
    check_layer(cfg, x, L.wr, L.bias, y, idx, w, counts, ox, n_sample=cfg.T)


def test_ragged_token_counts(layer20b, ox20b):
    """Token counts that are not multiples of the router block (32) or of the tile."""
    for T in (3, 37, 130):
        cfg = CFG20.with_T(T)
        layer20b.set_router(mi.draw_router(cfg), None)
        x = filtered_x(cfg, layer20b.wr, None)
        y, idx, w, counts = layer20b.forward(x)
        check_layer(cfg, x, layer20b.wr, None, y, idx, w, counts, ox20b, n_sample=6)


def test_zero_tokens_launches_nothing(layer20b):
    import torch
    n0 = layer20b.layer.launch_count()
    x = torch.empty((0, CFG20.d_model), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((0, CFG20.d_model), dtype=torch.bfloat16, device="cuda")
    layer20b.layer.forward(x, y)
    assert layer20b.layer.launch_count() == n0


def test_rows_are_independent(layer20b):
    cfg = CFG20.with_T(8)
    layer20b.set_router(mi.draw_router(cfg), None)
    x = filtered_x(cfg, layer20b.wr, None)
    y, _, _, _ = layer20b.forward(x)
    scale = np.abs(y).max()
    for t in range(8):
        yt, _, _, _ = layer20b.forward(x[t:t + 1])
        assert np.abs(yt[0] - y[t]).max() <= 1e-2 * scale


def test_grouping_is_stable_sort_by_expert(layer20b):
    import torch
    cfg = CFG20.with_T(100)
    layer20b.set_router(mi.draw_router(cfg), None)
    x = filtered_x(cfg, layer20b.wr, None)
    _, idx, w, counts = layer20b.forward(x)
    E, k = cfg.n_experts, cfg.top_k
    off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    rt = torch.empty(100 * k, dtype=torch.int32, device="cuda")
    rw = torch.empty(100 * k, dtype=torch.float32, device="cuda")
    layer20b.layer.get_grouping(off, rt, rw)
    torch.cuda.synchronize()
    off, rt, rw = off.cpu().numpy(), rt.cpu().numpy(), rw.cpu().numpy()
    np.testing.assert_array_equal(off, np.concatenate([[0], np.cumsum(counts)]))
    pairs = sorted(((int(idx[t, j]), t, j) for t in range(100) for j in range(k)))
    np.testing.assert_array_equal(rt, [t for _, t, _ in pairs])
    np.testing.assert_array_equal(rw, np.array([w[t, j] for _, t, j in pairs], np.float32))


def test_forward_host_matches_device(layer20b):
    import torch
    cfg = CFG20.with_T(16)
    layer20b.set_router(mi.draw_router(cfg), None)
    x = filtered_x(cfg, layer20b.wr, None)
    y_dev, idx_dev, w_dev, _ = layer20b.forward(x)
    xh = act_tensor(cfg, x, device="cpu").pin_memory()
    yh = torch.empty_like(xh).pin_memory()
    ih = torch.empty((16, cfg.top_k), dtype=torch.int32).pin_memory()
    wh = torch.empty((16, cfg.top_k), dtype=torch.float32).pin_memory()
    layer20b.layer.forward_host(xh, yh, ih, wh)
    np.testing.assert_array_equal(ih.numpy(), idx_dev)
    np.testing.assert_allclose(wh.numpy(), w_dev, atol=1e-7)
    assert np.abs(to_f64(yh) - y_dev).max() <= 1e-2 * np.abs(y_dev).max()


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("T", [1, 40, 200])
def test_router_ties_go_to_the_lower_index(dtype, T):
    """Experts 2 and 6 get identical router rows and a bias far above the rest,
    so every token's two best scores are exactly equal: expert 2 (the lower
    index) comes first, then 6, with weights 1/2 each.  T = 1, 40 and 200 take
    the top-k with 8, 4 and 1-2 lanes per token (and two router tiles at 200);
    fp32 layers score on the CUDA cores, bf16 layers on the tensor cores."""
    import mxfp4_expert_gemm_router_b200 as mx
    cfg = mi.MoeConfig("ties", T, 64, 128, 8, 2, dtype)
    L = GpuLayer(cfg, T, flags=mx.MOE_FLAG_UNFUSED_DECODE)
    wr = L.wr.copy()
    wr[6] = wr[2]
    bias = np.zeros(cfg.n_experts, np.float32)
    bias[2] = bias[6] = 50.0
    L.set_router(wr, bias)
    x = mi.draw_x(cfg)
    _, idx, w, counts = L.forward(x)
    assert (idx[:, 0] == 2).all() and (idx[:, 1] == 6).all(), idx[:4]
    np.testing.assert_allclose(w, 0.5, atol=1e-7)
    assert counts[2] == T and counts[6] == T and counts.sum() == 2 * T


def test_identity_experts_closed_form():
    """W_gate = a I, W_up = b I, W_down = c I (powers of two): y = sum_j w_j c a b x^2 sigma(a x)."""
    import torch
    import mxfp4_expert_gemm_router_b200 as mx
    d, E, k, T = 128, 4, 2, 40
    a, b, c = [0.5, 1.0, 2.0, 0.25], [1.0, 2.0, 0.5, 4.0], [2.0, 0.5, 1.0, 0.125]
    layer = mx.MoeMxfp4(d, d, E, k, T, "f32")
    I = torch.eye(d, device="cuda")
    for e in range(E):
        layer.quantize_expert(e, I * a[e], I * b[e], I * c[e])
    rng = np.random.default_rng(3)
    wr = (rng.standard_normal((E, d)) / np.sqrt(d)).astype(np.float32)
    x = rng.standard_normal((T, d)).astype(np.float32)
    cfg = mi.MoeConfig("ident", T, d, d, E, k, "f32")
    x, _ = mi.margin_filter(cfg, x, lambda r: oracle.router_logits(r, wr, None))
    layer.set_router(torch.from_numpy(wr).cuda())
    xt = torch.from_numpy(x).cuda()
    y = torch.empty_like(xt)
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    wt = torch.empty((T, k), dtype=torch.float32, device="cuda")
    layer.forward(xt, y, idx, wt)
    torch.cuda.synchronize()
    idx, wt, y = idx.cpu().numpy(), wt.cpu().numpy().astype(np.float64), y.cpu().numpy().astype(np.float64)
    x64 = x.astype(np.float64)
    ref = np.zeros_like(x64)
    for j in range(k):
        e = idx[:, j]
        A, B, C = (np.array(v)[e][:, None] for v in (a, b, c))
        ref += wt[:, j:j + 1] * C * A * B * x64 ** 2 / (1 + np.exp(-A * x64))
    assert np.abs(y - ref).max() <= 5e-3 * np.abs(ref).max()


def test_repeated_forward_is_stable(layer20b):
    cfg = CFG20.with_T(64)
    layer20b.set_router(mi.draw_router(cfg), None)
    x = filtered_x(cfg, layer20b.wr, None)
    y1, i1, w1, c1 = layer20b.forward(x)
    y2, i2, w2, c2 = layer20b.forward(x)
    np.testing.assert_array_equal(i1, i2)
    np.testing.assert_array_equal(c1, c2)
    np.testing.assert_array_equal(w1, w2)
    assert np.abs(y1 - y2).max() <= 1e-3 * np.abs(y1).max()


def test_pipeline_timeout_is_reported_not_hung():
    """A producer copy that never happens makes a consumer wait run out; the kernel
    returns, the status reports the timeout, and the context stays usable."""
    import torch
    import mxfp4_expert_gemm_router_b200 as mx
    cfg = mi.CONFIGS["tiny"]
    L = GpuLayer(cfg, cfg.T, flags=mx.MOE_FLAG_TEST_SKIP_FIRST_COPY, wait_timeout_ms=100)
    x = act_tensor(cfg, mi.draw_x(cfg))
    y = torch.empty((cfg.T, cfg.d_model), device="cuda")
    L.layer.forward(x, y)
    assert L.layer.status() == mx.MOE_ERR_TIMEOUT
    assert L.layer.status() == mx.MOE_OK  # cleared once read
    # the context still works: a normal handle runs and matches the oracle
    L2 = GpuLayer(cfg, cfg.T)
    xf = filtered_x(cfg, L2.wr, L2.bias)
    yy, idx, w, counts = L2.forward(xf)
    check_layer(cfg, xf, L2.wr, L2.bias, yy, idx, w, counts, OracleExperts(cfg), n_sample=cfg.T)


def test_scaled_activations_stay_within_tolerance(layer20b, ox20b):
    """x scaled by 16 (exact in bf16): H grows about 256-fold; it is formed and
    encoded in fp32 (no f16 range limit), so the layer still meets the bar."""
    cfg = CFG20
    wr = mi.draw_router(cfg)
    layer20b.set_router(wr, None)
    # scaling multiplies every selection margin by 16, so the filter still holds
    x = filtered_x(cfg, wr, None) * np.float32(16.0)
    y, idx, w, counts = layer20b.forward(x)
    check_layer(cfg, x, wr, None, y, idx, w, counts, ox20b, n_sample=16)


def test_quantize_weights_entry_point():
    """The whole-layer loader (all experts, the router and its bias in one
    call): exported codes and scales byte-for-byte equal to the oracle's
    quantiser for every expert, and the layer output matches the oracle
    (the Zipf-biased router at 256 tokens)."""
    import torch
    import mxfp4_expert_gemm_router_b200 as mx
    for cfg in (mi.CONFIGS["tiny"], mi.CONFIGS["zipf"].with_T(256)):
        E, d, f = cfg.n_experts, cfg.d_model, cfg.d_ff
        layer = mx.MoeMxfp4(d, f, E, cfg.top_k, cfg.T, cfg.act_dtype)
        wg = torch.empty((E, d, f), dtype=torch.float32, device="cuda")
        wu = torch.empty((E, d, f), dtype=torch.float32, device="cuda")
        wd = torch.empty((E, f, d), dtype=torch.float32, device="cuda")
        for e in range(E):
            g_, u_, d_ = mi.draw_expert(cfg, e)
            wg[e].copy_(torch.from_numpy(g_))
            wu[e].copy_(torch.from_numpy(u_))
            wd[e].copy_(torch.from_numpy(d_))
        wr = mi.draw_router(cfg)
        bias = mi.draw_bias(cfg)
        b_t = None if bias is None else torch.from_numpy(bias).cuda()
        layer.quantize_weights(wg, wu, wd, act_tensor(cfg, wr), b_t)
        torch.cuda.synchronize()
        del wg, wu, wd
        ox = OracleExperts(cfg)
        q = ox.ensure(range(E))
        for which, (rc, rs) in enumerate([(q.g_codes, q.g_scales), (q.u_codes, q.u_scales),
                                          (q.d_codes, q.d_scales)]):
            c, sc = _export(layer, cfg, which)
            np.testing.assert_array_equal(c, rc)
            np.testing.assert_array_equal(sc, rs)
        x = filtered_x(cfg, wr, bias)
        xt = act_tensor(cfg, x)
        y = torch.empty_like(xt)
        idx = torch.empty((cfg.T, cfg.top_k), dtype=torch.int32, device="cuda")
        w = torch.empty((cfg.T, cfg.top_k), dtype=torch.float32, device="cuda")
        counts = torch.empty((E,), dtype=torch.int32, device="cuda")
        layer.forward(xt, y, idx, w, counts)
        torch.cuda.synchronize()
        assert layer.status() == mx.MOE_OK
        check_layer(cfg, x, wr, bias, to_f64(y), idx.cpu().numpy(), w.cpu().numpy().astype(np.float64),
                    counts.cpu().numpy(), ox, n_sample=cfg.T)
        layer.close()


def test_misaligned_pointers_are_rejected_before_any_launch(layer20b):
    """x and y are read and written 16 bytes at a time: a pointer off that
    boundary returns INVALID_ARG and launches nothing (no misaligned access)."""
    import torch
    import mxfp4_expert_gemm_router_b200 as mx
    T, d = 8, CFG20.d_model
    L = mx.load()
    buf = torch.zeros((T + 1) * d, dtype=torch.bfloat16, device="cuda")
    good = buf.data_ptr()
    off = good + 2          # one bf16 element past a 16-byte boundary
    y = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty(T * CFG20.top_k + 1, dtype=torch.int32, device="cuda")
    n0 = layer20b.layer.launch_count()
    h = layer20b.layer.h
    s = torch.cuda.current_stream().cuda_stream
    assert L.moe_mxfp4_forward(h, off, T, y.data_ptr(), None, None, None, s) == mx.MOE_ERR_INVALID_ARG
    assert L.moe_mxfp4_forward(h, good, T, off, None, None, None, s) == mx.MOE_ERR_INVALID_ARG
    assert L.moe_mxfp4_forward(h, good, T, y.data_ptr(), idx.data_ptr() + 2, None, None,
                               s) == mx.MOE_ERR_INVALID_ARG
    assert layer20b.layer.launch_count() == n0
    # the handle still works
    assert L.moe_mxfp4_forward(h, good, T, y.data_ptr(), None, None, None, s) == mx.MOE_OK
    torch.cuda.synchronize()
    assert layer20b.layer.status() == mx.MOE_OK


# ------------------------------------------------------------------ fused decode path (T <= 16)

@pytest.mark.parametrize("name", ["dec1", "dec8"])
def test_decode_unfused_path_parity(layer20b_unfused, ox20b, name):
    """dec1 / dec8 through the multi-launch path (the default is the fused kernel)."""
    cfg = mi.CONFIGS[name]
    wr = mi.draw_router(cfg)
    layer20b_unfused.set_router(wr, None)
    x = filtered_x(cfg, wr, None)
    y, idx, w, counts = layer20b_unfused.forward(x)
    check_layer(cfg, x, wr, None, y, idx, w, counts, ox20b, n_sample=cfg.T)


def test_fused_decode_state_across_launches(layer20b, layer20b_unfused, ox20b):
    """The fused kernel keeps state between launches (epoch, counters, buffers
    alternating by parity that each launch clears for the next): a run of
    forwards of varying size must each match the oracle on every token and
    the multi-launch path."""
    wr = mi.draw_router(CFG20)
    layer20b.set_router(wr, None)
    layer20b_unfused.set_router(wr, None)
    for i, T in enumerate([8, 1, 16, 3, 16, 16, 2, 8]):
        cfg = CFG20.with_T(T)
        x = mi.draw_x(cfg.with_T(64))[8 * i: 8 * i + T] if T <= 8 else mi.draw_x(cfg)
        x, _ = mi.margin_filter(cfg, x, lambda r: oracle.router_logits(r, wr, None))
        y, idx, w, counts = layer20b.forward(x)
        check_layer(cfg, x, wr, None, y, idx, w, counts, ox20b, n_sample=T)
        y2, idx2, w2, _ = layer20b_unfused.forward(x)
        np.testing.assert_array_equal(idx, idx2)
        assert np.abs(w - w2).max() <= W_ABS_TOL
        assert np.abs(y - y2).max() <= 1e-2 * np.abs(y2).max()


@pytest.mark.parametrize("d,f_,E,k", [(192, 320, 4, 2), (96, 160, 5, 3), (64, 64, 256, 4), (2880, 2880, 128, 4)])
def test_fused_decode_ragged_shapes(d, f_, E, k):
    """The fused kernel on shapes with a short last feature tile, a short last
    K chunk (K a multiple of 32 but not of 64), 256 experts (eight per lane in
    the top-k) and 128 experts at full width, at 16 and 5 tokens."""
    for T in (16, 5):
        cfg = mi.MoeConfig("fused_ragged", T, d, f_, E, k, "bf16" if d == 2880 else "f32")
        L = GpuLayer(cfg, 16)
        ox = OracleExperts(cfg)
        x = filtered_x(cfg, L.wr, L.bias)
        y, idx, w, counts = L.forward(x)
        check_layer(cfg, x, L.wr, L.bias, y, idx, w, counts, ox, n_sample=cfg.T)
        L.layer.close()


def test_unfused_pipeline_timeout_is_reported_not_hung():
    """The timeout path of the multi-launch kernels (the fused kernel's is
    covered by test_pipeline_timeout_is_reported_not_hung at 16 tokens)."""
    import torch
    import mxfp4_expert_gemm_router_b200 as mx
    cfg = mi.CONFIGS["tiny"]
    L = GpuLayer(cfg, cfg.T, flags=mx.MOE_FLAG_TEST_SKIP_FIRST_COPY | mx.MOE_FLAG_UNFUSED_DECODE,
                 wait_timeout_ms=100)
    x = act_tensor(cfg, mi.draw_x(cfg))
    y = torch.empty((cfg.T, cfg.d_model), device="cuda")
    L.layer.forward(x, y)
    assert L.layer.status() == mx.MOE_ERR_TIMEOUT
    assert L.layer.status() == mx.MOE_OK


def test_forward_host_chunked_matches_device(layer20b):
    """At 12288 tokens the host-buffer entry point runs three chunks whose copies
    overlap the neighbouring forwards: same routing and output as one device
    forward of the whole batch."""
    import torch
    cfg = CFG20.with_T(12288)
    layer20b.set_router(mi.draw_router(cfg), None)
    x = mi.draw_x(cfg)
    y_dev, idx_dev, w_dev, _ = layer20b.forward(x)
    xh = act_tensor(cfg, x, device="cpu").pin_memory()
    yh = torch.empty_like(xh).pin_memory()
    ih = torch.empty((cfg.T, cfg.top_k), dtype=torch.int32).pin_memory()
    wh = torch.empty((cfg.T, cfg.top_k), dtype=torch.float32).pin_memory()
    layer20b.layer.forward_host(xh, yh, ih, wh)
    np.testing.assert_array_equal(ih.numpy(), idx_dev)
    np.testing.assert_allclose(wh.numpy(), w_dev, atol=1e-7)
    assert np.abs(to_f64(yh) - y_dev).max() <= 1e-2 * np.abs(y_dev).max()
