"""Seeded input generator: determinism, dtype rounding, per-tensor streams, margin filter."""
import numpy as np

import moe_inputs as mi
import oracle


def test_configs_match_workloads():
    c = mi.CONFIGS
    assert (c["tiny"].T, c["tiny"].d_model, c["tiny"].n_experts, c["tiny"].top_k, c["tiny"].d_ff) == (16, 64, 8, 2, 128)
    assert c["tiny"].act_dtype == "f32"
    for n, T in (("dec1", 1), ("dec8", 8), ("dec64", 64), ("pre4096", 4096)):
        assert (c[n].T, c[n].d_model, c[n].n_experts, c[n].top_k, c[n].d_ff, c[n].act_dtype) == (T, 2880, 32, 4, 2880, "bf16")
    assert (c["e128"].T, c["e128"].n_experts) == (8192, 128)
    assert (c["zipf"].T, c["zipf"].zipf_s) == (16384, 1.2)


def test_draws_are_deterministic_and_streams_independent():
    cfg = mi.CONFIGS["tiny"]
    np.testing.assert_array_equal(mi.draw_x(cfg), mi.draw_x(cfg))
    a = mi.draw_expert(cfg, 3)
    b = mi.draw_expert(cfg, 3)
    for u, v in zip(a, b):
        np.testing.assert_array_equal(u, v)
    c = mi.draw_expert(cfg, 4)
    assert not np.array_equal(a[0], c[0])
    assert not np.array_equal(a[0], a[1])
    # a longer draw starts with the shorter one (rows come from one stream)
    np.testing.assert_array_equal(mi.draw_x(cfg, 4), mi.draw_x(cfg, 16)[:4])


def test_distributions():
    cfg = mi.CONFIGS["tiny"]
    wg, wu, wd = mi.draw_expert(cfg, 0)
    assert wg.shape == (64, 128) and wd.shape == (128, 64)
    assert abs(np.concatenate([wg.ravel(), wu.ravel(), wd.ravel()]).std() - 0.02) < 0.001
    wr = mi.draw_router(mi.CONFIGS["dec1"])
    assert wr.shape == (32, 2880)
    assert abs(wr.std() * np.sqrt(2880) - 1) < 0.02


def test_bf16_rounding_ties_to_even():
    vals = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -9, -2.5, 1e-3], np.float32)
    r = mi.bf16_round(vals)
    assert r[0] == 1.0
    assert r[1] == 1.0                      # tie -> even (down)
    assert r[2] == 1.0 + 4 * 2 ** -8        # tie -> even (up)
    assert r[3] == 1.0
    assert r[4] == -2.5
    assert (r.view(np.uint32) & 0xFFFF == 0).all()
    assert np.abs(r[5] - 1e-3) <= 2 ** -9 * 1e-3
    x = mi.draw_x(mi.CONFIGS["dec8"])
    assert (x.view(np.uint32) & 0xFFFF == 0).all()
    np.testing.assert_array_equal(mi.bf16_bits(x).astype(np.uint32) << 16, x.view(np.uint32))


def test_zipf_bias_is_log_probability():
    cfg = mi.CONFIGS["zipf"]
    b = mi.draw_bias(cfg)
    assert b.shape == (32,)
    assert abs(np.exp(b.astype(np.float64)).sum() - 1) < 1e-5
    p = np.sort(np.exp(b.astype(np.float64)))[::-1]
    np.testing.assert_allclose(p[0] / p[1], 2 ** 1.2, rtol=1e-4)
    assert mi.draw_bias(mi.CONFIGS["dec1"]) is None


def test_margin_filter_removes_close_selections():
    cfg = mi.CONFIGS["tiny"]
    wr = mi.draw_router(cfg)
    x = mi.draw_x(cfg)
    fn = lambda rows: oracle.router_logits(rows, wr, None)
    # a huge margin forces redraws; the filtered rows all satisfy it
    xf, n = mi.margin_filter(cfg, x, fn, margin=0.05)
    lg = fn(xf)
    srt = -np.sort(-lg, axis=1)[:, :cfg.top_k + 1]
    assert (np.diff(-srt, axis=1) >= 0.05).all()
    assert n > 0
    # untouched rows keep their first draw
    same = (xf == x).all(axis=1)
    assert same.sum() >= 1
    xf2, n2 = mi.margin_filter(cfg, x, fn, margin=0.05)
    np.testing.assert_array_equal(xf, xf2)
    assert n2 == n
