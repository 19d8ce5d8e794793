"""Pins of the CPU oracle against what the pages and the mathematics fix.

Every test here runs on the CPU (no GPU marker).  Each pins one oracle function
to something other than the oracle itself: values the pages print, the MX
format table, hand-worked blocks, closed forms, brute force on tiny inputs, or
an independent dense computation.  A plausible slip in the oracle (a dropped
term, a swapped operand, a wrong sign, a wrong tie rule) fails at least one.
"""
import itertools
import math
import os

import numpy as np
import pytest

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _read_table(name):
    rows = []
    with open(os.path.join(GOLD, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line)
    return rows


def _figures():
    out = {}
    for line in _read_table("page_figures.txt"):
        k, v = line.split()
        out[k] = float(v)
    return out


# ---------------------------------------------------------------- MXFP4 format

def test_e2m1_decode_matches_format_table():
    for line in _read_table("e2m1_table.txt"):
        code, value = line.split()
        got = oracle.e2m1_decode(int(code))
        assert got == float(value), (code, got, value)
        assert math.copysign(1.0, got) == math.copysign(1.0, float(value))


def test_e8m0_decode():
    assert oracle.e8m0_decode(127) == 1.0
    assert oracle.e8m0_decode(0) == 2.0 ** -127
    assert oracle.e8m0_decode(254) == 2.0 ** 127
    assert oracle.e8m0_decode(130) == 8.0
    assert math.isnan(oracle.e8m0_decode(255))


def test_bits_per_parameter_is_4_25():
    fig = _figures()
    for K in (32, 64, 2880):
        w = np.zeros((3, K), np.float32)
        codes, scales = oracle.mxfp4_quantize_rows(w)
        bits = 8.0 * (codes.nbytes + scales.nbytes) / w.size
        assert bits == fig["bits_per_param"] == 4.25
        # 17/32 bytes per parameter exactly
        assert (codes.nbytes + scales.nbytes) * 32 == 17 * w.size


def test_hand_worked_blocks():
    for line in _read_table("mxfp4_blocks.txt"):
        name, vals, scale, codes = [p.strip() for p in line.split("|")]
        w = np.array([float(v) for v in vals.split()], np.float32)[None, :]
        assert w.shape == (1, 32), name
        exp_codes = [int(c) for c in codes.split()]
        c, s = oracle.mxfp4_quantize_rows(w)
        got = []
        for b in c[0]:
            got += [int(b) & 15, int(b) >> 4]
        assert int(s[0, 0]) == int(scale), (name, int(s[0, 0]), scale)
        assert got == exp_codes, (name, got, exp_codes)


def _all_values(scale_byte):
    return np.array([oracle.e2m1_decode(c) * oracle.e8m0_decode(scale_byte) for c in range(16)])


def test_rounding_is_nearest_with_ties_to_even_bruteforce():
    rng = np.random.default_rng(1)
    w = (rng.standard_normal((64, 32)) * rng.uniform(0.001, 10, (64, 1))).astype(np.float32)
    codes, scales = oracle.mxfp4_quantize_rows(w)
    deq = oracle.mxfp4_dequantize(codes, scales)
    for n in range(w.shape[0]):
        s = int(scales[n, 0])
        amax = float(np.abs(w[n]).max())
        # scale rule: largest power of two <= amax, divided by 4
        assert 2.0 ** (s - 127) == 2.0 ** math.floor(math.log2(amax)) / 4.0
        cand = _all_values(s)
        for i in range(32):
            dist = np.abs(cand - float(w[n, i]))
            best = dist.min()
            assert abs(deq[n, i] - float(w[n, i])) == best
            # tie -> even code
            ties = [c for c in range(16) if dist[c] == best and np.sign(cand[c]) in (0, np.sign(w[n, i]))]
            byte = codes[n, i // 2]
            code = (byte >> 4) if i & 1 else (byte & 15)
            if len({float(cand[c]) for c in ties}) > 1:
                assert (code & 1) == 0


def test_roundtrip_exact_on_grid():
    rng = np.random.default_rng(2)
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6], np.float64)
    for e in (-20, -7, 0, 5):
        v = grid[rng.integers(0, 8, 32)] * rng.choice([-1, 1], 32)
        v[0] = 6.0  # pins the block exponent to e
        w = (v * 2.0 ** e).astype(np.float32)[None, :]
        codes, scales = oracle.mxfp4_quantize_rows(w)
        assert int(scales[0, 0]) == e + 127
        np.testing.assert_array_equal(oracle.mxfp4_dequantize(codes, scales)[0], w[0].astype(np.float64))


def test_power_of_two_rescale_shifts_only_the_scale():
    rng = np.random.default_rng(3)
    w = (rng.standard_normal((8, 64)) * 0.02).astype(np.float32)
    c0, s0 = oracle.mxfp4_quantize_rows(w)
    for m in (-5, 1, 9):
        c1, s1 = oracle.mxfp4_quantize_rows((w * np.float32(2.0 ** m)).astype(np.float32))
        np.testing.assert_array_equal(c1, c0)
        np.testing.assert_array_equal(s1.astype(int), s0.astype(int) + m)


def test_negative_value_rounding_to_zero_keeps_sign_bit():
    w = np.zeros((1, 32), np.float32)
    w[0, 0] = 4.0          # e = 0
    w[0, 1] = -0.2         # rounds to zero
    codes, scales = oracle.mxfp4_quantize_rows(w)
    assert int(scales[0, 0]) == 127
    assert int(codes[0, 0]) >> 4 == 8


def test_matrix_quantiser_blocks_run_along_contraction_axis():
    rng = np.random.default_rng(4)
    W = (rng.standard_normal((64, 5)) * 0.02).astype(np.float32)   # y = x . W, K=64, N=5
    codes, scales = oracle.mxfp4_quantize_matrix(W)
    assert codes.shape == (5, 32) and scales.shape == (5, 2)
    c2, s2 = oracle.mxfp4_quantize_rows(np.ascontiguousarray(W.T))
    np.testing.assert_array_equal(codes, c2)
    np.testing.assert_array_equal(scales, s2)


# ---------------------------------------------------------------- Swish

def test_swish_closed_forms():
    assert oracle.swish(0.0) == 0.0
    for z in (0.3, 1.0, 2.5, 7.0):
        # sigma(z) + sigma(-z) = 1  =>  Swish(z) - Swish(-z) = z
        assert abs(oracle.swish(z) - oracle.swish(-z) - z) < 1e-15
        assert abs(oracle.swish(z) - z / (1 + math.exp(-z))) < 1e-15
    assert abs(oracle.swish(40.0) - 40.0) < 1e-12
    assert abs(oracle.swish(-40.0)) < 1e-12
    # sigma(0) = 1/2  =>  d/dz Swish at 0 is 1/2
    h = 1e-6
    assert abs((oracle.swish(h) - oracle.swish(-h)) / (2 * h) - 0.5) < 1e-9


# ---------------------------------------------------------------- router

def test_router_topk_matches_bruteforce_and_weights_sum_to_one():
    rng = np.random.default_rng(5)
    for trial in range(20):
        T, d = int(rng.integers(1, 17)), int(rng.integers(1, 12))
        E = int(rng.integers(2, 9))
        k = int(rng.integers(1, E + 1))
        x = rng.standard_normal((T, d))
        wr = rng.standard_normal((E, d))
        bias = rng.standard_normal(E) if trial % 2 else None
        logits, idx, w, counts = oracle.router(x, wr, bias, k)
        ref_logits = x @ wr.T + (0 if bias is None else bias)
        np.testing.assert_allclose(logits, ref_logits, rtol=0, atol=1e-12)
        for t in range(T):
            # brute force: the k-subset with the largest score sum, listed by score desc
            best = max(itertools.combinations(range(E), k),
                       key=lambda S: sum(ref_logits[t, list(S)]))
            want = sorted(best, key=lambda e: (-ref_logits[t, e], e))
            assert list(idx[t]) == want
            assert abs(w[t].sum() - 1.0) <= 1e-15 * k
            assert np.all(np.diff(w[t]) <= 0)
        assert counts.sum() == T * k
        np.testing.assert_array_equal(counts, np.bincount(idx.ravel(), minlength=E))


def test_router_tie_goes_to_lower_index():
    x = np.ones((1, 2))
    wr = np.array([[1.0, 0.0], [0.5, 0.5], [0.0, 1.0], [0.0, 0.0]])   # logits 1,1,1,0
    _, idx, w, _ = oracle.router(x, wr, None, 2)
    assert list(idx[0]) == [0, 1]
    np.testing.assert_allclose(w[0], [0.5, 0.5], atol=0)


def test_softmax_readings_agree():
    """Top-k then softmax over the k logits == softmax over all E, restricted to the
    top-k and renormalised (the two readings of the router method)."""
    rng = np.random.default_rng(6)
    x = rng.standard_normal((32, 16))
    wr = rng.standard_normal((8, 16)) / 4
    logits, idx, w, _ = oracle.router(x, wr, None, 3)
    full = np.exp(logits - logits.max(axis=1, keepdims=True))
    full /= full.sum(axis=1, keepdims=True)
    for t in range(32):
        order = np.argsort(-full[t], kind="stable")[:3]
        assert list(order) == list(idx[t])
        sel = full[t, idx[t]]
        np.testing.assert_allclose(w[t], sel / sel.sum(), rtol=1e-13)


def test_router_bias_adds_per_expert():
    rng = np.random.default_rng(7)
    x = rng.standard_normal((4, 8))
    wr = rng.standard_normal((5, 8))
    b = rng.standard_normal(5)
    l0 = oracle.router_logits(x, wr, None)
    l1 = oracle.router_logits(x, wr, b)
    np.testing.assert_allclose(l1 - l0, np.broadcast_to(b, l0.shape), atol=1e-13)


# ---------------------------------------------------------------- experts / layer

def _identity_experts(d, E, a, b, c):
    q = oracle.QuantExperts(d, d, E)
    I = np.eye(d, dtype=np.float32)
    for e in range(E):
        q.set_expert(e, I * a[e], I * b[e], I * c[e])
    return q


def test_identity_experts_closed_form():
    """W_gate = a I, W_up = b I, W_down = c I (powers of two, exact in MXFP4):
    y_i = sum_j w_j c a b x_i^2 sigma(a x_i)."""
    d, E, k = 64, 4, 2
    a = [2.0 ** p for p in (-1, 0, 1, -2)]
    b = [2.0 ** p for p in (0, 1, -1, 2)]
    c = [2.0 ** p for p in (1, -1, 0, -3)]
    q = _identity_experts(d, E, a, b, c)
    # a one-hot row quantises to code 6 (value 4) at scale a/4
    assert int(q.g_scales[0, 5, 0]) == 127 + int(math.log2(a[0])) - 2
    rng = np.random.default_rng(8)
    x = rng.standard_normal((6, d))
    wr = rng.standard_normal((E, d)) / 8
    _, idx, w, _ = oracle.router(x, wr, None, k)
    y = oracle.moe_forward(x, q, idx, w)
    sig = lambda z: 1.0 / (1.0 + np.exp(-z))
    for t in range(6):
        ref = np.zeros(d)
        for j in range(k):
            e = idx[t, j]
            ref += w[t, j] * c[e] * a[e] * b[e] * x[t] ** 2 * sig(a[e] * x[t])
        np.testing.assert_allclose(y[t], ref, rtol=1e-13, atol=1e-15)


def test_all_experts_equal_is_routing_independent():
    d, E = 32, 3
    q = _identity_experts(d, E, [0.5] * E, [2.0] * E, [1.0] * E)
    rng = np.random.default_rng(9)
    x = rng.standard_normal((5, d))
    for k in (1, 2, 3):
        _, idx, w, _ = oracle.router(x, rng.standard_normal((E, d)), None, k)
        y = oracle.moe_forward(x, q, idx, w)
        ref = 0.5 * 2.0 * x ** 2 / (1 + np.exp(-0.5 * x))
        np.testing.assert_allclose(y, ref, rtol=1e-13)


def _random_layer(d=64, f=96, E=4, T=7, k=2, seed=10):
    rng = np.random.default_rng(seed)
    q = oracle.QuantExperts(d, f, E)
    dense = []
    for e in range(E):
        wg = (rng.standard_normal((d, f)) * 0.1).astype(np.float32)
        wu = (rng.standard_normal((d, f)) * 0.1).astype(np.float32)
        wd = (rng.standard_normal((f, d)) * 0.1).astype(np.float32)
        q.set_expert(e, wg, wu, wd)
        dense.append((wg, wu, wd))
    x = rng.standard_normal((T, d))
    wr = rng.standard_normal((E, d)) / 8
    return q, x, wr, k


def test_expert_matches_independent_dense_computation():
    """Oracle expert (per-element decode, loops) vs dequantised dense matrices and numpy
    matmul in the y = x . W orientation: catches a transposed operand or a swapped
    gate/up pair."""
    q, x, _, _ = _random_layer()
    for e in range(q.E):
        Wg = oracle.mxfp4_dequantize(q.g_codes[e], q.g_scales[e]).T   # [d, f]
        Wu = oracle.mxfp4_dequantize(q.u_codes[e], q.u_scales[e]).T
        Wd = oracle.mxfp4_dequantize(q.d_codes[e], q.d_scales[e]).T   # [f, d]
        g, u = x @ Wg, x @ Wu
        h = g / (1 + np.exp(-g)) * u
        ref = h @ Wd
        for t in range(x.shape[0]):
            out, hh = oracle.expert(x[t], q, e, want_h=True)
            np.testing.assert_allclose(hh, h[t], rtol=1e-12, atol=1e-14)
            np.testing.assert_allclose(out, ref[t], rtol=1e-12, atol=1e-14)


def test_gate_and_up_are_not_interchangeable():
    q, x, _, _ = _random_layer(seed=11)
    out = oracle.expert(x[0], q, 0)
    q.g_codes[0], q.u_codes[0] = q.u_codes[0].copy(), q.g_codes[0].copy()
    q.g_scales[0], q.u_scales[0] = q.u_scales[0].copy(), q.g_scales[0].copy()
    assert np.abs(oracle.expert(x[0], q, 0) - out).max() > 1e-6


def test_doubling_down_weights_doubles_output():
    q, x, wr, k = _random_layer(seed=12)
    _, idx, w, _ = oracle.router(x, wr, None, k)
    y1 = oracle.moe_forward(x, q, idx, w)
    q.d_scales += 1
    y2 = oracle.moe_forward(x, q, idx, w)
    np.testing.assert_array_equal(y2, 2 * y1)


def test_rows_are_independent_and_thread_count_free():
    q, x, wr, k = _random_layer(seed=13)
    _, idx, w, _ = oracle.router(x, wr, None, k)
    y = oracle.moe_forward(x, q, idx, w, nthreads=3)
    for t in range(x.shape[0]):
        yt = oracle.moe_forward(x[t:t + 1], q, idx[t:t + 1], w[t:t + 1], nthreads=1)
        np.testing.assert_array_equal(yt[0], y[t])
    sub = oracle.moe_forward(x, q, idx, w, tokens=[4, 1], nthreads=2)
    np.testing.assert_array_equal(sub, y[[4, 1]])


def test_layer_is_weighted_sum_of_selected_experts():
    q, x, wr, k = _random_layer(seed=14)
    _, idx, w, _ = oracle.router(x, wr, None, k)
    y = oracle.moe_forward(x, q, idx, w)
    for t in range(x.shape[0]):
        ref = sum(w[t, j] * oracle.expert(x[t], q, int(idx[t, j])) for j in range(k))
        np.testing.assert_allclose(y[t], ref, rtol=1e-14, atol=1e-16)


# ---------------------------------------------------------------- page figures

def test_swiglu_parameter_count_matches_page_example():
    fig = _figures()
    dim = int(fig["swiglu_example_dim"])
    q = oracle.QuantExperts(dim, dim, 1)
    n_params = 2 * (q.g_codes[0].size + q.u_codes[0].size + q.d_codes[0].size)
    assert n_params == 3 * dim * dim == int(fig["swiglu_example_params"])
    # the classic two-layer module of that example: hidden = 4 * dim
    assert 2 * dim * (4 * dim) == int(fig["ffn_example_params"])


def test_active_expert_fraction():
    fig = _figures()
    assert fig["experts_active"] / fig["experts_total"] == fig["active_fraction"]


def test_expert_weights_dominate_the_20b_footprint():
    """12.8 GB total with MXFP4 experts (17/32 B/param) and 2-byte other params, of
    20.9e9 params: the expert share comes out above 90 %, consistent with the pages."""
    total, size = 20.9e9, 12.8e9
    p_exp = (2 * total - size) / (2 - 17 / 32)
    assert 0.90 < p_exp / total < 1.0


# ---------------------------------------------------------------- RMSNorm and the residual (N3)
# Page "GPT-OSS vs Qwen3 : comparaison détaillée", Adoption de RMSNorm: the
# block input is divided by its root mean square (no mean, no variance).

def test_rmsnorm_hand_worked_cases():
    for line in _read_table("rmsnorm_cases.txt"):
        name, xs, gs, eps, want = [p.strip() for p in line.split("|")]
        x = np.array([[float(v) for v in xs.split()]])
        g = None if gs == "-" else np.array([float(v) for v in gs.split()])
        got = oracle.rmsnorm(x, g, float(eps))[0]
        np.testing.assert_allclose(got, [float(v) for v in want.split()], rtol=1e-15, atol=0, err_msg=name)


def test_rmsnorm_is_scale_invariant_and_unit_rms():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((6, 96))
    base = oracle.rmsnorm(x, None, 0.0)
    for m in (-3, 1, 7):
        # powers of two scale the mean square by 4^m exactly: the result is bit-identical
        np.testing.assert_array_equal(oracle.rmsnorm(x * 2.0 ** m, None, 0.0), base)
    np.testing.assert_allclose((base ** 2).mean(axis=1), 1.0, rtol=1e-13)
    # the gain multiplies feature by feature
    g = rng.standard_normal(96)
    np.testing.assert_allclose(oracle.rmsnorm(x, g, 0.0), base * g, rtol=1e-14)
    # eps sits inside the root, added to the mean square
    e = 0.25
    np.testing.assert_allclose(oracle.rmsnorm(x, None, e),
                               x / np.sqrt((x ** 2).mean(axis=1, keepdims=True) + e), rtol=1e-14)


def _tiny_block_setup(seed=11, d=64, E=4, k=2, T=12):
    rng = np.random.default_rng(seed)
    wr = rng.standard_normal((E, d)) / np.sqrt(d)
    x = rng.standard_normal((T, d)) * 3.0
    gamma = 1.0 + 0.1 * rng.standard_normal(d)
    return rng, wr, x, gamma


def test_block_residual_with_zero_down_projection_is_the_input():
    rng, wr, x, gamma = _tiny_block_setup()
    d, E = x.shape[1], wr.shape[0]
    q = oracle.QuantExperts(d, d, E)
    for e in range(E):
        q.set_expert(e, rng.standard_normal((d, d)).astype(np.float32) * 0.02,
                     rng.standard_normal((d, d)).astype(np.float32) * 0.02, np.zeros((d, d), np.float32))
    y, _, _, _ = oracle.block_forward(x, q, wr, None, 2, gamma, 1e-5, residual=True)
    np.testing.assert_array_equal(y, x)
    y0, _, _, _ = oracle.block_forward(x, q, wr, None, 2, gamma, 1e-5, residual=False)
    np.testing.assert_array_equal(y0, 0.0)


def test_block_routes_on_the_normalised_input():
    """With the pre-norm, routing depends on x only through RMSNorm(x): scaling
    a token by a power of two (eps = 0) leaves its experts and weights as they
    were, while the routing of the raw input changes."""
    rng, wr, x, gamma = _tiny_block_setup()
    d, E = x.shape[1], wr.shape[0]
    q = oracle.QuantExperts(d, d, E)
    for e in range(E):
        q.set_expert(e, *(rng.standard_normal(s).astype(np.float32) * 0.02 for s in ((d, d), (d, d), (d, d))))
    _, i1, w1, _ = oracle.block_forward(x, q, wr, None, 2, gamma, 0.0, residual=False)
    _, i2, w2, _ = oracle.block_forward(x * 8.0, q, wr, None, 2, gamma, 0.0, residual=False)
    np.testing.assert_array_equal(i1, i2)
    np.testing.assert_allclose(w1, w2, rtol=1e-12)
    _, _, wraw1, _ = oracle.router(x, wr, None, 2)
    _, _, wraw2, _ = oracle.router(x * 8.0, wr, None, 2)
    assert np.abs(wraw1 - wraw2).max() > 1e-3


def test_block_identity_experts_closed_form_with_norm_and_residual():
    """W_gate = a I, W_up = b I, W_down = c I (powers of two, exact in MXFP4):
    y = x + sum_j w_j c a b h^2 sigma(a h) with h = RMSNorm(x) = x / rms * gamma."""
    rng, wr, x, gamma = _tiny_block_setup(d=64, E=4, k=2)
    d, E, k = 64, 4, 2
    a, b, c = [0.5, 1.0, 2.0, 0.25], [1.0, 2.0, 0.5, 4.0], [2.0, 0.5, 1.0, 0.125]
    q = oracle.QuantExperts(d, d, E)
    I = np.eye(d, dtype=np.float32)
    for e in range(E):
        q.set_expert(e, I * a[e], I * b[e], I * c[e])
    eps = 1e-5
    y, idx, w, _ = oracle.block_forward(x, q, wr, None, k, gamma, eps, residual=True)
    h = x / np.sqrt((x ** 2).mean(axis=1, keepdims=True) + eps) * gamma
    ref = x.copy()
    for j in range(k):
        e = idx[:, j]
        A, B, C = (np.array(v)[e][:, None] for v in (a, b, c))
        ref += w[:, j:j + 1] * C * A * B * h ** 2 / (1 + np.exp(-A * h))
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)
