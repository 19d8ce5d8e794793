"""Error budget of the activation encoding the expert GEMMs use (CPU only).

The block-scaled MMA multiplies MXFP4 by MXFP4, so the activations (x for
gate/up, H for down) are written as sums of MXFP4 terms: each term encodes the
residual of the previous ones in blocks of 32 along K, with the smallest scale
2^e such that max|v| <= 6 * 2^e and round-to-nearest, ties to the even code.
This file emulates that encoding in numpy (written from the definition above,
not from the kernels) on a small layer with the oracle's dequantised weights
and checks the design budget: one term misses the layer tolerance of
2e-2 * max|y| by far, three terms meet it with margin.
"""
import numpy as np

import moe_inputs as mi
import oracle

GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def e2m1_round(a):
    """Nearest E2M1 magnitude of a >= 0, ties to the even code."""
    d = np.abs(a[..., None] - GRID)
    d = d + (np.arange(8) & 1) * 1e-12          # at an exact midpoint the even code wins
    return GRID[np.argmin(d, axis=-1)]


def scale_exp(amax):
    """Smallest e with amax <= 6 * 2^e (amax > 0)."""
    e = np.ceil(np.log2(amax / 6.0))
    return np.where(amax <= 6.0 * 2.0 ** (e - 1), e - 1, e)   # guard the log's rounding


def encode_terms(v, terms):
    """Sum of `terms` MXFP4 terms approximating v [rows, K] (K % 32 == 0), blockwise along K."""
    R, K = v.shape
    r = v.reshape(R, K // 32, 32).astype(np.float64)
    acc = np.zeros_like(r)
    for _ in range(terms):
        amax = np.abs(r).max(axis=-1, keepdims=True)
        safe = np.where(amax > 0, amax, 1.0)
        s = 2.0 ** scale_exp(safe)
        q = np.where(amax > 0, np.sign(r) * e2m1_round(np.abs(r) / s) * s, 0.0)
        acc += q
        r = r - q
    return acc.reshape(R, K)


def test_scale_rule_values():
    amax = np.array([6.0, 6.0001, 4.0, 3.0, 3.01, 0.75, 1e-3])
    e = scale_exp(amax)
    assert (amax <= 6.0 * 2.0 ** e).all()
    assert (amax > 6.0 * 2.0 ** (e - 1)).all()          # the smallest such power of two
    assert e[0] == 0 and e[1] == 1 and e[2] == 0 and e[3] == -1 and e[4] == 0


def test_one_term_is_exact_on_the_grid():
    """A block of E2M1 values times one power of two is exact in one term, whatever
    its largest element: the chosen scale only rescales within the grid."""
    rng = np.random.default_rng(1)
    codes = rng.integers(1, 8, size=(6, 4, 32))
    signs = rng.choice([-1.0, 1.0], size=(6, 4, 32))
    scales = 2.0 ** rng.integers(-8, 8, size=(6, 4, 1))
    v = (signs * GRID[codes] * scales).reshape(6, 128)
    np.testing.assert_array_equal(encode_terms(v, 1), v)


def test_each_term_shrinks_the_residual():
    rng = np.random.default_rng(2)
    v = rng.standard_normal((16, 256))
    errs = [np.abs(encode_terms(v, t) - v).max() for t in (1, 2, 3)]
    assert errs[0] > errs[1] > errs[2]
    assert errs[2] < 1e-2 * np.abs(v).max()


def test_three_terms_meet_the_layer_tolerance():
    cfg = mi.MoeConfig("budget", 24, 256, 256, 4, 2, "bf16")
    x = mi.draw_x(cfg).astype(np.float64)
    wr, bias = mi.draw_router(cfg), mi.draw_bias(cfg)
    _, idx, w, _ = oracle.router(x.astype(np.float32), wr, bias, cfg.top_k)
    W = {}
    for e in range(cfg.n_experts):
        W[e] = [oracle.mxfp4_dequantize(*oracle.mxfp4_quantize_matrix(m)).T for m in mi.draw_expert(cfg, e)]

    def layer(terms):
        y = np.zeros((cfg.T, cfg.d_model))
        for e in range(cfg.n_experts):
            rows = np.argwhere(idx == e)
            if len(rows) == 0:
                continue
            t, j = rows[:, 0], rows[:, 1]
            xe = x[t] if terms is None else encode_terms(x[t], terms)
            g, u = xe @ W[e][0], xe @ W[e][1]
            h = g / (1.0 + np.exp(-g)) * u
            h = h if terms is None else encode_terms(h, terms)
            y[t] += w[t, j][:, None] * (h @ W[e][2])
        return y

    ref = layer(None)
    scale = np.abs(ref).max()
    err1 = np.abs(layer(1) - ref).max() / scale
    err3 = np.abs(layer(3) - ref).max() / scale
    assert err1 > 2e-2, err1      # one MXFP4 term alone misses the layer tolerance
    assert err3 < 1e-2, err3      # three terms pass it with margin
