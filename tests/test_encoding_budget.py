"""Error budget of the activation encoding the expert GEMMs use (CPU only).

The block-scaled MMA multiplies MXFP4 by MXFP4, so the activations (x for
gate/up, H for down) are written as sums of MXFP4 terms: each term encodes the
residual of the previous ones in blocks of 32 along K, with the smallest scale
2^e such that max|v| <= 6 * 2^e and round-to-nearest, ties to the even code.
This file emulates that encoding in numpy (written from the definition above,
not from the kernels) on a small layer with the oracle's dequantised weights
and checks the design budget: one term misses the layer tolerance of
2e-2 * max|y| by far, three terms meet it with margin.

The alternative format (two MXFP8 terms, E4M3 elements, scale rule max|v| <=
448 * 2^e) is emulated the same way: one E4M3 term misses the tolerance, two
meet it, with an error below that of three MXFP4 terms.
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


# E4M3 magnitudes by code 0..126 (code 127 is NaN): subnormal m/8 * 2^-6 for
# exponent field 0, else (1 + m/8) * 2^(E - 7); the largest is 448.
E4M3 = np.array([(c & 7) / 8.0 * 2.0 ** -6 if c >> 3 == 0 else (1 + (c & 7) / 8.0) * 2.0 ** ((c >> 3) - 7)
                 for c in range(127)])


def e4m3_round(a):
    """Nearest E4M3 magnitude of 0 <= a <= 448, ties to the even code (even mantissa)."""
    i = np.clip(np.searchsorted(E4M3, a), 1, 126)
    lo, hi = E4M3[i - 1], E4M3[i]
    pick_hi = (a - lo > hi - a) | ((a - lo == hi - a) & ((i & 1) == 0))
    return np.where(pick_hi, hi, lo)


def scale_exp8(amax):
    """Smallest e with amax <= 448 * 2^e (amax > 0)."""
    e = np.ceil(np.log2(amax / 448.0))
    return np.where(amax <= 448.0 * 2.0 ** (e - 1), e - 1, e)


def encode_terms(v, terms, fmt="mxfp4"):
    """Sum of `terms` MX terms (MXFP4, or MXFP8 E4M3 with fmt="mxfp8")
    approximating v [rows, K] (K % 32 == 0), blockwise along K."""
    R, K = v.shape
    r = v.reshape(R, K // 32, 32).astype(np.float64)
    acc = np.zeros_like(r)
    rnd, sexp = (e2m1_round, scale_exp) if fmt == "mxfp4" else (e4m3_round, scale_exp8)
    for _ in range(terms):
        amax = np.abs(r).max(axis=-1, keepdims=True)
        safe = np.where(amax > 0, amax, 1.0)
        s = 2.0 ** sexp(safe)
        q = np.where(amax > 0, np.sign(r) * rnd(np.abs(r) / s) * s, 0.0)
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


def test_e4m3_grid_and_rounding():
    """The E4M3 grid: 2^-9 the smallest subnormal, 2^-6 the smallest normal, 448
    the largest; spacing 2^(E-10) in binade E; ties go to the even mantissa."""
    assert E4M3[1] == 2.0 ** -9 and E4M3[8] == 2.0 ** -6 and E4M3[-1] == 448.0
    assert (np.diff(E4M3) > 0).all()
    np.testing.assert_array_equal(e4m3_round(E4M3), E4M3)
    # 1 + 1/16 lies between 1 (mantissa 0) and 1.125 (mantissa 1): even wins
    assert e4m3_round(np.array([1.0625]))[0] == 1.0
    assert e4m3_round(np.array([1.1875]))[0] == 1.25     # between 1.125 (odd) and 1.25 (even)
    assert e4m3_round(np.array([1.07]))[0] == 1.125
    np.testing.assert_array_equal(scale_exp8(np.array([448.0, 449.0, 224.0, 1.0])), [0, 1, -1, -8])


def test_one_mxfp8_term_is_exact_on_the_grid():
    rng = np.random.default_rng(3)
    codes = rng.integers(1, 127, size=(6, 4, 32))
    signs = rng.choice([-1.0, 1.0], size=(6, 4, 32))
    scales = 2.0 ** rng.integers(-8, 8, size=(6, 4, 1))
    v = (signs * E4M3[codes] * scales).reshape(6, 128)
    # the scale 2^e chosen for the block only shifts its codes up by a power of
    # two within the grid, so one term reproduces the block exactly
    np.testing.assert_array_equal(encode_terms(v, 1, "mxfp8"), v)


def _budget_layer():
    cfg = mi.MoeConfig("budget", 24, 256, 256, 4, 2, "bf16")
    x = mi.draw_x(cfg).astype(np.float64)
    wr, bias = mi.draw_router(cfg), mi.draw_bias(cfg)
    _, idx, w, _ = oracle.router(x.astype(np.float32), wr, bias, cfg.top_k)
    W = {}
    for e in range(cfg.n_experts):
        W[e] = [oracle.mxfp4_dequantize(*oracle.mxfp4_quantize_matrix(m)).T for m in mi.draw_expert(cfg, e)]

    def layer(terms, fmt="mxfp4"):
        y = np.zeros((cfg.T, cfg.d_model))
        for e in range(cfg.n_experts):
            rows = np.argwhere(idx == e)
            if len(rows) == 0:
                continue
            t, j = rows[:, 0], rows[:, 1]
            xe = x[t] if terms is None else encode_terms(x[t], terms, fmt)
            g, u = xe @ W[e][0], xe @ W[e][1]
            h = g / (1.0 + np.exp(-g)) * u
            h = h if terms is None else encode_terms(h, terms, fmt)
            y[t] += w[t, j][:, None] * (h @ W[e][2])
        return y

    ref = layer(None)
    return layer, ref, np.abs(ref).max()


def test_three_terms_meet_the_layer_tolerance():
    layer, ref, scale = _budget_layer()
    err1 = np.abs(layer(1) - ref).max() / scale
    err3 = np.abs(layer(3) - ref).max() / scale
    assert err1 > 2e-2, err1      # one MXFP4 term alone misses the layer tolerance
    assert err3 < 1e-2, err3      # three terms pass it with margin


def test_two_mxfp8_terms_meet_the_layer_tolerance():
    layer, ref, scale = _budget_layer()
    err1 = np.abs(layer(1, "mxfp8") - ref).max() / scale
    err2 = np.abs(layer(2, "mxfp8") - ref).max() / scale
    err3 = np.abs(layer(3) - ref).max() / scale
    assert err1 > 2e-2, err1      # one E4M3 term alone misses the layer tolerance
    assert err2 < 1e-2, err2      # two pass it with margin
    assert err2 < err3, (err2, err3)
