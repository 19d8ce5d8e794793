"""Shared set-up for the GPU parity tests: seeded inputs, the CUDA layer through
the C ABI, and the oracle's own quantisation of the same fp32 weights."""
from __future__ import annotations

import os
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

import moe_inputs as mi
import oracle

# tolerance on the layer output (bf16 activations, fp32 accumulation): max|gpu - ref| <= 2e-2 * max|ref|
Y_REL_TOL = 2e-2
# routing weights: |w_gpu - w_ref| <= 1e-6 (fp32 scores and softmax vs double)
W_ABS_TOL = 1e-6


def torch_mod():
    import torch
    return torch


def act_tensor(cfg, a: np.ndarray, device="cuda"):
    """float32 numpy holding act-dtype values -> torch tensor of the act dtype (bit-exact)."""
    torch = torch_mod()
    if cfg.act_dtype == "bf16":
        bits = mi.bf16_bits(a).view(np.int16)
        return torch.from_numpy(bits.copy()).to(device).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(device)


def to_f64(t) -> np.ndarray:
    torch = torch_mod()
    return t.detach().to(torch.float64).cpu().numpy()


class OracleExperts:
    """Oracle-quantised experts, filled lazily (only experts a test needs)."""

    def __init__(self, cfg: mi.MoeConfig):
        self.cfg = cfg
        self.q = oracle.QuantExperts(cfg.d_model, cfg.d_ff, cfg.n_experts)
        self.done = set()
        self.lock = threading.Lock()

    def _one(self, e):
        wg, wu, wd = mi.draw_expert(self.cfg, e)
        self.q.set_expert(e, wg, wu, wd)
        return e

    def ensure(self, experts):
        todo = sorted(set(int(e) for e in experts) - self.done)
        if not todo:
            return self.q
        with ThreadPoolExecutor(max_workers=min(len(todo), os.cpu_count() or 1)) as ex:
            for e in ex.map(self._one, todo):
                self.done.add(e)
        return self.q


class GpuLayer:
    """The CUDA layer for one weight set (router + experts drawn from cfg's seed)."""

    def __init__(self, cfg: mi.MoeConfig, max_tokens: int, flags: int = 0, wait_timeout_ms: int = 0,
                 quantize: bool = True, lib=None):
        import mxfp4_expert_gemm_router_b200 as mx
        torch = torch_mod()
        self.cfg = cfg
        self.layer = mx.MoeMxfp4(cfg.d_model, cfg.d_ff, cfg.n_experts, cfg.top_k, max_tokens, cfg.act_dtype,
                                 flags, wait_timeout_ms, lib=lib)
        self.wr = mi.draw_router(cfg)
        self.bias = mi.draw_bias(cfg)
        if quantize:
            for e in range(cfg.n_experts):
                wg, wu, wd = mi.draw_expert(cfg, e)
                self.layer.quantize_expert(e, torch.from_numpy(wg).cuda(), torch.from_numpy(wu).cuda(),
                                           torch.from_numpy(wd).cuda())
            self.set_router(self.wr, self.bias)
            torch.cuda.synchronize()

    def set_router(self, wr, bias):
        torch = torch_mod()
        self.wr, self.bias = wr, bias
        self._wr_t = act_tensor(self.cfg, wr)
        self._b_t = None if bias is None else torch.from_numpy(bias.astype(np.float32)).cuda()
        self.layer.set_router(self._wr_t, self._b_t)

    def forward(self, x_np: np.ndarray):
        torch = torch_mod()
        cfg = self.cfg
        T = x_np.shape[0]
        x = act_tensor(cfg, x_np)
        dt = torch.bfloat16 if cfg.act_dtype == "bf16" else torch.float32
        y = torch.empty((T, cfg.d_model), dtype=dt, device="cuda")
        idx = torch.empty((T, cfg.top_k), dtype=torch.int32, device="cuda")
        w = torch.empty((T, cfg.top_k), dtype=torch.float32, device="cuda")
        counts = torch.empty((cfg.n_experts,), dtype=torch.int32, device="cuda")
        self.layer.forward(x, y, idx, w, counts)
        torch.cuda.synchronize()
        assert self.layer.status() == 0, "device status not OK"
        return to_f64(y), idx.cpu().numpy(), w.cpu().numpy().astype(np.float64), counts.cpu().numpy()


def filtered_x(cfg: mi.MoeConfig, wr, bias, T=None):
    x = mi.draw_x(cfg, T)
    x, _ = mi.margin_filter(cfg, x, lambda rows: oracle.router_logits(rows, wr, bias))
    return x


def sample_tokens(idx: np.ndarray, counts_ref: np.ndarray, n: int, seed: int = 0):
    """Seeded sample of tokens plus the tokens routed to the most and least loaded experts."""
    T = idx.shape[0]
    if T <= n:
        return np.arange(T)
    rng = np.random.default_rng(seed)
    picks = set(rng.choice(T, size=n, replace=False).tolist())
    loaded = np.nonzero(counts_ref)[0]
    for e in (int(loaded[np.argmax(counts_ref[loaded])]), int(loaded[np.argmin(counts_ref[loaded])])):
        rows = np.nonzero((idx == e).any(axis=1))[0]
        picks.update(rows[:2].tolist())
    return np.array(sorted(picks))


def library_token_tile(T: int, k: int, E: int) -> int:
    """Token rows per expert-GEMM tile as the library picks them by default:
    about three times the mean rows per expert, rounded up to 16, within
    [16, 128].  Used only to choose which rows to check (tile boundaries)."""
    per_expert = -(-T * k // E)
    want = min(T, max(1, 3 * per_expert))
    return max(16, min(128, -(-want // 16) * 16))


def tile_boundary_tokens(idx: np.ndarray, counts_ref: np.ndarray, bn: int, max_full_experts=None, seed=0):
    """Tokens whose grouped rows lie in the tiles most likely to go wrong:
    every row of the first and the last token tile of the most-loaded expert,
    and every row of the last (ragged) tile of every expert.  The rows of an
    expert are its tokens in ascending order (a token picks an expert at most
    once), so tile m of expert e holds its tokens [m*bn, (m+1)*bn).  With
    max_full_experts set, only that many seeded experts (plus the most- and
    least-loaded) have their whole last tile checked; the others contribute
    that tile's first and last rows."""
    E = counts_ref.shape[0]
    picks = set()
    loaded = np.nonzero(counts_ref)[0]
    if loaded.size == 0:
        return np.array([], np.int64)
    most = int(loaded[np.argmax(counts_ref[loaded])])
    least = int(loaded[np.argmin(counts_ref[loaded])])
    full = set(range(E))
    if max_full_experts is not None and max_full_experts < loaded.size:
        rng = np.random.default_rng(seed)
        full = set(rng.choice(loaded, size=max_full_experts, replace=False).tolist()) | {most, least}
    for e in loaded.tolist():
        toks = np.nonzero((idx == e).any(axis=1))[0]
        n = toks.size
        last0 = ((n - 1) // bn) * bn
        last = toks[last0:]
        if e in full:
            picks.update(last.tolist())
        else:
            picks.update([int(last[0]), int(last[-1])])
        if e == most:
            picks.update(toks[:bn].tolist())
    return np.array(sorted(picks), np.int64)


def check_layer(cfg, x, wr, bias, y, idx, w, counts, ox: OracleExperts, n_sample=16, extra_tokens=None):
    """Router bit-exact over all tokens; layer output vs the oracle on a token
    sample (plus `extra_tokens`, e.g. tile-boundary rows)."""
    _, idx_ref, w_ref, counts_ref = oracle.router(x, wr, bias, cfg.top_k)
    np.testing.assert_array_equal(idx, idx_ref)
    np.testing.assert_array_equal(counts, counts_ref)
    w_err = np.abs(w - w_ref).max()
    assert w_err <= W_ABS_TOL, ("routing weight error", w_err)
    tok = sample_tokens(idx_ref, counts_ref, n_sample)
    if extra_tokens is not None and len(extra_tokens):
        tok = np.union1d(tok, np.asarray(extra_tokens, np.int64))
    q = ox.ensure(np.unique(idx_ref[tok]))
    y_ref = oracle.moe_forward(x, q, idx_ref, w_ref, tokens=tok)
    err = np.abs(y[tok] - y_ref).max()
    scale = np.abs(y_ref).max()
    assert err <= Y_REL_TOL * scale, (err, scale, err / scale)
    return err / scale


def filtered_x_norm(cfg: mi.MoeConfig, wr, bias, gamma, eps, T=None):
    """x drawn and margin-filtered on the scores of RMSNorm(x) (what the router sees)."""
    x = mi.draw_x(cfg, T)
    x, _ = mi.margin_filter(cfg, x, lambda rows: oracle.router_logits(oracle.rmsnorm(rows, gamma, eps), wr, bias))
    return x


def check_block(cfg, x, wr, bias, gamma, eps, residual, y, idx, w, counts, ox: OracleExperts, n_sample=16,
                extra_tokens=None):
    """The block with its adjacent steps: routing of RMSNorm(x) bit-exact over all
    tokens, output (with the residual) on a token sample vs the oracle."""
    h = oracle.rmsnorm(x, gamma, eps) if gamma is not None else np.asarray(x, np.float64)
    _, idx_ref, w_ref, counts_ref = oracle.router(h, wr, bias, cfg.top_k)
    np.testing.assert_array_equal(idx, idx_ref)
    np.testing.assert_array_equal(counts, counts_ref)
    w_err = np.abs(w - w_ref).max()
    assert w_err <= W_ABS_TOL, ("routing weight error", w_err)
    tok = sample_tokens(idx_ref, counts_ref, n_sample)
    if extra_tokens is not None and len(extra_tokens):
        tok = np.union1d(tok, np.asarray(extra_tokens, np.int64))
    q = ox.ensure(np.unique(idx_ref[tok]))
    y_ref, _, _, _ = oracle.block_forward(x, q, wr, bias, cfg.top_k, gamma, eps, residual, tokens=tok)
    err = np.abs(y[tok] - y_ref).max()
    # with the residual the bar applies to the MoE part (y - x): the residual is exact
    scale = np.abs(y_ref - (np.asarray(x, np.float64)[tok] if residual else 0.0)).max()
    assert err <= Y_REL_TOL * scale, (err, scale, err / scale)
    return err / scale
