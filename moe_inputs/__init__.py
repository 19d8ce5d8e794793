"""Seeded synthetic inputs for the MoE-MXFP4 feed-forward layer.

This module is shared by the tests, the benchmark and the oracle timing.  It
draws tensors and rounds them to the activation dtype; it holds none of the
layer's arithmetic (no router, no quantiser, no expert).  The one place that
needs router logits, the selection-margin filter, takes them from a callable
supplied by the caller.

Generator: numpy's Philox4x32-10 counter-based bit generator (Salmon et al.,
SC'11), keyed by (seed, stream, sub-stream ids), so each tensor -- and each
expert's weight matrices -- can be drawn on its own without drawing the rest.
Normal variates come from ``Generator.standard_normal`` in float32.

Workloads (shapes, distributions) follow the layer described on the pages
"GPT-OSS-20B : Architecture MoE & Résumé du Model Card" (§2.1 Qu'est-ce qu'un
modèle MoE ?, §3.1 Le Routeur, §3.2 Les Experts) with the sizes of the
gpt-oss-20b / 120b MoE blocks:

  tiny     T=16,    d_model=64,   d_ff=128,  E=8,   k=2, fp32 activations
  dec1/8/64  T=1/8/64, d_model=d_ff=2880, E=32, k=4, bf16 activations
  pre4096  T=4096,  2880/2880, E=32, k=4, bf16
  e128     T=8192,  2880/2880, E=128, k=4, bf16
  zipf     T=16384, 2880/2880, E=32, k=4, bf16, router bias so that expert
           popularity follows Zipf s=1.2

x ~ N(0,1); router weight ~ N(0, 1/d_model); expert weights ~ N(0, 0.02^2)
in fp32 (quantised to MXFP4 by the code under test and by the oracle).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Callable, Optional

import numpy as np

# Sub-stream ids, one per tensor.
STREAM_X = 1
STREAM_WR = 2
STREAM_BIAS = 3
STREAM_WG = 4
STREAM_WU = 5
STREAM_WD = 6
STREAM_GAMMA = 7

# RMSNorm epsilon of the optional pre-norm (the pages give none; a small
# positive constant keeps an all-zero token finite)
NORM_EPS = 1e-5

WEIGHT_STD = 0.02
MARGIN = 1e-4


@dataclasses.dataclass(frozen=True)
class MoeConfig:
    name: str
    T: int
    d_model: int
    d_ff: int
    n_experts: int
    top_k: int
    act_dtype: str  # "f32" or "bf16"
    zipf_s: Optional[float] = None
    seed: int = 0

    def with_T(self, T: int) -> "MoeConfig":
        return dataclasses.replace(self, T=T)


CONFIGS = {
    "tiny": MoeConfig("tiny", 16, 64, 128, 8, 2, "f32"),
    "dec1": MoeConfig("dec1", 1, 2880, 2880, 32, 4, "bf16"),
    "dec8": MoeConfig("dec8", 8, 2880, 2880, 32, 4, "bf16"),
    "dec64": MoeConfig("dec64", 64, 2880, 2880, 32, 4, "bf16"),
    "pre4096": MoeConfig("pre4096", 4096, 2880, 2880, 32, 4, "bf16"),
    "e128": MoeConfig("e128", 8192, 2880, 2880, 128, 4, "bf16"),
    "zipf": MoeConfig("zipf", 16384, 2880, 2880, 32, 4, "bf16", zipf_s=1.2),
}


def _rng(seed: int, stream: int, a: int = 0, b: int = 0) -> np.random.Generator:
    """Philox keyed by 4 x 32-bit words (seed, stream, a, b)."""
    key = ((seed & 0xFFFFFFFF) | ((stream & 0xFFFFFFFF) << 32)
           | ((a & 0xFFFFFFFF) << 64) | ((b & 0xFFFFFFFF) << 96))
    return np.random.Generator(np.random.Philox(key=key))


def bf16_round(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); returned as float32."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return r.astype(np.uint32).view(np.float32).reshape(a.shape)


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """Upper 16 bits of float32 values that are already bfloat16-representable."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    return (a.view(np.uint32) >> 16).astype(np.uint16)


def _act(cfg: MoeConfig, a: np.ndarray) -> np.ndarray:
    return bf16_round(a) if cfg.act_dtype == "bf16" else np.ascontiguousarray(a, np.float32)


def draw_x(cfg: MoeConfig, T: Optional[int] = None) -> np.ndarray:
    """Activations [T, d_model], N(0,1), rounded to the activation dtype (float32 container)."""
    T = cfg.T if T is None else T
    x = _rng(cfg.seed, STREAM_X).standard_normal((T, cfg.d_model), dtype=np.float32)
    return _act(cfg, x)


def redraw_x_row(cfg: MoeConfig, t: int, attempt: int) -> np.ndarray:
    """Replacement draw for token t (attempt >= 1), from its own sub-stream."""
    r = _rng(cfg.seed, STREAM_X, attempt, t).standard_normal(cfg.d_model, dtype=np.float32)
    return _act(cfg, r)


def draw_router(cfg: MoeConfig) -> np.ndarray:
    """Router weight [E, d_model], N(0, 1/d_model), rounded to the activation dtype."""
    w = _rng(cfg.seed, STREAM_WR).standard_normal((cfg.n_experts, cfg.d_model), dtype=np.float32)
    w *= np.float32(1.0 / math.sqrt(cfg.d_model))
    return _act(cfg, w)


def draw_bias(cfg: MoeConfig) -> Optional[np.ndarray]:
    """Per-expert router bias [E] (float32) or None.

    Zipf configs: b_e = ln p_e with p_e = r_e^-s / sum_r r^-s and r_e a seeded
    permutation of the ranks 1..E.  With logits near N(0,1) this gives roughly
    Zipf-shaped expert popularity; the achieved histogram is measured, not set.
    """
    if cfg.zipf_s is None:
        return None
    E = cfg.n_experts
    ranks = _rng(cfg.seed, STREAM_BIAS).permutation(E) + 1
    p = ranks.astype(np.float64) ** (-cfg.zipf_s)
    p /= p.sum()
    return np.log(p).astype(np.float32)


def draw_gamma(cfg: MoeConfig) -> np.ndarray:
    """Gain of the optional RMSNorm pre-norm [d_model], 1 + 0.1 N(0,1), float32."""
    g = _rng(cfg.seed, STREAM_GAMMA).standard_normal(cfg.d_model, dtype=np.float32)
    return (np.float32(1.0) + np.float32(0.1) * g).astype(np.float32)


def draw_expert(cfg: MoeConfig, e: int):
    """fp32 weights of expert e: (W_gate [d_model,d_ff], W_up [d_model,d_ff], W_down [d_ff,d_model]).

    Orientation: y = x . W, so the contraction dimension is the first axis.
    """
    d, f = cfg.d_model, cfg.d_ff
    s = np.float32(WEIGHT_STD)
    wg = _rng(cfg.seed, STREAM_WG, e).standard_normal((d, f), dtype=np.float32) * s
    wu = _rng(cfg.seed, STREAM_WU, e).standard_normal((d, f), dtype=np.float32) * s
    wd = _rng(cfg.seed, STREAM_WD, e).standard_normal((f, d), dtype=np.float32) * s
    return wg, wu, wd


def margin_filter(cfg: MoeConfig, x: np.ndarray,
                  logits_fn: Callable[[np.ndarray], np.ndarray],
                  margin: float = MARGIN, max_rounds: int = 64):
    """Redraw tokens whose top-(k+1) sorted logits have an adjacent gap below `margin`.

    `logits_fn(x_rows) -> [rows, E]` is supplied by the caller (the oracle's
    router).  Failing tokens are redrawn from their own sub-stream until none
    fails.  Returns (x, number_of_redraws).
    """
    x = np.array(x, dtype=np.float32, copy=True)
    k = cfg.top_k
    redraws = 0
    bad = np.arange(x.shape[0])
    attempt = 0
    for _ in range(max_rounds):
        if bad.size == 0:
            return x, redraws
        lg = np.asarray(logits_fn(x[bad]), dtype=np.float64)
        srt = -np.sort(-lg, axis=1)[:, : min(k + 1, lg.shape[1])]
        gaps = srt[:, :-1] - srt[:, 1:]
        fail = bad[(gaps < margin).any(axis=1)] if gaps.shape[1] else bad[:0]
        if fail.size == 0:
            return x, redraws
        attempt += 1
        for t in fail:
            x[t] = redraw_x_row(cfg, int(t), attempt)
        redraws += int(fail.size)
        bad = fail
    raise RuntimeError("margin filter did not converge")
