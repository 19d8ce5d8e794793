"""CPU oracle for the MoE feed-forward layer with MXFP4 experts (ctypes wrapper).

TEST INFRASTRUCTURE ONLY.  Only tests/, the smoke check and the benchmark's
CPU-baseline leg import this package.  It shares nothing with the CUDA
library: its arithmetic lives in oracle_moe.c (double precision), built with
gcc by oracle/build.py.

Sources (page "GPT-OSS-20B : Architecture MoE & Résumé du Model Card"):
§3.1 Le Routeur, §3.2 Les Experts, §2.1 (weighted aggregation), §4
Quantification MXFP4; page "GPT-OSS vs Qwen3 : comparaison détaillée",
Adoption de RMSNorm (the optional pre-norm of the block).  Parity pins for every function are in
tests/test_oracle_pins.py.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.POINTER
        d, i64, i32, u32 = ctypes.c_double, ctypes.c_int64, ctypes.c_int32, ctypes.c_uint32
        vp = ctypes.c_void_p
        L.oracle_e2m1_decode.argtypes = [u32]
        L.oracle_e2m1_decode.restype = d
        L.oracle_e8m0_decode.argtypes = [u32]
        L.oracle_e8m0_decode.restype = d
        L.oracle_swish.argtypes = [d]
        L.oracle_swish.restype = d
        L.oracle_mxfp4_quantize.argtypes = [vp, i64, i64, i64, i64, vp, vp]
        L.oracle_mxfp4_dequantize.argtypes = [vp, vp, i64, i64, i64, vp]
        L.oracle_router.argtypes = [vp, i64, i64, vp, i64, vp, i32, vp, vp, vp, vp]
        L.oracle_expert.argtypes = [vp, i64, i64, vp, vp, vp, vp, vp, vp, vp, vp]
        L.oracle_moe_forward.argtypes = [vp, i64, i64, i64, i32, vp, vp,
                                         vp, vp, vp, vp, vp, vp, vp, i64, vp, i32]
        L.oracle_rmsnorm.argtypes = [vp, i64, i64, vp, d, vp]
        _lib = L
    return _lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def e2m1_decode(code: int) -> float:
    return lib().oracle_e2m1_decode(int(code))


def e8m0_decode(s: int) -> float:
    return lib().oracle_e8m0_decode(int(s))


def swish(z: float) -> float:
    return lib().oracle_swish(float(z))


def mxfp4_quantize_rows(w_rows: np.ndarray):
    """Quantise rows of a [N, K] float32 array along K.  Returns (codes [N,K/2], scales [N,K/32])."""
    w = _c(w_rows, np.float32)
    N, K = w.shape
    assert K % 32 == 0
    codes = np.zeros((N, K // 2), np.uint8)
    scales = np.zeros((N, K // 32), np.uint8)
    lib().oracle_mxfp4_quantize(_ptr(w), N, K, K, 1, _ptr(codes), _ptr(scales))
    return codes, scales


def mxfp4_quantize_matrix(W: np.ndarray):
    """Quantise a weight matrix applied as y = x . W (W: [K, N], float32).

    Blocks run along the contraction axis K.  Returns canonical
    (codes [N, K/2], scales [N, K/32])."""
    W = np.asarray(W, dtype=np.float32)
    K, N = W.shape
    assert K % 32 == 0
    return mxfp4_quantize_rows(np.ascontiguousarray(W.T))


def mxfp4_dequantize(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    codes = _c(codes, np.uint8)
    scales = _c(scales, np.uint8)
    N, K2 = codes.shape
    out = np.zeros((N, K2 * 2), np.float64)
    lib().oracle_mxfp4_dequantize(_ptr(codes), _ptr(scales), K2 * 2, 0, N, _ptr(out))
    return out


def router(x: np.ndarray, wr: np.ndarray, bias: Optional[np.ndarray], k: int):
    """Returns (logits [T,E] f64, idx [T,k] i32, w [T,k] f64, counts [E] i64)."""
    x = _c(x, np.float64)
    wr = _c(wr, np.float64)
    T, d = x.shape
    E = wr.shape[0]
    b = None if bias is None else _c(bias, np.float64)
    logits = np.zeros((T, E), np.float64)
    idx = np.zeros((T, k), np.int32)
    w = np.zeros((T, k), np.float64)
    counts = np.zeros(E, np.int64)
    lib().oracle_router(_ptr(x), T, d, _ptr(wr), E, _ptr(b), k,
                        _ptr(logits), _ptr(idx), _ptr(w), _ptr(counts))
    return logits, idx, w, counts


def router_logits(x: np.ndarray, wr: np.ndarray, bias: Optional[np.ndarray]) -> np.ndarray:
    x = _c(x, np.float64)
    wr = _c(wr, np.float64)
    T, d = x.shape
    E = wr.shape[0]
    b = None if bias is None else _c(bias, np.float64)
    logits = np.zeros((T, E), np.float64)
    lib().oracle_router(_ptr(x), T, d, _ptr(wr), E, _ptr(b), 0,
                        _ptr(logits), None, None, None)
    return logits


class QuantExperts:
    """Canonical MXFP4 weights of all experts, quantised by the oracle."""

    def __init__(self, d_model: int, d_ff: int, E: int):
        self.d_model, self.d_ff, self.E = d_model, d_ff, E
        self.g_codes = np.zeros((E, d_ff, d_model // 2), np.uint8)
        self.g_scales = np.zeros((E, d_ff, d_model // 32), np.uint8)
        self.u_codes = np.zeros_like(self.g_codes)
        self.u_scales = np.zeros_like(self.g_scales)
        self.d_codes = np.zeros((E, d_model, d_ff // 2), np.uint8)
        self.d_scales = np.zeros((E, d_model, d_ff // 32), np.uint8)

    def set_expert(self, e: int, wg: np.ndarray, wu: np.ndarray, wd: np.ndarray):
        """wg, wu: [d_model, d_ff]; wd: [d_ff, d_model] (y = x . W)."""
        self.g_codes[e], self.g_scales[e] = mxfp4_quantize_matrix(wg)
        self.u_codes[e], self.u_scales[e] = mxfp4_quantize_matrix(wu)
        self.d_codes[e], self.d_scales[e] = mxfp4_quantize_matrix(wd)


def expert(x_row: np.ndarray, q: QuantExperts, e: int, want_h: bool = False):
    x = _c(x_row, np.float64)
    out = np.zeros(q.d_model, np.float64)
    h = np.zeros(q.d_ff, np.float64) if want_h else None
    lib().oracle_expert(_ptr(x), q.d_model, q.d_ff,
                        _ptr(q.g_codes[e]), _ptr(q.g_scales[e]),
                        _ptr(q.u_codes[e]), _ptr(q.u_scales[e]),
                        _ptr(q.d_codes[e]), _ptr(q.d_scales[e]), _ptr(out), _ptr(h))
    return (out, h) if want_h else out


def moe_forward(x: np.ndarray, q: QuantExperts, idx: np.ndarray, w: np.ndarray,
                tokens: Optional[Sequence[int]] = None, nthreads: Optional[int] = None):
    """Layer output for `tokens` (default all): [len(tokens), d_model] float64."""
    x = _c(x, np.float64)
    idx = _c(idx, np.int32)
    w = _c(w, np.float64)
    T = x.shape[0]
    k = idx.shape[1]
    tok = None if tokens is None else _c(np.asarray(tokens), np.int64)
    n = T if tok is None else tok.shape[0]
    y = np.zeros((n, q.d_model), np.float64)
    if nthreads is None:
        nthreads = os.cpu_count() or 1
    lib().oracle_moe_forward(_ptr(x), q.d_model, q.d_ff, q.E, k, _ptr(idx), _ptr(w),
                             _ptr(q.g_codes), _ptr(q.g_scales), _ptr(q.u_codes),
                             _ptr(q.u_scales), _ptr(q.d_codes), _ptr(q.d_scales),
                             _ptr(tok), n, _ptr(y), int(max(1, min(nthreads, max(n, 1)))))
    return y


def rmsnorm(x: np.ndarray, gamma: Optional[np.ndarray], eps: float) -> np.ndarray:
    """RMSNorm of each row of x [T, d] in double: x / sqrt(mean(x^2) + eps) * gamma."""
    x = _c(x, np.float64)
    T, d = x.shape
    g = None if gamma is None else _c(gamma, np.float64)
    out = np.zeros((T, d), np.float64)
    lib().oracle_rmsnorm(_ptr(x), T, d, _ptr(g), float(eps), _ptr(out))
    return out


def block_forward(x: np.ndarray, q: QuantExperts, wr: np.ndarray, bias: Optional[np.ndarray], k: int,
                  gamma: Optional[np.ndarray], eps: float, residual: bool,
                  tokens: Optional[Sequence[int]] = None, nthreads: Optional[int] = None):
    """The MoE block with its adjacent steps: h = RMSNorm(x) (when gamma is
    given), routing and experts on h, plus x when `residual`.  Returns
    (y [len(tokens), d], idx, w, counts) with the routing over all tokens."""
    x64 = _c(x, np.float64)
    h = rmsnorm(x64, gamma, eps) if gamma is not None else x64
    _, idx, w, counts = router(h, wr, bias, k)
    y = moe_forward(h, q, idx, w, tokens=tokens, nthreads=nthreads)
    if residual:
        y = y + (x64 if tokens is None else x64[np.asarray(tokens, np.int64)])
    return y, idx, w, counts
