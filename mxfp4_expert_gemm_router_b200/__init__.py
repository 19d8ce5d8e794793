"""Python binding of libmoe_mxfp4.so, the C-ABI library of the MoE feed-forward
layer with MXFP4 experts on B200 (sm_100a).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  The raw C functions are exposed under their C names
(``moe_mxfp4_create``, ``moe_mxfp4_forward`` ...); ``MoeMxfp4`` wraps a handle
and takes torch tensors (device pointers via ``data_ptr``) for convenience.

If the shared library is missing or cannot be loaded, every entry point raises
``RuntimeError`` -- there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmoe_mxfp4.so")

(MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_CUDA, MOE_ERR_NOT_QUANTIZED, MOE_ERR_TIMEOUT,
 MOE_ERR_BOUNDS) = range(7)
MOE_DTYPE_F32, MOE_DTYPE_BF16 = 0, 1
MOE_FLAG_TEST_SKIP_FIRST_COPY = 1 << 30
MOE_FLAG_TOKEN_TILE_SHIFT = 8
MOE_FLAG_TOKEN_TILE_MASK = 0xF << MOE_FLAG_TOKEN_TILE_SHIFT
MOE_FLAG_UNFUSED_DECODE = 1 << 12
MOE_FLAG_ACT_MXF8X2 = 1 << 13
MOE_FLAG_TEST_FAIL_ALLOC_SHIFT = 16
MOE_FLAG_TEST_FAIL_ALLOC_MASK = 0xFF << MOE_FLAG_TEST_FAIL_ALLOC_SHIFT


TOKEN_TILES = tuple(range(16, 129, 16))


def token_tile_flag(bn: int) -> int:
    """Config flag that forces BN token rows per expert-GEMM tile (16, 32, ..., 128)."""
    if bn not in TOKEN_TILES:
        raise ValueError("token tile must be a multiple of 16 from 16 to 128")
    return (bn // 16) << MOE_FLAG_TOKEN_TILE_SHIFT
MOE_NUM_STAGES = 7


class moe_mxfp4_config_t(ctypes.Structure):
    _fields_ = [("d_model", ctypes.c_int32), ("d_ff", ctypes.c_int32), ("n_experts", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("max_tokens", ctypes.c_int32), ("act_dtype", ctypes.c_int32),
                ("flags", ctypes.c_uint32), ("wait_timeout_ms", ctypes.c_int32)]


_VP = ctypes.c_void_p
_I32 = ctypes.c_int32
_ST = ctypes.c_int  # moe_status_t

# name -> (restype, argtypes); mirrors include/moe_mxfp4.h
SIGNATURES = {
    "moe_mxfp4_create": (_ST, [ctypes.POINTER(moe_mxfp4_config_t), ctypes.POINTER(_VP)]),
    "moe_mxfp4_destroy": (None, [_VP]),
    "moe_mxfp4_quantize_weights": (_ST, [_VP, _VP, _VP, _VP, _VP, _VP, _VP]),
    "moe_mxfp4_quantize_expert": (_ST, [_VP, _I32, _VP, _VP, _VP, _VP]),
    "moe_mxfp4_set_router": (_ST, [_VP, _VP, _VP, _VP]),
    "moe_mxfp4_set_norm_residual": (_ST, [_VP, _VP, ctypes.c_float, _I32, _VP]),
    "moe_mxfp4_forward": (_ST, [_VP, _VP, _I32, _VP, _VP, _VP, _VP, _VP]),
    "moe_mxfp4_forward_host": (_ST, [_VP, _VP, _I32, _VP, _VP, _VP, _VP]),
    "moe_mxfp4_export_weights": (_ST, [_VP, _I32, _VP, _VP, _VP]),
    "moe_mxfp4_get_grouping": (_ST, [_VP, _VP, _VP, _VP, _VP]),
    "moe_mxfp4_get_status": (_ST, [_VP]),
    "moe_mxfp4_status_string": (ctypes.c_char_p, [_ST]),
    "moe_mxfp4_set_profiling": (_ST, [_VP, _I32]),
    "moe_mxfp4_kernel_times": (_ST, [_VP, ctypes.POINTER(ctypes.c_float), _I32]),
    "moe_mxfp4_stage_name": (ctypes.c_char_p, [_I32]),
    "moe_mxfp4_launch_count": (ctypes.c_uint64, [_VP]),
    "moe_mxfp4_expert_param_count": (ctypes.c_int64, [ctypes.POINTER(moe_mxfp4_config_t)]),
    "moe_mxfp4_expert_weight_bytes": (ctypes.c_int64, [ctypes.POINTER(moe_mxfp4_config_t)]),
    "moe_mxfp4_route_noalloc": (_ST, [_VP, _VP, _VP, _I32, _I32, _I32, _I32, _I32, _VP, _VP, _VP, _VP]),
    "moe_mxfp4_check_guards": (_ST, [_VP]),
    "moe_mxfp4_test_write_guard": (_ST, [_VP, _I32]),
}

DEBUG_LIB_PATH = os.path.join(HERE, "libmoe_mxfp4_debug.so")

_lib = None
_debug_lib = None


def _open(path: str) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise RuntimeError(f"{path} not found: build it with mxfp4_expert_gemm_router_b200.build.build()")
    try:
        L = ctypes.CDLL(path)
    except OSError as e:
        raise RuntimeError(f"cannot load {path}: {e}") from e
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    return L


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the C-ABI library (raises RuntimeError if it is missing)."""
    global _lib
    if _lib is not None:
        return _lib
    _lib = _open(path)
    return _lib


def load_debug(path: str = DEBUG_LIB_PATH) -> ctypes.CDLL:
    """Load the debug build of the library (index checks, guard regions)."""
    global _debug_lib
    if _debug_lib is None:
        _debug_lib = _open(path)
    return _debug_lib


def __getattr__(name):
    # raw C entry points under their C names, e.g. moe_mxfp4_forward(...)
    if name in SIGNATURES:
        return getattr(load(), name)
    raise AttributeError(name)


MOE_ROUTE_NOALLOC_MAX_TOKENS = 256
MOE_ROUTE_NOALLOC_MAX_EXPERTS = 128


def route_noalloc(x, w_router, router_bias, top_k, topk_idx, topk_w, expert_counts=None, stream=None):
    """Router + top-k + softmax with no device allocation (see moe_mxfp4_route_noalloc)."""
    import torch
    dt = MOE_DTYPE_BF16 if x.dtype == torch.bfloat16 else MOE_DTYPE_F32
    T, d = int(x.shape[0]), int(x.shape[1])
    E = int(w_router.shape[0])
    check(load().moe_mxfp4_route_noalloc(_p(x), _p(w_router), _p(router_bias), T, d, E, int(top_k), dt,
                                         _p(topk_idx), _p(topk_w), _p(expert_counts), _stream(stream)),
          "route_noalloc")


class MoeError(RuntimeError):
    def __init__(self, status: int, what: str):
        msg = load().moe_mxfp4_status_string(status).decode()
        super().__init__(f"{what}: {msg} (status {status})")
        self.status = status


def check(status: int, what: str):
    if status != MOE_OK:
        raise MoeError(status, what)


def make_config(d_model, d_ff, n_experts, top_k, max_tokens, act_dtype="bf16", flags=0, wait_timeout_ms=0):
    dt = {"bf16": MOE_DTYPE_BF16, "f32": MOE_DTYPE_F32}[act_dtype] if isinstance(act_dtype, str) else act_dtype
    return moe_mxfp4_config_t(d_model, d_ff, n_experts, top_k, max_tokens, dt, flags, wait_timeout_ms)


def _p(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


class MoeMxfp4:
    """One layer handle.  Tensors are torch CUDA tensors on the handle's device."""

    def __init__(self, d_model, d_ff, n_experts, top_k, max_tokens, act_dtype="bf16", flags=0,
                 wait_timeout_ms=0, lib=None):
        """`lib`: the library to drive (default the release build; load_debug() for the debug build)."""
        self._L = lib if lib is not None else load()
        self.cfg = make_config(d_model, d_ff, n_experts, top_k, max_tokens, act_dtype, flags, wait_timeout_ms)
        self.act_dtype = act_dtype
        h = ctypes.c_void_p()
        check(self._L.moe_mxfp4_create(ctypes.byref(self.cfg), ctypes.byref(h)), "moe_mxfp4_create")
        self.h = h

    def close(self):
        if getattr(self, "h", None) is not None and self.h.value:
            self._L.moe_mxfp4_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def quantize_weights(self, w_gate, w_up, w_down, w_router, router_bias=None, stream=None):
        check(self._L.moe_mxfp4_quantize_weights(self.h, _p(w_gate), _p(w_up), _p(w_down), _p(w_router),
                                                _p(router_bias), _stream(stream)), "quantize_weights")

    def quantize_expert(self, e, w_gate, w_up, w_down, stream=None):
        check(self._L.moe_mxfp4_quantize_expert(self.h, int(e), _p(w_gate), _p(w_up), _p(w_down),
                                               _stream(stream)), "quantize_expert")

    def set_router(self, w_router, router_bias=None, stream=None):
        check(self._L.moe_mxfp4_set_router(self.h, _p(w_router), _p(router_bias), _stream(stream)), "set_router")

    def set_norm_residual(self, gamma=None, eps=1e-5, residual=False, stream=None):
        check(self._L.moe_mxfp4_set_norm_residual(self.h, _p(gamma), float(eps), 1 if residual else 0,
                                                 _stream(stream)), "set_norm_residual")

    def forward(self, x, y, topk_idx=None, topk_w=None, expert_counts=None, stream=None):
        T = int(x.shape[0]) if x is not None else 0
        check(self._L.moe_mxfp4_forward(self.h, _p(x), T, _p(y), _p(topk_idx), _p(topk_w), _p(expert_counts),
                                       _stream(stream)), "forward")

    def forward_host(self, x_host, y_host, topk_idx_host=None, topk_w_host=None, stream=None):
        T = int(x_host.shape[0])
        check(self._L.moe_mxfp4_forward_host(self.h, _p(x_host), T, _p(y_host), _p(topk_idx_host),
                                            _p(topk_w_host), _stream(stream)), "forward_host")

    def export_weights(self, which, codes, scales, stream=None):
        check(self._L.moe_mxfp4_export_weights(self.h, int(which), _p(codes), _p(scales), _stream(stream)),
              "export_weights")

    def get_grouping(self, offsets, row_token=None, row_weight=None, stream=None):
        check(self._L.moe_mxfp4_get_grouping(self.h, _p(offsets), _p(row_token), _p(row_weight),
                                            _stream(stream)), "get_grouping")

    def status(self) -> int:
        return self._L.moe_mxfp4_get_status(self.h)

    def set_profiling(self, enable: bool):
        check(self._L.moe_mxfp4_set_profiling(self.h, 1 if enable else 0), "set_profiling")

    def kernel_times(self):
        buf = (ctypes.c_float * MOE_NUM_STAGES)()
        check(self._L.moe_mxfp4_kernel_times(self.h, buf, MOE_NUM_STAGES), "kernel_times")
        return {self._L.moe_mxfp4_stage_name(i).decode(): float(buf[i]) for i in range(MOE_NUM_STAGES)}

    def launch_count(self) -> int:
        return int(self._L.moe_mxfp4_launch_count(self.h))

    def check_guards(self) -> int:
        return self._L.moe_mxfp4_check_guards(self.h)
