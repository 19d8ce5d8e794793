"""C-ABI library: it loads, exports every symbol include/moe_mxfp4.h declares,
and rejects bad arguments on the host (no GPU needed for any of these)."""
import ctypes
import os
import re

import pytest

import mxfp4_expert_gemm_router_b200 as mx
from mxfp4_expert_gemm_router_b200 import build as mxbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    mxbuild.build()
    return mx.load()


def _declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names.update(re.findall(r"\b(moe_mxfp4_\w+)\s*\(", src))
    return names


def test_every_declared_symbol_is_exported(lib):
    names = _declared_functions()
    assert len(names) >= 15
    for n in names:
        assert hasattr(lib, n), n
    assert names == set(mx.SIGNATURES), names ^ set(mx.SIGNATURES)


def test_status_strings(lib):
    for s in range(6):
        assert lib.moe_mxfp4_status_string(s)
    assert lib.moe_mxfp4_stage_name(2) == b"gate_up_swiglu"


def test_create_validates_arguments_before_touching_the_device(lib):
    h = ctypes.c_void_p()
    bad = [
        (mx.make_config(0, 128, 8, 2, 16, "f32"), mx.MOE_ERR_INVALID_ARG),
        (mx.make_config(64, 128, 8, 0, 16, "f32"), mx.MOE_ERR_INVALID_ARG),
        (mx.make_config(64, 128, 8, 2, 0, "f32"), mx.MOE_ERR_INVALID_ARG),
        (mx.make_config(64, 128, 8, 2, 16, 7), mx.MOE_ERR_INVALID_ARG),
        (mx.make_config(60, 128, 8, 2, 16, "f32"), mx.MOE_ERR_UNSUPPORTED),
        (mx.make_config(64, 100, 8, 2, 16, "f32"), mx.MOE_ERR_UNSUPPORTED),
        (mx.make_config(64, 128, 8, 9, 16, "f32"), mx.MOE_ERR_UNSUPPORTED),
        (mx.make_config(64, 128, 300, 2, 16, "f32"), mx.MOE_ERR_UNSUPPORTED),
    ]
    for cfg, want in bad:
        assert lib.moe_mxfp4_create(ctypes.byref(cfg), ctypes.byref(h)) == want
        assert not h.value
    assert lib.moe_mxfp4_create(None, ctypes.byref(h)) == mx.MOE_ERR_INVALID_ARG


def test_null_handles_are_rejected(lib):
    assert lib.moe_mxfp4_forward(None, None, 1, None, None, None, None, None) == mx.MOE_ERR_INVALID_ARG
    assert lib.moe_mxfp4_get_status(None) == mx.MOE_ERR_INVALID_ARG
    assert lib.moe_mxfp4_export_weights(None, 0, None, None, None) == mx.MOE_ERR_INVALID_ARG
    lib.moe_mxfp4_destroy(None)  # NULL-safe
    assert lib.moe_mxfp4_launch_count(None) == 0


def test_expert_size_matches_page_figures(lib):
    # SwiGLU expert with three d x d_ff matrices: 3,145,728 params at d = d_ff = 1024
    cfg = mx.make_config(1024, 1024, 1, 1, 1)
    assert lib.moe_mxfp4_expert_param_count(ctypes.byref(cfg)) == 3145728
    # 4.25 bits per parameter
    assert lib.moe_mxfp4_expert_weight_bytes(ctypes.byref(cfg)) * 8 == 3145728 * 4.25
    cfg = mx.make_config(2880, 2880, 32, 4, 1)
    assert lib.moe_mxfp4_expert_weight_bytes(ctypes.byref(cfg)) == 13219200


def test_binding_fails_loudly_without_the_library(tmp_path):
    import importlib
    m = importlib.import_module("mxfp4_expert_gemm_router_b200")
    saved = m._lib
    try:
        m._lib = None
        with pytest.raises(RuntimeError):
            m.load(str(tmp_path / "missing.so"))
    finally:
        m._lib = saved
