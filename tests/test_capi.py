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
    for s in range(7):
        assert lib.moe_mxfp4_status_string(s) != b"unknown status"
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


def _header_constants():
    """#define and enum constants of include/moe_mxfp4.h, evaluated."""
    src = open(os.path.join(ROOT, "include", "moe_mxfp4.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    consts = {}
    for name, val in re.findall(r"#define[ \t]+(MOE_\w+)[ \t]+([^\n]+)", src):
        consts[name] = val.strip()
    for name, val in re.findall(r"\b(MOE_\w+)\s*=\s*(\d+)", src):
        consts[name] = val
    out = {}
    for name, expr in consts.items():
        if not re.fullmatch(r"[\w\s()<>*+u-]+", expr):
            continue
        unsuffix = lambda e: re.sub(r"\b(0[xX][0-9A-Fa-f]+|\d+)[uU]\b", r"\1", e)
        expr = unsuffix(expr)
        for _ in range(3):
            expr = unsuffix(re.sub(r"\b(MOE_\w+)\b", lambda m: "(%s)" % consts.get(m.group(1), m.group(1)), expr))
        out[name] = eval(expr, {"__builtins__": {}})
    return out


def test_binding_constants_match_the_header():
    hdr = _header_constants()
    names = ["MOE_OK", "MOE_ERR_INVALID_ARG", "MOE_ERR_UNSUPPORTED", "MOE_ERR_CUDA", "MOE_ERR_NOT_QUANTIZED",
             "MOE_ERR_TIMEOUT", "MOE_ERR_BOUNDS", "MOE_DTYPE_F32", "MOE_DTYPE_BF16", "MOE_FLAG_TEST_SKIP_FIRST_COPY",
             "MOE_FLAG_TOKEN_TILE_SHIFT", "MOE_FLAG_TOKEN_TILE_MASK", "MOE_NUM_STAGES",
             "MOE_ROUTE_NOALLOC_MAX_TOKENS", "MOE_ROUTE_NOALLOC_MAX_EXPERTS", "MOE_FLAG_UNFUSED_DECODE",
             "MOE_FLAG_TEST_FAIL_ALLOC_SHIFT", "MOE_FLAG_TEST_FAIL_ALLOC_MASK", "MOE_FLAG_ACT_MXF8X2"]
    for n in names:
        assert getattr(mx, n) == hdr[n], n
    # the token-tile flag encodes BN / 16 in its field and rejects other sizes
    for bn in mx.TOKEN_TILES:
        f = mx.token_tile_flag(bn)
        assert (f & ~mx.MOE_FLAG_TOKEN_TILE_MASK) == 0 and 16 * (f >> mx.MOE_FLAG_TOKEN_TILE_SHIFT) == bn
    for bad in (0, 8, 24, 144):
        with pytest.raises(ValueError):
            mx.token_tile_flag(bad)


def test_route_noalloc_rejects_bad_arguments_before_touching_the_device(lib):
    """Sizes beyond the static array and misaligned pointers are refused on the
    host (the pointers here are never dereferenced)."""
    F32 = mx.MOE_DTYPE_F32
    ok = ctypes.c_void_p(4096)
    odd = ctypes.c_void_p(4096 + 8)      # 8 bytes past a 16-byte boundary
    odd4 = ctypes.c_void_p(4096 + 2)     # not even 4-byte aligned
    f = lib.moe_mxfp4_route_noalloc
    assert f(ok, ok, None, mx.MOE_ROUTE_NOALLOC_MAX_TOKENS + 1, 64, 8, 2, F32, ok, ok, None, None) == \
        mx.MOE_ERR_UNSUPPORTED
    assert f(ok, ok, None, 4, 64, mx.MOE_ROUTE_NOALLOC_MAX_EXPERTS + 1, 2, F32, ok, ok, None, None) == \
        mx.MOE_ERR_UNSUPPORTED
    assert f(ok, ok, None, 4, 60, 8, 2, F32, ok, ok, None, None) == mx.MOE_ERR_UNSUPPORTED
    assert f(ok, ok, None, 4, 64, 8, 9, F32, ok, ok, None, None) == mx.MOE_ERR_UNSUPPORTED
    assert f(odd, ok, None, 4, 64, 8, 2, F32, ok, ok, None, None) == mx.MOE_ERR_INVALID_ARG
    assert f(ok, odd, None, 4, 64, 8, 2, F32, ok, ok, None, None) == mx.MOE_ERR_INVALID_ARG
    assert f(ok, ok, odd4, 4, 64, 8, 2, F32, ok, ok, None, None) == mx.MOE_ERR_INVALID_ARG
    assert f(ok, ok, None, 4, 64, 8, 2, F32, odd4, ok, None, None) == mx.MOE_ERR_INVALID_ARG
    assert f(ok, ok, None, 4, 64, 8, 2, F32, ok, odd4, None, None) == mx.MOE_ERR_INVALID_ARG
    assert f(ok, ok, None, 4, 64, 8, 2, F32, ok, ok, odd4, None) == mx.MOE_ERR_INVALID_ARG
    assert f(None, ok, None, 4, 64, 8, 2, F32, ok, ok, None, None) == mx.MOE_ERR_INVALID_ARG
    assert f(ok, ok, None, 4, 64, 8, 2, 7, ok, ok, None, None) == mx.MOE_ERR_INVALID_ARG


def test_debug_library_exports_the_same_symbols():
    mxbuild.build_debug()
    L = mx.load_debug()
    for n in _declared_functions():
        assert hasattr(L, n), n
    assert L.moe_mxfp4_check_guards(None) == mx.MOE_ERR_INVALID_ARG
