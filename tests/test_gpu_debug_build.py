"""The debug build of the library (compiled with MOE_DEBUG_CHECKS): device
index checks on every index the kernels scatter or gather through that
another kernel wrote (grouped rows, token tiles, GEMM units, combine tokens),
and a guard region after every device buffer of a handle.  On the workloads
below no check may fire and no guard may change, and the layer still matches
the oracle; the guard checker is shown to detect a changed byte by writing one
from the host (no kernel writes out of bounds on purpose)."""
import numpy as np
import pytest

import moe_inputs as mi
from _layer import GpuLayer, OracleExperts, check_layer, filtered_x

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dlib():
    import mxfp4_expert_gemm_router_b200 as mx
    from mxfp4_expert_gemm_router_b200 import build as mxbuild
    mxbuild.build_debug()
    return mx.load_debug()


def _case(name, T):
    cfgs = {
        "tiny": mi.CONFIGS["tiny"],
        "ragged": mi.MoeConfig("ragged", T, 192, 320, 4, 2, "f32"),
        "wide": mi.CONFIGS["dec64"].with_T(T),
    }
    return cfgs[name].with_T(T)


@pytest.mark.parametrize("name,T,unfused", [("tiny", 16, False), ("tiny", 16, True), ("ragged", 40, True),
                                            ("ragged", 11, False), ("wide", 64, True), ("wide", 8, False),
                                            ("wide", 600, True)])
def test_debug_build_runs_clean(dlib, name, T, unfused):
    import mxfp4_expert_gemm_router_b200 as mx
    cfg = _case(name, T)
    flags = mx.MOE_FLAG_UNFUSED_DECODE if unfused else 0
    L = GpuLayer(cfg, T, flags=flags, lib=dlib)
    x = filtered_x(cfg, L.wr, L.bias)
    for _ in range(2):
        y, idx, w, counts = L.forward(x)    # asserts the device status is OK (no bounds check fired)
        assert L.layer.check_guards() == mx.MOE_OK
    check_layer(cfg, x, L.wr, L.bias, y, idx, w, counts, OracleExperts(cfg), n_sample=min(T, 24))
    L.layer.close()


def test_guard_checker_detects_a_changed_byte(dlib):
    import mxfp4_expert_gemm_router_b200 as mx
    cfg = mi.CONFIGS["tiny"]
    L = GpuLayer(cfg, cfg.T, lib=dlib)
    assert L.layer.check_guards() == mx.MOE_OK
    assert dlib.moe_mxfp4_test_write_guard(L.layer.h, 3) == mx.MOE_OK
    assert L.layer.check_guards() == mx.MOE_ERR_BOUNDS
    assert dlib.moe_mxfp4_test_write_guard(L.layer.h, 10_000) == mx.MOE_ERR_INVALID_ARG
    L.layer.close()


def test_release_build_has_no_guards():
    import mxfp4_expert_gemm_router_b200 as mx
    cfg = mi.CONFIGS["tiny"]
    L = GpuLayer(cfg, cfg.T, quantize=False)
    assert L.layer.check_guards() == mx.MOE_ERR_UNSUPPORTED
    assert mx.load().moe_mxfp4_test_write_guard(L.layer.h, 0) == mx.MOE_ERR_UNSUPPORTED
