"""Failure paths that need a device but fault nothing: an allocation in
moe_mxfp4_create that fails (a test flag makes the n-th allocation fail as if
cudaMalloc had) returns MOE_ERR_CUDA, leaves no handle and frees what was
already allocated."""
import ctypes

import pytest

pytestmark = pytest.mark.gpu


def test_failed_allocation_in_create_leaks_nothing():
    import torch
    import mxfp4_expert_gemm_router_b200 as mx
    lib = mx.load()
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    failures = 0
    for n in range(1, 255):
        cfg = mx.make_config(2880, 2880, 32, 4, 4096, "bf16",
                             flags=n << mx.MOE_FLAG_TEST_FAIL_ALLOC_SHIFT)
        h = ctypes.c_void_p()
        st = lib.moe_mxfp4_create(ctypes.byref(cfg), ctypes.byref(h))
        if st == mx.MOE_OK:
            assert h.value
            lib.moe_mxfp4_destroy(h)
            break
        assert st == mx.MOE_ERR_CUDA, (n, st)
        assert not h.value
        failures += 1
    else:
        pytest.fail("create never succeeded")
    # every device allocation of create was made to fail once (the fused-decode
    # workspace included)
    assert failures >= 30, failures
    torch.cuda.synchronize()
    free1 = torch.cuda.mem_get_info()[0]
    # the 2880-wide layer holds ~450 MB of weights and ~250 MB of workspace: a leak
    # of any large buffer would show; small ones are below the allocator granularity
    assert free0 - free1 < 64 << 20, (free0 - free1)
    lib.moe_mxfp4_destroy(None)
