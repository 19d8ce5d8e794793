"""The replica (N > 1) host path of bench.py on CPU: two gloo ranks.

The layer has no exchange step, so N GPUs run N independent replicas; the only
collective is the max over ranks of the per-rank device time.  This checks that
reduction and the whole-job throughput formula with world_size 2."""
import os
import socket

import pytest
import torch.multiprocessing as tmp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime
    import sys
    import torch
    import torch.distributed as dist
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        per_rank_ms = [12.5, 40.0][rank]
        m = bench.max_over_ranks(per_rank_ms, torch.device("cpu"), world)
        out[rank] = (m, bench.job_throughput(64, 10, world, m))
    finally:
        dist.destroy_process_group()


def test_two_rank_replica_timing():
    port = _free_port()
    with tmp.Manager() as mgr:
        out = mgr.dict()
        tmp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 40.0
    # 2 replicas x 10 steps x 64 tokens in 40 ms
    assert res[0][1] == pytest.approx(2 * 10 * 64 / 0.040)


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.0, None, 1) == 3.0
    assert bench.job_throughput(1, 5, 1, 10.0) == pytest.approx(500.0)


def test_roofline_bound_follows_machine_balance():
    """Decode-sized expert GEMMs are HBM-bound (each weight byte feeds a few
    FLOPs), prefill-sized ones with hundreds of rows per expert tensor-bound."""
    import bench
    import moe_inputs as mi

    peaks = {"hbm_gbs": 6500.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}
    dec = mi.CONFIGS["dec64"]
    w = bench.algorithmic_work(dec, dec.T, dec.n_experts)["gate_up_swiglu"]
    r = bench.roofline(w, 1e-4, peaks, "gate_up_swiglu", "f16")
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert abs(r["achieved"] - w["bytes"] / 1e-4 / 1e9) < 1e-6 * r["achieved"]
    pre = mi.CONFIGS["zipf"]
    w = bench.algorithmic_work(pre, pre.T, pre.n_experts)["gate_up_swiglu"]
    r = bench.roofline(w, 1e-3, peaks, "gate_up_swiglu", "f16")
    assert r["bound"] == "tensor" and r["peak"] == 1600.0
    # FP4 operands run at 4x the bf16 rate, which moves the balance point up
    r4 = bench.roofline(w, 1e-3, peaks, "gate_up_swiglu", "mxf4")
    assert r4["peak"] == 6400.0


def test_roofline_of_the_two_mxfp8_term_variant():
    """kind::mxf8f6f4 runs at the FP8 rate (2x bf16) and executes one MMA per
    activation term (two), and its operands carry 2 x 33/32 bytes per element
    against 3 x 17/32 for three MXFP4 terms."""
    import bench
    import moe_inputs as mi

    peaks = {"hbm_gbs": 6500.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}
    cfg = mi.CONFIGS["pre4096"]
    w4 = bench.algorithmic_work(cfg, cfg.T, cfg.n_experts, "mxf4x3")["gate_up_swiglu"]
    w8 = bench.algorithmic_work(cfg, cfg.T, cfg.n_experts, "mxf8x2")["gate_up_swiglu"]
    assert w8["flops"] == w4["flops"] and w8["bytes"] > w4["bytes"]
    rows = cfg.T * cfg.top_k
    extra = rows * (cfg.d_model + cfg.d_ff) * (2 * 33 / 32 - 3 * 17 / 32)
    assert abs((w8["bytes"] - w4["bytes"]) - extra) < 1e-6 * extra
    r = bench.roofline(w8, 1e-3, peaks, "gate_up_swiglu", "f8f6f4")
    assert r["bound"] == "tensor" and r["peak"] == 3200.0
    assert abs(r["executed_frac"] - 2 * w8["flops"] / 1e-3 / 1e12 / 3200.0) < 1e-12


def test_reference_arm_prints_one_json_line():
    """`bench.py --impl reference` (the oracle on the host cores) keeps the bench
    line's contract: one JSON line with the metric, its value and unit, the
    reference tag, the CPU-baseline description and a zero-copy e2e entry."""
    import json
    import os
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--config", "tiny",
                          "--steps", "1", "--warmup", "0"], capture_output=True, text=True, timeout=600, cwd=root)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["unit"] == "tokens/s" and rec["value"] > 0
    assert rec["higher_is_better"] is True and rec["steps"] == 1
    assert rec["cpu_baseline"]["kind"] == "oracle" and rec["cpu_baseline"]["value"] == rec["value"]
    assert rec["e2e"] == {"value": rec["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
