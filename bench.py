#!/usr/bin/env python3
"""Benchmark of the MoE-MXFP4 layer (router -> top-k -> softmax -> SwiGLU experts ->
weighted combine) on B200, through the C ABI.

Default workload: the largest single-GPU configuration, the skewed-routing
gpt-oss-20b-shaped layer at T=16384 tokens (d_model = d_ff = 2880, E = 32,
top-4, a router bias that makes expert popularity Zipf-shaped with s = 1.2,
bf16 activations, MXFP4 experts drawn N(0, 0.02) and quantised by the
library).  Other workloads (tiny, dec1, dec8, dec64, pre4096, e128) with
--config.  One step = one forward of the whole layer over one batch of T
tokens.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config zipf] [--impl ours|reference]

Prints ONE JSON line (rank 0).  Timing: W untimed warm-up steps, then K steps,
each preceded (outside its timed span) by a 256 MB L2 flush and bracketed by
CUDA events on the forward's stream; barrier + synchronize before and after
the timed region; the value uses the max over ranks.  Multi-GPU: independent
replicas (the layer has no exchange step), weak scaling.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import moe_inputs as mi  # noqa: E402

FLUSH_BYTES = 256 << 20
CSRC = os.path.join("mxfp4_expert_gemm_router_b200", "csrc")
# every CUDA source of the library (the hash ties a traffic record to the kernels it was taken on)
KERNEL_SOURCES = sorted(os.path.join(CSRC, f) for f in os.listdir(os.path.join(ROOT, CSRC))
                        if f.endswith((".cu", ".cuh")))


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for p in KERNEL_SOURCES:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ---------------------------------------------------------------- per-kernel algorithmic work

def algorithmic_work(cfg: mi.MoeConfig, T: int, touched: int, act_format: str = "mxf4x3"):
    """Bytes / flops each stage must move / do at minimum (per launch)."""
    d, f, E, k = cfg.d_model, cfg.d_ff, cfg.n_experts, cfg.top_k
    act = 2 if cfg.act_dtype == "bf16" else 4
    mx_bytes_per_param = 17 / 32
    # the grouped activation operands (x rows for gate/up, H rows for down) are
    # three MXFP4 terms per element (4 bits + a scale byte per 32), or two
    # MXFP8 terms (8 bits + a scale byte per 32)
    op_bytes = MXQ_TERMS * 17 / 32 if act_format == "mxf4x3" else MX8_TERMS * 33 / 32
    gu_w = touched * 2 * d * f * mx_bytes_per_param
    dn_w = touched * d * f * mx_bytes_per_param
    rows = T * k
    out = {
        "router_topk_schedule": {"bytes": T * d * act + E * d * act + rows * 8, "flops": 2.0 * T * d * E},
        "gate_up_swiglu": {"bytes": gu_w + rows * d * op_bytes + rows * f * op_bytes, "flops": 4.0 * rows * d * f},
        "down": {"bytes": dn_w + rows * f * op_bytes + rows * d * act, "flops": 2.0 * rows * d * f},
        "layer": {"bytes": gu_w + dn_w + 2 * T * d * act + E * d * act, "flops": 6.0 * rows * d * f + 2.0 * T * d * E},
    }
    # the fused decode kernel (at most 16 tokens) is the whole layer in one launch
    out["fused_decode"] = dict(out["layer"])
    return out


# ---------------------------------------------------------------- clocks sampler

class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            p = [s.strip() for s in ln.split(",")]
            if len(p) < 9:
                continue
            try:
                sm.append(float(p[1]))
                mx.append(float(p[2]))
            except ValueError:
                continue
            for n, v in zip(names, p[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


# ---------------------------------------------------------------- ranks

def max_over_ranks(value: float, device, world: int) -> float:
    """Max of a per-rank scalar over all ranks (replicas report the slowest one)."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_step: int, steps: int, world: int, max_total_ms: float) -> float:
    """Whole-job tokens/s: every replica processes tokens_per_step each step."""
    return tokens_per_step * steps * world / (max_total_ms / 1e3)


# ---------------------------------------------------------------- our arm

def build_layer(cfg: mi.MoeConfig, max_tokens: int, flags: int = 0):
    import torch
    import mxfp4_expert_gemm_router_b200 as mx
    from mxfp4_expert_gemm_router_b200 import build as mxbuild
    mxbuild.build()
    layer = mx.MoeMxfp4(cfg.d_model, cfg.d_ff, cfg.n_experts, cfg.top_k, max_tokens, cfg.act_dtype, flags)
    for e in range(cfg.n_experts):
        wg, wu, wd = mi.draw_expert(cfg, e)
        layer.quantize_expert(e, torch.from_numpy(wg).cuda(), torch.from_numpy(wu).cuda(),
                              torch.from_numpy(wd).cuda())
    wr = mi.draw_router(cfg)
    bias = mi.draw_bias(cfg)
    if cfg.act_dtype == "bf16":
        wr_t = torch.from_numpy(mi.bf16_bits(wr).view(np.int16).copy()).cuda().view(torch.bfloat16)
    else:
        wr_t = torch.from_numpy(wr).cuda()
    b_t = None if bias is None else torch.from_numpy(bias).cuda()
    layer.set_router(wr_t, b_t)
    torch.cuda.synchronize()
    return layer, (wr_t, b_t)


def act_tensor(cfg, a, device):
    import torch
    if cfg.act_dtype == "bf16":
        return torch.from_numpy(mi.bf16_bits(a).view(np.int16).copy()).to(device).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(device)


def uses_dependent_launches(cfg: mi.MoeConfig, T: int, act_format: str = "mxf4x3") -> bool:
    """The library launches a forward's kernels with programmatic (dependent)
    launches when it has at most 2048 grouped rows; stage events between the
    kernels would serialise those launches, so such forwards are timed without
    them and their stage times come from a second captured graph.  Forwards of
    at most 16 tokens are one launch (the fused decode kernel): its events sit
    outside it and ride in the timed graph (layers with two-MXFP8-term
    operands have no fused kernel)."""
    return (16 < T or act_format == "mxf8x2") and T * cfg.top_k <= 2048


def run_ours(args, cfg, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    T = cfg.T
    import mxfp4_expert_gemm_router_b200 as mx
    flags = mx.token_tile_flag(args.token_tile) if args.token_tile else 0
    if args.act_format == "mxf8x2":
        flags |= mx.MOE_FLAG_ACT_MXF8X2
    layer, _ = build_layer(cfg, T, flags)
    x = act_tensor(cfg, mi.draw_x(cfg), dev)
    y = torch.empty_like(x)
    counts = torch.empty(cfg.n_experts, dtype=torch.int32, device=dev)
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream(device=dev)

    def step():
        layer.forward(x, y, None, None, counts, stream)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            flush.fill_(1.0)
            step()
    torch.cuda.synchronize()
    # launches of one forward (the captured graph holds exactly these)
    n0 = layer.launch_count()
    with torch.cuda.stream(stream):
        step()
    torch.cuda.synchronize()
    launches_per_step = layer.launch_count() - n0

    def capture(with_stage_events: bool):
        # the forward never synchronises or allocates, so it can be captured once and replayed
        layer.set_profiling(with_stage_events)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            step()
        torch.cuda.synchronize()
        layer.set_profiling(False)
        return g

    # Stage events ride inside the timed graph (event-record nodes between the
    # kernels) unless the forward uses dependent launches, which the nodes would
    # serialise; then a second graph with the nodes gives the stage times.
    stages_in_timed = not uses_dependent_launches(cfg, T, args.act_format)
    graph = capture(stages_in_timed)
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            flush.fill_(1.0)
            graph.replay()
    torch.cuda.synchronize()

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    stage_ms = []
    clocks = ClockSampler(local_rank)
    if rank == 0 and not args.no_clocks:
        clocks.start()
        time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for i in range(args.steps):
            flush.fill_(float(i))
            starts[i].record(stream)
            graph.replay()
            ends[i].record(stream)
            if stages_in_timed:
                # read between steps, outside every step's event span
                stage_ms.append(layer.kernel_times())
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop() if rank == 0 and not args.no_clocks else None
    total_ms = max_over_ranks(sum(s.elapsed_time(e) for s, e in zip(starts, ends)), dev, world)
    del graph

    if not stages_in_timed:
        g2 = capture(True)
        with torch.cuda.stream(stream):
            for i in range(args.steps):
                flush.fill_(float(i))
                g2.replay()
                stage_ms.append(layer.kernel_times())
        torch.cuda.synchronize()
        del g2

    # end-to-end through the public host-buffer entry point
    xh = act_tensor(cfg, mi.draw_x(cfg), "cpu").pin_memory()
    yh = torch.empty_like(xh).pin_memory()
    for _ in range(max(1, args.warmup)):
        layer.forward_host(xh, yh, stream=stream)
    e_s = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    e_e = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    with torch.cuda.stream(stream):
        for i in range(args.steps):
            flush.fill_(float(i))
            e_s[i].record(stream)
            layer.forward_host(xh, yh, stream=stream)
            e_e[i].record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(sum(s.elapsed_time(e) for s, e in zip(e_s, e_e)), dev, world)
    touched = int((counts.cpu().numpy() > 0).sum())
    return {"total_ms": total_ms, "e2e_ms": e2e_ms, "stage_ms": stage_ms,
            "stage_timing": ("event-record nodes inside the timed graph replays" if stages_in_timed else
                             "a second captured graph with event-record nodes, replayed after the timed region "
                             "(the timed graph keeps its dependent launches)"),
            "launches": launches_per_step * args.steps, "clocks": clk, "touched": touched,
            "counts": counts.cpu().numpy().tolist(),
            "h2d": xh.numel() * xh.element_size(), "d2h": yh.numel() * yh.element_size()}


# ---------------------------------------------------------------- oracle (CPU) arm

def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def sample_tokens(cfg: mi.MoeConfig, n: int, seed: int = 1):
    """Seeded sample of n distinct token indices of the workload (all of them when n >= T)."""
    if n >= cfg.T:
        return np.arange(cfg.T)
    return np.sort(np.random.default_rng(seed).choice(cfg.T, size=n, replace=False))


class OracleLayer:
    """The oracle's layer for one workload: router weights, and every expert
    quantised by the oracle's own code (set-up, not timed)."""

    def __init__(self, cfg: mi.MoeConfig, nthreads: int):
        import oracle
        from concurrent.futures import ThreadPoolExecutor
        self.cfg, self.oracle = cfg, oracle
        self.wr = mi.draw_router(cfg)
        self.bias = mi.draw_bias(cfg)
        self.q = oracle.QuantExperts(cfg.d_model, cfg.d_ff, cfg.n_experts)
        with ThreadPoolExecutor(max_workers=nthreads) as ex:
            list(ex.map(lambda e: self.q.set_expert(e, *mi.draw_expert(cfg, e)), range(cfg.n_experts)))
        self.x = mi.draw_x(cfg)

    def time_tokens(self, tokens, nthreads: int) -> float:
        """Seconds for the oracle's router + experts over the given tokens."""
        x = self.x[tokens]
        t0 = time.perf_counter()
        _, idx, w, _ = self.oracle.router(x, self.wr, self.bias, self.cfg.top_k)
        self.oracle.moe_forward(x, self.q, idx, w, nthreads=nthreads)
        return time.perf_counter() - t0


# tokens per sample: all cores (about 10 s of CPU work on 16 host cores at the
# 2880-wide shape) and one core (about 5 s)
CPU_SAMPLE_ALL = 2048
CPU_SAMPLE_ONE = 64
# tokens per step of the reference arm (each step a bounded sample of the workload)
REF_STEP_TOKENS = 64


def cpu_baseline(cfg: mi.MoeConfig):
    nthreads = os.cpu_count() or 1
    ol = OracleLayer(cfg, nthreads)
    n_all = min(cfg.T, CPU_SAMPLE_ALL if cfg.d_model >= 1024 else cfg.T)
    n_one = min(cfg.T, CPU_SAMPLE_ONE if cfg.d_model >= 1024 else cfg.T)
    tok_all = sample_tokens(cfg, n_all)
    secs_all = ol.time_tokens(tok_all, nthreads)
    tok_one = sample_tokens(cfg, n_one, seed=2)
    secs_one = ol.time_tokens(tok_one, 1)
    return {"value": n_all / secs_all, "unit": "tokens/s", "cores": nthreads, "kind": "oracle",
            "sample": (f"seeded sample of {n_all} of the {cfg.T} tokens (router + experts in double, "
                       f"{nthreads} threads, {secs_all:.1f} s)"),
            "cpu_model": cpu_model(),
            "single_thread": {"value": n_one / secs_one, "unit": "tokens/s", "cores": 1,
                              "sample": f"seeded sample of {n_one} tokens, {secs_one:.1f} s"}}


def run_reference(args, cfg):
    nthreads = os.cpu_count() or 1
    ol = OracleLayer(cfg, nthreads)
    n = min(cfg.T, REF_STEP_TOKENS if cfg.d_model >= 1024 else cfg.T)
    for i in range(args.warmup):
        ol.time_tokens(sample_tokens(cfg, min(n, 8), seed=100 + i), nthreads)
    secs = 0.0
    toks = 0
    for i in range(args.steps):
        secs += ol.time_tokens(sample_tokens(cfg, n, seed=1000 + i), nthreads)
        toks += n
    value = toks / secs
    sample = (f"per step a seeded sample of {n} of the {cfg.T} tokens (router + experts in double, "
              f"{nthreads} threads), {args.steps} steps")
    return {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_dict(cfg, args), "impl": "reference",
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": nthreads, "kind": "oracle",
                             "sample": sample, "cpu_model": cpu_model()},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


METRIC = "MoE-MXFP4 layer tokens/s at 1 B200; % of HBM or FP4 tensor roofline"


def config_dict(cfg, args):
    return {"workload": f"gpt-oss-style MoE-MXFP4 layer '{cfg.name}': T={cfg.T}, d_model={cfg.d_model}, "
                        f"d_ff={cfg.d_ff}, E={cfg.n_experts}, top-{cfg.top_k}, {cfg.act_dtype} activations",
            "T": cfg.T, "d_model": cfg.d_model, "d_ff": cfg.d_ff, "n_experts": cfg.n_experts, "top_k": cfg.top_k,
            "seed": cfg.seed, "parallelism": f"replicas x{args.gpus}",
            "l2": "256 MB flush written between timed steps (outside each step's event span)",
            "launch": "forward captured once as a CUDA graph, replayed per timed step",
            "token_tile": getattr(args, "token_tile", 0) or "auto",
            "act_format": getattr(args, "act_format", "mxf4x3")}


# Dense tensor-core rate of the experts' MMA operand type relative to bf16
# (nominal dense ratios: f16 = bf16, fp8 2x, fp4 4x).  The expert GEMMs run
# kind::mxf4 (block-scaled FP4) with the activations as three MXFP4 terms, so
# the tensor cores execute MXQ_TERMS times the layer's useful FLOPs.
MMA_KIND = "mxf4"
MXQ_TERMS = 3
MX8_TERMS = 2
MMA_RATE_VS_BF16 = {"f16": 1.0, "f8f6f4": 2.0, "mxf4": 4.0}


def roofline(work_k, dur_s, peaks, kernel, mma_kind=None):
    """Roofline of one kernel launch: it is tensor-bound when its FLOP per byte
    exceeds the machine balance (tensor peak / HBM peak), else HBM-bound; the
    achieved rate is the algorithmic work of the launch over its duration."""
    kind = mma_kind or MMA_KIND
    # burst figure: each kernel is timed over a loop of well under a second with
    # the clocks at their maximum (the clock sampler records them)
    tflops_peak = peaks["bf16_tflops"] * MMA_RATE_VS_BF16[kind]
    # MMA flops executed per useful flop: one MMA per activation term
    terms = {"mxf4": MXQ_TERMS, "f8f6f4": MX8_TERMS}.get(kind, 1)
    t_tensor = terms * work_k["flops"] / (tflops_peak * 1e12)
    t_hbm = work_k["bytes"] / (peaks["hbm_gbs"] * 1e9)
    if t_tensor > t_hbm:
        return {"bound": "tensor", "achieved": work_k["flops"] / dur_s / 1e12, "peak": tflops_peak,
                "unit": "TFLOP/s", "kernel": kernel, "mma_kind": kind,
                "executed_frac": terms * work_k["flops"] / dur_s / 1e12 / tflops_peak}
    return {"bound": "hbm", "achieved": work_k["bytes"] / dur_s / 1e9, "peak": peaks["hbm_gbs"],
            "unit": "GB/s", "kernel": kernel, "mma_kind": kind}


def load_traffic_record():
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        return json.load(f)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="zipf", choices=sorted(mi.CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--act-format", default="mxf4x3", choices=["mxf4x3", "mxf8x2"],
                    help="activation operand format: three MXFP4 terms (kind::mxf4) or two MXFP8 terms "
                         "(kind::mxf8f6f4)")
    ap.add_argument("--token-tile", type=int, default=0, choices=[0, 16, 32, 48, 64, 80, 96, 112, 128],
                    help="token rows per expert-GEMM tile (0: chosen per forward)")
    args = ap.parse_args()
    cfg = mi.CONFIGS[args.config]

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args, cfg)), flush=True)
        return 0

    import torch
    import torch.distributed as dist
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    r = run_ours(args, cfg, rank, world, local_rank)
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0

    value = job_throughput(cfg.T, args.steps, world, r["total_ms"])
    e2e_value = job_throughput(cfg.T, args.steps, world, r["e2e_ms"])
    stages = {}
    for name in r["stage_ms"][0]:
        vals = [s[name] for s in r["stage_ms"]]
        stages[name] = sum(vals) / len(vals)
    work = algorithmic_work(cfg, cfg.T, r["touched"], args.act_format)
    peaks = measured_peaks()
    dominant = max(("gate_up_swiglu", "down", "router_topk_schedule", "fused_decode"),
                   key=lambda n: stages.get(n, 0.0))
    dur_s = stages[dominant] / 1e3
    roof = roofline(work[dominant], dur_s, peaks, dominant, "f8f6f4" if args.act_format == "mxf8x2" else "mxf4")
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["peak_source"] = peaks["source"]
    roof["algorithmic_per_launch"] = work[dominant]["bytes"] if roof["bound"] == "hbm" else work[dominant]["flops"]
    tr = load_traffic_record()
    roof["traffic"] = None
    if tr and tr.get("source_hash") == kernel_source_hash():
        # per-launch DRAM bytes of this workload's dominant kernel, from its ncu
        # capture (null when the kernels changed after the capture)
        roof["traffic"] = tr.get("per_config", {}).get(cfg.name, {}).get(dominant)
    layer_s = r["total_ms"] / 1e3 / args.steps
    out = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": r["total_ms"] / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": ("mxf4: MXFP4 weights as stored x activations as 3 MXFP4 terms, fp32 accumulate"
                  if args.act_format == "mxf4x3" else
                  "mxf8f6f4: MXFP4 weights as stored x activations as 2 MXFP8 (E4M3) terms, fp32 accumulate"),
        "data": "synthetic (seeded N(0,1) activations, N(0,0.02) experts quantised to MXFP4)",
        "config": config_dict(cfg, args),
        "roofline": roof,
        "layer_hbm": {"bytes": work["layer"]["bytes"], "GB/s": work["layer"]["bytes"] / layer_s / 1e9,
                      "frac_of_measured": work["layer"]["bytes"] / layer_s / 1e9 / peaks["hbm_gbs"],
                      "frac_of_8TBs": work["layer"]["bytes"] / layer_s / 8e12},
        "stage_ms": stages,
        "stage_timing": r["stage_timing"],
        "experts_touched": r["touched"],
        "gpu_launches": r["launches"],
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"]},
        "clocks": r["clocks"],
    }
    if world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(cfg)
    print(json.dumps(out), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
