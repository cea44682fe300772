#!/usr/bin/env python
"""Benchmark: quantized GEMV / MoE weight-stream GB/s on B200.

Headline workload (one "step"): one decode step's projections at TinyLlama-1.1B shape,
batch 1 — 22 layers of Q4_0 q/o 2048x2048, k/v 256x2048, gate/up 5632x2048, down
2048x5632 plus a Q8_0 LM head 32000x2048 (614,629,376 weight bytes) and the greedy token
(argmax of the head's logits), all in ONE qgemv_batched_argmax launch.  Inputs are seeded
synthetic tensors resident in HBM; the weights of a step (615 MB) are larger than L2
(126 MB), so no flush is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line on rank 0.  Under torchrun (N > 1) every rank runs an independent
replica on its own GPU (no data-path collective); time is the max over ranks.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "quantized GEMV/MoE weight-stream GB/s (% of HBM peak); us per MoE layer"
UNIT = "GB/s"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
KERNEL_SOURCES = ["common.cuh", "qgemv.cuh"]


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true")
    ap.add_argument("--no-glm", action="store_true", help="skip the 39 GB GLM-like MoE stack")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="budget of the CPU-baseline sample")
    return ap.parse_args()


# ---------------------------------------------------------------- helpers
def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def tensor_peak():
    """Dense fp16 tensor peak in TFLOP/s: the measured bf16 burst figure (fp16 and bf16 run at the
    same nominal rate on the tensor cores), else the fallback."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        if "bf16_tflops" in d:
            return float(d["bf16_tflops"])
    return FALLBACK_BF16_TFLOPS


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for name in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "block_quant_gemv_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def committed_traffic():
    """Per-launch DRAM bytes of the headline kernel from the committed ncu record
    (profiles/k_qgemv_tinyllama_decode.json), or None when it is missing or was taken on a
    different kernel source."""
    p = os.path.join(ROOT, "profiles", "k_qgemv_tinyllama_decode.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f)
    if rec.get("kernel_source_hash") != kernel_source_hash():
        return None
    try:
        return int(rec["traffic_bytes_per_launch"])
    except (KeyError, ValueError, TypeError):
        return None


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed region runs."""

    FIELDS = "clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown," \
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap"

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu), "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def wait_first(self, timeout: float = 15.0):
        """Blocks until nvidia-smi has printed its first sample: its start-up (driver
        initialisation) can stall this process's CUDA calls, so it must not overlap the timed
        region."""
        t0 = time.time()
        while self.proc is not None and not self.lines and time.time() - t0 < timeout:
            time.sleep(0.05)
        self.lines.clear()

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.t.join(timeout=5)
        if not self.lines:
            # a timed region shorter than the sampling period: one query right after it
            try:
                out = subprocess.run(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                      "-i", str(self.gpu)], capture_output=True, text=True, timeout=10).stdout
                self.lines = [ln.strip() for ln in out.splitlines() if ln.strip()]
            except (OSError, subprocess.SubprocessError):
                pass
        return self.summarize(self.lines)

    @staticmethod
    def summarize(lines):
        """Median SM clock, maximum SM clock and the throttle reasons seen in `FIELDS` records
        (malformed records are skipped)."""
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != 6:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[2:]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def physical_gpu(logical: int) -> str:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if not vis:
        return str(logical)
    ids = [v.strip() for v in vis.split(",") if v.strip()]
    return ids[logical] if logical < len(ids) else str(logical)


# ---------------------------------------------------------------- distributed plumbing
def dist_setup(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, world: int) -> float:
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------- CPU oracle leg
def oracle_sample(seconds: float, seed: int, threads: int = 1):
    """Time the float64 oracle (on `threads` BLAS threads) on whole matrices of the decode step,
    in execution order, until the time budget is used.  Returns (bytes, seconds, n_matrices)."""
    import numpy as np
    from threadpoolctl import threadpool_limits

    import synth
    from oracle import qgemv as oq
    from synth import workloads as wl

    specs = wl.decode_step_specs()
    done_bytes, t_total, n = 0, 0.0, 0
    xs = {}
    with threadpool_limits(threads):
        for s in specs:
            if s.x_name not in xs:
                xs[s.x_name] = wl.x_host(specs, s.x_name, seed).numpy().astype(np.float64)
            W = synth.matrix(s.fmt, s.rows, s.cols, seed, s.name).numpy()
            t0 = time.perf_counter()
            oq.qgemv(s.fmt, W, xs[s.x_name], s.rows, s.cols)
            t_total += time.perf_counter() - t0
            done_bytes += synth.weight_bytes(s.fmt, s.rows, s.cols) + 4 * (s.rows + s.cols)
            n += 1
            if t_total >= seconds:
                break
    return done_bytes, t_total, n


def run_reference(args, world, rank):
    """The oracle as the reference arm, on a bounded sample of the decode step: the first
    matrices in execution order (generated once, at least one), as many as fit a per-step
    budget that keeps the whole --steps/--warmup run near two and a half minutes of oracle
    time.  The same sample is timed at every step."""
    if rank != 0:
        return
    import numpy as np
    from threadpoolctl import threadpool_limits

    import synth
    from oracle import qgemv as oq
    from synth import workloads as wl

    specs = wl.decode_step_specs()
    per_step = min(5.0, 150.0 / max(1, args.steps + args.warmup))
    sample, xs = [], {}  # (spec, first row, end row, the rows' bytes)
    with threadpool_limits(1):
        t_pass = 0.0
        chunk = 64
        for s in specs:  # calibration: add row chunks in execution order until a pass fills the budget
            if s.x_name not in xs:
                xs[s.x_name] = wl.x_host(specs, s.x_name, args.seed).numpy().astype(np.float64)
            r0 = 0
            while r0 < s.rows and t_pass < per_step:
                r1 = min(s.rows, r0 + chunk)
                W = synth.matrix(s.fmt, s.rows, s.cols, args.seed, s.name, r0=r0, r1=r1).numpy()
                t0 = time.perf_counter()
                oq.qgemv(s.fmt, W, xs[s.x_name], r1 - r0, s.cols)
                t_pass += time.perf_counter() - t0
                sample.append((s, r0, r1, W))
                r0 = r1
                chunk = min(2 * chunk, 4096)
            if t_pass >= per_step:
                break

        def one_pass():
            t0 = time.perf_counter()
            for s, r0, r1, W in sample:
                oq.qgemv(s.fmt, W, xs[s.x_name], r1 - r0, s.cols)
            return time.perf_counter() - t0

        for _ in range(args.warmup):
            one_pass()
        tot_t = sum(one_pass() for _ in range(args.steps))
    pass_bytes = sum(synth.weight_bytes(s.fmt, r1 - r0, s.cols) + 4 * (r1 - r0 + s.cols) for s, r0, r1, _ in sample)
    gbs = pass_bytes * args.steps / tot_t / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": gbs, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot_t / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(),
        "cpu_baseline": {"value": gbs, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": f"float64 oracle, single thread: each timed step is the first "
                                   f"{pass_bytes / 1e6:.2f} MB of the decode step's matrices in execution order "
                                   f"({len(sample)} row chunks); ms_per_step is the time of that sample"},
        "e2e": {"value": gbs, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def oracle_moe_sample(seed: int, threads: int):
    """The float64 oracle on one Gemma-like MoE layer at one token (router, top-8, 8 routed
    experts and the shared expert): seconds and algorithmic bytes of that layer."""
    import numpy as np
    from threadpoolctl import threadpool_limits

    import synth
    from oracle import moe as om
    from synth import workloads as wl
    spec = wl.GEMMA_MOE
    x = wl.moe_tokens(spec, seed, 1).numpy().astype(np.float64)
    R = synth.normal_f32(seed, synth.stream_id(f"{spec.name}/L0/router"), spec.n_experts * spec.hidden,
                         std=0.02).view(spec.n_experts, spec.hidden).numpy()
    experts = {}

    def expert(e):
        if e not in experts:
            experts[e] = om.Expert(spec.expert_fmt, *[wl.expert_matrix(spec, seed, 0, e, w).numpy()
                                                      for w in ("gate", "up", "down")])
        return experts[e]
    shared = om.Expert(spec.shared_fmt, *[wl.shared_matrix(spec, seed, 0, w).numpy() for w in ("gate", "up", "down")])
    layer = om.Layer(spec.n_experts, spec.top_k, spec.hidden, spec.inter, spec.act, expert, shared, spec.shared_inter)
    idx, _ = om.router_topk(om.router_logits(R, x), spec.top_k)
    for e in idx.reshape(-1):
        expert(int(e))                          # generate the touched experts' bytes outside the timing
    with threadpool_limits(threads):
        t0 = time.perf_counter()
        idx, w = om.router_topk(om.router_logits(R, x), spec.top_k)
        om.moe_layer(layer, x, idx, w)
        t = time.perf_counter() - t0
    nbytes = 4 * spec.n_experts * spec.hidden + sum(spec.shared_bytes(m) for m in ("gate", "up", "down")) + \
        8 * sum(spec.mat_bytes(m) for m in ("gate", "up", "down"))
    return t, nbytes


def oracle_prefill_sample(seed: int, threads: int):
    """The float64 oracle on the prefill chunk at N = 1024 (128 x 1024 x 4096): seconds, FLOPs."""
    import numpy as np
    from threadpoolctl import threadpool_limits

    import synth
    from oracle import prefill as op
    t, n, k = 128, 1024, 4096
    W = synth.q4_0_matrix(n, k, seed, f"prefill/N{n}/copy0").numpy()
    X = synth.normal_f16(seed, synth.stream_id("prefill/X"), t * k).view(t, k).numpy()
    with threadpool_limits(threads):
        t0 = time.perf_counter()
        op.prefill(2, W, X, n, k)
        dt = time.perf_counter() - t0
    return dt, 2.0 * t * n * k


def cpu_baselines(args):
    """The oracle on one host core and on all of them (decode-step GB/s), plus one MoE layer and
    the N = 1024 prefill chunk."""
    cores = os.cpu_count() or 1
    out = {}
    for threads in (1, cores):
        b, t, n = oracle_sample(args.cpu_seconds / 2, args.seed, threads)
        out[threads] = {"value": b / t / 1e9, "unit": UNIT, "cores": threads, "kind": "oracle",
                        "sample": f"float64 oracle on {threads} thread(s), the first {n} whole matrices of the "
                                  f"decode step ({b / 1e6:.0f} MB in {t:.1f} s)"}
    mt, mb = oracle_moe_sample(args.seed, cores)
    pt, pf = oracle_prefill_sample(args.seed, cores)
    extra = {"moe_gemma_T1": {"us_per_layer": mt * 1e6, "GB/s": mb / mt / 1e9, "cores": cores},
             "prefill_N1024": {"us_per_call": pt * 1e6, "GFLOP/s": pf / pt / 1e9, "cores": cores}}
    return out[1], out[cores], extra


def synth_bytes(s):
    import synth
    return synth.weight_bytes(s.fmt, s.rows, s.cols)


def workload_config():
    return {"workload": "tinyllama_decode: 22 layers x Q4_0 (q,o 2048x2048; k,v 256x2048; gate,up 5632x2048; "
                        "down 2048x5632) + Q8_0 LM head 32000x2048 + greedy token (argmax of the head), batch 1, "
                        "x ~ N(0,1)",
            "weight_bytes_per_step": 614629376,
            "launch": "one qgemv_batched_argmax launch per step, captured once in a CUDA graph and replayed; "
                      "e2e calls the API eagerly",
            "l2": "inputs larger than L2 (615 MB of weights per step vs 126 MB L2); no flush",
            "parallelism": "replicas"}


# ---------------------------------------------------------------- GPU legs
def time_decode_step(args, world, dev):
    import torch

    import block_quant_gemv_b200 as bqg
    from synth import workloads as wl

    specs = wl.decode_step_specs()
    W = wl.build_gemv_workload(specs, seed=args.seed, device=dev)
    batch = bqg.GemvBatch(W.items())
    greedy = bqg.ArgmaxState(dev)
    head = len(specs) - 1

    def step_eager():
        batch.run(argmax=(head, greedy))

    # The decode step as an engine runs it: the public call captured once into a CUDA graph
    # (the pages' captured decode graph) and replayed per step, so the host's per-call
    # marshalling (155 descriptors, a 30 KB parameter block) does not starve the GPU.
    def capture(fn):
        cs = torch.cuda.Stream()
        cs.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(cs):
            fn()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cs):
            fn()
        torch.cuda.synchronize()
        return g
    g_step = capture(step_eager)
    g_plain = capture(batch.run)

    def step():
        g_step.replay()
    stream = torch.cuda.current_stream()
    clocks = ClockSampler(physical_gpu(torch.cuda.current_device()))
    clocks.start()
    clocks.wait_first()
    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    t_begin = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_push("timed")  # lets a profiler select exactly the timed launches
    t_begin.record(stream)
    for i in range(args.steps):
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    t_end.record(stream)
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    clk = clocks.stop()
    barrier(world)
    total_ms = t_begin.elapsed_time(t_end)
    launch_ms = statistics.mean(s.elapsed_time(e) for s, e in zip(starts, ends))
    total_ms = max_over_ranks(total_ms, world)

    # the same step without the greedy token (the cost of the fused argmax), same graph replay
    n_plain = max(20, min(args.steps, 500))
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    p0.record(stream)
    for _ in range(n_plain):
        g_plain.replay()
    p1.record(stream)
    torch.cuda.synchronize()
    plain_ms = p0.elapsed_time(p1) / n_plain

    # end to end through the public API: pinned host x -> device, step, greedy token (and its
    # logit) -> pinned host; the H2D and D2H legs are also timed on their own
    x_host = torch.empty(W.x_all.shape, dtype=torch.float32, pin_memory=True)
    x_host.copy_(W.x_all.cpu())
    tok_host = torch.empty(1, dtype=torch.int32, pin_memory=True)
    val_host = torch.empty(1, dtype=torch.float32, pin_memory=True)

    def e2e_step():  # eager: the public call itself every step
        W.x_all.copy_(x_host, non_blocking=True)
        step_eager()
        tok_host.copy_(greedy.token, non_blocking=True)
        val_host.copy_(greedy.value, non_blocking=True)
    e_steps = max(10, min(args.steps, 500))
    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    barrier(world)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
    ev[0].record(stream)
    for _ in range(e_steps):
        e2e_step()
    ev[1].record(stream)
    for _ in range(e_steps):
        W.x_all.copy_(x_host, non_blocking=True)
    ev[2].record(stream)
    for _ in range(e_steps):
        tok_host.copy_(greedy.token, non_blocking=True)
        val_host.copy_(greedy.value, non_blocking=True)
    ev[3].record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(ev[0].elapsed_time(ev[1]), world) / e_steps
    legs = {"h2d_us": ev[1].elapsed_time(ev[2]) * 1e3 / e_steps, "d2h_us": ev[2].elapsed_time(ev[3]) * 1e3 / e_steps}
    assert int(tok_host.item()) == int(torch.argmax(W.y(head)).item())
    barrier(world)
    del g_step, g_plain
    return dict(W=W, total_ms=total_ms, launch_ms=launch_ms, clocks=clk, e2e_ms=e2e_ms, plain_ms=plain_ms,
                legs=legs, h2d=x_host.numel() * 4, d2h=4 + 4)


def time_single_q8_0(dev, seed):
    """Single Q8_0 GEMV 2048x2048: 64 distinct weight copies (285 MB, over 2x L2) rotated in a
    captured CUDA graph; reports us per call and GB/s."""
    import torch

    import block_quant_gemv_b200 as bqg
    import synth
    copies = 64
    Ws = [synth.q8_0_matrix(2048, 2048, seed, f"cfg1/copy{c}", device=dev) for c in range(copies)]
    x = synth.normal_f32(seed, synth.stream_id("cfg1/x"), 2048).to(dev)
    y = torch.empty(2048, device=dev)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        for W in Ws:
            bqg.qgemv(bqg.Q8_0, W, x, 2048, 2048, y)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for W in Ws:
            bqg.qgemv(bqg.Q8_0, W, x, 2048, 2048, y)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    reps = 20
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / (reps * copies)
    nbytes = 2048 * 64 * 34 + 4 * 2048 * 2
    return {"workload": "q8_0 2048x2048 batch 1 (64 rotating weight copies, CUDA graph)",
            "us_per_call": us, "GB/s": nbytes / us / 1e3, "bytes_per_call": nbytes}


def time_single_row_scaled(dev, seed):
    """Single packed int4 and int2 GEMVs with a per-row scale, 6144x2048 (the GLM-like expert's down
    matrix): enough distinct weight copies rotated in one graph that a rotation reads >= 256 MB."""
    import torch

    import block_quant_gemv_b200 as bqg
    import synth
    rows, cols = 6144, 2048
    out = {"workload": "packed int4 / int2 with fp32 row scales, 6144x2048, batch 1 (rotating copies, CUDA graph)"}
    x = synth.normal_f32(seed, synth.stream_id("rowscaled/x"), cols).to(dev)
    y = torch.empty(rows, device=dev)
    for name, fmt in (("i4_row", bqg.I4_ROW), ("i2_row", bqg.I2_ROW)):
        wb = synth.weight_bytes(fmt, rows, cols)
        copies = max(1, -(-(256 << 20) // wb))
        Ws = [synth.matrix(fmt, rows, cols, seed, f"rowscaled/{name}/copy{c}", device=dev) for c in range(copies)]

        def fn():
            for W in Ws:
                bqg.qgemv(fmt, W, x, rows, cols, y)
        us = graph_us(fn, reps=10) / copies
        nbytes = wb + 4 * (rows + cols)
        out[name] = {"us_per_call": us, "GB/s": nbytes / us / 1e3, "bytes_per_call": nbytes, "rotating_copies": copies}
        del Ws
    return out


def graph_us(fn, reps: int = 20) -> float:
    """Device time of fn (a sequence of library calls) captured once in a CUDA graph: warm-up
    replays, then CUDA events around `reps` replays on the capture stream."""
    import torch
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        fn()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    # replay() launches on the current stream: the events go there too
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) * 1e3 / reps


def time_prefill(dev, seed, tensor_peak):
    """Q4_0 prefill-chunk GEMM, 128 tokens x K=4096, N in (14336, 4096, 1024): enough distinct
    weight copies rotated in one graph that a rotation touches >= 256 MB (2x L2)."""
    import torch

    import block_quant_gemv_b200 as bqg
    import synth
    out = {}
    t, k = 128, 4096
    X = synth.normal_f16(seed, synth.stream_id("prefill/X"), t * k).view(t, k).to(dev)
    for n in (14336, 4096, 1024):
        wb = synth.weight_bytes(bqg.Q4_0, n, k)
        copies = max(1, -(-(256 << 20) // wb))
        Ws = [synth.q4_0_matrix(n, k, seed, f"prefill/N{n}/copy{c}", device=dev) for c in range(copies)]
        Y = torch.empty(t, n, dtype=torch.float16, device=dev)

        def fn():
            for W in Ws:
                bqg.qgemm_prefill(bqg.Q4_0, W, X, n, k, Y)
        us = graph_us(fn, reps=10) / copies
        flops = 2.0 * t * n * k
        nbytes = wb + 2 * t * k + 2 * t * n
        out[f"N{n}"] = {"us_per_call": us, "TFLOP/s": flops / us / 1e6, "tensor_frac": flops / us / 1e6 / tensor_peak,
                        "GB/s": nbytes / us / 1e3, "rotating_copies": copies}
        del Ws
    out["workload"] = "prefill chunk 128 tokens x K=4096 fp16, Q4_0 W N x 4096, fp16 out"
    out["tensor_peak_TFLOP/s"] = tensor_peak
    return out


def moe_device_layer(T):
    import block_quant_gemv_b200 as bqg
    s = T.spec
    shared = None if T.shared is None else (s.shared_fmt, s.shared_inter) + tuple(T.shared)
    return bqg.MoELayer(s.n_experts, s.top_k, s.hidden, s.inter, s.expert_fmt, s.act, T.gate, T.up, T.down,
                        T.gate_stride, T.up_stride, T.down_stride, shared)


def time_moe_gemma(dev, seed, peak, copies=8):
    """Gemma-like MoE layer (router, top-8 of 128, grouped GeGLU experts, shared expert) at
    T = 1, 16, 128: `copies` independent layers rotated in one graph (>= 2x L2 of touched bytes
    at T = 1); us per layer includes the router."""
    import torch

    import block_quant_gemv_b200 as bqg
    from synth import workloads as wl
    spec = wl.GEMMA_MOE
    Ts = [wl.build_moe_layer(spec, seed, layer=l, device=dev) for l in range(copies)]
    Ls = [moe_device_layer(T) for T in Ts]
    shared_bytes = sum(spec.shared_bytes(w) for w in ("gate", "up", "down"))
    expert_bytes = sum(spec.mat_bytes(w) for w in ("gate", "up", "down"))
    router_bytes = 4 * spec.n_experts * spec.hidden
    out = {"workload": "gemma_moe: hidden 2816, 128 experts Q4_0 GeGLU 704, top-8, shared Q8_0 GeGLU 2112, "
                       f"fp32 router; {copies} layers rotated"}
    for T in (1, 16, 128):
        x = wl.moe_tokens(spec, seed, T).to(dev)
        logits = [torch.empty(T, spec.n_experts, device=dev) for _ in Ls]
        idx = [torch.empty(T, spec.top_k, dtype=torch.int32, device=dev) for _ in Ls]
        w = [torch.empty(T, spec.top_k, device=dev) for _ in Ls]
        y = torch.empty(T, spec.hidden, device=dev)
        ws = torch.empty(bqg.moe_workspace_size(Ls[0], T), dtype=torch.uint8, device=dev)

        def fn():
            for l in range(copies):
                bqg.moe_router_logits(Ts[l].R, x, logits[l])
                bqg.moe_router_topk(logits[l], spec.top_k, idx[l], w[l])
                bqg.moe_forward(Ls[l], x, idx[l], w[l], y, ws)
        us = graph_us(fn) / copies
        distinct = sum(int(torch.unique(i).numel()) for i in idx) / copies
        nbytes = router_bytes + shared_bytes + distinct * expert_bytes + 8 * T * spec.hidden
        out[f"T{T}"] = {"us_per_layer": us, "distinct_experts": distinct, "bytes_per_layer": nbytes,
                        "GB/s": nbytes / us / 1e3, "frac": nbytes / us / 1e3 / peak}
    del Ts, Ls
    torch.cuda.empty_cache()
    return out


def time_moe_glm(dev, seed, peak):
    """GLM-like stack: 8 resident layers of 256 int4-row SwiGLU experts (38.7 GB), given N(0,1)
    logits, top-8, run back to back, each layer on its own seeded N(0,1) input; T = 1, 8, 64."""
    import torch

    import block_quant_gemv_b200 as bqg
    from synth import workloads as wl
    spec = wl.GLM_MOE
    Ts = [wl.build_moe_layer(spec, seed, layer=l, device=dev) for l in range(wl.GLM_LAYERS)]
    Ls = [moe_device_layer(T) for T in Ts]
    expert_bytes = sum(spec.mat_bytes(w) for w in ("gate", "up", "down"))
    resident = sum(T.gate.numel() + T.up.numel() + T.down.numel() for T in Ts)
    out = {"workload": f"glm_moe: {wl.GLM_LAYERS} layers x 256 int4-row experts (hidden 6144, SwiGLU 2048), "
                       f"top-8 of given N(0,1) logits, layers back to back; {resident / 1e9:.1f} GB resident"}
    for T in (1, 8, 64):
        logits = [wl.moe_logits(spec, seed, l, T).to(dev) for l in range(len(Ls))]
        idx = [torch.empty(T, spec.top_k, dtype=torch.int32, device=dev) for _ in Ls]
        w = [torch.empty(T, spec.top_k, device=dev) for _ in Ls]
        xs = [wl.moe_tokens(spec, seed, T, layer=l).to(dev) for l in range(len(Ls))]
        ys = [torch.empty(T, spec.hidden, device=dev) for _ in Ls]
        ws = torch.empty(bqg.moe_workspace_size(Ls[0], T), dtype=torch.uint8, device=dev)

        def fn():
            for l in range(len(Ls)):
                bqg.moe_router_topk(logits[l], spec.top_k, idx[l], w[l])
                bqg.moe_forward(Ls[l], xs[l], idx[l], w[l], ys[l], ws)
        us = graph_us(fn, reps=5) / len(Ls)
        distinct = sum(int(torch.unique(i).numel()) for i in idx) / len(Ls)
        nbytes = distinct * expert_bytes + 8 * T * spec.hidden + 4 * T * spec.n_experts
        out[f"T{T}"] = {"us_per_layer": us, "distinct_experts": distinct, "bytes_per_layer": nbytes,
                        "GB/s": nbytes / us / 1e3, "frac": nbytes / us / 1e3 / peak}
    del Ts, Ls
    torch.cuda.empty_cache()
    return out


def time_moe_glm_i2(dev, seed, peak, layers=8):
    """The GLM-like stack with packed int2 experts (a quarter byte per weight): 8 resident layers
    of 256 experts (19.3 GB), given N(0,1) logits, top-8, run back to back; T = 1, 8, 64."""
    import dataclasses

    import torch

    import block_quant_gemv_b200 as bqg
    from synth import workloads as wl
    spec = dataclasses.replace(wl.GLM_MOE, name="glm_i2", expert_fmt=bqg.I2_ROW)
    Ts = [wl.build_moe_layer(spec, seed, layer=l, device=dev) for l in range(layers)]
    Ls = [moe_device_layer(T) for T in Ts]
    expert_bytes = sum(spec.mat_bytes(w) for w in ("gate", "up", "down"))
    resident = sum(T.gate.numel() + T.up.numel() + T.down.numel() for T in Ts)
    out = {"workload": f"glm_moe_i2: {layers} layers x 256 packed-int2 experts (hidden 6144, SwiGLU 2048), "
                       f"top-8 of given N(0,1) logits, layers back to back; {resident / 1e9:.1f} GB resident"}
    for T in (1, 8, 64):
        logits = [wl.moe_logits(spec, seed, l, T).to(dev) for l in range(len(Ls))]
        idx = [torch.empty(T, spec.top_k, dtype=torch.int32, device=dev) for _ in Ls]
        w = [torch.empty(T, spec.top_k, device=dev) for _ in Ls]
        xs = [wl.moe_tokens(spec, seed, T, layer=l).to(dev) for l in range(len(Ls))]
        ys = [torch.empty(T, spec.hidden, device=dev) for _ in Ls]
        ws = torch.empty(bqg.moe_workspace_size(Ls[0], T), dtype=torch.uint8, device=dev)

        def fn():
            for l in range(len(Ls)):
                bqg.moe_router_topk(logits[l], spec.top_k, idx[l], w[l])
                bqg.moe_forward(Ls[l], xs[l], idx[l], w[l], ys[l], ws)
        us = graph_us(fn, reps=5) / len(Ls)
        distinct = sum(int(torch.unique(i).numel()) for i in idx) / len(Ls)
        nbytes = distinct * expert_bytes + 8 * T * spec.hidden + 4 * T * spec.n_experts
        out[f"T{T}"] = {"us_per_layer": us, "distinct_experts": distinct, "bytes_per_layer": nbytes,
                        "GB/s": nbytes / us / 1e3, "frac": nbytes / us / 1e3 / peak}
    del Ts, Ls
    torch.cuda.empty_cache()
    return out


def time_expert_cache(dev, seed, n_host=64, n_slots=16, calls=10):
    """GLM-like experts (hidden 6144, int4 SwiGLU 2048, top-8) in pinned host memory, 16 device
    slots, one token per layer: us per layer and host-to-device bytes at 100 %, 50 % and 0 % hits.
    The routing is chosen to give those hit rates: the same 8 experts every call; 4 of them kept
    plus 4 taken in turn from the other experts; 8 new experts every call (blocks of 8 in turn,
    of which the slots hold two)."""
    import dataclasses

    import torch

    import block_quant_gemv_b200 as bqg
    from synth import workloads as wl
    spec = dataclasses.replace(wl.GLM_MOE, name="cache_glm", n_experts=n_host)
    L = wl.build_moe_layer(spec, seed, 0, device="cpu")
    host = [t.pin_memory() for t in (L.gate, L.up, L.down)]

    def new_cache():  # each case starts from empty slots
        return bqg.ExpertCache(spec.n_experts, spec.top_k, spec.hidden, spec.inter, spec.expert_fmt, spec.act,
                               *host, L.gate_stride, L.up_stride, L.down_stride, n_slots)
    cache = new_cache()
    x = wl.moe_tokens(spec, seed, 1).to(dev)
    w = torch.full((1, 8), 1.0 / 8, device=dev)
    y = torch.empty(1, spec.hidden, device=dev)
    ws = torch.empty(cache.workspace_size(1), dtype=torch.uint8, device=dev)
    expert_bytes = sum(spec.mat_bytes(m) for m in ("gate", "up", "down"))

    def routing(kind, i):
        if kind == "hit100":
            e = list(range(8))
        elif kind == "hit50":
            e = list(range(4)) + [8 + (4 * i + j) % (n_host - 8) for j in range(4)]
        else:
            e = [(8 * i + j) % n_host for j in range(8)]
        return torch.tensor([e], dtype=torch.int32)

    out = {"workload": f"glm-like experts (hidden 6144, int4 SwiGLU 2048, top-8), {n_host} on the host (pinned), "
                       f"{n_slots} device slots, 1 token per layer; {calls} timed calls per case"}
    stream = torch.cuda.current_stream()
    for kind in ("hit100", "hit50", "hit0"):
        cache = new_cache()
        for i in range(calls):  # warm-up: the same sequence, so the slots hold what the timed calls expect
            cache.forward(x, routing(kind, i), w, y, ws)
        torch.cuda.synchronize()
        before = cache.stats()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(calls):
            cache.forward(x, routing(kind, i + calls), w, y, ws)
        e1.record(stream)
        torch.cuda.synchronize()
        after = cache.stats()
        us = e0.elapsed_time(e1) * 1e3 / calls
        hits = after["hits"] - before["hits"]
        misses = after["misses"] - before["misses"]
        h2d = (after["bytes_copied"] - before["bytes_copied"]) / calls
        out[kind] = {"us_per_layer": us, "hit_rate": hits / max(1, hits + misses), "h2d_bytes_per_layer": h2d,
                     "h2d_GB/s": h2d / us / 1e3, "hbm_bytes_per_layer": 8 * expert_bytes}
    del cache, host, L
    torch.cuda.empty_cache()
    return out


def run_ours(args, world, rank, local):
    import torch
    assert torch.cuda.is_available(), "bench.py --impl ours needs a CUDA device"
    import block_quant_gemv_b200 as bqg
    bqg.lib()
    dev = torch.device("cuda", torch.cuda.current_device())
    peak, peak_kind = peaks()

    r = time_decode_step(args, world, dev)
    W = r["W"]
    step_bytes = W.weight_bytes + W.activation_bytes
    ms = r["total_ms"] / args.steps
    value = world * step_bytes / (ms * 1e-3) / 1e9
    achieved = step_bytes / (r["launch_ms"] * 1e-3) / 1e9
    e2e_gbs = world * step_bytes / (r["e2e_ms"] * 1e-3) / 1e9

    extras = {}
    if not args.no_extras:
        extras["q8_0_2048"] = time_single_q8_0(dev, args.seed)
        extras["row_scaled_6144x2048"] = time_single_row_scaled(dev, args.seed)
        extras["prefill"] = time_prefill(dev, args.seed, tensor_peak())
        extras["moe_gemma"] = time_moe_gemma(dev, args.seed, peak)
        if not args.no_glm:
            extras["moe_glm"] = time_moe_glm(dev, args.seed, peak)
            extras["moe_glm_i2"] = time_moe_glm_i2(dev, args.seed, peak)
        extras["expert_cache_glm"] = time_expert_cache(dev, args.seed)
    extras["decode_step_without_greedy_token"] = {
        "ms_per_step": r["plain_ms"], "GB/s": step_bytes / (r["plain_ms"] * 1e-3) / 1e9,
        "argmax_cost_frac": r["launch_ms"] / r["plain_ms"] - 1.0}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu, cpu_all, cpu_extra = cpu_baselines(args)
        cpu = dict(cpu, all_cores=cpu_all)
        extras["cpu_oracle"] = cpu_extra

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None,
            "dtype": "q4_0/q8_0 weights x fp32 activations held as 16-bit fixed point per 32/64 values inside "
                     "the kernel (exact int32 block sums), fp32 accumulate",
            "data": "synthetic", "config": workload_config(),
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "peak_kind": peak_kind, "traffic": committed_traffic(),
                         "kernel": "k_qgemv (qgemv_batched, 155 matrices)",
                         "algorithmic_bytes_per_launch": step_bytes},
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_gbs, "unit": UNIT, "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"],
                    "ms_per_step": r["e2e_ms"], "legs": r["legs"],
                    "result": "greedy token and its logit (8 bytes) read back every step"},
            "gpu_launches": args.steps,
            "clocks": r["clocks"],
            "extras": extras,
        }
        print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
