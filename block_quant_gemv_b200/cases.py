"""Runs one hot-path case a few times on cuda:0, for profilers (ncu) and quick timing.

    python -m block_quant_gemv_b200.cases decode  [--layers 22] [--argmax] [--iters 5]
    python -m block_quant_gemv_b200.cases prefill [--tokens 128] [--n 14336] [--k 4096] [--iters 5]
    python -m block_quant_gemv_b200.cases moe gemma|glm [--tokens 1] [--experts E] [--path P] [--iters 5]

decode:  one TinyLlama-shape decode step (7 Q4_0 projections per layer + the Q8_0 LM head),
         all matrices in one qgemv_batched launch per call.
prefill: qgemm_prefill of a Q4_0 [n x k] matrix with fp16 X [tokens x k].
moe:     one routed-expert layer: (router logits for the Gemma-like layer,) top-k routing
         and moe_forward; the GLM-like layer takes N(0,1) logits.
Inputs are the seeded synthetic tensors of the benchmark (seed 0).  Prints the mean time per
call (CUDA events, after two warm-up calls) and the device error bits.
"""
from __future__ import annotations

import argparse
import dataclasses
import os
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import block_quant_gemv_b200 as bqg  # noqa: E402
import synth  # noqa: E402
from synth import workloads as wl  # noqa: E402


def _time(fn, iters: int) -> float:
    for _ in range(2):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(iters):
        fn()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) * 1e3 / iters


def decode(args) -> str:
    W = wl.build_gemv_workload(wl.decode_step_specs(args.layers), seed=0, device="cuda")
    batch = bqg.GemvBatch(W.items())
    if args.argmax:  # the greedy token of the LM head (the last descriptor) in the same launch
        out = bqg.ArgmaxState("cuda")
        head = len(W.specs) - 1
        us = _time(lambda: batch.run(argmax=(head, out)), args.iters)
    else:
        us = _time(batch.run, args.iters)
    return (f"decode step ({args.layers} layers + head{' + greedy token' if args.argmax else ''}, "
            f"{W.weight_bytes} weight bytes): {us:.1f} us per call")


def prefill(args) -> str:
    t, n, k = args.tokens, args.n, args.k
    W = synth.q4_0_matrix(n, k, 0, f"prefill/N{n}/copy0", device="cuda")
    X = synth.normal_f16(0, synth.stream_id("prefill/X"), t * k).view(t, k).cuda()
    Y = torch.empty(t, n, dtype=torch.float16, device="cuda")
    us = _time(lambda: bqg.qgemm_prefill(bqg.Q4_0, W, X, n, k, Y), args.iters)
    return f"prefill {t}x{n}x{k}: {us:.1f} us per call, {2.0 * t * n * k / us / 1e6:.1f} TFLOP/s"


def moe(args) -> str:
    spec = wl.GEMMA_MOE if args.layer == "gemma" else wl.GLM_MOE
    if args.experts:  # the same layer geometry with fewer routed experts (a smaller footprint)
        spec = dataclasses.replace(spec, n_experts=args.experts)
    T = wl.build_moe_layer(spec, 0, layer=0, device="cuda")
    shared = None if T.shared is None else (spec.shared_fmt, spec.shared_inter) + tuple(T.shared)
    L = bqg.MoELayer(spec.n_experts, spec.top_k, spec.hidden, spec.inter, spec.expert_fmt, spec.act, T.gate, T.up,
                     T.down, T.gate_stride, T.up_stride, T.down_stride, shared, path=args.path)
    tok = args.tokens
    x = wl.moe_tokens(spec, 0, tok).cuda()
    logits = (torch.empty(tok, spec.n_experts, device="cuda") if spec.router
              else wl.moe_logits(spec, 0, 0, tok).cuda())
    idx = torch.empty(tok, spec.top_k, dtype=torch.int32, device="cuda")
    w = torch.empty(tok, spec.top_k, device="cuda")
    y = torch.empty(tok, spec.hidden, device="cuda")
    ws = torch.empty(bqg.moe_workspace_size(L, tok), dtype=torch.uint8, device="cuda")

    def step():
        if spec.router:
            bqg.moe_router_logits(T.R, x, logits)
        bqg.moe_router_topk(logits, spec.top_k, idx, w)
        bqg.moe_forward(L, x, idx, w, y, ws)
    us = _time(step, args.iters)
    return f"moe {spec.name} T={tok}: {us:.1f} us per layer (router included)"


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    sub = ap.add_subparsers(dest="case", required=True)
    d = sub.add_parser("decode")
    d.add_argument("--layers", type=int, default=22)
    d.add_argument("--argmax", action="store_true", help="also compute the greedy token of the LM head")
    p = sub.add_parser("prefill")
    p.add_argument("--tokens", type=int, default=128)
    p.add_argument("--n", type=int, default=14336)
    p.add_argument("--k", type=int, default=4096)
    m = sub.add_parser("moe")
    m.add_argument("layer", choices=["gemma", "glm"])
    m.add_argument("--tokens", type=int, default=1)
    m.add_argument("--experts", type=int, default=0, help="routed experts (default: the layer's own count)")
    m.add_argument("--path", type=int, default=0, help="0 automatic, 1 CUDA cores, 2 tensor cores")
    for s in (d, p, m):
        s.add_argument("--iters", type=int, default=5)
    args = ap.parse_args(argv)
    assert torch.cuda.is_available(), "needs a CUDA device"
    torch.cuda.set_device(0)
    bqg.lib()
    msg = {"decode": decode, "prefill": prefill, "moe": moe}[args.case](args)
    torch.cuda.synchronize()
    print(msg)
    print("device errors:", bqg.bqg_device_errors())


if __name__ == "__main__":
    main()
