"""Shapes of the synthetic workloads and builders for their seeded inputs.

The shapes stand in for the models the pages run (no model files are used):
* "q8_0_2048": one Q8_0 GEMV, W 2048 x 2048, x ~ N(0, 1)  (a Q8_0 projection of a
  TinyLlama-class model; Camelid README, "Supported models").
* "tinyllama_decode": one decode step's projections at TinyLlama-1.1B shape, batch 1:
  22 layers of Q4_0 q/o 2048x2048, k/v 256x2048, gate/up 5632x2048, down 2048x5632, and a
  Q8_0 LM head 32000x2048 (token-major rows; Camelid README, "Under the hood").  Each
  projection input is a fresh N(0, 1) vector: q/k/v share one, gate/up share one.
* MoE layers and the prefill chunk: see moe_workloads / prefill shapes below.

Nothing here computes any part of the method; it only draws inputs (see synth).
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional

import torch

from . import (FMT_I4_ROW, FMT_Q4_0, FMT_Q8_0, matrix, normal_f32, stream_id, weight_bytes)

TINYLLAMA = dict(hidden=2048, kv=256, inter=5632, layers=22, vocab=32000)


@dataclass
class GemvSpec:
    name: str
    fmt: int
    rows: int
    cols: int
    x_name: str


def decode_step_specs(layers: int = TINYLLAMA["layers"]) -> List[GemvSpec]:
    """The 7 projections of every layer (Q4_0) plus the Q8_0 LM head, in execution order."""
    H, KV, I = TINYLLAMA["hidden"], TINYLLAMA["kv"], TINYLLAMA["inter"]
    out = []
    for l in range(layers):
        p = f"tl/L{l}/"
        out += [GemvSpec(p + "q", FMT_Q4_0, H, H, p + "attn_in"),
                GemvSpec(p + "k", FMT_Q4_0, KV, H, p + "attn_in"),
                GemvSpec(p + "v", FMT_Q4_0, KV, H, p + "attn_in"),
                GemvSpec(p + "o", FMT_Q4_0, H, H, p + "o_in"),
                GemvSpec(p + "gate", FMT_Q4_0, I, H, p + "mlp_in"),
                GemvSpec(p + "up", FMT_Q4_0, I, H, p + "mlp_in"),
                GemvSpec(p + "down", FMT_Q4_0, H, I, p + "down_in")]
    out.append(GemvSpec("tl/head", FMT_Q8_0, TINYLLAMA["vocab"], H, "tl/head_in"))
    return out


@dataclass
class GemvWorkload:
    """Device tensors of a list of independent GEMVs: one uint8 buffer per matrix, all x
    vectors in one fp32 buffer and all y vectors in another (so host<->device transfers of a
    step are one copy each way)."""
    specs: List[GemvSpec]
    W: List[torch.Tensor]
    x_all: torch.Tensor
    y_all: torch.Tensor
    x_off: dict = field(default_factory=dict)   # x_name -> (offset, length)
    y_off: List[tuple] = field(default_factory=list)

    def x(self, name):
        o, n = self.x_off[name]
        return self.x_all[o:o + n]

    def y(self, i):
        o, n = self.y_off[i]
        return self.y_all[o:o + n]

    def items(self):
        return [(s.fmt, self.W[i], self.x(s.x_name), self.y(i), s.rows, s.cols) for i, s in enumerate(self.specs)]

    @property
    def weight_bytes(self) -> int:
        return sum(weight_bytes(s.fmt, s.rows, s.cols) for s in self.specs)

    @property
    def activation_bytes(self) -> int:
        return 4 * (self.x_all.numel() + self.y_all.numel())


def _pad4(n: int) -> int:
    return (n + 3) // 4 * 4          # keep every vector 16-byte aligned


def build_gemv_workload(specs: List[GemvSpec], seed: int, device="cuda") -> GemvWorkload:
    x_off, off = {}, 0
    for s in specs:
        if s.x_name not in x_off:
            x_off[s.x_name] = (off, s.cols)
            off += _pad4(s.cols)
    x_host = torch.zeros(off, dtype=torch.float32)
    for name, (o, n) in x_off.items():
        x_host[o:o + n] = normal_f32(seed, stream_id(name), n)
    y_off, yo = [], 0
    for s in specs:
        y_off.append((yo, s.rows))
        yo += _pad4(s.rows)
    W = [matrix(s.fmt, s.rows, s.cols, seed, s.name, device=device) for s in specs]
    return GemvWorkload(specs, W, x_host.to(device), torch.zeros(yo, dtype=torch.float32, device=device),
                        x_off, y_off)


def x_host(specs: List[GemvSpec], name: str, seed: int) -> torch.Tensor:
    """The host copy of one named input vector (identical to the workload's device copy)."""
    cols = next(s.cols for s in specs if s.x_name == name)
    return normal_f32(seed, stream_id(name), cols)


# ---------------------------------------------------------------- MoE layers
@dataclass
class MoESpec:
    """Shape of one routed-expert layer (see the MoE configurations)."""
    name: str
    n_experts: int
    top_k: int
    hidden: int
    inter: int
    expert_fmt: int
    act: int                      # 1 GeGLU (tanh GELU), 2 SwiGLU
    shared_inter: int = 0
    shared_fmt: int = 0
    router: bool = True           # fp32 router matrix R ~ N(0, 0.02); else logits are given

    def mat_bytes(self, which: str) -> int:
        if which == "down":
            return weight_bytes(self.expert_fmt, self.hidden, self.inter)
        return weight_bytes(self.expert_fmt, self.inter, self.hidden)

    def shared_bytes(self, which: str) -> int:
        if which == "down":
            return weight_bytes(self.shared_fmt, self.hidden, self.shared_inter)
        return weight_bytes(self.shared_fmt, self.shared_inter, self.hidden)


# Gemma-4-26B-A4B-like layer: hidden 2816, 128 experts, top-8, GeGLU experts of 704 in Q4_0,
# shared dense GeGLU expert of 2112 in Q8_0, fp32 router 128 x 2816.
GEMMA_MOE = MoESpec("gemma_moe", 128, 8, 2816, 704, FMT_Q4_0, 1, 2112, FMT_Q8_0, True)
# GLM-style layer: hidden 6144, 256 experts, top-8, SwiGLU experts of 2048 in packed int4 with
# fp32 row scales, no shared expert, logits given (N(0,1)); 8 such layers are stacked, resident
# together, and run back to back, each on its own seeded N(0,1) input (feeding a layer's output
# straight into the next, with no norm in between, overflows fp32 by the fifth layer).
GLM_MOE = MoESpec("glm_moe", 256, 8, 6144, 2048, FMT_I4_ROW, 2, 0, 0, False)
GLM_LAYERS = 8


def _align16(n: int) -> int:
    return (n + 15) // 16 * 16


def expert_matrix(spec: MoESpec, seed: int, layer: int, e: int, which: str, device="cpu") -> torch.Tensor:
    rows, cols = (spec.hidden, spec.inter) if which == "down" else (spec.inter, spec.hidden)
    return matrix(spec.expert_fmt, rows, cols, seed, f"{spec.name}/L{layer}/E{e}/{which}", device=device)


def shared_matrix(spec: MoESpec, seed: int, layer: int, which: str, device="cpu") -> torch.Tensor:
    rows, cols = (spec.hidden, spec.shared_inter) if which == "down" else (spec.shared_inter, spec.hidden)
    return matrix(spec.shared_fmt, rows, cols, seed, f"{spec.name}/L{layer}/shared/{which}", device=device)


@dataclass
class MoETensors:
    spec: MoESpec
    gate: torch.Tensor            # [E * stride] bytes, expert e at e * stride
    up: torch.Tensor
    down: torch.Tensor
    gate_stride: int
    up_stride: int
    down_stride: int
    shared: Optional[tuple] = None  # (s_gate, s_up, s_down)
    R: Optional[torch.Tensor] = None


def build_moe_layer(spec: MoESpec, seed: int, layer: int = 0, device="cuda") -> MoETensors:
    """All experts of one layer stacked per family (each expert padded to 16 bytes)."""
    strides = {w: _align16(spec.mat_bytes(w)) for w in ("gate", "up", "down")}
    fam = {}
    for w in ("gate", "up", "down"):
        t = torch.zeros(spec.n_experts * strides[w], dtype=torch.uint8, device=device)
        n = spec.mat_bytes(w)
        for e in range(spec.n_experts):
            t[e * strides[w]: e * strides[w] + n] = expert_matrix(spec, seed, layer, e, w, device=device)
        fam[w] = t
    shared = None
    if spec.shared_inter:
        shared = tuple(shared_matrix(spec, seed, layer, w, device=device) for w in ("gate", "up", "down"))
    R = None
    if spec.router:
        R = normal_f32(seed, stream_id(f"{spec.name}/L{layer}/router"), spec.n_experts * spec.hidden,
                       std=0.02).view(spec.n_experts, spec.hidden).to(device)
    return MoETensors(spec, fam["gate"], fam["up"], fam["down"], strides["gate"], strides["up"], strides["down"],
                      shared, R)


def moe_tokens(spec: MoESpec, seed: int, tokens: int, layer: Optional[int] = None) -> torch.Tensor:
    """Host fp32 activations x ~ N(0, 1), [tokens, hidden]; with `layer`, the input of that
    layer of a stack (each layer of the stack takes its own seeded input)."""
    name = f"{spec.name}/x/T{tokens}" if layer is None else f"{spec.name}/L{layer}/x/T{tokens}"
    return normal_f32(seed, stream_id(name), tokens * spec.hidden).view(tokens, spec.hidden)


def moe_logits(spec: MoESpec, seed: int, layer: int, tokens: int) -> torch.Tensor:
    """Host fp32 router logits ~ N(0, 1), [tokens, n_experts] (for layers whose logits are given)."""
    return normal_f32(seed, stream_id(f"{spec.name}/L{layer}/logits/T{tokens}"),
                      tokens * spec.n_experts).view(tokens, spec.n_experts)
