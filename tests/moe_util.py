"""Helpers shared by the MoE parity tests: device layers from the synthetic builders and the
matching oracle layers (whose expert bytes are regenerated on the host, independently)."""
import numpy as np

import block_quant_gemv_b200 as bqg
from synth import workloads as wl
from oracle import moe as om


def device_layer(T: wl.MoETensors, with_shared: bool = True) -> bqg.MoELayer:
    s = T.spec
    shared = None
    if with_shared and T.shared is not None:
        shared = (s.shared_fmt, s.shared_inter) + tuple(T.shared)
    return bqg.MoELayer(s.n_experts, s.top_k, s.hidden, s.inter, s.expert_fmt, s.act, T.gate, T.up, T.down,
                        T.gate_stride, T.up_stride, T.down_stride, shared)


def oracle_layer(spec: wl.MoESpec, seed: int, layer: int = 0, with_shared: bool = True) -> om.Layer:
    cache = {}

    def expert(e):
        if e not in cache:
            cache[e] = om.Expert(spec.expert_fmt,
                                 *[wl.expert_matrix(spec, seed, layer, e, w).numpy() for w in ("gate", "up", "down")])
        return cache[e]

    shared = None
    if with_shared and spec.shared_inter:
        shared = om.Expert(spec.shared_fmt, *[wl.shared_matrix(spec, seed, layer, w).numpy()
                                              for w in ("gate", "up", "down")])
    return om.Layer(spec.n_experts, spec.top_k, spec.hidden, spec.inter, spec.act, expert, shared,
                    spec.shared_inter if shared is not None else 0)


def oracle_router_logits(spec: wl.MoESpec, seed: int, layer: int, x: np.ndarray) -> np.ndarray:
    R = wl.normal_f32(seed, wl.stream_id(f"{spec.name}/L{layer}/router"), spec.n_experts * spec.hidden,
                      std=0.02).view(spec.n_experts, spec.hidden).numpy()
    return om.router_logits(R, x)


def tc_shapes_ok(spec: wl.MoESpec) -> bool:
    """Whether a tensor-core variant takes the layer (mirrors include/bqg.h): kind::i8 for int4 /
    int2 families with every dimension a multiple of 128, kind::f16 for layers without int2 with
    every dimension a multiple of 64."""
    dims = [spec.hidden, spec.inter] + ([spec.shared_inter] if spec.shared_inter else [])
    fmts = [spec.expert_fmt] + ([spec.shared_fmt] if spec.shared_inter else [])
    if all(f in (bqg.I4_ROW, bqg.I2_ROW) for f in fmts) and not any(d % 128 for d in dims):
        return True
    return bqg.I2_ROW not in fmts and not any(d % 64 for d in dims)


def expected_path(spec: wl.MoESpec, tokens: int) -> int:
    """The path the library's automatic choice takes for this layer: the tensor cores from
    MOE_TC_MIN_TOKENS tokens on when a variant takes the shapes, else the CUDA cores."""
    if tokens >= bqg.MOE_TC_MIN_TOKENS and tc_shapes_ok(spec):
        return bqg.MOE_PATH_TENSOR_CORES
    return bqg.MOE_PATH_CUDA_CORES
