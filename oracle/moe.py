"""Oracle: routed Mixture-of-Experts layer built on the block-quantized GEMVs, in float64.

Sources (page, section):
* 128 routed experts, top-8 per token, plus a dense shared expert branch —
  TurboFieldfare wiki, "메모리·전문가 스트리밍"; Camelid README, "Gemma 4"
  (dense shared-expert + sparse top-8 branch of the 26B-A4B row).
* 256 routed experts per MoE layer, int4 experts of about 19 MB — colibri wiki
  summary, "핵심 아이디어".
* GeGLU expert FFN — Camelid README, "Gemma 4" (list of implemented pieces).
* An exact expert-probability tie goes to the lower expert index — Camelid README,
  "Windows bring-up, perf & GPU" paragraph under "Experimental lanes".

Readings taken where the pages are silent:
* Router: logits l = R x; p = softmax(l) over all E experts; the selected set S is the
  k largest logits (ties to the lower index), listed in descending-logit order;
  weights w_j = p_{S_j} / sum_{S} p.  Ranking is done on the logits themselves, which in
  exact arithmetic orders experts exactly as p does.
* GeGLU uses the tanh form of GELU: 0.5 g (1 + tanh(sqrt(2/pi) (g + 0.044715 g^3)));
  the SwiGLU variant uses SiLU(g) = g / (1 + exp(-g)).
* Expert FFN: h = act(G x) * (U x), out = D h.  The shared expert's output is added
  with weight 1.  Norms and the residual are not part of the layer output.
* A stack of layers is chained: the next layer's input is this layer's output.

This module is test infrastructure: only tests, the smoke check and the
benchmark's CPU-baseline leg call it.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Callable, Optional

import numpy as np

from .qgemv import dequantize

ACT_GELU_TANH, ACT_SILU = 1, 2


def router_logits(R: np.ndarray, x: np.ndarray) -> np.ndarray:
    """l[t, e] = sum_h R[e, h] x[t, h] in float64.  R is [E, H], x is [T, H]."""
    return np.asarray(x, np.float64) @ np.asarray(R, np.float64).T


def topk_select(logits: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest logits per token, in descending order; equal logits are
    ordered by lower index first.  A full sort of the (-logit, index) pairs."""
    logits = np.asarray(logits)
    T, E = logits.shape
    idx = np.empty((T, k), dtype=np.int32)
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-float(logits[t, e]), e))
        idx[t] = order[:k]
    return idx


def softmax(l: np.ndarray) -> np.ndarray:
    """Softmax over the last axis in float64 (max subtracted before exponentiating)."""
    l = np.asarray(l, np.float64)
    z = np.exp(l - l.max(axis=-1, keepdims=True))
    return z / z.sum(axis=-1, keepdims=True)


def topk_weights(logits: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """w[t, j] = p[t, idx[t, j]] / sum_j' p[t, idx[t, j']] with p the softmax over all experts."""
    p = softmax(logits)
    sel = np.take_along_axis(p, np.asarray(idx, np.int64), axis=1)
    return sel / sel.sum(axis=1, keepdims=True)


def router_topk(logits: np.ndarray, k: int):
    """(idx int32 [T, k], w float64 [T, k]) for logits [T, E]."""
    idx = topk_select(logits, k)
    return idx, topk_weights(logits, idx)


def gelu_tanh(g):
    g = np.asarray(g, np.float64)
    return 0.5 * g * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (g + 0.044715 * g ** 3)))


def silu(g):
    g = np.asarray(g, np.float64)
    return g / (1.0 + np.exp(-g))


def activation(act: int):
    if act == ACT_GELU_TANH:
        return gelu_tanh
    if act == ACT_SILU:
        return silu
    raise ValueError(f"unknown activation {act}")


@dataclass
class Expert:
    """One gated FFN: gate and up are [inter, hidden], down is [hidden, inter] (raw bytes)."""
    fmt: int
    gate: np.ndarray
    up: np.ndarray
    down: np.ndarray


@dataclass
class Layer:
    n_experts: int
    top_k: int
    hidden: int
    inter: int
    act: int
    expert: Callable[[int], Expert]            # expert id -> its bytes (may regenerate lazily)
    shared: Optional[Expert] = None
    shared_inter: int = 0


def ffn_dense(ex: Expert, inter: int, hidden: int, act: int, X: np.ndarray) -> np.ndarray:
    """Gated FFN applied to the rows of X [n, hidden]: D (act(G x) * (U x)) per row, float64."""
    G = dequantize(ex.fmt, ex.gate, inter, hidden)
    U = dequantize(ex.fmt, ex.up, inter, hidden)
    D = dequantize(ex.fmt, ex.down, hidden, inter)
    X = np.asarray(X, np.float64).reshape(-1, hidden)
    h = activation(act)(X @ G.T) * (X @ U.T)
    return h @ D.T


def moe_layer(L: Layer, x: np.ndarray, idx: np.ndarray, w: np.ndarray,
              with_shared: bool = True) -> np.ndarray:
    """y_t = sum_{j=0..k-1} w[t, j] FFN_{idx[t, j]}(x_t) (+ shared FFN(x_t)), float64 [T, hidden].

    Each touched expert is dequantized once and applied to the tokens routed to it;
    the per-(token, slot) outputs are then summed over slots in slot order."""
    x = np.asarray(x, np.float64).reshape(-1, L.hidden)
    T, k = np.asarray(idx).shape
    out = np.zeros((T, k, L.hidden))
    for e in sorted(set(int(v) for v in np.asarray(idx).reshape(-1))):
        pairs = [(t, j) for t in range(T) for j in range(k) if int(idx[t, j]) == e]
        res = ffn_dense(L.expert(e), L.inter, L.hidden, L.act, x[[t for t, _ in pairs]])
        for n, (t, j) in enumerate(pairs):
            out[t, j] = res[n]
    y = np.zeros((T, L.hidden))
    for j in range(k):
        y += np.asarray(w, np.float64)[:, j:j + 1] * out[:, j]
    if with_shared and L.shared is not None:
        y += ffn_dense(L.shared, L.shared_inter, L.hidden, L.act, x)
    return y


def moe_stack(layers, x: np.ndarray, logits_per_layer) -> np.ndarray:
    """Chained layers: route layer l on its given logits, feed its output to layer l+1."""
    h = np.asarray(x, np.float64)
    for L, lg in zip(layers, logits_per_layer):
        idx, w = router_topk(lg, L.top_k)
        h = moe_layer(L, h, idx, w)
    return h
