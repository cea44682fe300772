"""Oracle: greedy token selection after the LM head (argmax of the logits), in plain Python.

Sources (page, section): Camelid README, "At a glance" (the "Apple Silicon path" row: GPU
decode with on-GPU greedy sampling) and "Supported models" (the first decoded token is the
argmax of the head's logits, compared against a CPU oracle).

Readings taken where the pages are silent:
* Greedy sampling picks the index of the largest logit.
* Logits are compared as IEEE values, so -0.0 and +0.0 are equal; among equal largest
  logits the lower index is chosen (the same tie rule the pages state for expert routing).
* Logits are finite (a precondition, as for every input of the path).
* The argmax is taken on the logits the head produced, in their own precision: a test gives
  this function the GPU's fp32 logits to check the GPU's index bit-exactly, and the float64
  oracle logits to check the head itself.

This module is test infrastructure: only tests, the smoke check and the benchmark's
CPU-baseline leg call it.
"""
from __future__ import annotations

import numpy as np

from .qgemv import qgemv


def argmax_lower(v) -> int:
    """Index of the largest value of v; equal largest values go to the lower index."""
    v = np.asarray(v).reshape(-1)
    if v.size == 0:
        raise ValueError("argmax of an empty vector")
    best = 0
    for i in range(1, v.size):
        if v[i] > v[best]:          # strictly greater: an equal value keeps the earlier index
            best = i
    return best


def lm_head_greedy(fmt: int, W, x, rows: int, cols: int):
    """(token, max logit) of the quantized LM head applied to x, in float64."""
    logits = qgemv(fmt, W, x, rows, cols)
    t = argmax_lower(logits)
    return t, float(logits[t])
