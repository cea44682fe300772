"""Oracle: the prefill-chunk product Y = X W^T with Q4_0 weights, in float64, rounded once to fp16.

Source (page, section): TurboFieldfare wiki, "메모리·전문가 스트리밍" — prefill runs in
chunks of at most 128 tokens so that each weight read serves every prompt row of the
chunk; Camelid README, "Engine status" (GPU-resident single-shot prefill).

Reading taken: X is fp16 [tokens, k] (row-major), W is a Q4_0 matrix [n, k] in the
block layout of oracle.qgemv, Y[t, j] = sum_i X[t, i] W[j, i] computed exactly enough
in float64 and rounded to fp16 with round-to-nearest-even.

This module is test infrastructure: only tests, the smoke check and the
benchmark's CPU-baseline leg call it.
"""
from __future__ import annotations

import numpy as np

from .qgemv import dequantize


def prefill_f64(fmt: int, W: np.ndarray, X: np.ndarray, n: int, k: int) -> np.ndarray:
    Wd = dequantize(fmt, W, n, k)
    X = np.asarray(X, dtype=np.float16).astype(np.float64).reshape(-1, k)
    return X @ Wd.T


def prefill(fmt: int, W: np.ndarray, X: np.ndarray, n: int, k: int) -> np.ndarray:
    """fp16 [tokens, n]."""
    return prefill_f64(fmt, W, X, n, k).astype(np.float16)
