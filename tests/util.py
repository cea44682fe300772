"""Shared helpers for the parity tests."""
import numpy as np
import torch

REL_TOL = 2e-3   # max|y - y_ref| <= REL_TOL * max|y_ref|  (float outputs)


def max_rel_err(y, y_ref) -> float:
    y = np.asarray(y.detach().cpu().numpy() if isinstance(y, torch.Tensor) else y, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    scale = np.max(np.abs(y_ref))
    if scale == 0:
        return float(np.max(np.abs(y)))
    return float(np.max(np.abs(y - y_ref)) / scale)


def assert_close(y, y_ref, tol: float = REL_TOL, what: str = ""):
    e = max_rel_err(y, y_ref)
    assert e <= tol, f"{what}: max|y - y_ref| / max|y_ref| = {e:.3e} > {tol:.1e}"
    return e


def need_gpu():
    if not torch.cuda.is_available():
        raise RuntimeError("this test needs a CUDA device (run with -m 'not gpu' on a CPU-only machine)")
