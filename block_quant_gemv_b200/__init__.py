"""Python binding of libbqg.so — block-quantized GEMV, MoE layer and prefill GEMM on B200.

Argument marshalling only: every step of the computation runs in the library's CUDA
kernels.  PyTorch provides device memory and the current stream.  There is no CPU
fallback: if the library is not built, every call raises.

The functions mirror the C ABI in include/bqg.h (same names):
    qgemv, qgemv_batched, qgemv_argmax, qgemv_batched_argmax (GemvBatch.run(argmax=...)),
    qgemm_prefill, moe_router_logits, moe_router_topk,
    moe_workspace_size, moe_forward, moe_forward_noalloc, bqg_status_string, bqg_weight_bytes,
    bqg_device_errors, bqg_selftest_wait_timeout
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

__all__ = [
    "Q8_0", "Q4_0", "I4_ROW", "ACT_GELU_TANH", "ACT_SILU", "BQGError",
    "MOE_PATH_AUTO", "MOE_PATH_CUDA_CORES", "MOE_PATH_TENSOR_CORES",
    "lib", "library_path", "bqg_status_string", "bqg_weight_bytes", "bqg_device_errors",
    "bqg_selftest_wait_timeout",
    "qgemv", "qgemv_batched", "GemvBatch", "qgemv_argmax", "ArgmaxState", "qgemm_prefill", "moe_router_logits",
    "moe_router_topk", "MoELayer", "moe_workspace_size", "moe_forward", "moe_forward_noalloc", "ExpertCache",
]

Q8_0, Q4_0, I4_ROW, I2_ROW = 1, 2, 3, 4
ACT_GELU_TANH, ACT_SILU = 1, 2
MOE_PATH_AUTO, MOE_PATH_CUDA_CORES, MOE_PATH_TENSOR_CORES = 0, 1, 2
MOE_TC_MIN_TOKENS = 8
MAX_COLS, MAX_BATCH, MAX_EXPERTS, MAX_TOPK, MAX_MOE_COLS = 15360, 256, 256, 8, 7168
DEVERR_TIMEOUT, DEVERR_EXPERT_ID = 0x1, 0x2

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libbqg.so")
_lib: Optional[ctypes.CDLL] = None

_vp, _i, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t


class BQGError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {bqg_status_string(status)} ({status})" if what else bqg_status_string(status))


class GemvDesc(ctypes.Structure):
    _fields_ = [("fmt", _i), ("rows", _i), ("cols", _i), ("reserved", _i),
                ("W", _vp), ("x", _vp), ("y", _vp)]


class MoELayerC(ctypes.Structure):
    _fields_ = [("n_experts", _i), ("top_k", _i), ("hidden", _i), ("inter", _i),
                ("expert_fmt", _i), ("act", _i),
                ("gate", _vp), ("up", _vp), ("down", _vp),
                ("gate_stride", _sz), ("up_stride", _sz), ("down_stride", _sz),
                ("shared_inter", _i), ("shared_fmt", _i),
                ("s_gate", _vp), ("s_up", _vp), ("s_down", _vp), ("path", _i)]


class ExpertCacheDesc(ctypes.Structure):
    _fields_ = [("layer", MoELayerC), ("n_slots", _i), ("slot_gate", _vp), ("slot_up", _vp), ("slot_down", _vp)]


class ExpertCacheStats(ctypes.Structure):
    _fields_ = [("calls", ctypes.c_longlong), ("hits", ctypes.c_longlong), ("misses", ctypes.c_longlong),
                ("evictions", ctypes.c_longlong), ("bytes_copied", ctypes.c_longlong)]


_SIGNATURES = {
    "bqg_status_string": (ctypes.c_char_p, [_i]),
    "bqg_version": (_i, []),
    "bqg_weight_bytes": (_sz, [_i, _i, _i]),
    "bqg_device_errors": (_i, [ctypes.POINTER(_i)]),
    "qgemv": (_i, [_i, _vp, _vp, _vp, _i, _i, _vp]),
    "qgemv_batched": (_i, [ctypes.POINTER(GemvDesc), _i, _vp]),
    "qgemv_argmax": (_i, [_i, _vp, _vp, _vp, _i, _i, _vp, _vp, _vp, _vp]),
    "qgemv_batched_argmax": (_i, [ctypes.POINTER(GemvDesc), _i, _i, _vp, _vp, _vp, _vp]),
    "qgemm_prefill": (_i, [_i, _vp, _vp, _vp, _i, _i, _i, _vp]),
    "moe_router_logits": (_i, [_vp, _vp, _vp, _i, _i, _i, _vp]),
    "moe_router_topk": (_i, [_vp, _i, _i, _i, _vp, _vp, _vp]),
    "moe_workspace_size": (_sz, [ctypes.POINTER(MoELayerC), _i]),
    "moe_forward": (_i, [ctypes.POINTER(MoELayerC), _vp, _vp, _vp, _vp, _i, _vp, _sz, _vp]),
    "moe_forward_noalloc": (_i, [ctypes.POINTER(MoELayerC), _vp, _vp, _vp, _vp, _i, _vp]),
    "bqg_selftest_wait_timeout": (_i, [_vp]),
    "bqg_expert_cache_create": (_i, [ctypes.POINTER(ExpertCacheDesc), ctypes.POINTER(_vp)]),
    "bqg_expert_cache_destroy": (None, [_vp]),
    "bqg_expert_cache_workspace_size": (_sz, [_vp, _i]),
    "bqg_expert_cache_forward": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _vp, _sz, _vp, _vp]),
    "bqg_expert_cache_get_stats": (_i, [_vp, ctypes.POINTER(ExpertCacheStats)]),
}


def library_path() -> str:
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    """The loaded library.  Raises if it has not been built (no fallback exists)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"{_LIB_PATH} is not built; run `python -m block_quant_gemv_b200.build` "
                               "(the CUDA library is required; there is no CPU fallback)")
        L = ctypes.CDLL(_LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            f = getattr(L, name, None)
            if f is None:
                continue
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def bqg_status_string(status: int) -> str:
    return lib().bqg_status_string(int(status)).decode()


def bqg_weight_bytes(fmt: int, rows: int, cols: int) -> int:
    return int(lib().bqg_weight_bytes(fmt, rows, cols))


def bqg_device_errors() -> int:
    """Reads and clears the device error bits (synchronises the device)."""
    bits = _i(0)
    _check(lib().bqg_device_errors(ctypes.byref(bits)), "bqg_device_errors")
    return int(bits.value)


def bqg_selftest_wait_timeout() -> None:
    """Launches the failure-detection self-test on the current device: one wait that nothing
    completes gives up after its bound (2 s) and sets DEVERR_TIMEOUT (read it with
    bqg_device_errors)."""
    _check(lib().bqg_selftest_wait_timeout(_vp(torch.cuda.current_stream().cuda_stream)), "bqg_selftest_wait_timeout")


def _check(status: int, what: str):
    if status != 0:
        raise BQGError(status, what)


def _stream(t: torch.Tensor) -> _vp:
    return _vp(torch.cuda.current_stream(t.device).cuda_stream)


def _ptr(t: Optional[torch.Tensor]) -> _vp:
    return _vp(0 if t is None else t.data_ptr())


def _need_cuda(name: str, t: torch.Tensor, dtype: torch.dtype):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


# ---------------------------------------------------------------- GEMV
def qgemv(fmt: int, W: torch.Tensor, x: torch.Tensor, rows: int, cols: int,
          y: Optional[torch.Tensor] = None) -> torch.Tensor:
    """y = W x for a quantized matrix W (uint8 bytes in the canonical layout of `fmt`)."""
    _need_cuda("W", W, torch.uint8)
    _need_cuda("x", x, torch.float32)
    if y is None:
        y = torch.empty(rows, dtype=torch.float32, device=x.device)
    _need_cuda("y", y, torch.float32)
    if W.numel() < bqg_weight_bytes(fmt, rows, cols) or x.numel() < cols or y.numel() < rows:
        raise ValueError("tensor smaller than the shape requires")
    _check(lib().qgemv(fmt, _ptr(W), _ptr(x), _ptr(y), rows, cols, _stream(x)), "qgemv")
    return y


class ArgmaxState:
    """Device outputs and working state of the fused greedy argmax: token (int32), its logit
    (fp32) and the 16-byte state the kernel leaves zeroed after every call."""

    def __init__(self, device):
        self.token = torch.zeros(1, dtype=torch.int32, device=device)
        self.value = torch.zeros(1, dtype=torch.float32, device=device)
        self.state = torch.zeros(2, dtype=torch.int64, device=device)

    def ptrs(self):
        return _ptr(self.token), _ptr(self.value), _ptr(self.state)


def qgemv_argmax(fmt: int, W: torch.Tensor, x: torch.Tensor, rows: int, cols: int,
                 y: Optional[torch.Tensor] = None, out: Optional[ArgmaxState] = None):
    """y = W x and the greedy token argmax(y) (ties to the lower index) in one launch.
    Returns (y, ArgmaxState); read .token / .value on the device."""
    _need_cuda("W", W, torch.uint8)
    _need_cuda("x", x, torch.float32)
    if y is None:
        y = torch.empty(rows, dtype=torch.float32, device=x.device)
    _need_cuda("y", y, torch.float32)
    if W.numel() < bqg_weight_bytes(fmt, rows, cols) or x.numel() < cols or y.numel() < rows:
        raise ValueError("tensor smaller than the shape requires")
    out = out if out is not None else ArgmaxState(x.device)
    _check(lib().qgemv_argmax(fmt, _ptr(W), _ptr(x), _ptr(y), rows, cols, *out.ptrs(), _stream(x)), "qgemv_argmax")
    return y, out


class GemvBatch:
    """A prepared list of independent GEMVs (fmt, W, x, y, rows, cols) launched as one
    qgemv_batched call.  Keeps the tensors alive and the descriptor array ready."""

    def __init__(self, items: Sequence[tuple]):
        if not 1 <= len(items) <= MAX_BATCH:
            raise ValueError(f"1..{MAX_BATCH} descriptors")
        self.items = list(items)
        self.descs = (GemvDesc * len(items))()
        for d, (fmt, W, x, y, rows, cols) in zip(self.descs, self.items):
            _need_cuda("W", W, torch.uint8)
            _need_cuda("x", x, torch.float32)
            _need_cuda("y", y, torch.float32)
            if W.numel() < bqg_weight_bytes(fmt, rows, cols) or x.numel() < cols or y.numel() < rows:
                raise ValueError("tensor smaller than the shape requires")
            d.fmt, d.rows, d.cols, d.reserved = fmt, rows, cols, 0
            d.W, d.x, d.y = W.data_ptr(), x.data_ptr(), y.data_ptr()
        self.device = self.items[0][2].device

    def run(self, stream: Optional[torch.cuda.Stream] = None, argmax: Optional[tuple] = None):
        """One launch over every descriptor; with argmax = (index, ArgmaxState) also the greedy
        token of descriptor `index`'s y."""
        s = stream if stream is not None else torch.cuda.current_stream(self.device)
        if argmax is None:
            _check(lib().qgemv_batched(self.descs, len(self.descs), _vp(s.cuda_stream)), "qgemv_batched")
        else:
            index, out = argmax
            _check(lib().qgemv_batched_argmax(self.descs, len(self.descs), index, *out.ptrs(), _vp(s.cuda_stream)),
                   "qgemv_batched_argmax")


def qgemv_batched(items: Sequence[tuple]) -> None:
    """Every (fmt, W, x, y, rows, cols) item's y = W x, in one launch."""
    GemvBatch(items).run()


# ---------------------------------------------------------------- prefill GEMM
def qgemm_prefill(fmt: int, W: torch.Tensor, X: torch.Tensor, n: int, k: int,
                  Y: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Y[tokens, n] = X[tokens, k] W^T with fp16 X and Y (tensor cores, fp32 accumulation)."""
    _need_cuda("W", W, torch.uint8)
    _need_cuda("X", X, torch.float16)
    tokens = X.shape[0]
    if Y is None:
        Y = torch.empty(tokens, n, dtype=torch.float16, device=X.device)
    _need_cuda("Y", Y, torch.float16)
    if X.numel() != tokens * k or Y.numel() < tokens * n or W.numel() < bqg_weight_bytes(fmt, n, k):
        raise ValueError("tensor shapes do not match")
    _check(lib().qgemm_prefill(fmt, _ptr(W), _ptr(X), _ptr(Y), tokens, n, k, _stream(X)), "qgemm_prefill")
    return Y


# ---------------------------------------------------------------- router
def moe_router_logits(R: torch.Tensor, x: torch.Tensor, logits: Optional[torch.Tensor] = None) -> torch.Tensor:
    _need_cuda("R", R, torch.float32)
    _need_cuda("x", x, torch.float32)
    if R.dim() != 2:
        raise ValueError("R must be [n_experts, hidden]")
    n_experts, hidden = R.shape
    tokens = x.numel() // hidden
    if tokens < 1 or x.numel() != tokens * hidden:
        raise ValueError(f"x must hold whole tokens of {hidden} values")
    if logits is None:
        logits = torch.empty(tokens, n_experts, dtype=torch.float32, device=x.device)
    _need_cuda("logits", logits, torch.float32)
    if logits.numel() < tokens * n_experts:
        raise ValueError(f"logits must hold tokens x n_experts = {tokens} x {n_experts} values")
    _check(lib().moe_router_logits(_ptr(R), _ptr(x), _ptr(logits), tokens, n_experts, hidden, _stream(x)),
           "moe_router_logits")
    return logits


def moe_router_topk(logits: torch.Tensor, k: int, idx: Optional[torch.Tensor] = None,
                    weights: Optional[torch.Tensor] = None):
    _need_cuda("logits", logits, torch.float32)
    if logits.dim() != 2:
        raise ValueError("logits must be [tokens, n_experts]")
    tokens, n_experts = logits.shape
    if idx is None:
        idx = torch.empty(tokens, k, dtype=torch.int32, device=logits.device)
    if weights is None:
        weights = torch.empty(tokens, k, dtype=torch.float32, device=logits.device)
    _need_cuda("idx", idx, torch.int32)
    _need_cuda("weights", weights, torch.float32)
    if idx.numel() < tokens * k or weights.numel() < tokens * k:
        raise ValueError(f"idx and weights must hold tokens x k = {tokens} x {k} values")
    _check(lib().moe_router_topk(_ptr(logits), tokens, n_experts, k, _ptr(idx), _ptr(weights), _stream(logits)),
           "moe_router_topk")
    return idx, weights


# ---------------------------------------------------------------- MoE layer
class MoELayer:
    """Device tensors of one MoE layer plus its C description.

    gate/up/down: uint8 tensors holding n_experts matrices each, expert e at byte offset
    e * <name>_stride.  shared: optional (fmt, inter, gate, up, down) uint8 tensors."""

    def __init__(self, n_experts: int, top_k: int, hidden: int, inter: int, expert_fmt: int, act: int,
                 gate: torch.Tensor, up: torch.Tensor, down: torch.Tensor,
                 gate_stride: int, up_stride: int, down_stride: int, shared=None, path: int = 0):
        self.tensors = [gate, up, down]

        def need(name, t, fmt, rows, cols, count=1, stride=0):
            # `count` matrices of rows x cols in fmt, `stride` bytes apart, must lie inside t
            nb = bqg_weight_bytes(fmt, rows, cols)
            if nb == 0:
                return  # invalid shape or format: the library's own checks report it
            if count > 1 and stride < nb:
                raise ValueError(f"{name}: stride {stride} is smaller than one matrix ({nb} bytes)")
            if t.numel() * t.element_size() < (count - 1) * stride + nb:
                raise ValueError(f"{name}: {t.numel() * t.element_size()} bytes, "
                                 f"{count} matrices need {(count - 1) * stride + nb}")
        need("gate", gate, expert_fmt, inter, hidden, n_experts, gate_stride)
        need("up", up, expert_fmt, inter, hidden, n_experts, up_stride)
        need("down", down, expert_fmt, hidden, inter, n_experts, down_stride)
        c = MoELayerC()
        c.n_experts, c.top_k, c.hidden, c.inter = n_experts, top_k, hidden, inter
        c.expert_fmt, c.act = expert_fmt, act
        c.gate, c.up, c.down = gate.data_ptr(), up.data_ptr(), down.data_ptr()
        c.gate_stride, c.up_stride, c.down_stride = gate_stride, up_stride, down_stride
        if shared is not None:
            sfmt, sinter, sg, su, sd = shared
            need("shared gate", sg, sfmt, sinter, hidden)
            need("shared up", su, sfmt, sinter, hidden)
            need("shared down", sd, sfmt, hidden, sinter)
            self.tensors += [sg, su, sd]
            c.shared_inter, c.shared_fmt = sinter, sfmt
            c.s_gate, c.s_up, c.s_down = sg.data_ptr(), su.data_ptr(), sd.data_ptr()
        c.path = path
        self.c = c
        self.hidden, self.top_k, self.n_experts = hidden, top_k, n_experts

    def with_path(self, path: int) -> "MoELayer":
        """The same layer (same tensors) with another expert path (MOE_PATH_*)."""
        other = object.__new__(MoELayer)
        other.__dict__.update(self.__dict__)
        c = MoELayerC()
        ctypes.memmove(ctypes.byref(c), ctypes.byref(self.c), ctypes.sizeof(c))
        c.path = path
        other.c = c
        return other


def moe_workspace_size(layer: MoELayer, tokens: int) -> int:
    return int(lib().moe_workspace_size(ctypes.byref(layer.c), tokens))


def _moe_tokens(layer: MoELayer, x: torch.Tensor, idx: torch.Tensor, w: torch.Tensor, y: torch.Tensor) -> int:
    tokens = x.numel() // layer.hidden
    if tokens < 1 or x.numel() != tokens * layer.hidden:
        raise ValueError(f"x must hold whole tokens of hidden = {layer.hidden} values")
    if idx.numel() < tokens * layer.top_k or w.numel() < tokens * layer.top_k:
        raise ValueError(f"idx and w must hold tokens x top_k = {tokens} x {layer.top_k} values")
    if y.numel() < tokens * layer.hidden:
        raise ValueError(f"y must hold tokens x hidden = {tokens} x {layer.hidden} values")
    return tokens


def moe_forward(layer: MoELayer, x: torch.Tensor, idx: torch.Tensor, w: torch.Tensor,
                y: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    _need_cuda("x", x, torch.float32)
    _need_cuda("idx", idx, torch.int32)
    _need_cuda("w", w, torch.float32)
    if y is None:
        y = torch.empty(max(x.numel() // layer.hidden, 1), layer.hidden, dtype=torch.float32, device=x.device)
    _need_cuda("y", y, torch.float32)
    tokens = _moe_tokens(layer, x, idx, w, y)
    need = moe_workspace_size(layer, tokens)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=x.device)
    _need_cuda("workspace", workspace, torch.uint8)
    _check(lib().moe_forward(ctypes.byref(layer.c), _ptr(x), _ptr(idx), _ptr(w), _ptr(y), tokens,
                             _ptr(workspace), workspace.numel(), _stream(x)), "moe_forward")
    return y


NOALLOC_SCRATCH_BYTES = 32 << 20


def moe_forward_noalloc(layer: MoELayer, x: torch.Tensor, idx: torch.Tensor, w: torch.Tensor,
                        y: torch.Tensor) -> torch.Tensor:
    """moe_forward with the library's fixed scratch array instead of a caller workspace: for
    callers that cannot allocate device memory around the call.  y must be preallocated; calls
    that could overlap on the GPU share the scratch and must not be issued."""
    _need_cuda("x", x, torch.float32)
    _need_cuda("idx", idx, torch.int32)
    _need_cuda("w", w, torch.float32)
    _need_cuda("y", y, torch.float32)
    tokens = _moe_tokens(layer, x, idx, w, y)
    _check(lib().moe_forward_noalloc(ctypes.byref(layer.c), _ptr(x), _ptr(idx), _ptr(w), _ptr(y), tokens, _stream(x)),
           "moe_forward_noalloc")
    return y


# ---------------------------------------------------------------- host-resident experts
class ExpertCache:
    """Routed experts of one layer in pinned host memory, `n_slots` of them resident in device
    slots (LFU replacement with a recency tie-break).  forward() takes the routing ids on the
    host and computes the layer exactly as moe_forward would.

    gate/up/down: pinned host uint8 tensors with n_experts matrices each (expert e at
    e * <name>_stride); shared: optional (fmt, inter, gate, up, down) DEVICE uint8 tensors."""

    def __init__(self, n_experts: int, top_k: int, hidden: int, inter: int, expert_fmt: int, act: int,
                 gate: torch.Tensor, up: torch.Tensor, down: torch.Tensor,
                 gate_stride: int, up_stride: int, down_stride: int, n_slots: int, shared=None, device="cuda",
                 path: int = 0):
        for name, t in (("gate", gate), ("up", up), ("down", down)):
            if t.is_cuda or t.dtype != torch.uint8 or not t.is_contiguous():
                raise TypeError(f"{name} must be a contiguous uint8 HOST tensor (pinned for asynchronous copies)")
        if not 1 <= n_slots <= min(n_experts, MAX_EXPERTS):
            raise ValueError(f"n_slots must be in 1..{min(n_experts, MAX_EXPERTS)}")
        # the host stacks, described as a layer (the library checks them like any MoE layer)
        self.host = MoELayer.__new__(MoELayer)
        c = MoELayerC()
        c.n_experts, c.top_k, c.hidden, c.inter, c.expert_fmt, c.act = n_experts, top_k, hidden, inter, expert_fmt, act
        c.gate, c.up, c.down = gate.data_ptr(), up.data_ptr(), down.data_ptr()
        c.gate_stride, c.up_stride, c.down_stride = gate_stride, up_stride, down_stride
        c.path = path
        for name, t, rows, cols, stride in (("gate", gate, inter, hidden, gate_stride), ("up", up, inter, hidden, up_stride),
                                            ("down", down, hidden, inter, down_stride)):
            nb = bqg_weight_bytes(expert_fmt, rows, cols)
            if nb == 0 or stride < nb or t.numel() < (n_experts - 1) * stride + nb:
                raise ValueError(f"{name}: host tensor or stride too small for {n_experts} experts")
        self.tensors = [gate, up, down]
        if shared is not None:
            sfmt, sinter, sg, su, sd = shared
            for t in (sg, su, sd):
                _need_cuda("shared expert", t, torch.uint8)
            c.shared_inter, c.shared_fmt = sinter, sfmt
            c.s_gate, c.s_up, c.s_down = sg.data_ptr(), su.data_ptr(), sd.data_ptr()
            self.tensors += [sg, su, sd]
        self.slots = [torch.empty(n_slots * st, dtype=torch.uint8, device=device)
                      for st in (gate_stride, up_stride, down_stride)]
        d = ExpertCacheDesc()
        d.layer = c
        d.n_slots = n_slots
        d.slot_gate, d.slot_up, d.slot_down = [t.data_ptr() for t in self.slots]
        self.desc = d
        h = _vp()
        _check(lib().bqg_expert_cache_create(ctypes.byref(d), ctypes.byref(h)), "bqg_expert_cache_create")
        self.handle = h
        self.hidden, self.top_k, self.n_experts, self.n_slots = hidden, top_k, n_experts, n_slots
        self.device = torch.device(device)
        self.copy_stream = torch.cuda.Stream(device=self.device)

    def __del__(self):
        h = getattr(self, "handle", None)
        if h is not None and h.value:
            lib().bqg_expert_cache_destroy(h)
            self.handle = None

    def workspace_size(self, tokens: int) -> int:
        return int(lib().bqg_expert_cache_workspace_size(self.handle, tokens))

    def forward(self, x: torch.Tensor, idx_host: torch.Tensor, w: torch.Tensor, y: Optional[torch.Tensor] = None,
                workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
        """y for routing ids idx_host (int32 HOST tensor [tokens, top_k]) and weights w (device)."""
        _need_cuda("x", x, torch.float32)
        _need_cuda("w", w, torch.float32)
        if idx_host.is_cuda or idx_host.dtype != torch.int32 or not idx_host.is_contiguous():
            raise TypeError("idx_host must be a contiguous int32 HOST tensor")
        tokens = x.numel() // self.hidden
        if tokens < 1 or x.numel() != tokens * self.hidden:
            raise ValueError(f"x must hold whole tokens of hidden = {self.hidden} values")
        if idx_host.numel() < tokens * self.top_k or w.numel() < tokens * self.top_k:
            raise ValueError(f"idx_host and w must hold tokens x top_k = {tokens} x {self.top_k} values")
        if y is None:
            y = torch.empty(tokens, self.hidden, dtype=torch.float32, device=x.device)
        _need_cuda("y", y, torch.float32)
        if y.numel() < tokens * self.hidden:
            raise ValueError("y too small")
        need = self.workspace_size(tokens)
        if workspace is None:
            workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=x.device)
        _need_cuda("workspace", workspace, torch.uint8)
        _check(lib().bqg_expert_cache_forward(self.handle, _ptr(x), idx_host.data_ptr(), _ptr(w), _ptr(y), tokens,
                                              _ptr(workspace), workspace.numel(), _stream(x),
                                              _vp(self.copy_stream.cuda_stream)), "bqg_expert_cache_forward")
        return y

    def stats(self) -> dict:
        st = ExpertCacheStats()
        _check(lib().bqg_expert_cache_get_stats(self.handle, ctypes.byref(st)), "bqg_expert_cache_get_stats")
        return {name: int(getattr(st, name)) for name, _ in ExpertCacheStats._fields_}
