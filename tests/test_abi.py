"""The C-ABI library on the host: it builds, loads, exports every symbol include/bqg.h
declares, and rejects invalid arguments with typed errors before touching a device."""
import ctypes
import os
import re
import subprocess

import pytest

import synth
from tests.conftest import ROOT

HEADER = os.path.join(ROOT, "include", "bqg.h")


@pytest.fixture(scope="module")
def L():
    from block_quant_gemv_b200 import build
    build.build()
    import block_quant_gemv_b200 as bqg
    return bqg


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:BQG_API\s+)?(?:const\s+)?(?:int|size_t|char\s*\*|void)\s*\*?\s*(\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_api():
    names = declared_functions()
    for want in ["qgemv", "qgemv_batched", "qgemm_prefill", "moe_router_logits", "moe_router_topk",
                 "moe_workspace_size", "moe_forward", "moe_forward_noalloc", "bqg_status_string", "bqg_weight_bytes",
                 "bqg_device_errors", "bqg_version", "bqg_selftest_wait_timeout", "qgemv_argmax",
                 "qgemv_batched_argmax", "bqg_expert_cache_create", "bqg_expert_cache_destroy",
                 "bqg_expert_cache_workspace_size", "bqg_expert_cache_forward", "bqg_expert_cache_get_stats"]:
        assert want in names


def test_library_exports_every_declared_symbol(L):
    so = ctypes.CDLL(L.library_path())
    for name in declared_functions():
        assert hasattr(so, name), f"{name} declared in bqg.h but not exported"
    out = subprocess.run(["nm", "-D", "--defined-only", L.library_path()], capture_output=True, text=True).stdout
    exported = set(line.split()[-1] for line in out.splitlines() if " T " in line)
    for name in declared_functions():
        assert name in exported


def test_status_strings(L):
    for s in range(0, -9, -1):
        assert L.bqg_status_string(s).startswith("BQG")
    assert L.lib().bqg_version() >= 100


def test_weight_bytes_agrees_with_generator(L):
    for fmt in (1, 2, 3):
        for rows, cols in [(1, 32), (7, 96), (2048, 2048), (6144, 2048), (3, 704)]:
            assert L.bqg_weight_bytes(fmt, rows, cols) == synth.weight_bytes(fmt, rows, cols)
    assert L.bqg_weight_bytes(9, 4, 32) == 0
    assert L.bqg_weight_bytes(1, 4, 33) == 0
    assert L.bqg_weight_bytes(1, 0, 32) == 0


def test_qgemv_argument_errors_before_any_launch(L):
    f = L.lib().qgemv
    A = 0x10000  # a 16-byte aligned fake address; nothing is dereferenced on these paths
    assert f(9, A, A, A, 4, 32, None) == -2                # unknown format
    assert f(1, None, A, A, 4, 32, None) == -1             # null W
    assert f(1, A, A, A, 0, 32, None) == -1                # rows < 1
    assert f(1, A, A, A, 4, 33, None) == -3                # cols % 32
    assert f(2, A, A, A, 4, 15360 + 32, None) == -3        # cols above the maximum
    assert f(2, A + 2, A, A, 4, 32, None) == -4            # W not 16-byte aligned
    assert f(2, A, A + 4, A, 4, 32, None) == -4            # x not 16-byte aligned
    assert f(2, A, A, A + 2, 4, 32, None) == -4            # y not 4-byte aligned


def test_qgemv_batched_argument_errors(L):
    f = L.lib().qgemv_batched
    D = (L.GemvDesc * 300)()
    for d in D:
        d.fmt, d.rows, d.cols, d.W, d.x, d.y = 2, 4, 32, 0x10000, 0x10000, 0x10000
    assert f(None, 1, None) == -1
    assert f(D, 0, None) == -1
    assert f(D, 300, None) == -8
    D[3].cols = 48
    assert f(D, 5, None) == -3
    D[3].cols = 32
    D[1].reserved = 1
    assert f(D, 5, None) == -1


def test_valid_call_without_gpu_fails_loudly(L):
    """With no usable device, a valid call returns an error: there is no CPU fallback."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert L.lib().qgemv(2, 0x10000, 0x10000, 0x10000, 4, 32, None) in (-6, -7)


def test_router_argument_errors(L):
    lg, tk = L.lib().moe_router_logits, L.lib().moe_router_topk
    A = 0x10000
    assert lg(None, A, A, 1, 128, 2816, None) == -1
    assert lg(A, A, A, 1, 300, 2816, None) == -8          # more than 256 experts
    assert lg(A, A, A, 1, 128, 2818, None) == -3          # hidden % 4
    assert lg(A + 4, A, A, 1, 128, 2816, None) == -4
    assert tk(A, 1, 128, 9, A, A, None) == -8              # k above 8
    assert tk(A, 1, 4, 8, A, A, None) == -3                # k > n_experts
    assert tk(A, 0, 128, 8, A, A, None) == -1
    assert tk(A + 2, 1, 128, 8, A, A, None) == -4


def test_only_the_c_abi_is_exported(L):
    """Internal symbols (kernels, per-device caches) are hidden, so two copies of the library
    loaded in one process cannot share internal state."""
    out = subprocess.run(["nm", "-D", "--defined-only", L.library_path()], capture_output=True, text=True).stdout
    exported = set(line.split()[-1] for line in out.splitlines() if line.split()[1:2] and line.split()[1] in "TBDVWu")
    assert exported <= set(declared_functions()) | {"_init", "_fini"}, exported - set(declared_functions())


def test_prefill_argument_errors(L):
    f = L.lib().qgemm_prefill
    A = 0x10000
    assert f(1, A, A, A, 128, 1024, 4096, None) == -2        # only Q4_0
    assert f(2, A, A, A, 129, 1024, 4096, None) == -3        # more than 128 tokens
    assert f(2, A, A, A, 128, 1000, 4096, None) == -3        # n % 16
    assert f(2, A, A, A, 128, 1024, 4000, None) == -3        # k % 256
    assert f(2, A + 8, A, A, 128, 1024, 4096, None) == -4
    assert f(2, None, A, A, 128, 1024, 4096, None) == -1


def test_moe_argument_errors(L):
    import block_quant_gemv_b200 as bqg
    c = bqg.MoELayerC()
    c.n_experts, c.top_k, c.hidden, c.inter, c.expert_fmt, c.act = 128, 8, 2816, 704, 2, 1
    c.gate = c.up = c.down = 0x10000
    c.gate_stride = c.up_stride = c.down_stride = synth.weight_bytes(2, 704, 2816) + 16 - synth.weight_bytes(2, 704, 2816) % 16
    size = L.lib().moe_workspace_size(ctypes.byref(c), 16)
    assert size > 0
    A = 0x10000
    fwd = L.lib().moe_forward
    assert fwd(ctypes.byref(c), A, A, A, A, 16, A, size - 1, None) == -5   # workspace too small
    assert fwd(ctypes.byref(c), A, A, A, A, 16, A + 16, size, None) == -4  # workspace alignment
    c.top_k = 9
    assert fwd(ctypes.byref(c), A, A, A, A, 16, A, size, None) == -8
    c.top_k, c.act = 8, 7
    assert fwd(ctypes.byref(c), A, A, A, A, 16, A, size, None) == -1
    c.act, c.hidden = 1, 2820
    assert L.lib().moe_workspace_size(ctypes.byref(c), 16) == 0


def test_binding_limits_match_header():
    import re
    import block_quant_gemv_b200 as bqg
    text = open(os.path.join(ROOT, "include", "bqg.h")).read()
    for name, val in (("BQG_MAX_COLS", bqg.MAX_COLS), ("BQG_MAX_BATCH", bqg.MAX_BATCH),
                      ("BQG_MAX_EXPERTS", bqg.MAX_EXPERTS), ("BQG_MAX_TOPK", bqg.MAX_TOPK),
                      ("BQG_MAX_MOE_COLS", bqg.MAX_MOE_COLS)):
        m = re.search(rf"#define {name} (\d+)", text)
        assert m and int(m.group(1)) == val, name


def test_moe_layer_binding_rejects_short_tensors():
    """The binding checks every stacked expert tensor against n_experts x stride before any
    pointer reaches the library (the C ABI cannot see buffer sizes)."""
    import block_quant_gemv_b200 as bqg
    from synth import workloads as wl
    from tests.moe_util import device_layer
    spec = wl.MoESpec("abi_small", 4, 2, 64, 32, bqg.Q4_0, bqg.ACT_GELU_TANH, 32, bqg.Q8_0, False)
    T = wl.build_moe_layer(spec, 0, device="cpu")
    device_layer(T)  # the builder's layout passes
    with pytest.raises(ValueError):
        bqg.MoELayer(4, 2, 64, 32, bqg.Q4_0, 1, T.gate[:-1], T.up, T.down, T.gate_stride, T.up_stride, T.down_stride)
    with pytest.raises(ValueError):  # stride below one matrix
        bqg.MoELayer(4, 2, 64, 32, bqg.Q4_0, 1, T.gate, T.up, T.down, T.gate_stride - 16, T.up_stride, T.down_stride)
    short_shared = (bqg.Q8_0, 32, T.shared[0], T.shared[1], T.shared[2][:-2])
    with pytest.raises(ValueError):
        bqg.MoELayer(4, 2, 64, 32, bqg.Q4_0, 1, T.gate, T.up, T.down, T.gate_stride, T.up_stride, T.down_stride,
                     short_shared)


def _layer_c(spec, path=0):
    import block_quant_gemv_b200 as bqg
    c = bqg.MoELayerC()
    c.n_experts, c.top_k, c.hidden, c.inter, c.expert_fmt, c.act = (spec.n_experts, spec.top_k, spec.hidden,
                                                                     spec.inter, spec.expert_fmt, spec.act)
    c.gate = c.up = c.down = 0x10000
    c.gate_stride = c.up_stride = (synth.weight_bytes(spec.expert_fmt, spec.inter, spec.hidden) + 15) // 16 * 16
    c.down_stride = (synth.weight_bytes(spec.expert_fmt, spec.hidden, spec.inter) + 15) // 16 * 16
    if spec.shared_inter:
        c.shared_inter, c.shared_fmt = spec.shared_inter, spec.shared_fmt
        c.s_gate = c.s_up = c.s_down = 0x20000
    c.path = path
    return c


def test_noalloc_scratch_covers_the_listed_configs(L):
    """moe_forward_noalloc's fixed scratch holds the workspace of every listed MoE configuration:
    the Gemma-like layer at 1, 16 and 128 tokens and the GLM-like layer at 1, 8 and 64 tokens."""
    import re
    import block_quant_gemv_b200 as bqg
    from synth import workloads as wl
    m = re.search(r"#define BQG_NOALLOC_SCRATCH_BYTES \((\d+)u << (\d+)\)", open(HEADER).read())
    limit = int(m.group(1)) << int(m.group(2))
    assert limit == bqg.NOALLOC_SCRATCH_BYTES
    for spec, Ts in ((wl.GEMMA_MOE, (1, 16, 128)), (wl.GLM_MOE, (1, 8, 64))):
        for T in Ts:
            for path in (0, 1, 2):
                need = L.lib().moe_workspace_size(ctypes.byref(_layer_c(spec, path)), T)
                assert 0 < need <= limit, (spec.name, T, path, need)


def test_moe_workspace_covers_fewer_tokens(L):
    """A workspace sized for T tokens serves every call with fewer tokens, whichever path the
    automatic choice takes for them."""
    from synth import workloads as wl
    for spec in (wl.GEMMA_MOE, wl.GLM_MOE):
        c = _layer_c(spec)
        sizes = [L.lib().moe_workspace_size(ctypes.byref(c), T) for T in range(1, 70)]
        assert all(a <= b for a, b in zip(sizes, sizes[1:]))


def test_moe_path_argument_errors(L):
    """An unknown path value is refused; forcing the tensor cores on shapes they cannot take
    (inter not a multiple of 64) gives BQG_ERR_SHAPE before any launch."""
    from synth import workloads as wl
    A = 0x10000
    c = _layer_c(wl.GEMMA_MOE, 7)
    assert L.lib().moe_workspace_size(ctypes.byref(c), 16) == 0
    assert L.lib().moe_forward(ctypes.byref(c), A, A, A, A, 16, A, 1 << 30, None) == -1
    spec = wl.MoESpec("odd", 8, 2, 128, 96, 2, 1, 0, 0, False)
    c = _layer_c(spec, 2)
    assert L.lib().moe_forward(ctypes.byref(c), A, A, A, A, 16, A, 1 << 30, None) == -3
    c.path = 0
    assert L.lib().moe_workspace_size(ctypes.byref(c), 16) > 0


def test_argmax_argument_errors(L):
    f = L.lib().qgemv_argmax
    A = 0x10000
    assert f(2, A, A, A, 4, 32, None, None, A, None) == -1          # no token pointer
    assert f(2, A, A, A, 4, 32, A, None, None, None) == -1          # no state
    assert f(2, A, A, A, 4, 32, A, None, A + 4, None) == -4         # state not 8-byte aligned
    assert f(2, A, A, A, 4, 32, A + 2, None, A, None) == -4         # token not 4-byte aligned
    g = L.lib().qgemv_batched_argmax
    D = (L.GemvDesc * 3)()
    for d in D:
        d.fmt, d.rows, d.cols, d.W, d.x, d.y = 2, 4, 32, A, A, A
    assert g(D, 3, 3, A, None, A, None) == -1                       # index outside the batch
    assert g(D, 3, -1, A, None, A, None) == -1


def test_expert_cache_argument_errors(L):
    """Creation is refused for bad slot counts or a slot layer that is not a valid MoE layer,
    before any device call."""
    import block_quant_gemv_b200 as bqg
    from synth import workloads as wl
    d = bqg.ExpertCacheDesc()
    d.layer = _layer_c(wl.GLM_MOE)
    d.n_slots = 16
    d.slot_gate = d.slot_up = d.slot_down = 0x40000
    h = ctypes.c_void_p()
    f = L.lib().bqg_expert_cache_create
    d.n_slots = 0
    assert f(ctypes.byref(d), ctypes.byref(h)) == -1
    d.n_slots = 300
    assert f(ctypes.byref(d), ctypes.byref(h)) == -8
    d.n_slots = 16
    d.slot_up = 0x40008                                          # slot buffer not 16-byte aligned
    assert f(ctypes.byref(d), ctypes.byref(h)) == -4
    d.slot_up = None
    assert f(ctypes.byref(d), ctypes.byref(h)) == -1
    assert L.lib().bqg_expert_cache_forward(None, 0x1000, 0x1000, 0x1000, 0x1000, 1, 0x1000, 1 << 20, None, None) == -1
