"""moe_forward_noalloc, the MoE entry point that allocates nothing.

Some callers cannot allocate device memory around a call: a component whose work is captured
into a CUDA graph by someone else, a runtime that forbids cudaMalloc once it has started, or a
plugin that a host framework hands only its input and output buffers.  This entry point runs
the same kernels as moe_forward with their scratch in a fixed array inside the library.  The
test calls it through the C ABI twice in a row (with different inputs, so stale scratch from
the first call cannot leak into the second) and checks each result against moe_forward, the
entry point that takes a caller workspace.  This file is collected last on purpose.
"""
import pytest
import torch

import block_quant_gemv_b200 as bqg
from synth import workloads as wl
from tests.moe_util import device_layer
from tests.util import assert_close, need_gpu

pytestmark = pytest.mark.gpu


def _inputs(spec, L, seed, tokens):
    x = wl.moe_tokens(spec, seed, tokens).cuda()
    if L.R is not None:
        logits = bqg.moe_router_logits(L.R, x)
    else:
        logits = wl.moe_logits(spec, seed, 0, tokens).cuda()
    idx, w = bqg.moe_router_topk(logits, spec.top_k)
    return x, idx, w


@pytest.mark.parametrize("spec,tokens", [
    (wl.GEMMA_MOE, 16),
    (wl.MoESpec("na_small", 8, 2, 128, 64, bqg.Q4_0, bqg.ACT_GELU_TANH, 96, bqg.Q8_0, False), 5),
], ids=["gemma_like_T16", "small_shared"])
def test_noalloc_matches_workspace_entry_point_twice(spec, tokens):
    need_gpu()
    L = wl.build_moe_layer(spec, 3, 0, device="cuda")
    lay = device_layer(L)
    assert bqg.moe_workspace_size(lay, tokens) <= bqg.NOALLOC_SCRATCH_BYTES
    for call, seed in enumerate((11, 12)):
        x, idx, w = _inputs(spec, L, seed, tokens)
        y_ref = bqg.moe_forward(lay, x, idx, w)
        y = torch.full_like(y_ref, float("nan"))
        bqg.moe_forward_noalloc(lay, x, idx, w, y)
        torch.cuda.synchronize()
        assert torch.isfinite(y).all(), f"call {call}"
        assert_close(y, y_ref.cpu().numpy(), what=f"noalloc call {call}")


def test_noalloc_rejects_sizes_beyond_the_scratch():
    need_gpu()
    spec = wl.MoESpec("na_limit", 4, 2, 2048, 2048, bqg.Q4_0, bqg.ACT_SILU, 0, 0, False)
    L = wl.build_moe_layer(spec, 0, 0, device="cuda")
    lay = device_layer(L)
    tokens = 4096  # 8192 pairs of per-pair rows of 2048 values: far beyond the fixed scratch
    assert bqg.moe_workspace_size(lay, tokens) > bqg.NOALLOC_SCRATCH_BYTES
    x = torch.zeros(tokens, spec.hidden, device="cuda")
    idx = torch.zeros(tokens, 2, dtype=torch.int32, device="cuda")
    w = torch.zeros(tokens, 2, device="cuda")
    y = torch.zeros(tokens, spec.hidden, device="cuda")
    with pytest.raises(bqg.BQGError) as e:
        bqg.moe_forward_noalloc(lay, x, idx, w, y)
    assert e.value.status == -8
