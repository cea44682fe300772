"""GPU parity of the router (logits GEMV, softmax/top-k/renormalise) against the oracle."""
import numpy as np
import pytest
import torch

import block_quant_gemv_b200 as bqg
import synth
from oracle import moe as om
from tests.util import assert_close, need_gpu

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("tokens,E,H", [(1, 128, 2816), (16, 128, 2816), (128, 128, 2816), (3, 256, 6144),
                                        (13, 37, 64), (300, 8, 2048)])
def test_router_logits(tokens, E, H):
    need_gpu()
    R = synth.normal_f32(0, synth.stream_id(f"R{E}x{H}"), E * H, std=0.02).view(E, H)
    x = synth.normal_f32(0, synth.stream_id(f"x{tokens}x{H}"), tokens * H).view(tokens, H)
    got = bqg.moe_router_logits(R.cuda(), x.cuda())
    ref = om.router_logits(R.numpy(), x.numpy())
    assert_close(got, ref, what="router logits")
    assert_close(got, ref, tol=1e-5, what="router logits (fp32 accuracy)")


@pytest.mark.parametrize("tokens,E,k", [(1, 128, 8), (16, 128, 8), (128, 128, 8), (64, 256, 8), (5, 8, 8),
                                        (33, 37, 3), (7, 256, 1), (1, 1, 1)])
def test_topk_bit_exact_indices(tokens, E, k):
    """Both sides rank the same fp32 logits: indices must match exactly."""
    need_gpu()
    lg = synth.normal_f32(1, synth.stream_id(f"lg{tokens}x{E}"), tokens * E).view(tokens, E)
    idx, w = bqg.moe_router_topk(lg.cuda(), k)
    ridx, rw = om.router_topk(lg.numpy(), k)
    assert np.array_equal(idx.cpu().numpy(), ridx)
    assert_close(w, rw, what="topk weights")
    assert_close(w, rw, tol=1e-5, what="topk weights (fp32 accuracy)")


@pytest.mark.parametrize("E", [8, 128, 256])
def test_topk_ties_go_to_lower_index(E):
    need_gpu()
    tokens = 200
    # logits drawn from 3 values: many exact ties at every rank
    w = synth.words(2, E, tokens * E)
    lg = ((w % 3).to(torch.float32) - 1.0).view(tokens, E)
    idx, wt = bqg.moe_router_topk(lg.cuda(), 8)
    ridx, rw = om.router_topk(lg.numpy(), 8)
    assert np.array_equal(idx.cpu().numpy(), ridx)
    assert_close(wt, rw, tol=1e-5, what="tied weights")


def test_topk_all_equal_uniform():
    need_gpu()
    lg = torch.full((4, 8), 0.7, device="cuda")
    idx, w = bqg.moe_router_topk(lg, 8)
    assert (idx.cpu() == torch.arange(8)).all()
    assert torch.allclose(w.cpu(), torch.full((4, 8), 0.125), atol=1e-7)


def test_topk_weights_sum_to_one():
    need_gpu()
    lg = synth.normal_f32(3, 4, 512 * 256, std=4.0).view(512, 256).cuda()
    _, w = bqg.moe_router_topk(lg, 8)
    assert torch.allclose(w.sum(dim=1), torch.ones(512, device="cuda"), atol=1e-6)
    assert bool((w[:, :-1] >= w[:, 1:]).all())


def test_binding_rejects_short_buffers():
    """Buffers smaller than the shape needs are refused by the binding before any launch."""
    need_gpu()
    R = torch.zeros(8, 64, device="cuda")
    with pytest.raises(ValueError):  # not a whole number of tokens
        bqg.moe_router_logits(R, torch.zeros(100, device="cuda"))
    with pytest.raises(ValueError):
        bqg.moe_router_logits(R, torch.zeros(3, 64, device="cuda"), torch.empty(3, 7, device="cuda"))
    lg = torch.zeros(3, 8, device="cuda")
    with pytest.raises(ValueError):
        bqg.moe_router_topk(lg, 2, torch.empty(3, 1, dtype=torch.int32, device="cuda"))
    with pytest.raises(ValueError):
        bqg.moe_router_topk(lg, 2, None, torch.empty(5, device="cuda"))
