"""GPU parity at the documented limits of the C ABI (include/bqg.h), against the oracle:
the largest descriptor count of qgemv_batched, the widest MoE rows, the longest prefill k and
router rows, with 256 experts."""
import numpy as np
import pytest
import torch

import block_quant_gemv_b200 as bqg
import synth
from synth import workloads as wl
from oracle import moe as om
from oracle import prefill as op
from oracle import qgemv as oq
from tests.moe_util import device_layer, oracle_layer
from tests.util import assert_close, need_gpu

pytestmark = pytest.mark.gpu


def test_qgemv_batched_max_descriptors():
    """BQG_MAX_BATCH (256) independent matrices of all three formats in one launch."""
    need_gpu()
    rng = np.random.default_rng(7)
    items, host = [], []
    for i in range(bqg.MAX_BATCH):
        fmt = (bqg.Q8_0, bqg.Q4_0, bqg.I4_ROW)[i % 3]
        rows, cols = int(rng.integers(1, 40)), 32 * int(rng.integers(1, 12))
        W = synth.matrix(fmt, rows, cols, 7, f"lim/b/{i}")
        x = synth.normal_f32(7, 1000 + i, cols)
        y = torch.empty(rows, device="cuda")
        items.append((fmt, W.cuda(), x.cuda(), y, rows, cols))
        host.append((fmt, W, x, rows, cols))
    with pytest.raises(ValueError):
        bqg.GemvBatch(items + items[:1])
    bqg.qgemv_batched(items)
    torch.cuda.synchronize()
    for (fmt, W, x, rows, cols), it in zip(host, items):
        ref = oq.qgemv(fmt, W.numpy(), x.numpy().astype(np.float64), rows, cols)
        assert_close(it[3], ref, what=f"fmt {fmt} {rows}x{cols}")


def test_moe_widest_rows():
    """hidden = BQG_MAX_MOE_COLS (7168, 224 one-block units per row) with a shared expert."""
    need_gpu()
    spec = wl.MoESpec("lim_wide", 4, 2, bqg.MAX_MOE_COLS, 64, bqg.Q4_0, bqg.ACT_GELU_TANH, 96, bqg.Q8_0, False)
    L = wl.build_moe_layer(spec, 5, 0, device="cuda")
    for tokens in (1, 3):
        x = wl.moe_tokens(spec, 5, tokens)
        lg = wl.moe_logits(spec, 5, 0, tokens)
        idx, w = bqg.moe_router_topk(lg.cuda(), spec.top_k)
        y = bqg.moe_forward(device_layer(L), x.cuda(), idx, w)
        torch.cuda.synchronize()
        ridx, rw = om.router_topk(lg.numpy(), spec.top_k)
        assert np.array_equal(idx.cpu().numpy(), ridx)
        ref = om.moe_layer(oracle_layer(spec, 5, 0), x.numpy(), ridx, rw)
        assert_close(y, ref, what=f"hidden {spec.hidden} T={tokens}")
    c = bqg.MoELayerC()
    c.n_experts, c.top_k, c.hidden, c.inter, c.expert_fmt, c.act = 4, 2, bqg.MAX_MOE_COLS + 32, 64, bqg.Q4_0, 1
    c.gate = c.up = c.down = L.gate.data_ptr()
    c.gate_stride = c.up_stride = c.down_stride = 1 << 20
    assert bqg.lib().moe_workspace_size(c, 1) == 0  # rejected: BQG_ERR_LIMIT on the call


@pytest.mark.parametrize("fmt,shared_fmt,shared_inter,tol", [
    (bqg.Q4_0, bqg.Q8_0, 192, 1e-3),  # kind::f16 variant
    (bqg.I4_ROW, 0, 0, 3e-4),         # kind::i8 variant: int32 sums over k = 7168
    (bqg.I2_ROW, bqg.I4_ROW, 128, 3e-4),
], ids=["f16_q4_shared_q8", "i8_i4", "i8_i2_shared_i4"])
def test_moe_widest_rows_tensor_cores(fmt, shared_fmt, shared_inter, tol):
    """hidden = BQG_MAX_MOE_COLS (7168) on the tensor-core path (20 tokens, every token compared)."""
    need_gpu()
    spec = wl.MoESpec("lim_wide_tc", 4, 2, bqg.MAX_MOE_COLS, 256, fmt, bqg.ACT_SILU, shared_inter, shared_fmt, False)
    L = wl.build_moe_layer(spec, 6, 0, device="cuda")
    tokens = 20
    assert tokens >= bqg.MOE_TC_MIN_TOKENS
    x = wl.moe_tokens(spec, 6, tokens)
    lg = wl.moe_logits(spec, 6, 0, tokens)
    idx, w = bqg.moe_router_topk(lg.cuda(), spec.top_k)
    y = bqg.moe_forward(device_layer(L).with_path(bqg.MOE_PATH_TENSOR_CORES), x.cuda(), idx, w)
    torch.cuda.synchronize()
    ridx, rw = om.router_topk(lg.numpy(), spec.top_k)
    ref = om.moe_layer(oracle_layer(spec, 6, 0), x.numpy(), ridx, rw)
    assert_close(y, ref, what=f"hidden {spec.hidden} tensor cores")
    assert_close(y, ref, tol=tol, what=f"hidden {spec.hidden} tensor cores (strict)")
    assert bqg.bqg_device_errors() == 0


def test_prefill_longest_k():
    """k = BQG_MAX_COLS (15360 = 60 chunks of 256) with ragged tokens and features."""
    need_gpu()
    tokens, n, k = 3, 144, bqg.MAX_COLS
    W = synth.q4_0_matrix(n, k, 0, "lim/pf")
    X = synth.normal_f16(0, 11, tokens * k).view(tokens, k)
    Y = bqg.qgemm_prefill(bqg.Q4_0, W.cuda(), X.cuda(), n, k)
    torch.cuda.synchronize()
    assert_close(Y.float(), op.prefill_f64(bqg.Q4_0, W.numpy(), X.numpy(), n, k), what="prefill k=15360")


def test_router_widest():
    """256 experts, hidden = BQG_MAX_COLS; top-8 indices bit-exact on the same fp32 logits."""
    need_gpu()
    E, H, T = bqg.MAX_EXPERTS, bqg.MAX_COLS, 3
    R = synth.normal_f32(0, 12, E * H, std=0.02).view(E, H)
    x = synth.normal_f32(0, 13, T * H).view(T, H)
    lg = bqg.moe_router_logits(R.cuda(), x.cuda())
    assert_close(lg, om.router_logits(R.numpy(), x.numpy()), what="router logits")
    idx, w = bqg.moe_router_topk(lg, 8)
    ridx, rw = om.router_topk(lg.cpu().numpy(), 8)
    assert np.array_equal(idx.cpu().numpy(), ridx)
    assert_close(w, rw, what="top-k weights")
