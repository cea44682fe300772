"""GPU: the LM-head GEMV with the fused greedy argmax (qgemv_argmax, qgemv_batched_argmax),
through the C ABI.  The token must equal the oracle's argmax of the same fp32 logits the GPU
wrote, bit for bit (ties to the lower index); the logits themselves are checked against the
float64 oracle within the GEMV tolerance."""
import numpy as np
import pytest
import torch

import block_quant_gemv_b200 as bqg
import synth
from oracle import argmax as oa
from oracle import qgemv as oq
from synth import workloads as wl
from tests.util import assert_close, need_gpu

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("fmt,rows,cols", [
    (bqg.Q8_0, 32000, 2048),     # the TinyLlama-shape LM head
    (bqg.Q4_0, 32000, 2048),
    (bqg.I4_ROW, 4099, 4096),
    (bqg.Q8_0, 7, 96),
    (bqg.Q4_0, 1, 64),
    (bqg.I4_ROW, 300, 1056),
])
def test_token_is_the_argmax_of_the_written_logits(fmt, rows, cols):
    need_gpu()
    W = synth.matrix(fmt, rows, cols, 0, f"am/{fmt}/{rows}x{cols}")
    out = bqg.ArgmaxState("cuda")
    for call, seed in enumerate((1, 2)):  # twice in a row: the state is left zeroed by the first call
        x = synth.normal_f32(seed, 9, cols)
        y, out = bqg.qgemv_argmax(fmt, W.cuda(), x.cuda(), rows, cols, out=out)
        torch.cuda.synchronize()
        yg = y.cpu().numpy()
        tok = int(out.token.item())
        assert tok == oa.argmax_lower(yg), f"call {call}"
        assert out.value.item() == yg[tok]
        assert torch.count_nonzero(out.state) == 0
        ref = oq.qgemv(fmt, W.numpy(), x.numpy().astype(np.float64), rows, cols)
        assert_close(yg, ref, what=f"logits fmt {fmt} {rows}x{cols}")
        # the head's own greedy token, unless the top two float64 logits are within fp32 error
        t_ref, _ = oa.lm_head_greedy(fmt, W.numpy(), x.numpy().astype(np.float64), rows, cols)
        if tok != t_ref:
            assert abs(ref[tok] - ref[t_ref]) <= 2e-4 * np.max(np.abs(ref))


@pytest.mark.parametrize("fmt", [bqg.Q8_0, bqg.Q4_0, bqg.I4_ROW])
def test_exact_ties_go_to_the_lower_index(fmt):
    """Copies of the winning row at other positions give bit-identical logits (the kernel's sum
    order does not depend on the row): the token must be the lowest of those positions."""
    need_gpu()
    rows, cols = 5000, 2048
    W = synth.matrix(fmt, rows, cols, 3, f"am/tie/{fmt}").clone()
    x = synth.normal_f32(4, 9, cols)
    y = bqg.qgemv(fmt, W.cuda(), x.cuda(), rows, cols).cpu().numpy()
    m = int(np.argmax(y))
    rb = synth.weight_bytes(fmt, 1, cols) if fmt != bqg.I4_ROW else cols // 2
    copies = sorted({(m + 1777) % rows, (m + 3) % rows, 17, rows - 1} - {m})
    for c in copies:
        W[c * rb:(c + 1) * rb] = W[m * rb:(m + 1) * rb]
        if fmt == bqg.I4_ROW:
            off = synth.i4_row_scale_offset(rows, cols)
            W[off + 4 * c: off + 4 * c + 4] = W[off + 4 * m: off + 4 * m + 4]
    y2, out = bqg.qgemv_argmax(fmt, W.cuda(), x.cuda(), rows, cols)
    torch.cuda.synchronize()
    yg = y2.cpu().numpy()
    winners = [i for i in [m] + copies if yg[i] == yg.max()]
    assert len(winners) >= 2, "the copies must tie exactly"
    assert int(out.token.item()) == min(winners) == oa.argmax_lower(yg)


def test_decode_step_with_greedy_token():
    """The full TinyLlama-shape decode step (155 GEMVs in one launch) with the greedy token of
    the LM head computed in the same launch."""
    need_gpu()
    specs = wl.decode_step_specs()
    Wk = wl.build_gemv_workload(specs, seed=0, device="cuda")
    batch = bqg.GemvBatch(Wk.items())
    out = bqg.ArgmaxState("cuda")
    head = len(specs) - 1
    for _ in range(2):
        batch.run(argmax=(head, out))
    torch.cuda.synchronize()
    yh = Wk.y(head).cpu().numpy()
    assert int(out.token.item()) == oa.argmax_lower(yh)
    assert out.value.item() == yh.max()
    assert torch.count_nonzero(out.state) == 0
    # the other outputs are unchanged by the argmax: same bits as a plain launch
    y_with = Wk.y_all.clone()
    batch.run()
    torch.cuda.synchronize()
    assert torch.equal(y_with, Wk.y_all)
