"""Failure detection on the GPU without a fault: a bounded wait that nothing completes gives up,
reports BQG_DEVERR_TIMEOUT through the device error word, and leaves the context usable."""
import time

import numpy as np
import pytest
import torch

import block_quant_gemv_b200 as bqg
import synth
from oracle import qgemv as oq
from tests.util import assert_close, need_gpu

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_reports():
    need_gpu()
    assert bqg.bqg_device_errors() == 0
    t0 = time.time()
    bqg.bqg_selftest_wait_timeout()
    bits = bqg.bqg_device_errors()  # synchronises, reads and clears
    elapsed = time.time() - t0
    assert bits == bqg.DEVERR_TIMEOUT
    assert 1.5 < elapsed < 60.0, elapsed  # the 2 s bound, not an early return
    assert bqg.bqg_device_errors() == 0   # cleared by the read
    # the context is still usable: a normal call right after gives the oracle's rows
    rows, cols = 300, 2048
    W = synth.q4_0_matrix(rows, cols, 0, "failure/W")
    x = synth.normal_f32(0, 21, cols)
    y = bqg.qgemv(bqg.Q4_0, W.cuda(), x.cuda(), rows, cols)
    torch.cuda.synchronize()
    assert_close(y, oq.qgemv(bqg.Q4_0, W.numpy(), x.numpy().astype(np.float64), rows, cols), what="after the timeout")
