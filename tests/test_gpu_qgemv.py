"""GPU parity of qgemv / qgemv_batched against the float64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import block_quant_gemv_b200 as bqg
import synth
from synth import workloads as wl
from oracle import qgemv as oq
from tests.util import assert_close, need_gpu

pytestmark = pytest.mark.gpu

FMTS = [bqg.Q8_0, bqg.Q4_0, bqg.I4_ROW]
# (rows, cols): single block, odd block counts (unpaired units), ragged rows, several
# stages per CTA, rows not 16-byte aligned (cols 704 / 2112), the largest cols.
SHAPES = [(1, 32), (3, 64), (37, 96), (5, 160), (130, 704), (300, 2112), (77, 5632),
          (1000, 2048), (2048, 2048), (4099, 256), (64, 15360), (513, 2816)]


def _run(fmt, rows, cols, seed=0):
    need_gpu()
    name = f"t/{fmt}/{rows}x{cols}"
    W_host = synth.matrix(fmt, rows, cols, seed, name)
    x_host = synth.normal_f32(seed, synth.stream_id(name + "/x"), cols)
    y = bqg.qgemv(fmt, W_host.cuda(), x_host.cuda(), rows, cols)
    torch.cuda.synchronize()
    ref = oq.qgemv(fmt, W_host.numpy(), x_host.numpy().astype(np.float64), rows, cols)
    return y, ref


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("rows,cols", SHAPES)
def test_qgemv_matches_oracle(fmt, rows, cols):
    y, ref = _run(fmt, rows, cols)
    assert_close(y, ref, what=f"fmt {fmt} {rows}x{cols}")
    # Exact integer block sums; the only approximation is x in 16-bit fixed point per unit of
    # 32/64 values (|x_i - s X_i| <= max|x| / 65534, about 3e-5 of a typical |y|), so outputs
    # of many rows stay far inside the tolerance; 2e-4 still catches any misread weight.
    if rows >= 64:
        assert_close(y, ref, tol=2e-4, what=f"fmt {fmt} {rows}x{cols} (x fixed-point accuracy)")


def test_q8_0_2048_config_seed0():
    """The single Q8_0 GEMV configuration: W 2048x2048, seed 0."""
    y, ref = _run(bqg.Q8_0, 2048, 2048, seed=0)
    assert_close(y, ref, what="q8_0 2048x2048")


@pytest.mark.parametrize("fmt", FMTS)
def test_qgemv_deterministic(fmt):
    need_gpu()
    W = synth.matrix(fmt, 999, 2048, 1, "det").cuda()
    x = synth.normal_f32(1, 2, 2048).cuda()
    a = bqg.qgemv(fmt, W, x, 999, 2048)
    b = bqg.qgemv(fmt, W, x, 999, 2048)
    assert torch.equal(a, b)


def test_qgemv_special_inputs():
    """x = 0 gives exactly 0; all-zero scales give 0; a unit vector reads one column."""
    need_gpu()
    rows, cols = 64, 256
    for fmt in FMTS:
        W = synth.matrix(fmt, rows, cols, 2, "sp")
        y0 = bqg.qgemv(fmt, W.cuda(), torch.zeros(cols, device="cuda"), rows, cols)
        assert torch.count_nonzero(y0) == 0
        e = torch.zeros(cols)
        e[37] = 1.0
        y1 = bqg.qgemv(fmt, W.cuda(), e.cuda(), rows, cols).cpu().numpy()
        ref = oq.dequantize(fmt, W.numpy(), rows, cols)[:, 37]
        np.testing.assert_allclose(y1, ref, rtol=1e-6, atol=1e-9)
    # zero scales in Q8_0 / Q4_0
    for fmt, blk in ((bqg.Q8_0, 34), (bqg.Q4_0, 18)):
        W = synth.matrix(fmt, rows, cols, 3, "zs").view(-1, blk).clone()
        W[:, 0:2] = 0
        y = bqg.qgemv(fmt, W.reshape(-1).cuda(), synth.normal_f32(3, 4, cols).cuda(), rows, cols)
        assert torch.count_nonzero(y) == 0


def test_qgemv_batched_mixed_matches_oracle():
    need_gpu()
    shapes = [(bqg.Q4_0, 2048, 2048), (bqg.Q4_0, 256, 2048), (bqg.Q8_0, 300, 2112), (bqg.I4_ROW, 129, 6144),
              (bqg.Q4_0, 2816, 704), (bqg.Q8_0, 7, 96), (bqg.Q4_0, 33, 5632), (bqg.I4_ROW, 5, 32)]
    host, items = [], []
    for i, (fmt, rows, cols) in enumerate(shapes):
        W = synth.matrix(fmt, rows, cols, 5, f"b{i}")
        x = synth.normal_f32(5, 100 + i, cols)
        y = torch.full((rows,), float("nan"), device="cuda")
        host.append((fmt, W, x, rows, cols))
        items.append((fmt, W.cuda(), x.cuda(), y, rows, cols))
    bqg.qgemv_batched(items)
    torch.cuda.synchronize()
    for (fmt, W, x, rows, cols), it in zip(host, items):
        ref = oq.qgemv(fmt, W.numpy(), x.numpy().astype(np.float64), rows, cols)
        assert_close(it[3], ref, what=f"batched fmt {fmt} {rows}x{cols}")


def test_generator_same_bytes_on_gpu_and_cpu():
    need_gpu()
    for fmt in FMTS:
        a = synth.matrix(fmt, 300, 2112 if fmt != bqg.I4_ROW else 2048, 9, "xdev")
        b = synth.matrix(fmt, 300, 2112 if fmt != bqg.I4_ROW else 2048, 9, "xdev", device="cuda")
        assert torch.equal(a, b.cpu())


def test_tinyllama_decode_step_full_size_sampled():
    """The decode-step workload at full size in the benchmark's launch configuration (one
    qgemv_batched call over all 155 matrices): sampled rows of every matrix against the
    oracle on rows regenerated on the host."""
    need_gpu()
    specs = wl.decode_step_specs()
    W = wl.build_gemv_workload(specs, seed=0, device="cuda")
    W.y_all.fill_(float("nan"))
    batch = bqg.GemvBatch(W.items())
    batch.run()
    torch.cuda.synchronize()
    for i, s in enumerate(specs):  # every row of every matrix written (static ranges and claimed tail)
        assert torch.isfinite(W.y(i)).all(), s.name
    rng = np.random.default_rng(0)
    xs = {}
    for i, s in enumerate(specs):
        if s.x_name not in xs:
            xs[s.x_name] = wl.x_host(specs, s.x_name, 0).numpy().astype(np.float64)
        sel = sorted(set([0, s.rows - 1] + rng.integers(0, s.rows, 6).tolist()))
        y = W.y(i).cpu().numpy()[sel]
        ref = np.array([oq.qgemv(s.fmt, synth.matrix(s.fmt, s.rows, s.cols, 0, s.name, r0=r, r1=r + 1).numpy(),
                                 xs[s.x_name], 1, s.cols)[0] for r in sel])
        assert_close(y, ref, what=s.name)
        assert_close(y, ref, tol=2e-4, what=s.name + " (x fixed-point accuracy)")
    assert W.weight_bytes == 614_629_376


def test_repeated_launches_and_graph_replays():
    """Thousands of back-to-back launches, and replays of a captured graph of launches, all
    give the same rows (no state is carried from one launch to the next)."""
    need_gpu()
    rows, cols = 3000, 2048
    W = synth.q4_0_matrix(rows, cols, 0, "sched/W").cuda()
    x = synth.normal_f32(0, 11, cols).cuda()
    ref = bqg.qgemv(bqg.Q4_0, W, x, rows, cols).clone()
    ys = [torch.empty(rows, device="cuda") for _ in range(4)]
    for i in range(4200):
        bqg.qgemv(bqg.Q4_0, W, x, rows, cols, ys[i % 4])
        if i % 700 == 0 or i >= 4196:
            torch.cuda.synchronize()
            assert torch.equal(ys[i % 4], ref), f"launch {i}"
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for y in ys:
            bqg.qgemv(bqg.Q4_0, W, x, rows, cols, y)
    for rep in range(5):
        for y in ys:
            y.zero_()
        g.replay()
        torch.cuda.synchronize()
        for y in ys:
            assert torch.equal(y, ref), f"replay {rep}"
    assert bqg.bqg_device_errors() == 0


# ---------------------------------------------------------------- packed int2 with a per-row scale
I2_SHAPES = [(1, 64), (37, 128), (130, 704), (300, 2112), (77, 5632), (1000, 2048), (2048, 2048),
             (4099, 256), (64, 15360), (513, 2816)]


@pytest.mark.parametrize("rows,cols", I2_SHAPES)
def test_qgemv_i2_row_matches_oracle(rows, cols):
    y, ref = _run(bqg.I2_ROW, rows, cols)
    assert_close(y, ref, what=f"i2_row {rows}x{cols}")
    if rows >= 64:
        assert_close(y, ref, tol=2e-4, what=f"i2_row {rows}x{cols} (x fixed-point accuracy)")


def test_qgemv_i2_row_unit_probes_and_determinism():
    """x = e_j reads column j (s_r * q_rj exactly); two calls give identical bits; cols not a
    multiple of 64 is refused."""
    need_gpu()
    rows, cols = 96, 1024
    W = synth.matrix(bqg.I2_ROW, rows, cols, 5, "i2probe")
    deq = oq.dequantize(bqg.I2_ROW, W.numpy(), rows, cols)
    for j in (0, 1, 2, 3, 4, 63, 64, 511, 1023):
        e = torch.zeros(cols)
        e[j] = 1.0
        y = bqg.qgemv(bqg.I2_ROW, W.cuda(), e.cuda(), rows, cols).cpu().numpy()
        np.testing.assert_allclose(y, deq[:, j], rtol=1e-6, atol=1e-9)
    x = synth.normal_f32(5, 6, cols).cuda()
    assert torch.equal(bqg.qgemv(bqg.I2_ROW, W.cuda(), x, rows, cols), bqg.qgemv(bqg.I2_ROW, W.cuda(), x, rows, cols))
    with pytest.raises(bqg.BQGError) as e:
        bqg.qgemv(bqg.I2_ROW, W.cuda(), x, rows, 992)
    assert e.value.status == -3


def test_qgemv_batched_mixed_with_i2_row():
    """int2 matrices inside a mixed-format batch (one launch)."""
    need_gpu()
    specs = [(bqg.I2_ROW, 700, 2048), (bqg.Q4_0, 300, 2048), (bqg.I2_ROW, 2048, 704), (bqg.Q8_0, 64, 128),
             (bqg.I4_ROW, 129, 640)]
    items, refs = [], []
    for i, (fmt, rows, cols) in enumerate(specs):
        W = synth.matrix(fmt, rows, cols, 0, f"mix2/{i}")
        x = synth.normal_f32(0, 100 + i, cols)
        y = torch.empty(rows, device="cuda")
        items.append((fmt, W.cuda(), x.cuda(), y, rows, cols))
        refs.append(oq.qgemv(fmt, W.numpy(), x.numpy().astype(np.float64), rows, cols))
    bqg.qgemv_batched(items)
    torch.cuda.synchronize()
    for (fmt, _, _, y, rows, cols), ref in zip(items, refs):
        assert_close(y, ref, tol=2e-4, what=f"mixed batch fmt {fmt} {rows}x{cols}")
