"""The seeded input generator: determinism, counter addressing, value ranges, layout sizes."""
import numpy as np
import torch

import synth


def test_words_are_counter_based():
    a = synth.words(3, 7, 1000)
    b = synth.words(3, 7, 400, start=600)
    assert torch.equal(a[600:], b)
    assert not torch.equal(synth.words(3, 8, 1000), a)
    assert int(a.min()) >= 0 and int(a.max()) < 2 ** 32
    # far counters (above 2**32) are reachable and distinct from low ones
    hi = synth.words(3, 7, 4, start=2 ** 33)
    assert not torch.equal(hi, a[:4])


def test_fmix32_scalar_and_tensor_agree():
    vals = [0, 1, 0xDEADBEEF, 0xFFFFFFFF, 123456789]
    t = synth._fmix32_t(torch.tensor(vals, dtype=torch.int64))
    assert t.tolist() == [synth._fmix32_i(v) for v in vals]
    # MurmurHash3 fmix32 known answers
    assert synth._fmix32_i(0) == 0
    assert synth._fmix32_i(1) == 0x514E28B7


def test_q8_0_values_and_layout():
    W = synth.q8_0_matrix(64, 256, 0, "t").numpy().reshape(64 * 8, 34)
    d = W[:, :2].copy().view(np.float16).astype(np.float64)
    q = W[:, 2:].view(np.int8)
    assert d.min() >= 1e-3 - 1e-6 and d.max() <= 1e-2 + 1e-5
    assert q.min() >= -127 and q.max() <= 127
    assert q.min() == -127 and q.max() == 127      # both ends drawn at this size
    assert len(synth.q8_0_matrix(2, 64, 0, "t")) == synth.weight_bytes(synth.FMT_Q8_0, 2, 64) == 136


def test_q4_0_and_i4_row_layout():
    assert len(synth.q4_0_matrix(3, 96, 0, "t")) == synth.weight_bytes(synth.FMT_Q4_0, 3, 96) == 3 * 3 * 18
    W = synth.i4_row_matrix(3, 10, 0, "t")
    off = synth.i4_row_scale_offset(3, 10)
    assert off == 16 and len(W) == 16 + 12
    assert torch.all(W[15:16] == 0)
    s = W[off:].numpy().view("<f4")
    assert np.all((s >= 1e-3) & (s <= 1e-2))


def test_normals_are_standard():
    z = synth.normal(0, 1, 200000).numpy()
    assert abs(z.mean()) < 0.01 and abs(z.std() - 1) < 0.01


def test_uniform_f16_is_rounded_f32():
    a = synth.uniform_f32(1, 2, 1000, 1e-3, 1e-2)
    b = synth.uniform_f16(1, 2, 1000, 1e-3, 1e-2)
    assert torch.equal(a.to(torch.float16), b)
