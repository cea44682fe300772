"""Pins for the oracle's block decoding and y = W x (CPU only).

Each test checks the oracle against something other than itself: hand-worked blocks
stored under tests/golden, exact rational brute force, unit-vector probes of bytes
packed here from chosen element values, and algebraic invariants."""
import json
import os
import struct
from fractions import Fraction

import numpy as np
import pytest

from oracle import qgemv as oq



def _load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- packing helpers (test side)
def pack_q8_0_block(d_bits: int, q) -> bytes:
    q = list(q)
    assert len(q) == 32
    return struct.pack("<H", d_bits) + bytes((v & 0xFF) for v in q)


def pack_q4_0_block(d_bits: int, nibbles) -> bytes:
    """Element 2j -> low nibble of qs[j], element 2j+1 -> high nibble."""
    nib = list(nibbles)
    assert len(nib) == 32
    qs = bytes((nib[2 * j] & 0xF) | ((nib[2 * j + 1] & 0xF) << 4) for j in range(16))
    return struct.pack("<H", d_bits) + qs


def fp16_bits(v: float) -> int:
    return int(np.array(v, dtype=np.float16).view(np.uint16))


# ---------------------------------------------------------------- golden hand blocks
def _expand_q(spec):
    if spec == "ramp_minus_16":
        return [i - 16 for i in range(32)]
    if isinstance(spec, list) and len(spec) == 1:
        return spec * 32
    return spec


def _x(spec, cols):
    if spec == "ones":
        return np.ones(cols)
    if spec == "ones_then_twos":
        return np.concatenate([np.ones(32), 2 * np.ones(cols - 32)])
    return np.asarray(spec, dtype=np.float64)


def test_q8_0_golden_cases(golden_dir):
    g = _load(golden_dir, "q8_0_hand_blocks.json")
    for case in g["cases"]:
        raw = b"".join(pack_q8_0_block(int(b["d_bits"], 16), _expand_q(b["q"]))
                       for row in case["blocks"] for b in row)
        W = np.frombuffer(raw, dtype=np.uint8)
        y = oq.qgemv(oq.FMT_Q8_0, W, _x(case["x"], case["cols"]), case["rows"], case["cols"])
        assert y.tolist() == case["y"], case["name"]


def test_q8_0_golden_probe(golden_dir):
    g = _load(golden_dir, "q8_0_hand_blocks.json")
    W = np.frombuffer(pack_q8_0_block(0x3800, [i - 16 for i in range(32)]), dtype=np.uint8)
    for j, want in enumerate(g["probe"]["y_for_e_j"]):
        x = np.zeros(32)
        x[j] = 1.0
        assert oq.qgemv(oq.FMT_Q8_0, W, x, 1, 32)[0] == want


def test_q4_0_golden_cases(golden_dir):
    g = _load(golden_dir, "q4_0_hand_blocks.json")
    for case in g["cases"]:
        raw = struct.pack("<H", int(case["d_bits"], 16)) + bytes(int(b, 16) for b in case["qs"])
        W = np.frombuffer(raw, dtype=np.uint8)
        y = oq.qgemv(oq.FMT_Q4_0, W, _x(case["x"], 32), 1, 32)
        assert y[0] == case["y"], case["name"]


def test_q4_0_golden_probe_pins_nibble_order(golden_dir):
    g = _load(golden_dir, "q4_0_hand_blocks.json")
    case = g["cases"][0]
    raw = struct.pack("<H", int(case["d_bits"], 16)) + bytes(int(b, 16) for b in case["qs"])
    W = np.frombuffer(raw, dtype=np.uint8)
    for j, want in enumerate(g["probe"]["y_for_e_j"]):
        x = np.zeros(32)
        x[j] = 1.0
        assert oq.qgemv(oq.FMT_Q4_0, W, x, 1, 32)[0] == want


def test_i4_row_golden(golden_dir):
    g = _load(golden_dir, "i4_row_hand.json")
    W = np.frombuffer(bytes.fromhex(g["bytes_hex"]), dtype=np.uint8)
    y = oq.qgemv(oq.FMT_I4_ROW, W, np.array(g["x"]), g["rows"], g["cols"])
    assert y.tolist() == g["y"]


# ---------------------------------------------------------------- exact brute force
def _brute_q8_0(blocks_d, blocks_q, x):
    """Exact rational y for Q8_0 / Q4_0-like data given per-block d (fp16 value) and signed ints."""
    rows = len(blocks_d)
    y = []
    for r in range(rows):
        acc = Fraction(0)
        for b, (d, q) in enumerate(zip(blocks_d[r], blocks_q[r])):
            for i in range(32):
                acc += Fraction(d) * q[i] * Fraction(float(x[32 * b + i]))
        y.append(acc)
    return y


@pytest.mark.parametrize("fmt", [oq.FMT_Q8_0, oq.FMT_Q4_0])
def test_random_tiny_matches_exact_rational(fmt):
    rng = np.random.default_rng(7)
    rows, cols = 3, 96
    raw, ds, qs = b"", [], []
    for r in range(rows):
        rd, rq = [], []
        for b in range(cols // 32):
            d = float(np.float16(rng.uniform(-2, 2)))
            if fmt == oq.FMT_Q8_0:
                q = [int(v) for v in rng.integers(-128, 128, 32)]
                raw += pack_q8_0_block(fp16_bits(d), q)
                rq.append(q)
            else:
                nib = [int(v) for v in rng.integers(0, 16, 32)]
                raw += pack_q4_0_block(fp16_bits(d), nib)
                rq.append([v - 8 for v in nib])
            rd.append(d)
        ds.append(rd)
        qs.append(rq)
    x = rng.standard_normal(cols).astype(np.float32)
    want = _brute_q8_0(ds, qs, x)
    got = oq.qgemv(fmt, np.frombuffer(raw, dtype=np.uint8), x, rows, cols)
    for g_, w_ in zip(got, want):
        assert abs(Fraction(g_) - w_) <= Fraction(1, 10 ** 9) * (1 + abs(w_))


def test_i4_row_random_tiny_matches_exact_rational():
    rng = np.random.default_rng(11)
    rows, cols = 5, 10
    vals = rng.integers(-8, 8, (rows, cols))
    s = rng.uniform(-1, 1, rows).astype(np.float32)
    packed = bytearray()
    for r in range(rows):
        for j in range(cols // 2):
            packed.append((int(vals[r, 2 * j]) & 0xF) | ((int(vals[r, 2 * j + 1]) & 0xF) << 4))
    off = (len(packed) + 15) // 16 * 16
    raw = bytes(packed) + bytes(off - len(packed)) + s.astype("<f4").tobytes()
    x = rng.standard_normal(cols).astype(np.float32)
    got = oq.qgemv(oq.FMT_I4_ROW, np.frombuffer(raw, dtype=np.uint8), x, rows, cols)
    for r in range(rows):
        want = Fraction(float(s[r])) * sum(int(vals[r, i]) * Fraction(float(x[i])) for i in range(cols))
        assert abs(Fraction(got[r]) - want) <= Fraction(1, 10 ** 9) * (1 + abs(want))


# ---------------------------------------------------------------- probes, special cases, invariants
def test_q4_0_unit_probes_random_nibbles():
    rng = np.random.default_rng(3)
    nib = [int(v) for v in rng.integers(0, 16, 32)]
    d = 0.375
    W = np.frombuffer(pack_q4_0_block(fp16_bits(d), nib), dtype=np.uint8)
    for j in range(32):
        x = np.zeros(32)
        x[j] = 1.0
        assert oq.qgemv(oq.FMT_Q4_0, W, x, 1, 32)[0] == d * (nib[j] - 8)


def test_i4_row_nibble_values():
    # byte 0x8F: element 0 = 0xF -> -1, element 1 = 0x8 -> -8; byte 0x07: element 2 = 7, element 3 = 0
    raw = bytes([0x8F, 0x07]) + bytes(14) + struct.pack("<f", 1.0)
    W = np.frombuffer(raw, dtype=np.uint8)
    for j, want in enumerate([-1.0, -8.0, 7.0, 0.0]):
        x = np.zeros(4)
        x[j] = 1.0
        assert oq.qgemv(oq.FMT_I4_ROW, W, x, 1, 4)[0] == want


def test_q8_0_unit_scale_is_integer_matvec():
    rng = np.random.default_rng(5)
    rows, cols = 4, 64
    q = rng.integers(-127, 128, (rows, cols))
    raw = b"".join(pack_q8_0_block(0x3C00, q[r, 32 * b:32 * b + 32]) for r in range(rows) for b in range(2))
    x = rng.integers(-5, 6, cols).astype(np.float64)
    got = oq.qgemv(oq.FMT_Q8_0, np.frombuffer(raw, dtype=np.uint8), x, rows, cols)
    want = [sum(int(q[r, i]) * int(x[i]) for i in range(cols)) for r in range(rows)]
    assert got.tolist() == want


def test_zero_scale_block_contributes_nothing():
    rng = np.random.default_rng(9)
    for fmt, pack in ((oq.FMT_Q8_0, pack_q8_0_block), (oq.FMT_Q4_0, pack_q4_0_block)):
        lo, hi = (-127, 128) if fmt == oq.FMT_Q8_0 else (0, 16)
        good = pack(fp16_bits(0.5), rng.integers(lo, hi, 32))
        z1 = pack(0x0000, rng.integers(lo, hi, 32))
        z2 = pack(0x0000, rng.integers(lo, hi, 32))
        x = rng.standard_normal(64)
        a = oq.qgemv(fmt, np.frombuffer(good + z1, dtype=np.uint8), x, 1, 64)
        b = oq.qgemv(fmt, np.frombuffer(good + z2, dtype=np.uint8), x, 1, 64)
        c = oq.qgemv(fmt, np.frombuffer(good, dtype=np.uint8), x[:32], 1, 32)
        assert a[0] == b[0] == c[0]


def test_q4_0_offset_closed_form():
    """sum_b d (sum_i q x - 8 sum_i x) equals the oracle's sum_b d sum_i (q - 8) x."""
    rng = np.random.default_rng(13)
    rows, cols = 6, 128
    nib = rng.integers(0, 16, (rows, cols))
    ds = rng.uniform(1e-3, 1e-2, (rows, cols // 32)).astype(np.float16)
    raw = b"".join(pack_q4_0_block(int(ds[r, b].view(np.uint16)), nib[r, 32 * b:32 * b + 32])
                   for r in range(rows) for b in range(cols // 32))
    x = rng.standard_normal(cols)
    got = oq.qgemv(oq.FMT_Q4_0, np.frombuffer(raw, dtype=np.uint8), x, rows, cols)
    xb = x.reshape(-1, 32)
    want = [sum(float(ds[r, b]) * (float(np.dot(nib[r, 32 * b:32 * b + 32], xb[b])) - 8.0 * float(xb[b].sum()))
                for b in range(cols // 32)) for r in range(rows)]
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("fmt", [oq.FMT_Q8_0, oq.FMT_Q4_0, oq.FMT_I4_ROW])
def test_linearity_and_rows_subset(fmt):
    import synth
    rows, cols = 37, 192
    W = synth.matrix(fmt, rows, cols, 1, "lin").numpy()
    x1 = synth.normal(1, 11, cols).numpy()
    x2 = synth.normal(1, 12, cols).numpy()
    y1 = oq.qgemv(fmt, W, x1, rows, cols)
    y2 = oq.qgemv(fmt, W, x2, rows, cols)
    y12 = oq.qgemv(fmt, W, 2.0 * x1 - 0.5 * x2, rows, cols)
    np.testing.assert_allclose(y12, 2.0 * y1 - 0.5 * y2, rtol=1e-12, atol=1e-12)
    sel = [0, 5, 36]
    np.testing.assert_allclose(oq.qgemv_rows(fmt, W, x1, rows, cols, sel), y1[sel], rtol=1e-14, atol=1e-14)
    # dequantize() agrees with the block formula
    np.testing.assert_allclose(oq.dequantize(fmt, W, rows, cols) @ x1, y1, rtol=1e-12, atol=1e-12)


def test_i4_row_scale_factors_out():
    import synth
    rows, cols = 8, 64
    W = synth.i4_row_matrix(rows, cols, 2, "sc").numpy().copy()
    x = synth.normal(2, 3, cols).numpy()
    y = oq.qgemv(oq.FMT_I4_ROW, W, x, rows, cols)
    off = oq.i4_row_scale_offset(rows, cols)
    s = W[off:off + 4 * rows].view("<f4").copy()
    W2 = W.copy()
    W2[off:off + 4 * rows] = np.ones(rows, dtype="<f4").view(np.uint8)
    y_int = oq.qgemv(oq.FMT_I4_ROW, W2, x, rows, cols)
    np.testing.assert_allclose(y, s.astype(np.float64) * y_int, rtol=1e-14)


# ---------------------------------------------------------------- packed int2 with a per-row scale
def _i2_pack_row(vals):
    """Bytes of one row of 2-bit two's-complement values, element 4j+k in bits 2k..2k+1 of byte j
    (written out by shifting each value into place, independently of the oracle's decoder)."""
    out = bytearray()
    for j in range(len(vals) // 4):
        b = 0
        for k in range(4):
            b |= (int(vals[4 * j + k]) & 0x3) << (2 * k)
        out.append(b)
    return bytes(out)


def test_i2_row_golden_probes(golden_dir):
    g = _load(golden_dir, "i2_row_hand.json")
    for p in g["probes"]:
        raw = bytes([p["byte"]]) + bytes(15) + struct.pack("<f", 1.0)
        W = np.frombuffer(raw, dtype=np.uint8)
        for j, want in enumerate(p["values"]):
            x = np.zeros(4)
            x[j] = 1.0
            assert oq.qgemv(oq.FMT_I2_ROW, W, x, 1, 4)[0] == want, (p, j)
    h = g["hand_row"]
    raw = bytes(h["bytes"]) + bytes(12) + struct.pack("<f", h["scale"])
    y = oq.qgemv(oq.FMT_I2_ROW, np.frombuffer(raw, dtype=np.uint8), np.ones(16), 1, 16)
    assert y[0] == h["y"]


def test_i2_row_random_tiny_matches_exact_rational():
    rng = np.random.default_rng(21)
    rows, cols = 6, 16
    vals = rng.integers(-2, 2, (rows, cols))
    s = rng.uniform(-1, 1, rows).astype(np.float32)
    packed = b"".join(_i2_pack_row(vals[r]) for r in range(rows))
    off = (len(packed) + 15) // 16 * 16
    raw = packed + bytes(off - len(packed)) + s.astype("<f4").tobytes()
    x = rng.standard_normal(cols).astype(np.float32)
    got = oq.qgemv(oq.FMT_I2_ROW, np.frombuffer(raw, dtype=np.uint8), x, rows, cols)
    for r in range(rows):
        want = Fraction(float(s[r])) * sum(int(vals[r, i]) * Fraction(float(x[i])) for i in range(cols))
        assert abs(Fraction(got[r]) - want) <= Fraction(1, 10 ** 9) * (1 + abs(want))


def test_i2_row_unit_probes_pin_the_order():
    """x = e_j returns s_r * q_rj for every j of a random row."""
    rng = np.random.default_rng(23)
    cols = 64
    vals = rng.integers(-2, 2, cols)
    raw = _i2_pack_row(vals) + bytes(0) + struct.pack("<f", 0.25)
    for j in range(cols):
        x = np.zeros(cols)
        x[j] = 1.0
        assert oq.qgemv(oq.FMT_I2_ROW, np.frombuffer(raw, dtype=np.uint8), x, 1, cols)[0] == 0.25 * vals[j]


def test_i2_row_unit_scale_is_integer_matvec_and_scale_factors_out():
    import synth
    rows, cols = 9, 128
    W = synth.i2_row_matrix(rows, cols, 4, "i2sc").numpy().copy()
    x = synth.normal(4, 5, cols).numpy()
    off = oq.i2_row_scale_offset(rows, cols)
    s = W[off:off + 4 * rows].view("<f4").copy().astype(np.float64)
    W1 = W.copy()
    W1[off:off + 4 * rows] = np.ones(rows, dtype="<f4").view(np.uint8)
    xi = np.arange(cols, dtype=np.float64) % 7 - 3
    # naive integer matvec from the raw bytes by explicit bit extraction
    rb = cols // 4
    want = []
    for r in range(rows):
        acc = 0
        for i in range(cols):
            c = (int(W[r * rb + i // 4]) >> (2 * (i % 4))) & 3
            acc += (c - 4 if c >= 2 else c) * int(xi[i])
        want.append(acc)
    assert oq.qgemv(oq.FMT_I2_ROW, W1, xi, rows, cols).tolist() == want
    np.testing.assert_allclose(oq.qgemv(oq.FMT_I2_ROW, W, x, rows, cols),
                               s * oq.qgemv(oq.FMT_I2_ROW, W1, x, rows, cols), rtol=1e-14)
    np.testing.assert_allclose(oq.dequantize(oq.FMT_I2_ROW, W, rows, cols) @ x,
                               oq.qgemv(oq.FMT_I2_ROW, W, x, rows, cols), rtol=1e-12, atol=1e-12)


def test_i2_row_expert_size():
    """A GLM-like expert (gate, up 2048 x 6144, down 6144 x 2048) in packed int2: a quarter byte per
    weight plus fp32 row scales."""
    import synth
    b = 2 * synth.weight_bytes(oq.FMT_I2_ROW, 2048, 6144) + synth.weight_bytes(oq.FMT_I2_ROW, 6144, 2048)
    assert b == 3 * 2048 * 6144 // 4 + 4 * (2048 + 2048 + 6144)
