"""Oracle: block-quantized matrix-vector products, dequantized exactly and accumulated in float64.

Sources (page, section):
* Q8_0 — Camelid README, "Engine status" table (Q8_0 inference row) and the model
  rows quantized Q8_0; Camelid README, "Gemma 4" (Q8_0 projection GEMVs).
* Q4_0 — Camelid README, "Gemma 4" (Q4_0 projections decoded on the GPU by
  parity-gated GEMVs) and "Experimental lanes" (per-kernel q4_0 GEMV unit tests).
* packed int4 and packed int2 with a per-row scale — colibri wiki summary, "구현 범위"
  (int8 / packed int4 / packed int2 quantization with per-row scale).

The pages name the formats but print no byte layout.  Readings taken (each pinned
by a test under tests/):
* Q8_0 block = 34 bytes: little-endian fp16 scale d, then 32 int8 q; value = d*q.
* Q4_0 block = 18 bytes: fp16 d, then 16 bytes qs; element 2j is the LOW nibble of
  qs[j], element 2j+1 the HIGH nibble; value = (q - 8)*d with q in 0..15.
* i4_row: row r is cols/2 bytes, element 2j in the low nibble of byte j, nibbles are
  two's complement (-8..7); after all rows, zero padding to a 16-byte boundary, then
  one little-endian fp32 scale per row; y_r = s_r * sum_i q_ri x_i.
* i2_row: row r is cols/4 bytes, element 4j+k in bits 2k..2k+1 of byte j (lowest bits first),
  two's complement (0b00 = 0, 0b01 = 1, 0b10 = -2, 0b11 = -1); after all rows, zero padding to a
  16-byte boundary, then one little-endian fp32 scale per row; y_r = s_r * sum_i q_ri x_i.
* Rows are stored one after another; row r holds its cols/32 blocks in order.

This module is test infrastructure: only tests, the smoke check and the
benchmark's CPU-baseline leg call it.
"""
from __future__ import annotations

import numpy as np

FMT_Q8_0, FMT_Q4_0, FMT_I4_ROW, FMT_I2_ROW = 1, 2, 3, 4
QK = 32  # weights per block


def _fp16_to_f64(lo_hi: np.ndarray) -> np.ndarray:
    """Two little-endian bytes -> the fp16 value they encode, as float64 (exact)."""
    bits = lo_hi[..., 0].astype(np.uint16) | (lo_hi[..., 1].astype(np.uint16) << 8)
    return bits.view(np.float16).astype(np.float64)


def q8_0_decode(W: np.ndarray, rows: int, cols: int):
    """Split a Q8_0 matrix into scales d[rows, nb] (float64) and quants q[rows, nb, 32] (int64)."""
    nb = cols // QK
    blk = np.asarray(W, dtype=np.uint8)[: rows * nb * 34].reshape(rows, nb, 34)
    d = _fp16_to_f64(blk[:, :, 0:2])
    q = blk[:, :, 2:34].view(np.int8).astype(np.int64)
    return d, q


def q4_0_decode(W: np.ndarray, rows: int, cols: int):
    """Split a Q4_0 matrix into d[rows, nb] and the raw nibbles q[rows, nb, 32] in 0..15.

    Element 2j of a block is the low nibble of qs[j]; element 2j+1 the high nibble."""
    nb = cols // QK
    blk = np.asarray(W, dtype=np.uint8)[: rows * nb * 18].reshape(rows, nb, 18)
    d = _fp16_to_f64(blk[:, :, 0:2])
    qs = blk[:, :, 2:18].astype(np.int64)
    q = np.empty((rows, nb, QK), dtype=np.int64)
    q[:, :, 0::2] = qs & 0x0F
    q[:, :, 1::2] = qs >> 4
    return d, q


def i4_row_scale_offset(rows: int, cols: int) -> int:
    return (rows * (cols // 2) + 15) // 16 * 16


def i4_row_decode(W: np.ndarray, rows: int, cols: int):
    """Split an i4_row matrix into signed nibbles q[rows, cols] in -8..7 and fp32 scales s[rows]."""
    W = np.asarray(W, dtype=np.uint8)
    packed = W[: rows * (cols // 2)].reshape(rows, cols // 2).astype(np.int64)
    u = np.empty((rows, cols), dtype=np.int64)
    u[:, 0::2] = packed & 0x0F
    u[:, 1::2] = packed >> 4
    q = np.where(u >= 8, u - 16, u)              # two's complement nibble
    off = i4_row_scale_offset(rows, cols)
    s = W[off: off + 4 * rows].view("<f4").astype(np.float64)
    return q, s


def i2_row_scale_offset(rows: int, cols: int) -> int:
    return (rows * (cols // 4) + 15) // 16 * 16


def i2_row_decode(W: np.ndarray, rows: int, cols: int):
    """Split an i2_row matrix into signed 2-bit values q[rows, cols] in -2..1 and fp32 scales s[rows]."""
    W = np.asarray(W, dtype=np.uint8)
    packed = W[: rows * (cols // 4)].reshape(rows, cols // 4).astype(np.int64)
    u = np.empty((rows, cols), dtype=np.int64)
    for k in range(4):                            # element 4j+k: bits 2k..2k+1 of byte j
        u[:, k::4] = (packed >> (2 * k)) & 0x3
    q = np.where(u >= 2, u - 4, u)                # two's complement
    off = i2_row_scale_offset(rows, cols)
    s = W[off: off + 4 * rows].view("<f4").astype(np.float64)
    return q, s


def dequantize(fmt: int, W: np.ndarray, rows: int, cols: int) -> np.ndarray:
    """Every weight as a float64 value (exact: an fp16 or fp32 scale times a small integer)."""
    if fmt == FMT_Q8_0:
        d, q = q8_0_decode(W, rows, cols)
        return (d[:, :, None] * q).reshape(rows, cols)
    if fmt == FMT_Q4_0:
        d, q = q4_0_decode(W, rows, cols)
        return (d[:, :, None] * (q - 8)).reshape(rows, cols)
    if fmt == FMT_I4_ROW:
        q, s = i4_row_decode(W, rows, cols)
        return s[:, None] * q
    if fmt == FMT_I2_ROW:
        q, s = i2_row_decode(W, rows, cols)
        return s[:, None] * q
    raise ValueError(f"unknown format {fmt}")


def qgemv(fmt: int, W: np.ndarray, x: np.ndarray, rows: int, cols: int) -> np.ndarray:
    """y = W x in float64, written as the block formula of each format.

    Q8_0:  y_r = sum_b d_rb * sum_i q_rbi * x_{32b+i}
    Q4_0:  y_r = sum_b d_rb * sum_i (q_rbi - 8) * x_{32b+i}
    i4_row, i2_row: y_r = s_r * sum_i q_ri * x_i
    """
    x = np.asarray(x, dtype=np.float64).reshape(cols)
    if fmt in (FMT_Q8_0, FMT_Q4_0):
        nb = cols // QK
        xb = x.reshape(nb, QK)
        if fmt == FMT_Q8_0:
            d, q = q8_0_decode(W, rows, cols)
        else:
            d, q = q4_0_decode(W, rows, cols)
            q = q - 8
        inner = np.einsum("rbi,bi->rb", q.astype(np.float64), xb)   # sum over the 32 weights of each block
        return (d * inner).sum(axis=1)
    if fmt == FMT_I4_ROW:
        q, s = i4_row_decode(W, rows, cols)
        return s * (q.astype(np.float64) @ x)
    if fmt == FMT_I2_ROW:
        q, s = i2_row_decode(W, rows, cols)
        return s * (q.astype(np.float64) @ x)
    raise ValueError(f"unknown format {fmt}")


def qgemv_rows(fmt: int, W: np.ndarray, x: np.ndarray, rows: int, cols: int, sel) -> np.ndarray:
    """Selected outputs y[sel] only (rows decoded one at a time), for spot checks of large matrices."""
    x = np.asarray(x, dtype=np.float64).reshape(cols)
    W = np.asarray(W, dtype=np.uint8)
    out = []
    for r in np.asarray(sel).reshape(-1):
        r = int(r)
        if fmt == FMT_Q8_0:
            rb = (cols // QK) * 34
            out.append(qgemv(fmt, W[r * rb:(r + 1) * rb], x, 1, cols)[0])
        elif fmt == FMT_Q4_0:
            rb = (cols // QK) * 18
            out.append(qgemv(fmt, W[r * rb:(r + 1) * rb], x, 1, cols)[0])
        elif fmt in (FMT_I4_ROW, FMT_I2_ROW):
            rb = cols // 2 if fmt == FMT_I4_ROW else cols // 4
            sofs = i4_row_scale_offset if fmt == FMT_I4_ROW else i2_row_scale_offset
            off = sofs(rows, cols)
            one = np.zeros(sofs(1, cols) + 4, dtype=np.uint8)
            one[:rb] = W[r * rb:(r + 1) * rb]
            soff = sofs(1, cols)
            one[soff:soff + 4] = W[off + 4 * r: off + 4 * r + 4]
            out.append(qgemv(fmt, one, x, 1, cols)[0])
        else:
            raise ValueError(f"unknown format {fmt}")
    return np.array(out, dtype=np.float64)
