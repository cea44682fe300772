"""Seeded synthetic inputs shared by the CUDA path's tests/benchmark and the CPU oracle.

This module holds no arithmetic of the method itself (no dequantisation, no dot
products, no routing).  It only draws random numbers and lays them out in the
byte formats the method consumes:

* ``q8_0``  : rows x (cols/32) blocks of 34 bytes ``{fp16 d; int8 q[32]}``
* ``q4_0``  : rows x (cols/32) blocks of 18 bytes ``{fp16 d; uint8 qs[16]}``
* ``i4_row``: rows x (cols/2) packed bytes, zero padding to a 16-byte boundary,
  then ``rows`` little-endian fp32 scales.
* ``i2_row``: rows x (cols/4) packed bytes (four 2-bit values per byte), zero padding to a
  16-byte boundary, then ``rows`` little-endian fp32 scales.

Randomness comes from a counter-based generator: every 32-bit word is a pure
function of ``(seed, stream, index)``, so any tensor (or any single expert of a
39 GB stack) can be regenerated on its own, on the host or on the GPU, with
identical bytes.  The word function is the MurmurHash3 32-bit finaliser
("fmix32", Austin Appleby, public domain) applied twice to the counter xor a
per-stream key.  Integer torch ops are exact on every device, so the same code
gives the same bytes on CPU and CUDA.

Gaussian values (activations, router matrices, logits) are drawn on the host
only (Box-Muller in float64) and moved to the device by the caller, so there is
no cross-device floating-point difference.
"""
from __future__ import annotations

import math
import zlib
from typing import Optional

import torch

M32 = 0xFFFFFFFF
_GOLDEN = 0x9E3779B9


# ---------------------------------------------------------------- word generator
def _mul32_t(h: torch.Tensor, c: int) -> torch.Tensor:
    """(h * c) mod 2**32 for int64 tensors with 0 <= h < 2**32, without int64 overflow."""
    c_lo, c_hi = c & 0xFFFF, c >> 16
    return (h * c_lo + (((h * c_hi) & 0xFFFF) << 16)) & M32


def _fmix32_t(h: torch.Tensor) -> torch.Tensor:
    h = h ^ (h >> 16)
    h = _mul32_t(h, 0x85EBCA6B)
    h = h ^ (h >> 13)
    h = _mul32_t(h, 0xC2B2AE35)
    return h ^ (h >> 16)


def _fmix32_i(h: int) -> int:
    h &= M32
    h ^= h >> 16
    h = (h * 0x85EBCA6B) & M32
    h ^= h >> 13
    h = (h * 0xC2B2AE35) & M32
    return h ^ (h >> 16)


def stream_id(name: str) -> int:
    """Stable 32-bit stream id for a named tensor role (CRC-32 of the name)."""
    return zlib.crc32(name.encode()) & M32


def _keys(seed: int, stream: int) -> tuple[int, int]:
    k1 = _fmix32_i((seed & M32) ^ _fmix32_i(stream ^ _GOLDEN))
    k2 = _fmix32_i(k1 ^ ((seed >> 32) & M32) ^ 0x7F4A7C15)
    return k1, k2


def words(seed: int, stream: int, n: int, device="cpu", start: int = 0) -> torch.Tensor:
    """n pseudo-random 32-bit words (int64 tensor, values in [0, 2**32)) for counters start..start+n-1."""
    k1, k2 = _keys(seed, stream)
    i = torch.arange(start, start + n, dtype=torch.int64, device=device)
    h = _fmix32_t((i & M32) ^ k1)
    return _fmix32_t(h ^ (((i >> 32) + k2) & M32))


def _words_as_bytes(w: torch.Tensor) -> torch.Tensor:
    """Little-endian bytes of 32-bit words (uint8 tensor of 4*len(w))."""
    w32 = torch.where(w >= 2**31, w - 2**32, w).to(torch.int32)
    return w32.view(torch.uint8)


def random_bytes(seed: int, stream: int, nbytes: int, device="cpu", start: int = 0) -> torch.Tensor:
    """Bytes start..start+nbytes-1 of the stream (byte b is byte b%4 of word b//4)."""
    w0 = start // 4
    nw = (start + nbytes + 3) // 4 - w0
    b = _words_as_bytes(words(seed, stream, nw, device, start=w0))
    return b[start - 4 * w0: start - 4 * w0 + nbytes]


def uniform_f32(seed: int, stream: int, n: int, lo: float, hi: float, device="cpu", start: int = 0) -> torch.Tensor:
    """float32 values lo + (hi-lo)*u with u = k/2**24, k uniform in [0, 2**24).

    Every step is a single correctly rounded fp32 operation on fp32 tensors, so the
    result is bit-identical on CPU and GPU."""
    u = (words(seed, stream, n, device, start=start) >> 8).to(torch.float32) * (2.0 ** -24)
    span = torch.tensor(hi - lo, dtype=torch.float32, device=device)
    base = torch.tensor(lo, dtype=torch.float32, device=device)
    return u * span + base


def uniform_f16(seed: int, stream: int, n: int, lo: float, hi: float, device="cpu", start: int = 0) -> torch.Tensor:
    """fp16 scale values: the fp32 uniform value rounded to fp16 (round-to-nearest-even)."""
    return uniform_f32(seed, stream, n, lo, hi, device, start).to(torch.float16)


def int8_uniform(seed: int, stream: int, n: int, lo: int = -127, hi: int = 127, device="cpu",
                 start: int = 0) -> torch.Tensor:
    span = hi - lo + 1
    return ((words(seed, stream, n, device, start=start) % span) + lo).to(torch.int8)


# ---------------------------------------------------------------- gaussians (host only)
def normal(seed: int, stream: int, n: int, std: float = 1.0) -> torch.Tensor:
    """Host float64 N(0, std^2) draws by the Box-Muller transform, returned as float64."""
    w = words(seed, stream, 2 * n, "cpu").view(n, 2).to(torch.float64)
    u1 = (w[:, 0] + 1.0) * (2.0 ** -32)          # (0, 1]
    u2 = w[:, 1] * (2.0 ** -32)                  # [0, 1)
    z = torch.sqrt(-2.0 * torch.log(u1)) * torch.cos(2.0 * math.pi * u2)
    return z * std


def normal_f32(seed: int, stream: int, n: int, std: float = 1.0) -> torch.Tensor:
    return normal(seed, stream, n, std).to(torch.float32)


def normal_f16(seed: int, stream: int, n: int, std: float = 1.0) -> torch.Tensor:
    return normal(seed, stream, n, std).to(torch.float16)


# ---------------------------------------------------------------- block layouts
Q8_0_BLOCK = 34
Q4_0_BLOCK = 18
FMT_Q8_0, FMT_Q4_0, FMT_I4_ROW, FMT_I2_ROW = 1, 2, 3, 4


def weight_bytes(fmt: int, rows: int, cols: int) -> int:
    """Byte size of a rows x cols matrix in the canonical layout of ``fmt``."""
    if fmt == FMT_Q8_0:
        return rows * (cols // 32) * Q8_0_BLOCK
    if fmt == FMT_Q4_0:
        return rows * (cols // 32) * Q4_0_BLOCK
    if fmt == FMT_I4_ROW:
        return i4_row_scale_offset(rows, cols) + 4 * rows
    if fmt == FMT_I2_ROW:
        return i2_row_scale_offset(rows, cols) + 4 * rows
    raise ValueError(f"unknown format {fmt}")


def i4_row_scale_offset(rows: int, cols: int) -> int:
    """Byte offset of the fp32 row scales inside an i4_row matrix (packed data padded to 16 B)."""
    packed = rows * (cols // 2)
    return (packed + 15) // 16 * 16


def i2_row_scale_offset(rows: int, cols: int) -> int:
    """Byte offset of the fp32 row scales inside an i2_row matrix (packed data padded to 16 B)."""
    packed = rows * (cols // 4)
    return (packed + 15) // 16 * 16


def q8_0_matrix(rows: int, cols: int, seed: int, name: str, device="cpu",
                d_range=(1e-3, 1e-2), q_range=(-127, 127), r0: int = 0, r1: Optional[int] = None) -> torch.Tensor:
    """Q8_0 matrix bytes: per block an fp16 scale d ~ U[d_range] and 32 int8 q ~ U{q_range}.
    With r0/r1, only rows r0..r1-1 of the same matrix (as a standalone matrix)."""
    assert cols % 32 == 0
    r1 = rows if r1 is None else r1
    nb = cols // 32
    b0, nblk = r0 * nb, (r1 - r0) * nb
    s = stream_id(name)
    d = uniform_f16(seed, s ^ 0x1, nblk, *d_range, device=device, start=b0).view(torch.uint8).view(nblk, 2)
    q = int8_uniform(seed, s ^ 0x2, nblk * 32, *q_range, device=device, start=32 * b0)
    q = q.view(torch.uint8).view(nblk, 32)
    return torch.cat([d, q], dim=1).reshape(-1)


def q4_0_matrix(rows: int, cols: int, seed: int, name: str, device="cpu",
                d_range=(1e-3, 1e-2), r0: int = 0, r1: Optional[int] = None) -> torch.Tensor:
    """Q4_0 matrix bytes: per block an fp16 scale d ~ U[d_range] and 16 uniformly random bytes
    (each byte holds two independent nibbles uniform in 0..15).
    With r0/r1, only rows r0..r1-1 of the same matrix (as a standalone matrix)."""
    assert cols % 32 == 0
    r1 = rows if r1 is None else r1
    nb = cols // 32
    b0, nblk = r0 * nb, (r1 - r0) * nb
    s = stream_id(name)
    d = uniform_f16(seed, s ^ 0x1, nblk, *d_range, device=device, start=b0).view(torch.uint8).view(nblk, 2)
    qs = random_bytes(seed, s ^ 0x2, nblk * 16, device=device, start=16 * b0).view(nblk, 16)
    return torch.cat([d, qs], dim=1).reshape(-1)


def i4_row_matrix(rows: int, cols: int, seed: int, name: str, device="cpu",
                  s_range=(1e-3, 1e-2), r0: int = 0, r1: Optional[int] = None) -> torch.Tensor:
    """i4_row matrix bytes: uniformly random packed nibbles (two's-complement values -8..7),
    zero padding to 16 B, then fp32 row scales ~ U[s_range].
    With r0/r1, only rows r0..r1-1 of the same matrix (as a standalone matrix)."""
    assert cols % 2 == 0
    r1 = rows if r1 is None else r1
    n = r1 - r0
    s = stream_id(name)
    rb = cols // 2
    packed = n * rb
    off = i4_row_scale_offset(n, cols)
    out = torch.zeros(off + 4 * n, dtype=torch.uint8, device=device)
    out[:packed] = random_bytes(seed, s ^ 0x2, packed, device=device, start=r0 * rb)
    out[off:] = uniform_f32(seed, s ^ 0x1, n, *s_range, device=device, start=r0).view(torch.uint8)
    return out


def i2_row_matrix(rows: int, cols: int, seed: int, name: str, device="cpu",
                  s_range=(1e-3, 1e-2), r0: int = 0, r1: Optional[int] = None) -> torch.Tensor:
    """i2_row matrix bytes: uniformly random bytes (four independent 2-bit values each),
    zero padding to 16 B, then fp32 row scales ~ U[s_range].
    With r0/r1, only rows r0..r1-1 of the same matrix (as a standalone matrix)."""
    assert cols % 4 == 0
    r1 = rows if r1 is None else r1
    n = r1 - r0
    s = stream_id(name)
    rb = cols // 4
    packed = n * rb
    off = i2_row_scale_offset(n, cols)
    out = torch.zeros(off + 4 * n, dtype=torch.uint8, device=device)
    out[:packed] = random_bytes(seed, s ^ 0x2, packed, device=device, start=r0 * rb)
    out[off:] = uniform_f32(seed, s ^ 0x1, n, *s_range, device=device, start=r0).view(torch.uint8)
    return out


def matrix(fmt: int, rows: int, cols: int, seed: int, name: str, device="cpu",
           r0: int = 0, r1: Optional[int] = None) -> torch.Tensor:
    if fmt == FMT_Q8_0:
        return q8_0_matrix(rows, cols, seed, name, device, r0=r0, r1=r1)
    if fmt == FMT_Q4_0:
        return q4_0_matrix(rows, cols, seed, name, device, r0=r0, r1=r1)
    if fmt == FMT_I4_ROW:
        return i4_row_matrix(rows, cols, seed, name, device, r0=r0, r1=r1)
    if fmt == FMT_I2_ROW:
        return i2_row_matrix(rows, cols, seed, name, device, r0=r0, r1=r1)
    raise ValueError(f"unknown format {fmt}")
