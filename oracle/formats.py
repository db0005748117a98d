"""Byte formats of the indexer caches, decoded from their definitions (fp64).

* bf16: the upper 16 bits of an IEEE-754 binary32 value.
* fp8 e4m3 ("fn" variant, as the 128 B indexer key of "03 long context",
  section "The Architectural Answer: Read Less of the Past"): 1 sign bit,
  4 exponent bits with bias 7, 3 mantissa bits; exponent field 0 encodes
  subnormals m/8 * 2^-6; codes 0x7F / 0xFF are NaN; there is no infinity.
* int8: two's complement.
* fp16 (IEEE-754 binary16, the PQ codebook entries): 1 sign bit, 5 exponent
  bits with bias 15, 10 mantissa bits; exponent 0 encodes subnormals
  m/1024 * 2^-14; exponent 31 encodes infinities (m = 0) and NaN.
* PQ compact key (LeanSparse podcast transcript, 07:12-07:34, 32-byte
  compact keys): 32 one-byte codes, code m selecting row code[m] of the
  m-th codebook [256][4]; the decoded key is the 32 selected 4-vectors laid
  end to end.

Scaled formats multiply the decoded value by the per-key fp32 scale (the 4 B
scale beside the 128 B key, same section).
"""

from __future__ import annotations

import numpy as np


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float64, exactly."""
    b = np.asarray(bits).astype(np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def e4m3_to_f64(codes: np.ndarray) -> np.ndarray:
    """fp8 e4m3 codes (uint8) -> float64, exactly, from the field layout."""
    c = np.asarray(codes).astype(np.int64)
    sign = np.where((c >> 7) & 1, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    normal = (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0)
    sub = (m / 8.0) * 2.0 ** -6
    val = sign * np.where(e == 0, sub, normal)
    return np.where((e == 15) & ((c & 7) == 7), np.nan, val)


def f16_to_f64(bits: np.ndarray) -> np.ndarray:
    """fp16 bit patterns (uint16) -> float64, exactly, from the field layout."""
    b = np.asarray(bits).astype(np.int64)
    sign = np.where((b >> 15) & 1, -1.0, 1.0)
    e = (b >> 10) & 0x1F
    m = (b & 0x3FF).astype(np.float64)
    normal = (1.0 + m / 1024.0) * np.exp2(e.astype(np.float64) - 15.0)
    sub = (m / 1024.0) * 2.0 ** -14
    val = sign * np.where(e == 0, sub, normal)
    val = np.where(e == 31, np.where(m == 0, sign * np.inf, np.nan), val)
    return val


def pq_decode(codes: np.ndarray, books_bits: np.ndarray) -> np.ndarray:
    """[..., 32] uint8 PQ codes and [32][256][4] fp16 codebooks -> [..., 128]
    float64 keys: sub-vector m is codebook m's row codes[..., m]."""
    books = f16_to_f64(books_bits)                       # [32, 256, 4]
    c = np.asarray(codes).astype(np.int64)
    parts = [books[m][c[..., m]] for m in range(c.shape[-1])]  # each [..., 4]
    return np.concatenate(parts, axis=-1)


def int8_to_f64(codes: np.ndarray) -> np.ndarray:
    return np.asarray(codes).astype(np.int8).astype(np.float64)


def dequant(codes: np.ndarray, scale: np.ndarray, fmt: str) -> np.ndarray:
    """[..., d] codes and [...] fp32 scales -> [..., d] float64 key values."""
    if fmt == "bf16":
        return bf16_to_f64(codes)
    s = np.asarray(scale, dtype=np.float32).astype(np.float64)[..., None]
    if fmt == "e4m3":
        return e4m3_to_f64(codes) * s
    if fmt == "int8":
        return int8_to_f64(codes) * s
    raise ValueError(fmt)
