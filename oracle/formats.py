"""Byte formats of the indexer caches, decoded from their definitions (fp64).

* bf16: the upper 16 bits of an IEEE-754 binary32 value.
* fp8 e4m3 ("fn" variant, as the 128 B indexer key of "03 long context",
  section "The Architectural Answer: Read Less of the Past"): 1 sign bit,
  4 exponent bits with bias 7, 3 mantissa bits; exponent field 0 encodes
  subnormals m/8 * 2^-6; codes 0x7F / 0xFF are NaN; there is no infinity.
* int8: two's complement.

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
