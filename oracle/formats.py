"""Number formats of the FP4 main-KV cache, from their closed-form definitions.

The cache stores E2M1 codes with one E4M3 scale per 16 channels, NVFP4 style
but without the tensor-wide scale (ai-wave.ru, "DeepSeek V4.1-Flash: 1M
контекст, FP4 KV-кэш ...", fourth paragraph; globalfeed.ai, "DeepSeek-V4.1-Flash
çıktı ...", section "Mimari tarafında ne değişti"; agentnet.co.il, "דיפסיק
משיקה את V4.1-פלאש ...", section "קוונטיזציה ופריסה: FP4 ו-DRAM במקום SSD").
The pages name the formats only; their bit layouts are the OCP
microscaling-format definitions: E2M1 = sign, 2 exponent bits (bias 1), 1
mantissa bit, no inf/NaN; E4M3 ("FN") = sign, 4 exponent bits (bias 7), 3
mantissa bits, no inf, NaN at S.1111.111.

Pinned by tests/test_oracle_formats.py (printed value tables of the formats,
extreme values, code counts).
"""
from __future__ import annotations

import numpy as np


def e2m1_value(code: int) -> float:
    """Value of a 4-bit E2M1 code (bit 3 sign, bits 2..1 exponent, bit 0 mantissa)."""
    sign = -1.0 if code & 0x8 else 1.0
    e = (code >> 1) & 0x3
    m = code & 0x1
    if e == 0:
        mag = m * 0.5                      # subnormal: m/2 * 2^(1-1)
    else:
        mag = (1.0 + m / 2.0) * 2.0 ** (e - 1)
    return sign * mag


def e4m3_value(byte: int) -> float:
    """Value of an 8-bit E4M3 (FN) byte; NaN for S.1111.111."""
    sign = -1.0 if byte & 0x80 else 1.0
    e = (byte >> 3) & 0xF
    m = byte & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        mag = (m / 8.0) * 2.0 ** -6          # subnormal
    else:
        mag = (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return sign * mag


E2M1_VALUES = np.array([e2m1_value(c) for c in range(16)], dtype=np.float64)
E4M3_VALUES = np.array([e4m3_value(b) for b in range(256)], dtype=np.float64)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns (uint16) -> float64 (exact)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    with np.errstate(invalid="ignore"):
        return b.view(np.float32).astype(np.float64)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns (uint16) -> float32 (exact)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32)


def f32_to_bf16(x: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns, round to nearest, ties to even."""
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    nan = (u & 0x7FFFFFFF) > 0x7F800000
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    r = np.where(nan, (u >> 16) | 0x40, r)
    return r.astype(np.uint16)
