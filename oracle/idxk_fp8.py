"""FP8 indexer keys: 64 E4M3 codes and one fp32 scale per token (68 B).

The pages give the global cache's size, 890 B per token (ai-wave.ru, "DeepSeek
V4.1-Flash: 1M контекст ...", first paragraph; news.hamidun.com, "В
DeepSeek-V4.1-Flash KV-кэш в HBM сократили до 890 байт ...", lead), but not
its parts.  One accounting reproduces it exactly: the decoder's main KV row
(288 B) plus three encoder Full layers' rows at compression ratio 2, each row
with an FP8 indexer key of 64 B and a 4-B scale:
(288 + 68) + 3 (288 + 68) / 2 = 890.  This module is that key format.

Readings (the pages say nothing about the indexer key's number format):

* the FP8 key quantises the bf16 key that the bf16 format would store (the
  key itself at ratio 1, the bf16-rounded pair mean at ratio 2);
* scale s = fl32(amax / 448), amax = max_d |k_d| (448 = the largest E4M3
  value), IEEE fp32 division;
* code_d = the E4M3 value nearest to fl32(k_d / s), ties to the even code,
  saturating at 448, sign kept (a negative value that rounds to zero is
  0x80); s = 0 stores 0x00 in every slot;
* dequantised key d = fl32(s x value(code_d));
* score against a query q: fl32(s x score(q, value(codes))), the fp32 score
  of the code values scaled once -- s >= 0 factors out of the ReLU, so this
  is the score of the dequantised key up to rounding;
* block keys are built from the dequantised keys (same rule as for bf16 keys).

Page layout: 64 tokens x 64 code bytes (4096 B) then 64 fp32 scales (256 B)
= 4352 B per page; code byte d of a token is dimension d.

Pinned by tests/test_oracle_idxk_fp8.py: the E4M3 rounding against a
brute-force nearest search and against torch's float8_e4m3fn conversion,
saturation and signed zero, the error bound of the quantised key, the
890-byte accounting, scores against an fp64 evaluation on the dequantised key.
"""
from __future__ import annotations

import numpy as np

from .codec import E4M3_MIDS
from .formats import E4M3_VALUES, bf16_to_f32

IDX_DIM = 64
E4M3_MAX = 448.0
CODE_BYTES = IDX_DIM                 # 64
SCALE_BYTES = 4
ROW_BYTES = CODE_BYTES + SCALE_BYTES    # 68
PAGE_TOKENS = 64
PAGE_BYTES = PAGE_TOKENS * ROW_BYTES    # 4352
SCALE_OFFSET = PAGE_TOKENS * CODE_BYTES  # 4096: scales follow the page's codes


def e4m3_code(t: np.ndarray) -> np.ndarray:
    """E4M3 byte of fp32 values t: nearest value, ties to the even code,
    saturating at 448, sign bit kept."""
    t = np.asarray(t, dtype=np.float32)
    mag = np.abs(t.astype(np.float64))
    below = np.sum(E4M3_MIDS < mag[..., None], axis=-1)
    tie = np.any(E4M3_MIDS == mag[..., None], axis=-1)
    code = below + (tie & (below % 2 == 1))
    return (code | (np.signbit(t).astype(np.int64) << 7)).astype(np.uint8)


def quantize(key_bits: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """bf16 keys [n, 64] -> (codes uint8 [n, 64], scales float32 [n])."""
    k = bf16_to_f32(np.asarray(key_bits, dtype=np.uint16))
    amax = np.max(np.abs(k), axis=-1).astype(np.float32)
    s = (amax / np.float32(E4M3_MAX)).astype(np.float32)
    codes = np.zeros(k.shape, dtype=np.uint8)
    nz = s != 0
    t = (k[nz] / s[nz, None]).astype(np.float32)
    codes[nz] = e4m3_code(t)
    return codes, s


def code_values(codes: np.ndarray) -> np.ndarray:
    """float32 values of E4M3 codes (exact)."""
    return E4M3_VALUES[np.asarray(codes, dtype=np.int64)].astype(np.float32)


def dequantize(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """float32 [n, 64]: fl32(s x value(code))."""
    return (np.asarray(scales, dtype=np.float32)[..., None] * code_values(codes)).astype(np.float32)


class Fp8Keys:
    """A sequence's FP8 indexer keys: codes [n, 64] and scales [n]; indexable
    by position arrays like a key matrix."""

    def __init__(self, codes: np.ndarray, scales: np.ndarray):
        self.codes = np.asarray(codes, dtype=np.uint8)
        self.scales = np.asarray(scales, dtype=np.float32)

    @classmethod
    def from_bf16(cls, key_bits: np.ndarray) -> "Fp8Keys":
        return cls(*quantize(key_bits))

    def __len__(self) -> int:
        return self.codes.shape[0]

    def __getitem__(self, idx) -> "Fp8Keys":
        return Fp8Keys(self.codes[idx], self.scales[idx])

    def dequantized(self) -> np.ndarray:
        return dequantize(self.codes, self.scales)

    def pack(self) -> np.ndarray:
        """The bytes of whole pages (n a multiple of 64): [pages, 4352] uint8."""
        n = len(self)
        assert n % PAGE_TOKENS == 0
        pages = n // PAGE_TOKENS
        out = np.empty((pages, PAGE_BYTES), dtype=np.uint8)
        out[:, :SCALE_OFFSET] = self.codes.reshape(pages, SCALE_OFFSET)
        out[:, SCALE_OFFSET:] = self.scales.reshape(pages, PAGE_TOKENS).view(np.uint8).reshape(pages, -1)
        return out
