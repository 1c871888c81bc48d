"""FP4 main-KV codec: E2M1 codes with one E4M3 scale per 16 channels.

What the pages fix: the main KV is stored as E2M1 values with a single E4M3
scale for every 16 channels, following NVFP4 without its global scale
(agentnet.co.il, "דיפסיק משיקה את V4.1-פלאש ...", section "קוונטיזציה ופריסה:
FP4 ו-DRAM במקום SSD"; ai-wave.ru, "DeepSeek V4.1-Flash: 1M контекст ...",
fourth paragraph; globalfeed.ai, "DeepSeek-V4.1-Flash çıktı ...", section
"Mimari tarafında ne değişti").

Readings taken where the pages are silent (the NVFP4 convention):

* scale  = the E4M3 value nearest to amax/6 (amax = max |x| over the group,
  6 = the largest E2M1 magnitude), ties to the even code, saturating at 448;
* code   = sign bit of x | the E2M1 magnitude nearest to |x|/scale, ties to
  the even code, saturating at 6 (a negative value that rounds to zero keeps
  its sign: code 0x8);
* a group whose scale rounds to 0 stores code 0x0 in all 16 slots;
* channel 2j goes to the low nibble of byte j, channel 2j+1 to the high one;
* one 512-channel row = 256 code bytes followed by 32 scale bytes = 288 B.

Both roundings are written as the plain definition (nearest point of a finite
grid, compared exactly against the grid's midpoints in fp64, where every
product below is exact).

Pinned by tests/test_oracle_codec.py: exhaustive comparison with a brute-force
nearest-value search over all bf16 inputs and all scales, the division form
used by hardware converters, round trips on grid values, error bounds and the
288-byte accounting.
"""
from __future__ import annotations

import numpy as np

from .formats import E2M1_VALUES, E4M3_VALUES, bf16_to_f64, f32_to_bf16, bf16_to_f32

D = 512                 # latent channels per token (K = V)
GROUP = 16              # channels per E4M3 scale
N_GROUPS = D // GROUP   # 32
CODE_BYTES = D // 2     # 256
ROW_BYTES = CODE_BYTES + N_GROUPS   # 288

# non-negative finite E4M3 values, codes 0x00..0x7E, ascending with the code
E4M3_GRID = E4M3_VALUES[:127].copy()
E4M3_MIDS = (E4M3_GRID[:-1] + E4M3_GRID[1:]) / 2.0          # 126 midpoints, exact
E2M1_GRID = E2M1_VALUES[:8].copy()                          # 0, .5, 1, 1.5, 2, 3, 4, 6
E2M1_MIDS = (E2M1_GRID[:-1] + E2M1_GRID[1:]) / 2.0          # .25 .75 1.25 1.75 2.5 3.5 5


def _round_to_grid(t: np.ndarray, thresholds: np.ndarray) -> np.ndarray:
    """Index of the grid point nearest to t, ties to the even index, given the
    grid's midpoints `thresholds` (ascending along the last axis, broadcast
    against t[..., None]).  Values past the last midpoint saturate."""
    t = np.asarray(t, dtype=np.float64)[..., None]
    below = np.sum(thresholds < t, axis=-1)                 # midpoints strictly below t
    tie = np.any(thresholds == t, axis=-1)                  # t exactly on a midpoint
    return below + (tie & (below % 2 == 1))


def scale_code(amax: np.ndarray) -> np.ndarray:
    """E4M3 code (0..126) of the scale for a group with absolute maximum amax.

    Nearest E4M3 value to amax/6, ties to even, saturating: compared as
    amax against 6 x midpoint, which is exact in fp64."""
    return _round_to_grid(amax, 6.0 * E4M3_MIDS).astype(np.uint8)


def e2m1_code(x: np.ndarray, s: np.ndarray) -> np.ndarray:
    """4-bit codes of values x under scale values s (s > 0, broadcast to x)."""
    x = np.asarray(x, dtype=np.float64)
    s = np.broadcast_to(np.asarray(s, dtype=np.float64), x.shape)
    mag = _round_to_grid(np.abs(x), s[..., None] * E2M1_MIDS)
    return (mag | (np.signbit(x).astype(np.int64) << 3)).astype(np.uint8)


def quantize_rows(x: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Quantize rows of 512 exact values (bf16 or fp32 inputs, given as fp64).

    Returns (codes [n,512] uint8 nibbles, scales [n,32] uint8 E4M3 bytes)."""
    x = np.asarray(x, dtype=np.float64)
    n = x.shape[0]
    g = x.reshape(n, N_GROUPS, GROUP)
    amax = np.abs(g).max(axis=-1)
    sc = scale_code(amax)
    s = E4M3_GRID[sc]
    codes = e2m1_code(g, s[..., None])
    codes = np.where((s == 0.0)[..., None], np.uint8(0), codes)
    return codes.reshape(n, D).astype(np.uint8), sc


def pack_rows(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """[n,512] nibbles + [n,32] scale bytes -> [n,288] cache rows."""
    codes = np.asarray(codes, dtype=np.uint8)
    packed = (codes[:, 0::2] & 0xF) | ((codes[:, 1::2] & 0xF) << 4)
    return np.concatenate([packed.astype(np.uint8), np.asarray(scales, dtype=np.uint8)], axis=1)


def unpack_rows(rows: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """[n,288] cache rows -> ([n,512] nibbles, [n,32] scale bytes)."""
    rows = np.asarray(rows, dtype=np.uint8)
    packed = rows[:, :CODE_BYTES]
    codes = np.empty((rows.shape[0], D), dtype=np.uint8)
    codes[:, 0::2] = packed & 0xF
    codes[:, 1::2] = packed >> 4
    return codes, rows[:, CODE_BYTES:ROW_BYTES].copy()


def dequantize(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Decoded values [n,512] in fp64 (exact: every product has <= 6 significant bits)."""
    n = codes.shape[0]
    v = E2M1_VALUES[np.asarray(codes, dtype=np.int64)].reshape(n, N_GROUPS, GROUP)
    s = E4M3_VALUES[np.asarray(scales, dtype=np.int64)]
    return (v * s[..., None]).reshape(n, D)


def encode_bf16_rows(kv_bits: np.ndarray) -> np.ndarray:
    """bf16 rows [n,512] -> packed 288-byte cache rows (ratio-1 path)."""
    codes, scales = quantize_rows(bf16_to_f64(kv_bits))
    return pack_rows(codes, scales)


# ---------------------------------------------------------------------------
# 2:1 sequence compression (encoder layers, compression ratio 2)
# ---------------------------------------------------------------------------
# The encoder's CSA2 layers run at compression ratio 2 (agentnet.co.il,
# section "CSA2: דחיסה לאורך ציר השכבות"; globalfeed.ai, section "Mimari
# tarafında ne değişti").  The pages do not say how two tokens become one entry;
# the reading taken is the mean of the adjacent pair (2c, 2c+1), in fp32.

def compress_pairs_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 rows [2m, C] -> fp32 [m, C]: (x[2c] + x[2c+1]) * 0.5 in fp32."""
    x = bf16_to_f32(bits)
    a = x[0::2]
    b = x[1::2]
    return ((a + b).astype(np.float32) * np.float32(0.5)).astype(np.float32)


def encode_entries(kv_bits: np.ndarray, compress: int) -> np.ndarray:
    """Raw bf16 rows -> packed cache rows for compression ratio 1 or 2."""
    if compress == 1:
        return encode_bf16_rows(kv_bits)
    if compress == 2:
        codes, scales = quantize_rows(compress_pairs_f32(kv_bits).astype(np.float64))
        return pack_rows(codes, scales)
    raise ValueError(compress)


def idxk_entries(idxk_bits: np.ndarray, compress: int) -> np.ndarray:
    """Raw bf16 indexer keys -> stored bf16 keys (pair mean rounded to bf16 at ratio 2)."""
    if compress == 1:
        return np.asarray(idxk_bits, dtype=np.uint16).copy()
    if compress == 2:
        return f32_to_bf16(compress_pairs_f32(idxk_bits))
    raise ValueError(compress)
