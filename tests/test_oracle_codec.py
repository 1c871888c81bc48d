"""Pins for the FP4 codec oracle: exhaustive brute force, division form, round trips,
byte accounting and the 2:1 compression special cases."""
import json
import os

import numpy as np
import pytest

from oracle import codec, formats

CONST = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_constants.json")))


def _all_finite_bf16():
    b = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    v = formats.bf16_to_f64(b)
    return b, v[np.isfinite(v)]


def _nearest_even(target, grid):
    """Brute force: index of the grid value nearest to target, ties to the even
    index, by direct distance comparison (no midpoints)."""
    d = np.abs(target[:, None] - grid[None, :])
    best = d.min(axis=1, keepdims=True)
    hits = d == best
    idx = np.argmax(hits, axis=1)                      # lowest index at the min distance
    two = hits.sum(axis=1) > 1
    nxt = idx + 1
    idx = np.where(two & (idx % 2 == 1), nxt, idx)
    return idx


def test_e2m1_code_exhaustive_vs_brute_force_and_division_form():
    _, x = _all_finite_bf16()
    grid = codec.E2M1_GRID
    for sc in range(1, 127):                           # every positive finite scale
        s = codec.E4M3_GRID[sc]
        ours = codec.e2m1_code(x, s)
        mag = ours & 7
        sign = ours >> 3
        # brute force on |x|/s done in fp64 (distance to every grid point)
        t = np.abs(x) / s
        want = _nearest_even(t, grid)
        # values past 6 saturate to 6 (code 7)
        want = np.where(t > 6.0, 7, want)
        np.testing.assert_array_equal(mag, want, err_msg=f"scale code {sc}")
        np.testing.assert_array_equal(sign, np.signbit(x).astype(np.uint8))
        # the hardware-converter form: fp32 quotient, then nearest grid value
        with np.errstate(over="ignore"):
            q32 = (np.abs(x).astype(np.float32) / np.float32(s)).astype(np.float64)
        want32 = np.where(q32 > 6.0, 7, _nearest_even(q32, grid))
        np.testing.assert_array_equal(mag, want32, err_msg=f"fp32 division form, scale {sc}")


def test_scale_code_exhaustive_bf16_and_fp32_division_form():
    _, x = _all_finite_bf16()
    amax = np.unique(np.abs(x))
    ours = codec.scale_code(amax)
    grid = codec.E4M3_GRID
    want = _nearest_even(amax / 6.0, grid)
    want = np.where(amax / 6.0 > 448.0, 126, want)
    np.testing.assert_array_equal(ours, want)
    # fp32 amax/6 followed by nearest-even onto the grid gives the same code
    q32 = (amax.astype(np.float32) / np.float32(6.0)).astype(np.float64)
    want32 = np.where(q32 > 448.0, 126, _nearest_even(q32, grid))
    np.testing.assert_array_equal(ours, want32)
    # also for arbitrary fp32 group maxima (the ratio-2 path quantizes fp32 values)
    rng = np.random.default_rng(1)
    a32 = np.abs(rng.standard_normal(400000) * np.exp(rng.uniform(-12, 8, 400000))).astype(np.float32)
    q = (a32 / np.float32(6.0)).astype(np.float64)
    np.testing.assert_array_equal(codec.scale_code(a32.astype(np.float64)),
                                  np.where(q > 448.0, 126, _nearest_even(q, grid)))


def test_round_trip_on_grid_values():
    for sc in range(1, 127):
        s = codec.E4M3_GRID[sc]
        for c in range(16):
            v = formats.E2M1_VALUES[c] * s
            got = int(codec.e2m1_code(np.array([v]), s)[0])
            assert got == c, (sc, c, v, got)


def test_quantize_rows_properties():
    rng = np.random.default_rng(2)
    x32 = (rng.standard_normal((64, 512)) * np.exp(rng.uniform(-6, 6, (64, 1)))).astype(np.float32)
    x = formats.bf16_to_f64(formats.f32_to_bf16(x32))
    codes, scales = codec.quantize_rows(x)
    assert codes.shape == (64, 512) and scales.shape == (64, 32)
    y = codec.dequantize(codes, scales)
    g = x.reshape(64, 32, 16)
    s = formats.E4M3_VALUES[scales][..., None]
    yg = y.reshape(64, 32, 16)
    # every decoded value is the nearest point of s*{grid} (checked by brute force)
    cand = s[..., None] * codec.E2M1_GRID            # [64,32,1,8]
    dist = np.abs(np.abs(g)[..., None] - cand)
    assert np.all(np.abs(np.abs(yg) - np.abs(g)) <= dist.min(axis=-1) + 0.0)
    # the group's maximum never saturates by more than the scale rounding allows
    amax = np.abs(g).max(-1)
    normal = (amax / 6.0 >= 2.0 ** -6) & (amax / 6.0 <= 448.0)
    assert normal.sum() > 1000
    assert np.all((6.0 * s[..., 0] >= amax * (1 - 2.0 ** -4))[normal])
    # ... and the scale puts the group maximum next to the largest E2M1 magnitude (6)
    assert np.all((6.0 * s[..., 0] <= amax * (1 + 2.0 ** -4))[normal])


def test_zero_scale_and_saturation():
    x = np.zeros((2, 512))
    x[0, :16] = 2.0 ** -20          # amax/6 rounds to E4M3 zero
    x[0, 16] = -1e-30
    x[1, :] = 1e6                   # amax/6 far above 448: scale saturates
    x[1, 1] = -1e6
    codes, scales = codec.quantize_rows(x)
    assert scales[0, 0] == 0 and np.all(codes[0, :16] == 0)
    assert scales[0, 1] == 0 and codes[0, 16] == 0        # zero scale -> code 0x0, sign dropped
    assert np.all(scales[1] == 126)
    assert codes[1, 0] == 7 and codes[1, 1] == 15           # saturate to +-6


def test_row_bytes_and_nibble_order():
    assert codec.ROW_BYTES == 512 // 2 + 512 // CONST["scale_group_channels"]["value"] == 288
    assert codec.ROW_BYTES * 64 == 18432                   # 64-token page
    assert (4 * 1024 ** 3) // (codec.ROW_BYTES * 64) == 233016
    # 1M tokens x 288 B x 4 sequences ~ 1.2 GB (the long-context workload's total)
    assert abs(4 * 1048576 * 288 / 1e9 - 1.21) < 0.01
    codes = np.zeros((1, 512), dtype=np.uint8)
    codes[0, 0] = 0x3
    codes[0, 1] = 0xA
    codes[0, 511] = 0x7
    row = codec.pack_rows(codes, np.arange(32, dtype=np.uint8)[None])
    assert row.shape == (1, 288)
    assert row[0, 0] == 0xA3 and row[0, 255] == 0x70
    assert list(row[0, 256:]) == list(range(32))
    c2, s2 = codec.unpack_rows(row)
    np.testing.assert_array_equal(c2, codes)


def test_compression_special_cases():
    rng = np.random.default_rng(3)
    a = formats.f32_to_bf16(rng.standard_normal((6, 512)).astype(np.float32))
    pairs = np.repeat(a, 2, axis=0)                       # (a, a) pairs
    np.testing.assert_array_equal(codec.encode_entries(pairs, 2), codec.encode_entries(a, 1))
    neg = np.empty((12, 512), dtype=np.uint16)
    neg[0::2] = a
    neg[1::2] = a ^ np.uint16(0x8000)                     # (a, -a) pairs average to zero
    rows = codec.encode_entries(neg, 2)
    assert np.all(rows[:, 256:] == 0) and np.all(rows[:, :256] == 0)
    k = formats.f32_to_bf16(rng.standard_normal((8, 64)).astype(np.float32))
    np.testing.assert_array_equal(codec.idxk_entries(np.repeat(k, 2, axis=0), 2), k)


def test_decoded_values_exact_in_bf16():
    # every (code, scale) product is a bf16 value: the dequantized row is exact in bf16
    v = (formats.E2M1_VALUES[:, None] * codec.E4M3_GRID[None, :]).reshape(-1)
    b = formats.f32_to_bf16(v.astype(np.float32))
    np.testing.assert_array_equal(formats.bf16_to_f64(b), v)


def test_compress_pairs_hand_values():
    """2:1 compression is the mean of adjacent rows: hand-computed pairs, and on
    random bf16 pairs in the normal range the fp32 result equals the exact mean
    (fp64) rounded to fp32 (halving is exact, so fl32(a + b) / 2 = fl32((a + b) / 2))."""
    def bits(vals):
        return formats.f32_to_bf16(np.asarray(vals, dtype=np.float32)).reshape(len(vals), 1)
    got = codec.compress_pairs_f32(bits([1.0, 2.0, -3.0, 3.0, 0.5, 0.25, -0.0, 0.0]))
    np.testing.assert_array_equal(got[:, 0], np.array([1.5, 0.0, 0.375, 0.0], dtype=np.float32))
    rng = np.random.default_rng(11)
    x = formats.f32_to_bf16((rng.standard_normal((4096, 8)) * np.exp2(rng.integers(-20, 20, (4096, 8))))
                            .astype(np.float32))
    got = codec.compress_pairs_f32(x)
    xf = formats.bf16_to_f64(x)
    want = ((xf[0::2] + xf[1::2]) / 2.0).astype(np.float32)
    np.testing.assert_array_equal(got, want)
