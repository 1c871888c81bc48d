"""Pins for the oracle's number formats: printed format tables and library conversions."""
import json
import os

import numpy as np
import torch

from oracle import formats

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "formats.json")))


def test_e2m1_table_matches_format_definition():
    want = np.array(GOLD["e2m1_values_by_code"])
    np.testing.assert_array_equal(formats.E2M1_VALUES, want)
    # code 8 is negative zero, not +0
    assert np.signbit(formats.E2M1_VALUES[8]) and not np.signbit(formats.E2M1_VALUES[0])


def test_e4m3_extremes_and_counts():
    e = GOLD["e4m3"]
    for name in ("max_normal", "min_normal", "min_subnormal", "max_subnormal", "one"):
        assert formats.E4M3_VALUES[e[name]["code"]] == e[name]["value"], name
    for c in e["nan_codes"]:
        assert np.isnan(formats.E4M3_VALUES[c])
    finite = formats.E4M3_VALUES[~np.isnan(formats.E4M3_VALUES)]
    assert finite.size == 254
    assert np.nanmax(formats.E4M3_VALUES) == 448.0
    pos = formats.E4M3_VALUES[:127]
    assert pos.size == e["finite_nonnegative_count"]
    assert np.all(np.diff(pos) > 0)            # code order == value order
    np.testing.assert_array_equal(formats.E4M3_VALUES[128:255], -pos)


def test_e4m3_matches_torch_float8():
    # independent decoder: torch's float8_e4m3fn bit reinterpretation
    b = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    t = b.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ok = ~np.isnan(formats.E4M3_VALUES)
    np.testing.assert_array_equal(t[ok], formats.E4M3_VALUES[ok])
    assert np.all(np.isnan(t[~ok]))


def test_bf16_conversion_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.standard_normal(100000).astype(np.float32),
        (rng.standard_normal(100000) * 1e30).astype(np.float32),
        np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -1.0 - 2.0 ** -8, 0.0, -0.0,
                  3.0e38, 1e-40], dtype=np.float32),
    ])
    ours = formats.f32_to_bf16(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref)
    back = formats.bf16_to_f32(ours)
    np.testing.assert_array_equal(back, torch.from_numpy(ours.view(np.int16)).view(
        torch.bfloat16).to(torch.float32).numpy())
    # ties go to the even mantissa
    assert formats.f32_to_bf16(np.float32(1.0 + 2.0 ** -8)) == 0x3F80
    assert formats.f32_to_bf16(np.float32(1.0 + 3 * 2.0 ** -8)) == 0x3F82
