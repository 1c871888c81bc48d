"""Pins for the attention oracle: textbook dense attention via torch (fp64), closed-form
special cases and the selected-set / window union rule."""
import json
import os

import numpy as np
import torch

from oracle import attention, codec, formats

CONST = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_constants.json")))


def _rows(rng, n):
    bits = formats.f32_to_bf16(rng.standard_normal((n, 512)).astype(np.float32))
    c, s = codec.quantize_rows(formats.bf16_to_f64(bits))
    return codec.dequantize(c, s)


def test_window_constant():
    assert attention.WINDOW == CONST["swa_window"]["value"]


def test_dense_when_window_covers_context():
    rng = np.random.default_rng(0)
    for L in (1, 5, 77, 128):
        rows = _rows(rng, L)
        q = formats.f32_to_bf16((rng.standard_normal((16, 512)) / np.sqrt(512)).astype(np.float32))
        idx = np.full(512, -1)
        pos = attention.attended_positions(idx, L)
        np.testing.assert_array_equal(pos, np.arange(L))
        ours = attention.attend(q, rows[pos], sm_scale=0.7)
        qt = torch.from_numpy(formats.bf16_to_f64(q))[None, :, None, :]    # [1,H,1,D]
        kt = torch.from_numpy(rows)[None, None].expand(1, 16, L, 512)
        ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, kt, scale=0.7)[0, :, 0]
        np.testing.assert_allclose(ours, ref.numpy(), rtol=1e-12, atol=1e-13)


def test_closed_forms():
    rng = np.random.default_rng(1)
    rows = _rows(rng, 9)
    q = formats.f32_to_bf16(rng.standard_normal((4, 512)).astype(np.float32))
    # one attended row: the output is that row for every head
    np.testing.assert_array_equal(attention.attend(q, rows[3:4]), np.repeat(rows[3:4], 4, axis=0))
    # zero query: uniform weights, the output is the mean row
    z = np.zeros((2, 512), dtype=np.uint16)
    np.testing.assert_allclose(attention.attend(z, rows), np.repeat(rows.mean(0, keepdims=True), 2, 0),
                               rtol=1e-12, atol=1e-14)
    # empty set: zero output
    assert np.all(attention.attend(q, rows[:0]) == 0)
    # a dominant logit puts all weight on its row
    big = np.zeros((1, 512), dtype=np.float64)
    r = np.zeros((3, 512))
    r[1, 0] = 1.0
    qb = formats.f32_to_bf16(np.array([[1000.0] + [0.0] * 511], dtype=np.float32))
    np.testing.assert_allclose(attention.attend(qb, r)[0], r[1], atol=1e-300)


def test_union_of_selection_and_window():
    L = 1000
    idx = np.array([0, 5, 900, 950, 999] + [-1] * 507)
    pos = attention.attended_positions(idx, L)
    want = np.concatenate([[0, 5], np.arange(872, 1000)])
    np.testing.assert_array_equal(pos, want)
    assert pos.size == 130                                  # duplicates counted once
    # a full selection far from the window: 512 + 128 rows
    idx = np.arange(0, 1024, 2)
    pos = attention.attended_positions(idx, 100000)
    assert pos.size == 640


def test_prefill_visibility():
    # entry c averages raw tokens 2c, 2c+1: visible once token 2c+1 exists
    assert [attention.prefill_visible(p, 2) for p in range(6)] == [0, 1, 1, 2, 2, 3]
    assert attention.prefill_visible(131071, 2) == 65536
    assert [attention.prefill_visible(p, 1) for p in range(3)] == [1, 2, 3]
