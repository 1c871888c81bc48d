"""Pins for the C oracle (oracle/c/csa2_oracle.c): the format tables the pages'
formats define, brute-force rounding over every bf16 input, the row layout,
closed-form scores and block keys, brute-force top-k and hierarchy, textbook
attention through torch in fp64, the Reuse / Reindex invariants of a decode
step -- and agreement with the numpy oracle, an independent implementation."""
import json
import os

import numpy as np
import pytest
import torch

import workload as wl
from oracle import attention as oattn
from oracle import c_oracle as co
from oracle import codec as ocodec
from oracle import formats
from oracle import indexer as oidx
from oracle import modes as omodes

HERE = os.path.dirname(__file__)
FORMATS = json.load(open(os.path.join(HERE, "golden", "formats.json")))
CONST = json.load(open(os.path.join(HERE, "golden", "page_constants.json")))


def _bf16(x):
    return formats.f32_to_bf16(np.asarray(x, dtype=np.float32))


def _nearest_even(target, grid):
    """Brute force: index of the grid value nearest to each target (direct
    distances to every point), ties to the even index."""
    d = np.abs(np.asarray(target, np.float64)[:, None] - np.asarray(grid, np.float64)[None, :])
    best = d.min(axis=1, keepdims=True)
    hits = d == best
    idx = np.argmax(hits, axis=1)
    two = hits.sum(axis=1) > 1
    return np.where(two & (idx % 2 == 1), idx + 1, idx)


def test_format_tables_from_the_golden_values():
    for c, v in enumerate(FORMATS["e2m1_values_by_code"]):
        got = co.e2m1_value(c)
        assert got == v and np.signbit(got) == np.signbit(v), c
    e = FORMATS["e4m3"]
    for name in ("max_normal", "min_normal", "min_subnormal", "max_subnormal", "one"):
        assert co.e4m3_value(e[name]["code"]) == e[name]["value"], name
    for c in e["nan_codes"]:
        assert np.isnan(co.e4m3_value(c))
    finite = [co.e4m3_value(c) for c in range(128)]
    assert sum(1 for v in finite if np.isfinite(v)) == e["finite_nonnegative_count"]
    # and every byte against torch's float8_e4m3fn decoding (a library conversion)
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = np.array([co.e4m3_value(b) for b in range(256)])
    fin = np.isfinite(ref)
    np.testing.assert_array_equal(ours[fin], ref[fin])
    assert np.all(np.isnan(ours[~fin]))


def _all_finite_bf16():
    b = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    return b[np.isfinite(formats.bf16_to_f64(b))]


def test_scale_byte_of_every_bf16_group_maximum():
    # a group [a, 0 x 15]: its scale byte is E4M3-nearest(fp32(a / 6)), ties even, saturating
    a = np.unique(np.abs(formats.bf16_to_f64(_all_finite_bf16())))
    grid = np.array([co.e4m3_value(c) for c in range(127)])
    n = a.size
    rows = np.zeros((n, 512), np.uint16)
    rows[:, 0] = _bf16(a)
    got = co.encode_rows(rows)[:, 256]
    q32 = (a.astype(np.float32) / np.float32(6.0)).astype(np.float64)
    want = np.where(q32 > 448.0, 126, _nearest_even(q32, grid))
    np.testing.assert_array_equal(got, want)


def test_codes_of_every_bf16_value_under_every_scale():
    """Groups led by 6 x scale (which selects that scale) holding every finite
    bf16 value up to it: each code is sign | E2M1-nearest(|x| / scale), ties even."""
    x = formats.bf16_to_f64(_all_finite_bf16())
    mag = np.array([co.e2m1_value(c) for c in range(8)])
    for sc in range(1, 127):
        s = co.e4m3_value(sc)
        vals = x[np.abs(x) <= 6.0 * s]
        pad = (-vals.size) % 15
        vals = np.concatenate([vals, np.zeros(pad)]).reshape(-1, 15)
        lead = np.full((vals.shape[0], 1), 6.0 * s)
        groups = np.concatenate([lead, vals], axis=1).reshape(-1)
        groups = np.concatenate([groups, np.zeros((-groups.size) % 512)]).reshape(-1, 512)
        rows = co.encode_rows(_bf16(groups))
        ng = rows.shape[0] * 32
        scales = rows[:, 256:].reshape(-1)
        full = np.arange(ng) < vals.shape[0]
        assert np.all(scales[full] == sc), sc
        packed = rows[:, :256]
        codes = np.empty((rows.shape[0], 512), np.uint8)
        codes[:, 0::2] = packed & 15
        codes[:, 1::2] = packed >> 4
        codes = codes.reshape(-1, 16)[full][:, 1:].reshape(-1)
        v = vals.reshape(-1)
        want = _nearest_even(np.abs(v) / s, mag) | (np.signbit(v).astype(np.int64) << 3)
        np.testing.assert_array_equal(codes, want, err_msg=f"scale code {sc}")


def test_row_layout_zero_scale_and_saturation():
    x = np.zeros((3, 512), np.float32)
    x[0, 0], x[0, 1] = 6.0, -1.0            # group 0: scale 1.0 (byte 56), codes 7 and 0xA
    x[1, :16] = 2.0 ** -20                  # scale rounds to zero: every code 0
    x[1, 16] = -1e-30
    x[2, :] = 1e6                           # scale saturates at 448, codes at +-6
    x[2, 1] = -1e6
    rows = co.encode_rows(_bf16(x))
    assert rows.shape == (3, 288) and 288 == 512 // 2 + 512 // CONST["scale_group_channels"]["value"]
    assert rows[0, 0] == 0xA7 and rows[0, 256] == 56 and np.all(rows[0, 1:256] == 0)
    assert rows[1, 256] == 0 and rows[1, 257] == 0 and np.all(rows[1, :16] == 0)
    assert np.all(rows[2, 256:] == 126) and rows[2, 0] == 0xF7


def test_decode_is_code_value_times_scale_and_round_trips_grid_values():
    for sc in (1, 8, 56, 100, 126):
        s = co.e4m3_value(sc)
        x = np.zeros((1, 512))
        x[0, :16] = [6.0 * s] + [co.e2m1_value(c) * s for c in range(1, 16)]
        dec = co.decode_rows(co.encode_rows(_bf16(x)))
        np.testing.assert_array_equal(dec[0, :16], x[0, :16])


def test_scores_closed_forms_and_fp64_bound():
    rng = np.random.default_rng(1)
    k = _bf16(rng.standard_normal((300, 64)))
    kf = formats.bf16_to_f32(k)
    for d in (0, 17, 63):
        q = np.zeros((4, 64), np.uint16)
        q[0, d] = 0x3F80                                   # 1.0 in head 0
        np.testing.assert_array_equal(co.index_scores(q, k), np.maximum(kf[:, d], 0.0))
        q[0, d] = 0xBF80                                   # -1.0: the ReLU of the negation
        np.testing.assert_array_equal(co.index_scores(q, k), np.maximum(-kf[:, d], 0.0))
        q3 = np.zeros((4, 64), np.uint16)
        q3[2, d] = 0x3F80
        w = np.array([0, 0, 3.0, 0], np.float32)
        np.testing.assert_array_equal(co.index_scores(q3, k, w),
                                      (np.float32(3.0) * np.maximum(kf[:, d], 0)).astype(np.float32))
    q = _bf16(rng.standard_normal((4, 64)))
    k = _bf16(rng.standard_normal((4000, 64)))
    w = np.array([1.0, 0.5, 2.0, 0.25], np.float32)
    ours = co.index_scores(q, k, w).astype(np.float64)
    qf, kf = formats.bf16_to_f64(q), formats.bf16_to_f64(k)
    ref = (np.maximum(np.einsum("hd,nd->nh", qf, kf), 0) * w).sum(1)
    bound = 1e-5 * (np.einsum("hd,nd->nh", np.abs(qf), np.abs(kf)) * w).sum(1)
    assert np.all(np.abs(ours - ref) <= bound + 1e-30)


def test_block_key_identities():
    rng = np.random.default_rng(2)
    k = _bf16(rng.standard_normal((40, 64)))
    np.testing.assert_array_equal(co.block_keys(k, 1), k[:1])
    np.testing.assert_array_equal(co.block_keys(np.repeat(k[:1], 8, 0), 8), k[:1])
    t = np.zeros((11, 64), np.uint16)
    t[8:11] = _bf16(np.array([1.0, 2.0, 3.0]))[:, None]
    kb = co.block_keys(t, 11)
    assert kb.shape == (2, 64)
    np.testing.assert_array_equal(formats.bf16_to_f64(kb[1]), 2.0)
    np.testing.assert_array_equal(co.block_keys(k ^ np.uint16(0x8000), 40),
                                  co.block_keys(k, 40) ^ np.uint16(0x8000))
    ints = _bf16(np.arange(16, dtype=np.float32)[:, None] * np.ones((1, 64)))
    np.testing.assert_array_equal(formats.bf16_to_f64(co.block_keys(ints, 16))[:, 0], [3.5, 11.5])


def _brute_topk(s, k):
    items = sorted((-float(s[i]), i) for i in range(len(s)))
    chosen = sorted(i for _, i in items[:k])
    return chosen + [-1] * (k - len(chosen))


def test_topk_brute_force_ties_and_padding():
    rng = np.random.default_rng(3)
    for _ in range(300):
        n, k = int(rng.integers(0, 60)), int(rng.integers(1, 20))
        s = rng.integers(-3, 4, n).astype(np.float32) * np.float32(0.5)   # many ties
        assert list(co.top_k(s, k)) == _brute_topk(s, k)
    np.testing.assert_array_equal(co.top_k(np.full(2000, 7.0, np.float32), 512), np.arange(512))
    out = co.top_k(np.arange(10, dtype=np.float32), 16)
    assert list(out[:10]) == list(range(10)) and np.all(out[10:] == -1)


def test_hierarchy_brute_force():
    rng = np.random.default_rng(4)
    # up to 2,048 blocks every token is a candidate: the set is the flat top-512
    for L in (1, 300, 4096, 16384):
        keys = _bf16(rng.standard_normal((L, 64)))
        q = _bf16(rng.standard_normal((4, 64)))
        pool, idx = co.full_indexer(q, keys, L)
        nb = (L + 7) // 8
        np.testing.assert_array_equal(pool, np.where(np.arange(2048) < nb, np.arange(2048), -1))
        assert list(idx) == _brute_topk(co.index_scores(q, keys), 512)
    # beyond: the pool is the top 2,048 block keys, the set the top 512 of their tokens
    L = 20011
    keys = _bf16(rng.standard_normal((L, 64)))
    q = _bf16(rng.standard_normal((4, 64)))
    pool, idx = co.full_indexer(q, keys, L)
    bs = co.index_scores(q, co.block_keys(keys, L))
    assert list(pool) == _brute_topk(bs, 2048)
    cand = np.array([b * 8 + t for b in pool for t in range(8) if b * 8 + t < L])
    sel = _brute_topk(co.index_scores(q, keys[cand]), 512)
    assert list(idx) == [int(cand[i]) if i >= 0 else -1 for i in sel]
    # Reindex with the Full layer's own query reproduces the Full set
    np.testing.assert_array_equal(co.reindex_indexer(q, keys, L, pool), idx)


def test_attention_textbook_closed_forms_and_union():
    rng = np.random.default_rng(5)
    for L in (1, 77, 128):
        rows = co.decode_rows(co.encode_rows(_bf16(rng.standard_normal((L, 512)))))
        q = _bf16(rng.standard_normal((16, 512)) / np.sqrt(512))
        pos = co.attended_positions(np.full(512, -1), L)
        np.testing.assert_array_equal(pos, np.arange(L))
        ours = co.attend(q, rows[pos], 0.7)
        qt = torch.from_numpy(formats.bf16_to_f64(q))[None, :, None, :]
        kt = torch.from_numpy(rows)[None, None].expand(1, 16, L, 512)
        ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, kt, scale=0.7)[0, :, 0]
        np.testing.assert_allclose(ours, ref.numpy(), rtol=1e-12, atol=1e-13)
    rows = co.decode_rows(co.encode_rows(_bf16(rng.standard_normal((9, 512)))))
    q = _bf16(rng.standard_normal((4, 512)))
    np.testing.assert_array_equal(co.attend(q, rows[3:4]), np.repeat(rows[3:4], 4, 0))
    np.testing.assert_allclose(co.attend(np.zeros((2, 512), np.uint16), rows),
                               np.repeat(rows.mean(0, keepdims=True), 2, 0), rtol=1e-12, atol=1e-14)
    assert np.all(co.attend(q, rows[:0]) == 0)
    r = np.zeros((3, 512))                     # a dominant logit puts all weight on its row
    r[1, 0] = 1.0
    qb = _bf16(np.array([[1000.0] + [0.0] * 511]))
    np.testing.assert_allclose(co.attend(qb, r)[0], r[1], atol=1e-300)
    idx = np.array([0, 5, 900, 950, 999] + [-1] * 507)
    np.testing.assert_array_equal(co.attended_positions(idx, 1000),
                                  np.concatenate([[0, 5], np.arange(872, 1000)]))
    assert co.attended_positions(np.arange(0, 1024, 2), 100000).size == 640
    with pytest.raises(ValueError):
        co.attended_positions(np.array([1000] + [-1] * 511), 1000)


def _decode_inputs(seed, lengths, layers, heads):
    out = []
    for s, L in enumerate(lengths):
        out.append({"L": L, "seq": s, "keys": wl.idxk_rows(seed, s, 0, L),
                    "iq": {l: wl.idxq_rows(seed, l, s) for l, m in enumerate(layers) if m != "R"},
                    "q": {l: wl.q_rows(seed, l, s, heads) for l in range(len(layers))},
                    "new": wl.kv_rows(seed, s, L - 1, 1)})
    return out


def test_decode_steps_invariants_and_agreement_with_the_numpy_oracle():
    layers = ["F", "R", "RI", "R"]
    seed, heads, scale = 3, 16, 0.044
    seqs = _decode_inputs(seed, [20011, 3000, 130], layers, heads)
    ds = co.DecodeSteps(layers, heads, seed, seqs, scale)
    ds.step(3)
    for i, s in enumerate(seqs):
        L = s["L"]
        # Reuse layers keep their set; each layer's output is its set's attention
        np.testing.assert_array_equal(ds.idx[i][1], ds.idx[i][0])
        np.testing.assert_array_equal(ds.idx[i][3], ds.idx[i][2])
        for l in range(4):
            pos = co.attended_positions(ds.idx[i][l], L)
            rows = co.decode_rows(co.encode_rows(np.concatenate([wl.kv_rows(seed, i, int(p), 1) for p in pos])))
            np.testing.assert_array_equal(ds.out[i][l], co.attend(s["q"][l], rows, scale))
        # the numpy oracle (independent code) gives the same sets and outputs
        res = omodes.run_layers(
            layers, L, s["keys"], lambda l, s=s: s["iq"][l], lambda l, s=s: s["q"][l],
            lambda pos, i=i: ocodec.dequantize(*ocodec.unpack_rows(ocodec.encode_bf16_rows(
                np.concatenate([wl.kv_rows(seed, i, int(p), 1) for p in pos])))), scale)
        for l, r in enumerate(res):
            np.testing.assert_array_equal(ds.idx[i][l], r["idx"])
            np.testing.assert_allclose(ds.out[i][l], r["out"], rtol=1e-12, atol=1e-14)
    # a second step draws nothing new and gives the same results
    before = [o.copy() for o in ds.out]
    ds.step(2)
    for a, b in zip(before, ds.out):
        np.testing.assert_array_equal(a, b)


def test_codec_and_indexer_agree_with_the_numpy_oracle():
    rng = np.random.default_rng(6)
    x = (rng.standard_normal((300, 512)) * np.exp(rng.uniform(-10, 10, (300, 1)))).astype(np.float32)
    kv = _bf16(x)
    rows = co.encode_rows(kv)
    np.testing.assert_array_equal(rows, ocodec.encode_bf16_rows(kv))
    np.testing.assert_array_equal(co.decode_rows(rows), ocodec.dequantize(*ocodec.unpack_rows(rows)))
    keys = _bf16(rng.standard_normal((40000, 64)))
    q = _bf16(rng.standard_normal((4, 64)))
    np.testing.assert_array_equal(co.block_keys(keys, 40000), oidx.block_keys(keys, 40000))
    np.testing.assert_array_equal(co.index_scores(q, keys), oidx.index_scores(q, keys))
    pool, idx = co.full_indexer(q, keys, 40000)
    p2, i2, _ = oidx.full_indexer(q, keys, 40000)
    np.testing.assert_array_equal(pool, p2)
    np.testing.assert_array_equal(idx, i2)
    np.testing.assert_array_equal(co.attended_positions(idx, 40000), oattn.attended_positions(i2, 40000))


def test_ratio2_entries_pins_and_agreement():
    rng = np.random.default_rng(7)
    a = _bf16(rng.standard_normal((6, 512)))
    # (a, a) pairs are entries a; (a, -a) pairs average to zero rows
    np.testing.assert_array_equal(co.encode_entries(np.repeat(a, 2, axis=0), 2), co.encode_rows(a))
    neg = np.empty((12, 512), np.uint16)
    neg[0::2], neg[1::2] = a, a ^ np.uint16(0x8000)
    assert np.all(co.encode_entries(neg, 2) == 0)
    k = _bf16(rng.standard_normal((8, 64)))
    np.testing.assert_array_equal(co.key_entries(np.repeat(k, 2, axis=0), 2), k)
    # hand values: the pair (1, 2) averages to 1.5 in every channel
    pair = np.stack([_bf16(np.ones(512)), _bf16(np.full(512, 2.0))])
    np.testing.assert_array_equal(co.decode_rows(co.encode_entries(pair, 2)), co.decode_rows(co.encode_rows(
        _bf16(np.full((1, 512), 1.5)))))
    # against the numpy oracle on wide-range pairs
    raw = _bf16(rng.standard_normal((800, 512)) * np.exp(rng.uniform(-8, 8, (800, 1))))
    np.testing.assert_array_equal(co.encode_entries(raw, 2), ocodec.encode_entries(raw, 2))
    kr = _bf16(rng.standard_normal((800, 64)))
    np.testing.assert_array_equal(co.key_entries(kr, 2), ocodec.idxk_entries(kr, 2))


def test_flat_indexer_brute_force():
    rng = np.random.default_rng(8)
    keys = _bf16(rng.standard_normal((3000, 64)))
    q = _bf16(rng.standard_normal((4, 64)))
    for v in (0, 1, 511, 512, 513, 3000):
        assert list(co.flat_indexer(q, keys, v)) == _brute_topk(co.index_scores(q, keys[:v]), 512)


def test_prefill_queries_and_append_agree_with_the_numpy_oracle():
    rng = np.random.default_rng(9)
    n_raw, heads, nl = 4000, 16, 3
    raw_kv = _bf16(rng.standard_normal((n_raw, 512)))
    raw_k = _bf16(rng.standard_normal((n_raw, 64)))
    keys = ocodec.idxk_entries(raw_k, 2)
    qs = [{"P": P, "iq": _bf16(rng.standard_normal((4, 64))),
           "q": _bf16(rng.standard_normal((nl, heads, 512)) / np.sqrt(512))} for P in (0, 1, 2, 255, 2047, 3999)]
    pq = co.PrefillQueries(nl, heads, 2, keys, raw_kv, raw_k, qs, 0.5)
    pq.append(3)
    np.testing.assert_array_equal(pq.rows_out, ocodec.encode_entries(raw_kv, 2))
    np.testing.assert_array_equal(pq.keys_out, keys)
    pq.queries(2)
    rows_all = ocodec.dequantize(*ocodec.unpack_rows(ocodec.encode_entries(raw_kv, 2)))
    for i, qq in enumerate(qs):
        v = oattn.prefill_visible(qq["P"], 2)
        idx, _ = oidx.flat_indexer(qq["iq"], keys, v)
        np.testing.assert_array_equal(pq.idx[i], idx)
        pos = oattn.attended_positions(idx, v)
        for l in range(nl):
            np.testing.assert_allclose(pq.out[i][l], oattn.attend(qq["q"][l], rows_all[pos], 0.5),
                                       rtol=1e-12, atol=1e-14)
        if v == 0:
            assert np.all(pq.out[i] == 0)


def test_ragged_steps_agree_with_the_numpy_oracle():
    seed, heads = 4, 16
    lengths, ri, miss = [20011, 3000, 130, 1], [True, False, True, False], [True, True, False, False]
    seqs = []
    for s, L in enumerate(lengths):
        keys = wl.idxk_rows(seed, s, 0, L)
        pool, idx, _ = oidx.full_indexer(wl.idxq_rows(seed, 0, s), keys, L)
        n = min(128, L)
        kv_last = np.zeros((128, 512), np.uint16)
        kv_last[128 - n:] = wl.kv_rows(seed, s, L - n, n)
        seqs.append({"L": L, "seq": s, "ri": ri[s], "miss": miss[s], "kv_last": kv_last, "keys": keys,
                     "pool": pool, "set": idx, "iq": wl.idxq_rows(seed, 1, s), "q": wl.q_rows(seed, 1, s, heads)})
    rs = co.RaggedSteps(heads, seed, seqs, 0.7)
    rs.step(3)
    for i, s in enumerate(seqs):
        _, want_rows = omodes.replay_entries(s["kv_last"], s["L"], s["miss"])
        np.testing.assert_array_equal(rs.replayed_rows(i), want_rows)
        want = oidx.reindex_indexer(s["iq"], s["keys"], s["L"], s["pool"])[0] if s["ri"] else s["set"]
        np.testing.assert_array_equal(rs.idx[i], want)
        pos = oattn.attended_positions(want, s["L"])
        rows = ocodec.dequantize(*ocodec.unpack_rows(ocodec.encode_bf16_rows(
            np.concatenate([wl.kv_rows(seed, i, int(p), 1) for p in pos]))))
        np.testing.assert_allclose(rs.out[i], oattn.attend(s["q"], rows, 0.7), rtol=1e-12, atol=1e-14)
