"""Pins for the FP8 indexer-key oracle: the E4M3 rounding against brute force and
torch's float8_e4m3fn conversion, saturation and signed zero, the quantised key's
error bound, the 890-byte accounting, and scores, block keys and index sets
against the bf16 path on keys that FP8 holds exactly."""
import numpy as np
import pytest
import torch

from oracle import codec, formats, idxk_fp8, indexer

GRID = formats.E4M3_VALUES[:127]          # non-negative finite values, codes 0..126


def _bf16(x):
    return formats.f32_to_bf16(np.asarray(x, dtype=np.float32))


def _brute_code(t: float) -> int:
    """Nearest finite E4M3 value by exhaustive search; ties to the even code; beyond 448 -> 448."""
    mag = min(abs(float(t)), 448.0)
    d = np.abs(GRID - mag)
    best = np.nonzero(d == d.min())[0]
    code = int(best[0]) if best.size == 1 else int(best[best % 2 == 0][0])
    return code | (0x80 if np.signbit(t) else 0)


def test_every_e4m3_value_encodes_to_itself():
    vals = formats.E4M3_VALUES
    codes = np.arange(256)
    finite = ~np.isnan(vals)
    got = idxk_fp8.e4m3_code(vals[finite].astype(np.float32))
    np.testing.assert_array_equal(got, codes[finite])    # -0.0 -> 0x80 included


def test_rounding_against_brute_force_on_all_bf16_magnitudes():
    bits = np.arange(0, 0x7F80, dtype=np.uint16)           # every finite non-negative bf16
    t = formats.bf16_to_f32(bits)
    t = t[(t <= 512.0)]
    got = idxk_fp8.e4m3_code(t)
    want = np.array([_brute_code(x) for x in t])
    np.testing.assert_array_equal(got, want)
    np.testing.assert_array_equal(idxk_fp8.e4m3_code(-t), want | 0x80)


def test_midpoints_round_to_even_and_match_torch():
    mids = ((GRID[:-1] + GRID[1:]) / 2).astype(np.float32)
    got = idxk_fp8.e4m3_code(mids)
    assert np.all(got % 2 == 0)
    # torch's conversion rounds to nearest even; compared inside the finite range
    rng = np.random.default_rng(0)
    t = np.concatenate([mids, (rng.standard_normal(20000) * np.exp2(rng.integers(-12, 8, 20000))),
                        GRID * 1.0000001, GRID * 0.9999999]).astype(np.float32)
    t = t[np.abs(t) <= 448.0]
    ref = torch.from_numpy(t).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(idxk_fp8.e4m3_code(t), ref)


def test_saturation():
    np.testing.assert_array_equal(idxk_fp8.e4m3_code(np.array([448.0, 460.0, 464.0, 1e6, 3e38], np.float32)),
                                  [0x7E] * 5)
    np.testing.assert_array_equal(idxk_fp8.e4m3_code(np.array([-500.0, -1e30], np.float32)), [0xFE] * 2)


def test_quantised_key_error_bound_and_degenerate_keys():
    rng = np.random.default_rng(1)
    k = _bf16(rng.standard_normal((4000, 64)) * np.exp2(rng.integers(-20, 20, (4000, 1))))
    codes, s = idxk_fp8.quantize(k)
    kf = formats.bf16_to_f32(k).astype(np.float64)
    amax = np.abs(kf).max(axis=1)
    np.testing.assert_array_equal(s, (amax.astype(np.float32) / np.float32(448.0)).astype(np.float32))
    deq = idxk_fp8.dequantize(codes, s).astype(np.float64)
    # half a unit in the last place: 2^-4 relative for normals, 2^-10 s for subnormals,
    # plus the fp32 quotient's and product's roundings
    bound = np.maximum(np.abs(kf) * 2.0 ** -4, s[:, None].astype(np.float64) * 2.0 ** -10) * 1.0001
    assert np.all(np.abs(deq - kf) <= bound)
    # each key's largest element comes back within rounding of the scale
    i = np.arange(k.shape[0])
    j = np.argmax(np.abs(kf), axis=1)
    assert np.all(np.abs(np.abs(deq[i, j]) - amax) <= amax * 2.0 ** -20)
    # all-zero key: scale 0 and zero codes; tiny negatives next to a large value keep their sign
    z, sz = idxk_fp8.quantize(np.zeros((1, 64), np.uint16))
    assert sz[0] == 0 and np.all(z == 0)
    x = np.zeros(64, np.float32)
    x[0], x[1], x[2] = 1000.0, -1e-3, 1e-3
    c, sx = idxk_fp8.quantize(_bf16(x)[None])
    assert c[0, 0] == 0x7E and c[0, 1] == 0x80 and c[0, 2] == 0x00


def test_890_byte_accounting():
    main, key = codec.ROW_BYTES, idxk_fp8.ROW_BYTES
    assert (main + key) + 3 * (main + key) // 2 == 890 and 3 * (main + key) % 2 == 0
    assert idxk_fp8.PAGE_BYTES == 64 * 64 + 64 * 4


def test_page_packing():
    rng = np.random.default_rng(2)
    keys = idxk_fp8.Fp8Keys.from_bf16(_bf16(rng.standard_normal((128, 64))))
    pages = keys.pack()
    assert pages.shape == (2, 4352)
    np.testing.assert_array_equal(pages[1, 5 * 64:(5 + 1) * 64], keys.codes[64 + 5])
    assert pages[1, 4096 + 5 * 4:4096 + 6 * 4].view(np.float32)[0] == keys.scales[64 + 5]


def _exact_fp8_keys(rng, n):
    """bf16 keys that FP8 holds exactly: E4M3 grid values x 2^-8 whose largest
    magnitude is 448 (so the scale is 2^-8 and every quotient is a grid value)."""
    codes = rng.integers(0, 255, (n, 64)).astype(np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x10           # no NaN codes
    codes[:, rng.integers(0, 64)] = 0x7E           # 448 somewhere in every key
    vals = formats.E4M3_VALUES[codes] * 2.0 ** -8
    return _bf16(vals), codes


def test_exactly_representable_keys_round_trip_and_score_like_bf16():
    rng = np.random.default_rng(3)
    kb, codes = _exact_fp8_keys(rng, 3000)
    keys = idxk_fp8.Fp8Keys.from_bf16(kb)
    assert np.all(keys.scales == np.float32(2.0 ** -8))
    np.testing.assert_array_equal(keys.codes, np.where(codes == 0x80, 0x80, codes))
    q = _bf16(rng.standard_normal((4, 64)))
    w = np.array([1.0, 0.5, 2.0, 0.25], np.float32)
    # a power-of-two scale commutes with every fp32 rounding: the scores are equal
    np.testing.assert_array_equal(indexer.index_scores(q, keys, w), indexer.index_scores(q, kb, w))
    np.testing.assert_array_equal(indexer.block_keys(keys, 2999), indexer.block_keys(kb, 2999))
    a = indexer.full_indexer(q, keys, 3000, w, hierarchical=False)
    b = indexer.full_indexer(q, kb, 3000, w, hierarchical=False)
    np.testing.assert_array_equal(a[1], b[1])


def test_scores_against_fp64_on_the_dequantised_key():
    rng = np.random.default_rng(4)
    keys = idxk_fp8.Fp8Keys.from_bf16(_bf16(rng.standard_normal((5000, 64))))
    q = _bf16(rng.standard_normal((4, 64)))
    w = np.array([1.0, -0.5, 2.0, 0.25], np.float32)
    ours = indexer.index_scores(q, keys, w).astype(np.float64)
    qf = formats.bf16_to_f64(q)
    kf = formats.E4M3_VALUES[keys.codes] * keys.scales[:, None].astype(np.float64)   # exact
    dots = np.einsum("hd,nd->nh", qf, kf)
    ref = (np.maximum(dots, 0.0) * w.astype(np.float64)).sum(axis=1)
    bound = 1e-5 * (np.einsum("hd,nd->nh", np.abs(qf), np.abs(kf)) * np.abs(w)).sum(axis=1)
    assert np.all(np.abs(ours - ref) <= bound + 1e-30)


@pytest.mark.parametrize("L", [100, 20000])
def test_fp8_index_sets_are_top_k_of_fp8_scores(L):
    """Full indexer over FP8 keys against a direct top-k of the FP8 scores of all
    candidates (flat) and of the pool tokens (hierarchical)."""
    rng = np.random.default_rng(L)
    keys = idxk_fp8.Fp8Keys.from_bf16(_bf16(rng.standard_normal((L, 64))))
    q = _bf16(rng.standard_normal((4, 64)))
    pool, idx, info = indexer.full_indexer(q, keys, L)
    cand = info["candidates"]
    s = indexer.index_scores(q, keys[cand])
    order = np.lexsort((cand, -s.astype(np.float64)))[:512]
    np.testing.assert_array_equal(idx[idx >= 0], np.sort(cand[order]))
