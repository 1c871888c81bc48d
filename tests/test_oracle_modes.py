"""Pins for the layer-mode and replay oracle: the pages' mode invariants and group patterns."""
import json
import os

import numpy as np
import pytest

from oracle import codec, formats, indexer, modes

CONST = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_constants.json")))


def _bf16(x):
    return formats.f32_to_bf16(np.asarray(x, dtype=np.float32))


def test_group_patterns():
    dec = modes.DECODER_PATTERN
    c = CONST["decoder_layers"]
    assert len(dec) == c["value"] == c["groups"] * c["group_size"]
    assert dec[0] == "F" and dec.count("F") == 1 and dec.count("RI") == c["groups"] - 1
    for g in range(c["groups"]):
        grp = dec[g * 4:(g + 1) * 4]
        assert grp[0] in ("F", "RI") and grp[1:] == ["R", "R", "R"]
    enc = modes.ENCODER_PATTERN
    e = CONST["encoder_csa2_layers"]
    assert len(enc) == e["value"] and enc.count("F") == e["groups"] and enc.count("R") == 15
    assert modes.REPLAY == CONST["replay_tokens"]["value"]


def _setup(L, seed=0):
    rng = np.random.default_rng(seed)
    kv_bits = _bf16(rng.standard_normal((L, 512)))
    c, s = codec.quantize_rows(formats.bf16_to_f64(kv_bits))
    rows = codec.dequantize(c, s)
    keys = _bf16(rng.standard_normal((L, 64)))
    return rng, rows, keys


@pytest.mark.parametrize("L", [3000, 20000])
def test_reuse_and_reindex_invariants(L):
    rng, rows, keys = _setup(L)
    layers = ["F", "R", "R", "R", "RI", "R"]
    iq = {l: _bf16(rng.standard_normal((4, 64))) for l in range(len(layers))}
    qq = {l: _bf16(rng.standard_normal((8, 512)) / np.sqrt(512)) for l in range(len(layers))}
    res = modes.run_layers(layers, L, keys, lambda l: iq[l], lambda l: qq[l], lambda p: rows[p])
    # Reuse layers consume exactly the preceding Full / Reindex layer's indices
    for l in (1, 2, 3):
        np.testing.assert_array_equal(res[l]["idx"], res[0]["idx"])
    np.testing.assert_array_equal(res[5]["idx"], res[4]["idx"])
    # the Reindex layer ranks the Full layer's pool: same candidates, its own choice
    np.testing.assert_array_equal(res[4]["pool"], res[0]["pool"])
    assert not np.array_equal(res[4]["idx"], res[0]["idx"])
    # Reindex shares K but not Q: fed the Full layer's query it reproduces the Full set
    same = modes.run_layers(["F", "RI"], L, keys, lambda l: iq[0], lambda l: qq[0],
                            lambda p: rows[p])
    np.testing.assert_array_equal(same[1]["idx"], same[0]["idx"])
    # a Reuse layer with the Full layer's attention query reproduces its output
    again = modes.run_layers(["F", "R"], L, keys, lambda l: iq[0], lambda l: qq[0],
                             lambda p: rows[p])
    np.testing.assert_array_equal(again[1]["out"], again[0]["out"])


def test_mode_order_errors():
    rng, rows, keys = _setup(100)
    q = lambda l: _bf16(np.zeros((4, 64)))
    with pytest.raises(ValueError):
        modes.run_layers(["R"], 100, keys, q, q, lambda p: rows[p])
    with pytest.raises(ValueError):
        modes.run_layers(["RI"], 100, keys, q, q, lambda p: rows[p])


def test_replay_positions():
    p, r = modes.replay_positions(1000, True)
    np.testing.assert_array_equal(p, np.arange(872, 1000))
    np.testing.assert_array_equal(r, np.arange(128))
    p, r = modes.replay_positions(50, True)
    np.testing.assert_array_equal(p, np.arange(50))
    np.testing.assert_array_equal(r, np.arange(78, 128))
    p, r = modes.replay_positions(1000, False)
    assert list(p) == [999] and list(r) == [127]
    assert modes.replay_positions(0, True)[0].size == 0


def test_replay_idempotent_and_restores_poisoned_rows():
    rng = np.random.default_rng(7)
    L = 300
    kv_bits = _bf16(rng.standard_normal((L, 512)))
    cache = codec.encode_bf16_rows(kv_bits)
    poisoned = cache.copy()
    poisoned[L - 128:] = 0xFF
    pos, src = modes.replay_positions(L, True)
    last = kv_bits[L - 128:]
    poisoned[pos] = codec.encode_bf16_rows(last[src])
    np.testing.assert_array_equal(poisoned, cache)
    again = poisoned.copy()
    again[pos] = codec.encode_bf16_rows(last[src])
    np.testing.assert_array_equal(again, cache)
