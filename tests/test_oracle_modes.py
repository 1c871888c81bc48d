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


@pytest.mark.parametrize("L", [300, 50, 128, 1])
def test_ratio2_replay_of_an_intact_sequence_reproduces_its_entries(L):
    """Encoder replay at compression ratio 2: the supplied block holds the raw
    rows of the last 128 entries (two per entry, zero rows ahead of a short
    sequence); re-encoding them gives back the entries the append made."""
    rng = np.random.default_rng(L)
    raw = _bf16(rng.standard_normal((2 * L, 512)))
    rawk = _bf16(rng.standard_normal((2 * L, 64)))
    entries = codec.encode_entries(raw, 2)
    keys = codec.idxk_entries(rawk, 2)
    n = min(128, L)
    block = np.zeros((256, 512), np.uint16)
    block[256 - 2 * n:] = raw[2 * (L - n):]
    kblock = np.zeros((256, 64), np.uint16)
    kblock[256 - 2 * n:] = rawk[2 * (L - n):]
    for miss in (True, False):
        pos, rows = modes.replay_entries(block, L, miss, compress=2)
        kpos, krows = modes.replay_keys(kblock, L, miss, compress=2)
        np.testing.assert_array_equal(pos, np.arange(L - n, L) if miss else [L - 1])
        np.testing.assert_array_equal(kpos, pos)
        np.testing.assert_array_equal(rows, entries[pos])
        np.testing.assert_array_equal(krows, keys[pos])


def test_ratio2_replay_of_duplicated_rows_equals_ratio1():
    """The pair mean of two equal bf16 rows is the row itself (exact in fp32),
    so a block whose raw rows come in equal pairs replays to the ratio-1
    encoding of one row of each pair."""
    rng = np.random.default_rng(3)
    x = _bf16(rng.standard_normal((128, 512)) * rng.uniform(0.01, 50, (128, 1)))
    k = _bf16(rng.standard_normal((128, 64)))
    pos, rows = modes.replay_entries(np.repeat(x, 2, axis=0), 700, True, compress=2)
    np.testing.assert_array_equal(pos, np.arange(572, 700))
    np.testing.assert_array_equal(rows, codec.encode_bf16_rows(x))
    _, krows = modes.replay_keys(np.repeat(k, 2, axis=0), 700, True, compress=2)
    np.testing.assert_array_equal(krows, k)
    # ratio 1 reads the block row by row
    _, rows1 = modes.replay_entries(x, 700, True, compress=1)
    np.testing.assert_array_equal(rows1, codec.encode_bf16_rows(x))


def test_window_store_holds_the_last_128_entries():
    """Against a first-in first-out queue of capacity 128 fed one entry at a
    time: the store's positions are the queue's content, each in its own slot,
    and the attended positions read from the store are exactly those."""
    import collections
    fifo = collections.deque(maxlen=128)
    for L in range(1, 700):
        fifo.append(L - 1)
        if L in (1, 2, 127, 128, 129, 255, 256, 300, 699):
            pos, slot = modes.window_store_slots(L)
            np.testing.assert_array_equal(pos, np.array(fifo))
            assert len(set(slot.tolist())) == pos.size and slot.min() >= 0 and slot.max() < 128
            probe = np.arange(L)
            np.testing.assert_array_equal(modes.from_window_store(probe, L), np.isin(probe, list(fifo)))


def test_window_store_is_a_ring_filled_from_slot_zero():
    """Appending moves nothing: an entry keeps its slot for as long as it is in
    the window, and the one appended takes the slot its evicted predecessor
    left.  An empty store fills its first slots first.  Together these fix the
    layout (by induction, slot of position p = p mod 128)."""
    slot_of = {}
    for L in range(1, 600):
        pos, slot = modes.window_store_slots(L)
        cur = dict(zip(pos.tolist(), slot.tolist()))
        for p_, s_ in cur.items():
            if p_ in slot_of:
                assert slot_of[p_] == s_, (L, p_)            # no entry moves
        if L <= 128:
            assert cur[L - 1] == L - 1                       # filled from slot 0 in order
        else:
            assert cur[L - 1] == slot_of[L - 1 - 128]        # takes the evicted entry's slot
        slot_of.update(cur)
