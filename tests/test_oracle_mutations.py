"""Planted mistakes: each test replaces one oracle function with a plausible slip
(a dropped term, a wrong sign or index, an off-by-one, a reversed tie-break) and
checks that at least one of the oracle's pins fails.  The slips are planted in the
oracle only, on the CPU, through monkeypatch, so the oracle itself is untouched."""
import numpy as np
import pytest

from oracle import attention, codec, indexer
from oracle.formats import bf16_to_f32, bf16_to_f64, f32_to_bf16
from tests import test_oracle_attention as pin_attn
from tests import test_oracle_codec as pin_codec
from tests import test_oracle_indexer as pin_idx


def _some_pin_fails(pins) -> list[str]:
    """Names of the pins that fail, with the exception type."""
    failed = []
    for pin in pins:
        try:
            pin()
        except Exception as e:   # an assertion, or the slip breaking a pin's assumptions
            failed.append(f"{pin.__name__}: {type(e).__name__}")
    return failed


ATTN_PINS = [pin_attn.test_dense_when_window_covers_context, pin_attn.test_closed_forms,
             pin_attn.test_union_of_selection_and_window]
INDEXER_PINS = [pin_idx.test_scores_against_fp64_einsum, pin_idx.test_scores_closed_forms,
                pin_idx.test_block_key_identities, pin_idx.test_topk_against_brute_force_loops,
                pin_idx.test_topk_tie_break_and_padding, pin_idx.test_hierarchy_brute_force_on_shrunken_sizes,
                pin_idx.test_pool_tokens_expansion_and_clipping, pin_idx.test_select_tokens_brute_force,
                pin_idx.test_block_max_scores_brute_force]
CODEC_PINS = [pin_codec.test_e2m1_code_exhaustive_vs_brute_force_and_division_form,
              pin_codec.test_scale_code_exhaustive_bf16_and_fp32_division_form,
              pin_codec.test_round_trip_on_grid_values, pin_codec.test_quantize_rows_properties,
              pin_codec.test_zero_scale_and_saturation, pin_codec.test_row_bytes_and_nibble_order,
              pin_codec.test_compression_special_cases, pin_codec.test_compress_pairs_hand_values]


def _caught(pins) -> bool:
    """True when some pin fails on one of its own checks (an assertion), not
    merely because the slip broke the call."""
    return any(f.endswith("AssertionError") for f in _some_pin_fails(pins))


def test_pins_pass_unmodified():
    assert _some_pin_fails(ATTN_PINS + INDEXER_PINS + CODEC_PINS) == []


# ---- attention ----

def _attend_without_scale(q_bits, rows, sm_scale=1.0):
    q = bf16_to_f64(q_bits)
    rows = np.asarray(rows, dtype=np.float64)
    if rows.shape[0] == 0:
        return np.zeros((q.shape[0], q.shape[1]))
    s = q @ rows.T                                   # slip: sm_scale dropped
    p = np.exp(s - s.max(axis=1, keepdims=True))
    return (p / p.sum(axis=1, keepdims=True)) @ rows


def _attend_without_max(q_bits, rows, sm_scale=1.0):
    q = bf16_to_f64(q_bits)
    rows = np.asarray(rows, dtype=np.float64)
    if rows.shape[0] == 0:
        return np.zeros((q.shape[0], q.shape[1]))
    with np.errstate(over="ignore", invalid="ignore"):
        p = np.exp(sm_scale * (q @ rows.T))          # slip: no max subtraction
        return (p / p.sum(axis=1, keepdims=True)) @ rows


def _attend_reversed_values(q_bits, rows, sm_scale=1.0):
    q = bf16_to_f64(q_bits)
    rows = np.asarray(rows, dtype=np.float64)
    if rows.shape[0] == 0:
        return np.zeros((q.shape[0], q.shape[1]))
    s = sm_scale * (q @ rows.T)
    p = np.exp(s - s.max(axis=1, keepdims=True))
    return (p / p.sum(axis=1, keepdims=True)) @ rows[::-1]   # slip: values paired with the wrong rows


def _window_off_by_one(idx, visible, window=attention.WINDOW):
    sel = np.asarray(idx, dtype=np.int64)
    sel = sel[sel >= 0]
    w0 = max(0, visible - window + 1)                # slip: a 127-token window
    return np.union1d(sel, np.arange(w0, visible, dtype=np.int64))


@pytest.mark.parametrize("name,fn", [("attend", _attend_without_scale), ("attend", _attend_without_max),
                                     ("attend", _attend_reversed_values),
                                     ("attended_positions", _window_off_by_one)])
def test_attention_slips_are_caught(monkeypatch, name, fn):
    monkeypatch.setattr(attention, name, fn)
    assert _caught(ATTN_PINS)


# ---- indexer ----

def _scores_without_relu(q, k, w):
    wv = np.ones(q.shape[0], dtype=np.float32) if w is None else np.asarray(w, dtype=np.float32)
    dots = (k.astype(np.float32) @ q.T.astype(np.float32)).astype(np.float32)   # [n, heads]
    return (dots * wv).sum(axis=1).astype(np.float32)                           # slip: no ReLU


def _scores_without_weights(q, k, w):
    dots = (k.astype(np.float32) @ q.T.astype(np.float32)).astype(np.float32)
    return np.maximum(dots, 0).sum(axis=1).astype(np.float32)                  # slip: w ignored


def _scores_transposed_dims(q, k, w):
    wv = np.ones(q.shape[0], dtype=np.float32) if w is None else np.asarray(w, dtype=np.float32)
    dots = (k.astype(np.float32) @ q[:, ::-1].T.astype(np.float32)).astype(np.float32)   # slip: dims reversed
    return (np.maximum(dots, 0) * wv).sum(axis=1).astype(np.float32)


def _top_k_highest_index_wins(scores, valid, k):
    pos = np.nonzero(np.asarray(valid, dtype=bool))[0]
    s = np.asarray(scores, dtype=np.float64)[pos]
    order = np.lexsort((-pos, -s))                   # slip: ties go to the highest position
    chosen = np.sort(pos[order[:k]])
    out = np.full(k, -1, dtype=np.int64)
    out[:chosen.size] = chosen
    return out


def _top_k_unsorted_output(scores, valid, k):
    pos = np.nonzero(np.asarray(valid, dtype=bool))[0]
    s = np.asarray(scores, dtype=np.float64)[pos]
    chosen = pos[np.lexsort((pos, -s))[:k]]          # slip: listed by score, not ascending
    out = np.full(k, -1, dtype=np.int64)
    out[:chosen.size] = chosen
    return out


def _block_keys_sum(key_bits, length, block=indexer.BLOCK):
    k = bf16_to_f32(np.asarray(key_bits)[:length])
    nb = (length + block - 1) // block
    acc = np.zeros((nb, k.shape[1]), dtype=np.float32)
    for t in range(block):
        rows = np.arange(nb) * block + t
        present = rows < length
        acc[present] = (acc[present] + k[rows[present]]).astype(np.float32)
    return f32_to_bf16(acc)                          # slip: sum instead of mean


def _block_keys_full_count(key_bits, length, block=indexer.BLOCK):
    k = bf16_to_f32(np.asarray(key_bits)[:length])
    nb = (length + block - 1) // block
    acc = np.zeros((nb, k.shape[1]), dtype=np.float32)
    for t in range(block):
        rows = np.arange(nb) * block + t
        present = rows < length
        acc[present] = (acc[present] + k[rows[present]]).astype(np.float32)
    return f32_to_bf16((acc / np.float32(block)).astype(np.float32))   # slip: a ragged block divided by 8


def _pool_tokens_unclipped(pool_blocks, length, block=indexer.BLOCK):
    b = np.asarray(pool_blocks)
    b = b[b >= 0]
    return (b[:, None] * block + np.arange(block)[None, :]).reshape(-1)   # slip: not clipped to the context


def _block_max_first_token(q_bits, key_bits, length, w=None, block=indexer.BLOCK):
    ts = indexer.index_scores(q_bits, np.asarray(key_bits)[:length], w)
    return ts[::block].astype(np.float32)            # slip: the block's first token, not its maximum


@pytest.mark.parametrize("name,fn", [("_scores_f32", _scores_without_relu), ("_scores_f32", _scores_without_weights),
                                     ("_scores_f32", _scores_transposed_dims),
                                     ("top_k", _top_k_highest_index_wins), ("top_k", _top_k_unsorted_output),
                                     ("block_keys", _block_keys_sum), ("block_keys", _block_keys_full_count),
                                     ("pool_tokens", _pool_tokens_unclipped),
                                     ("block_max_scores", _block_max_first_token)])
def test_indexer_slips_are_caught(monkeypatch, name, fn):
    monkeypatch.setattr(indexer, name, fn)
    assert _caught(INDEXER_PINS)


# ---- codec ----

def _scale_code_over_four(amax):
    return codec._round_to_grid(amax, 4.0 * codec.E4M3_MIDS).astype(np.uint8)   # slip: amax / 4


def _pack_rows_swapped_nibbles(codes, scales):
    codes = np.asarray(codes, dtype=np.uint8)
    packed = (codes[:, 1::2] & 0xF) | ((codes[:, 0::2] & 0xF) << 4)          # slip: nibble order
    return np.concatenate([packed.astype(np.uint8), np.asarray(scales, dtype=np.uint8)], axis=1)


def _e2m1_code_without_sign(x, s):
    x = np.asarray(x, dtype=np.float64)
    s = np.broadcast_to(np.asarray(s, dtype=np.float64), x.shape)
    return codec._round_to_grid(np.abs(x), s[..., None] * codec.E2M1_MIDS).astype(np.uint8)   # slip: sign lost


def _compress_first_of_pair(bits):
    return bf16_to_f32(bits)[0::2].astype(np.float32)                        # slip: no averaging


@pytest.mark.parametrize("name,fn", [("scale_code", _scale_code_over_four), ("pack_rows", _pack_rows_swapped_nibbles),
                                     ("e2m1_code", _e2m1_code_without_sign),
                                     ("compress_pairs_f32", _compress_first_of_pair)])
def test_codec_slips_are_caught(monkeypatch, name, fn):
    monkeypatch.setattr(codec, name, fn)
    assert _caught(CODEC_PINS)


# ---- FP8 indexer keys ----

from oracle import idxk_fp8, modes                     # noqa: E402
from tests import test_oracle_idxk_fp8 as pin_fp8       # noqa: E402
from tests import test_oracle_modes as pin_modes        # noqa: E402

FP8_PINS = [pin_fp8.test_every_e4m3_value_encodes_to_itself,
            pin_fp8.test_rounding_against_brute_force_on_all_bf16_magnitudes,
            pin_fp8.test_midpoints_round_to_even_and_match_torch, pin_fp8.test_saturation,
            pin_fp8.test_quantised_key_error_bound_and_degenerate_keys,
            pin_fp8.test_exactly_representable_keys_round_trip_and_score_like_bf16,
            pin_fp8.test_scores_against_fp64_on_the_dequantised_key]


def _e4m3_ties_away(t):
    t = np.asarray(t, dtype=np.float32)
    mag = np.abs(t.astype(np.float64))
    code = np.sum(idxk_fp8.E4M3_MIDS <= mag[..., None], axis=-1)   # slip: ties round up, not to even
    return (code | (np.signbit(t).astype(np.int64) << 7)).astype(np.uint8)


def _e4m3_sign_dropped(t):
    t = np.asarray(t, dtype=np.float32)
    mag = np.abs(t.astype(np.float64))
    below = np.sum(idxk_fp8.E4M3_MIDS < mag[..., None], axis=-1)
    tie = np.any(idxk_fp8.E4M3_MIDS == mag[..., None], axis=-1)
    return (below + (tie & (below % 2 == 1))).astype(np.uint8)     # slip: the sign bit lost


def _quantize_scale_240(key_bits):
    k = bf16_to_f32(np.asarray(key_bits, dtype=np.uint16))
    amax = np.max(np.abs(k), axis=-1).astype(np.float32)
    s = (amax / np.float32(240.0)).astype(np.float32)                # slip: the E4M3 maximum taken as 240
    codes = np.zeros(k.shape, dtype=np.uint8)
    nz = s != 0
    codes[nz] = idxk_fp8.e4m3_code((k[nz] / s[nz, None]).astype(np.float32))
    return codes, s


@pytest.mark.parametrize("name,fn", [("e4m3_code", _e4m3_ties_away), ("e4m3_code", _e4m3_sign_dropped),
                                     ("quantize", _quantize_scale_240)])
def test_fp8_key_slips_are_caught(monkeypatch, name, fn):
    monkeypatch.setattr(idxk_fp8, name, fn)
    assert _caught(FP8_PINS)


# ---- replay and the sliding-window store ----

MODES_PINS = [pin_modes.test_replay_positions, pin_modes.test_replay_idempotent_and_restores_poisoned_rows,
              pin_modes.test_ratio2_replay_of_duplicated_rows_equals_ratio1,
              pin_modes.test_window_store_holds_the_last_128_entries,
              pin_modes.test_window_store_is_a_ring_filled_from_slot_zero,
              lambda: pin_modes.test_ratio2_replay_of_an_intact_sequence_reproduces_its_entries(300)]


def _replay_one_short(length, miss, window=modes.REPLAY):
    if length <= 0:
        return np.zeros(0, np.int64), np.zeros(0, np.int64)
    if miss:
        n = min(window - 1, length)                                  # slip: 127 entries replayed
        return np.arange(length - n, length), np.arange(window - n, window)
    return np.array([length - 1]), np.array([window - 1])


def _replay_wrong_rows(length, miss, window=modes.REPLAY):
    if length <= 0:
        return np.zeros(0, np.int64), np.zeros(0, np.int64)
    if miss:
        n = min(window, length)
        return np.arange(length - n, length), np.arange(0, n)        # slip: the block's first rows, not its last
    return np.array([length - 1]), np.array([window - 1])


def _store_slots_shifted(length, window=modes.REPLAY):
    pos = np.arange(max(0, length - window), length, dtype=np.int64)
    return pos, (pos + 1) % window                                   # slip: slots shifted by one


@pytest.mark.parametrize("name,fn", [("replay_positions", _replay_one_short), ("replay_positions", _replay_wrong_rows),
                                     ("window_store_slots", _store_slots_shifted)])
def test_replay_slips_are_caught(monkeypatch, name, fn):
    monkeypatch.setattr(modes, name, fn)
    assert _caught(MODES_PINS)


# ---- the layer schedule ----

def _run_layers_with(slip):
    """run_layers with one schedule slip: "ri_own_pool" (a Reindex layer builds
    its own pool), "reuse_recomputes" (a Reuse layer selects with its own query),
    "ri_reuses" (a Reindex layer keeps the previous set)."""
    def run(layers, length, key_bits, idxq_fn, q_fn, rows_fn, sm_scale=1.0, hierarchical=True, w=None):
        results, pool, latest = [], None, None
        for layer, mode in enumerate(layers):
            if mode == "F" or (mode == "RI" and slip == "ri_own_pool") or (mode == "R" and slip == "reuse_recomputes"):
                pool, latest, _ = indexer.full_indexer(idxq_fn(layer), key_bits, length, w, hierarchical)
            elif mode == "RI" and slip != "ri_reuses":
                latest, _ = indexer.reindex_indexer(idxq_fn(layer), key_bits, length, pool, w)
            pos = attention.attended_positions(latest, length)
            out = attention.attend(q_fn(layer), rows_fn(pos), sm_scale)
            results.append({"mode": mode, "idx": latest.copy(), "pool": None if pool is None else pool.copy(),
                            "out": out})
        return results
    return run


@pytest.mark.parametrize("slip", ["ri_own_pool", "reuse_recomputes", "ri_reuses"])
def test_schedule_slips_are_caught(monkeypatch, slip):
    monkeypatch.setattr(modes, "run_layers", _run_layers_with(slip))
    assert _caught([lambda: pin_modes.test_reuse_and_reindex_invariants(20000)])


def test_schedule_reimplementation_without_slip_passes(monkeypatch):
    monkeypatch.setattr(modes, "run_layers", _run_layers_with(None))
    assert _some_pin_fails([lambda: pin_modes.test_reuse_and_reindex_invariants(20000)]) == []
