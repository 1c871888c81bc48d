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
