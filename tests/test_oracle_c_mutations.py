"""Sensitivity of the C oracle's pins: each plausible slip, planted in a copy of
oracle/c/csa2_oracle.c compiled on the CPU, must make some pin of
tests/test_oracle_c.py fail (the unmodified source passes them all)."""
import ctypes
import os
import subprocess

import pytest

from oracle import c_oracle as co
from tests import test_oracle_c as pins

# fast pins first: a slip usually fails one of them
PINS = [pins.test_row_layout_zero_scale_and_saturation, pins.test_decode_is_code_value_times_scale_and_round_trips_grid_values,
        pins.test_scores_closed_forms_and_fp64_bound, pins.test_block_key_identities,
        pins.test_topk_brute_force_ties_and_padding, pins.test_attention_textbook_closed_forms_and_union,
        pins.test_hierarchy_brute_force, pins.test_decode_steps_invariants_and_agreement_with_the_numpy_oracle,
        pins.test_ratio2_entries_pins_and_agreement, pins.test_flat_indexer_brute_force,
        pins.test_ragged_steps_agree_with_the_numpy_oracle,
        pins.test_scale_byte_of_every_bf16_group_maximum, pins.test_codes_of_every_bf16_value_under_every_scale]

SLIPS = {
    "ties to the odd grid point": ("(d == bd && (i & 1) == 0)", "(d == bd && (i & 1) == 1)"),
    "scale from amax / 4": ("scale6[c] = 6.0 * csa2o_e4m3_value(c)", "scale6[c] = 4.0 * csa2o_e4m3_value(c)"),
    "nibbles swapped": ("(code[2 * j] | (code[2 * j + 1] << 4))", "(code[2 * j + 1] | (code[2 * j] << 4))"),
    "sign lost": ("nearest_even(fabs((double)v), grid, 8) | (signbit(v) ? 8 : 0)",
                  "nearest_even(fabs((double)v), grid, 8)"),
    "scale byte of the next group": ("row[CODE_BYTES + c / GROUP]", "row[CODE_BYTES + (c / GROUP + 1) % N_GROUPS]"),
    "ReLU dropped": ("dot > 0.0f ? dot : 0.0f", "dot"),
    "head weight dropped": ("const float t = wh * relu;", "const float t = relu;"),
    "key dimensions reversed": ("bf16_to_float(k[d])", "bf16_to_float(k[IDX_DIM - 1 - d])"),
    "ties to the highest position": ("return x->i < y->i ? -1 : (x->i > y->i ? 1 : 0);",
                                     "return x->i > y->i ? -1 : (x->i < y->i ? 1 : 0);"),
    "selection left unsorted": ("qsort(out, (size_t)m, sizeof(int64_t), by_value);", ""),
    "block key divided by 8": ("float_to_bf16(acc / cnt)", "float_to_bf16(acc / 8.0f)"),
    "pool tokens not clipped": ("if (p < L) cand[n++] = p;", "cand[n++] = p;"),
    "127-token window": ("#define WINDOW 128", "#define WINDOW 127"),
    "sm_scale dropped": ("s[t] = sm_scale * dot;", "s[t] = dot;"),
    "no max subtraction": ("s[t] = exp(s[t] - m);", "s[t] = exp(s[t]);"),
    "Reuse selects again": ("} else if (m != 'R' || !have_set) {",
                            "} else if (m == 'R' && have_set) {\n      csa2o_full_indexer(iq, NULL, sq->keys, sq->L, pool, latest);\n      fresh = 1;\n    } else {"),
    "no pair averaging": ("x[c] = sum * 0.5f;", "x[c] = a;"),
    "flat indexer sees one position too many": ("for (int64_t p = 0; p < visible; ++p) cand[p] = p;\n  select_tokens(q, w, keys, cand, visible, idx);",
                                                "for (int64_t p = 0; p < visible; ++p) cand[p] = p;\n  select_tokens(q, w, keys, cand, visible > 0 ? visible - 1 : 0, idx);"),
    "replay window of 127": ("(sq->L < REPLAY ? sq->L : REPLAY)", "(sq->L < REPLAY - 1 ? sq->L : REPLAY - 1)"),
    "Reindex builds its own pool": ("csa2o_reindex_indexer(iq, NULL, sq->keys, sq->L, pool, latest);",
                                    "csa2o_full_indexer(iq, NULL, sq->keys, sq->L, pool, latest);"),
}


def _build_variant(tmp_path, src_text, name):
    src = tmp_path / f"{name}.c"
    lib = tmp_path / f"lib{name}.so"
    src.write_text(src_text)
    subprocess.check_call(["gcc", *co.CFLAGS, "-o", str(lib), str(src), "-lm"])
    return str(lib)


def _with_lib(path, fn):
    saved = co.lib()
    L = ctypes.CDLL(path)
    for name in dir(saved):
        if name.startswith("csa2o_"):
            f, g = getattr(saved, name), getattr(L, name)
            g.restype, g.argtypes = f.restype, f.argtypes
    co._lib = L
    try:
        return fn()
    finally:
        co._lib = saved


def _failing_pin():
    for pin in PINS:
        try:
            pin()
        except (AssertionError, ValueError):
            return pin.__name__
    return None


def test_pins_pass_on_an_unmodified_copy(tmp_path):
    text = open(co.SRC).read()
    assert _with_lib(_build_variant(tmp_path, text, "same"), _failing_pin) is None


@pytest.mark.parametrize("slip", sorted(SLIPS))
def test_each_slip_fails_a_pin(tmp_path, slip):
    old, new = SLIPS[slip]
    text = open(co.SRC).read()
    assert text.count(old) == 1, f"slip site not found: {slip}"
    lib = _build_variant(tmp_path, text.replace(old, new), "mutant")
    caught = _with_lib(lib, _failing_pin)
    assert caught is not None, f"no pin fails with the slip: {slip}"
