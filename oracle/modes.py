"""CSA2 layer modes (Full / Reindex / Reuse) and SWA bounded replay.

What the pages fix (agentnet.co.il, "דיפסיק משיקה את V4.1-פלאש ...", section
"CSA2: דחיסה לאורך ציר השכבות"; ai-wave.ru, "DeepSeek V4.1-Flash: 1M
контекст ...", third paragraph; tgviewer.app, "DeepSeek V4.1 Flash: новая
архитектура ...", section "Слои больше не хранят всё независимо"):

* each CSA2 layer has one static mode;
* Full computes the main KV, projects indexer K and selects fresh indices;
* Reindex reuses the last Full layer's main KV and indexer K but ranks them
  with its own indexer Q;
* Reuse reuses the main KV and the latest indices and skips the indexer;
* decoder: 20 layers in five groups of four -- the first group Full + 3 Reuse,
  the others Reindex + 3 Reuse; encoder: 18 layers at compression ratio 2 in
  three groups of six, each 1 Full + 5 Reuse.

Bounded replay: on a cache miss only the last 128 tokens are recomputed
(ai-wave.ru, second paragraph; agentnet.co.il, sections "ארכיטקטורה שחותכת
בחצי את הפריפיל" and "קוונטיזציה ופריסה: FP4 ו-DRAM במקום SSD"), in the
decoder and in the encoder (the latter section: 128 tokens instead of layers
x window).  Reading: a flagged sequence rewrites its last min(128, L) entries
from freshly supplied bf16 rows; an unflagged one writes only its newest entry
(position L-1).  At compression ratio 2 (encoder) an entry is made of two raw
rows, so the supplied block holds 2 x 128 raw rows.

Sliding-window store: the window's KV is kept apart from the global cache
(ai-wave.ru, fourth paragraph; agentnet.co.il, section "קוונטיזציה ופריסה: FP4
ו-DRAM במקום SSD": a separate pool with a short lifetime, never written to
disk).  Reading: the store holds each sequence's last 128 entries, entry p in
slot p mod 128, in the cache's FP4 row format; attention reads those entries
from the store and every older entry from the global cache; replay with a
store rewrites only the store.

Pinned by tests/test_oracle_modes.py (Reuse reproduces the preceding set
exactly; Reindex with the Full layer's own query reproduces the Full set;
group patterns; replay idempotence and poisoned-row restore; ratio-2 replay of
an intact sequence reproduces its entries, and of duplicated raw rows equals
ratio 1; the store's slots against a first-in first-out queue of the last 128
appended entries).
"""
from __future__ import annotations

import numpy as np

from . import attention as attn_mod
from . import codec as codec_mod
from . import indexer as idx_mod

DECODER_PATTERN = ["F", "R", "R", "R"] + ["RI", "R", "R", "R"] * 4
ENCODER_PATTERN = (["F"] + ["R"] * 5) * 3
REPLAY = 128


def run_layers(layers, length, key_bits, idxq_fn, q_fn, rows_fn, sm_scale=1.0,
               hierarchical=True, w=None):
    """Run a static layer schedule for one decode query.

    idxq_fn(layer) -> indexer query bits [4,64]; q_fn(layer) -> attention query
    bits [H,512]; rows_fn(positions) -> fp64 decoded rows.  Returns a list of
    per-layer dicts {mode, idx, pool, out}."""
    results = []
    pool = None
    latest = None
    for layer, mode in enumerate(layers):
        if mode == "F":
            pool, latest, _ = idx_mod.full_indexer(idxq_fn(layer), key_bits, length, w,
                                                   hierarchical)
        elif mode == "RI":
            if pool is None:
                raise ValueError("Reindex layer before any Full layer")
            latest, _ = idx_mod.reindex_indexer(idxq_fn(layer), key_bits, length, pool, w)
        elif mode == "R":
            if latest is None:
                raise ValueError("Reuse layer before any Full or Reindex layer")
        else:
            raise ValueError(mode)
        pos = attn_mod.attended_positions(latest, length)
        out = attn_mod.attend(q_fn(layer), rows_fn(pos), sm_scale)
        results.append({"mode": mode, "idx": latest.copy(), "pool": None if pool is None
                        else pool.copy(), "out": out})
    return results


def replay_positions(length: int, miss: bool, window: int = REPLAY) -> tuple[np.ndarray, np.ndarray]:
    """(cache positions rewritten, rows of the supplied last-128 block used) for
    one sequence of length `length`."""
    if length <= 0:
        return np.zeros(0, np.int64), np.zeros(0, np.int64)
    if miss:
        n = min(window, length)
        return np.arange(length - n, length), np.arange(window - n, window)
    return np.array([length - 1]), np.array([window - 1])


def replay_entries(kv_last_bits: np.ndarray, length: int, miss: bool, compress: int = 1,
                   window: int = REPLAY) -> tuple[np.ndarray, np.ndarray]:
    """(entry positions rewritten, their packed 288-B rows) for one sequence.
    kv_last_bits: the raw bf16 rows [window * compress, 512] behind the
    sequence's last `window` entries; entry r is made of raw rows
    [compress r, compress r + compress)."""
    pos, used = replay_positions(length, miss, window)
    raw = np.asarray(kv_last_bits, dtype=np.uint16).reshape(window, compress, -1)[used]
    return pos, codec_mod.encode_entries(raw.reshape(-1, raw.shape[-1]), compress)


def replay_keys(idxk_last_bits: np.ndarray, length: int, miss: bool, compress: int = 1,
                window: int = REPLAY) -> tuple[np.ndarray, np.ndarray]:
    """(entry positions rewritten, their stored bf16 indexer keys) for one
    sequence replayed without a sliding-window store."""
    pos, used = replay_positions(length, miss, window)
    raw = np.asarray(idxk_last_bits, dtype=np.uint16).reshape(window, compress, -1)[used]
    return pos, codec_mod.idxk_entries(raw.reshape(-1, raw.shape[-1]), compress)


def window_store_slots(length: int, window: int = REPLAY) -> tuple[np.ndarray, np.ndarray]:
    """(entry positions the sliding-window store holds for a sequence of
    `length` entries, their slots)."""
    pos = np.arange(max(0, length - window), length, dtype=np.int64)
    return pos, pos % window


def from_window_store(positions, length: int, window: int = REPLAY) -> np.ndarray:
    """Mask of the attended positions that are read from the sliding-window
    store rather than the global cache."""
    return np.asarray(positions, dtype=np.int64) >= length - window
