"""CSA2 sparse attention over the selected tokens and the sliding window.

What the pages fix: every layer runs sliding-window attention over the last
128 tokens (ai-wave.ru, "DeepSeek V4.1-Flash: 1M контекст ...", second
paragraph; agentnet.co.il, "דיפסיק משיקה את V4.1-פלאש ...", section
"ארכיטקטורה שחותכת בחצי את הפריפיל"), and a CSA2 layer attends over 512
selected indices (same page, section "CSA2: דחיסה לאורך ציר השכבות").

Readings taken where the pages are silent:

* the attended set is the union of the selected positions and the window
  [max(0, v-128), v), each position counted once (v = visible length);
* the latent is shared by K and V (MQA over a 512-d latent): K = V = the
  decoded FP4 rows;
* logits = sm_scale * q . k, exact softmax over the set, output = sum p_t k_t;
  an empty set gives a zero output;
* in a causal prefill at compression ratio 2 a query at raw position P sees
  the compressed entries [0, floor((P+1)/2)) -- entry c averages raw tokens
  2c and 2c+1 and is complete once token 2c+1 exists -- and its window is the
  last 128 visible entries.

Arithmetic is fp64 (the GPU path is bf16 x bf16 with fp32 accumulation; the
comparison tolerance covers the difference).

Pinned by tests/test_oracle_attention.py: dense textbook attention through
torch's scaled_dot_product_attention in fp64 when the window covers the
context, a single-row set returns that row, a zero query returns the mean,
and the union/dedup rule on hand-made sets.
"""
from __future__ import annotations

import numpy as np

from .formats import bf16_to_f64

WINDOW = 128


def attended_positions(idx: np.ndarray, visible: int, window: int = WINDOW) -> np.ndarray:
    """Selected positions (>= 0) joined with the window, ascending and unique."""
    sel = np.asarray(idx, dtype=np.int64)
    sel = sel[sel >= 0]
    if sel.size and sel.max() >= visible:
        raise ValueError("selected position beyond the visible context")
    w0 = max(0, visible - window)
    return np.union1d(sel, np.arange(w0, visible, dtype=np.int64))


def attend(q_bits: np.ndarray, rows: np.ndarray, sm_scale: float = 1.0) -> np.ndarray:
    """Exact softmax attention of q [H,512] (bf16 bits) over rows [T,512] (fp64)."""
    q = bf16_to_f64(q_bits)
    rows = np.asarray(rows, dtype=np.float64)
    if rows.shape[0] == 0:
        return np.zeros((q.shape[0], q.shape[1]), dtype=np.float64)
    s = sm_scale * (q @ rows.T)
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p = p / p.sum(axis=1, keepdims=True)
    return p @ rows


def prefill_visible(raw_pos: int, compress: int) -> int:
    """Compressed entries visible to a query at raw token position raw_pos."""
    return (raw_pos + 1) // compress
