"""CSA2 indexer: block keys, indexer scores, top-k, hierarchical candidate pool.

What the pages fix (agentnet.co.il, "דיפסיק משיקה את V4.1-פלאש ...", section
"CSA2: דחיסה לאורך ציר השכבות"; ai-wave.ru, "DeepSeek V4.1-Flash: 1M
контекст ...", third paragraph; globalfeed.ai, section "Mimari tarafında ne
değişti"):

* a Full layer projects indexer K and selects 512 fresh indices;
* a Reindex layer ranks the last Full layer's indexer K with its own indexer Q;
* in the decoder a hierarchical sparse indexer lets the Full layer build a
  candidate pool of up to 16,384 positions = 2,048 blocks of 8 tokens, so that
  later Reindex layers rank a bounded set instead of the whole context.

Readings taken where the pages are silent:

* indexer: 4 query heads x 64 dims, one shared 64-d bf16 key per token;
* score(q, k) = sum_h w_h * max(0, q_h . k), fp32, accumulated over d
  ascending inside each head and then over h ascending (w_h = 1 by default);
* block key of block j = bf16(mean of the stored keys of tokens
  8j .. min(8j+8, L)-1), summed in fp32 in ascending token order, divided by
  the token count in fp32, rounded to nearest-even bf16;
* the pool is used only when the context has more than 2,048 blocks; up to
  that size every token is a candidate (the flat case);
* ranking is by score descending, then position ascending (lowest position
  wins a tie); fewer candidates than k -> all of them, padded with -1; the
  output set is listed in ascending position order;
* Reindex ranks the tokens of the pool that the Full layer built.
* block score: the pages do not give it.  Default ("mean"): the score of the
  block key (mean-pooled keys) -- a real hierarchy that reads L/8 keys.
  Alternative ("max"): the largest score of the block's present tokens.  It
  reads every key, and it is lossless: a token of the flat top-k lies in a
  block that fewer than pool_blocks blocks can beat (each of those holds a
  token that beats it), so the pool's top-k equals the flat top-k.

Keys are bf16 bit patterns [n, 64] or FP8 keys (oracle.idxk_fp8.Fp8Keys):
an FP8 key's score is its scale times the score of its code values, and
block keys are built from the dequantised keys.

The score arithmetic is fp32, as in the kernels, because its result decides
integer outcomes (which positions are selected).

Pinned by tests/test_oracle_indexer.py: closed-form scores (unit queries,
ReLU, head weights) against an fp64 einsum, block-key identities, brute-force
top-k with explicit loops, hierarchy == flat up to 16,384 tokens, and a
brute-force pool on shrunken sizes.
"""
from __future__ import annotations

import numpy as np

from .formats import bf16_to_f32, f32_to_bf16
from .idxk_fp8 import Fp8Keys, code_values

IDX_HEADS = 4
IDX_DIM = 64
BLOCK = 8          # tokens per indexer block
POOL_BLOCKS = 2048  # blocks in the candidate pool
TOP_K = 512         # indices selected per query


def block_keys(key_bits, length: int, block: int = BLOCK) -> np.ndarray:
    """Mean-pooled block keys (bf16 bits [ceil(L/block), 64]) of the first
    `length` stored keys (bf16 bits, or FP8 keys through their dequantised values)."""
    if isinstance(key_bits, Fp8Keys):
        k = key_bits[:length].dequantized()
    else:
        k = bf16_to_f32(np.asarray(key_bits)[:length])
    nb = (length + block - 1) // block
    acc = np.zeros((nb, k.shape[1]), dtype=np.float32)
    cnt = np.zeros(nb, dtype=np.float32)
    for t in range(block):                      # ascending token order inside a block
        rows = np.arange(nb) * block + t
        present = rows < length
        acc[present] = (acc[present] + k[rows[present]]).astype(np.float32)
        cnt[present] += np.float32(1.0)
    mean = (acc / cnt[:, None]).astype(np.float32)
    return f32_to_bf16(mean)


def index_scores(q_bits: np.ndarray, key_bits, w: np.ndarray | None = None) -> np.ndarray:
    """fp32 scores [n] of one indexer query q [4,64] against keys [n,64]
    (bf16 bits, or FP8 keys: fl32(scale x score of the code values))."""
    if isinstance(key_bits, Fp8Keys):
        total = _scores_f32(bf16_to_f32(q_bits), code_values(key_bits.codes), w)
        return (key_bits.scales * total).astype(np.float32)
    return _scores_f32(bf16_to_f32(q_bits), bf16_to_f32(key_bits), w)


def _scores_f32(q: np.ndarray, k: np.ndarray, w) -> np.ndarray:
    heads = q.shape[0]
    wv = np.ones(heads, dtype=np.float32) if w is None else np.asarray(w, dtype=np.float32)
    total = np.zeros(k.shape[0], dtype=np.float32)
    for h in range(heads):
        dot = np.zeros(k.shape[0], dtype=np.float32)
        for d in range(q.shape[1]):
            dot = (dot + (q[h, d] * k[:, d]).astype(np.float32)).astype(np.float32)
        relu = np.maximum(dot, np.float32(0.0))
        total = (total + (wv[h] * relu).astype(np.float32)).astype(np.float32)
    return total


def top_k(scores: np.ndarray, valid: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k best valid entries by (score desc, index asc), listed
    ascending, padded with -1 to length k."""
    pos = np.nonzero(np.asarray(valid, dtype=bool))[0]
    s = np.asarray(scores, dtype=np.float64)[pos]
    order = np.lexsort((pos, -s))
    chosen = np.sort(pos[order[:k]])
    out = np.full(k, -1, dtype=np.int64)
    out[:chosen.size] = chosen
    return out


def pool_tokens(pool_blocks: np.ndarray, length: int, block: int = BLOCK) -> np.ndarray:
    """Token positions covered by the pool's blocks, ascending, clipped to the context."""
    b = np.asarray(pool_blocks)
    b = b[b >= 0]
    toks = (b[:, None] * block + np.arange(block)[None, :]).reshape(-1)
    return toks[toks < length]


def select_tokens(q_bits, key_bits, candidates: np.ndarray, w=None, k: int = TOP_K):
    """Top-k token positions among `candidates` (ascending positions)."""
    cand = np.asarray(candidates, dtype=np.int64)
    keys = key_bits if isinstance(key_bits, Fp8Keys) else np.asarray(key_bits)
    s = index_scores(q_bits, keys[cand], w)
    sel = top_k(s, np.ones(cand.size, dtype=bool), k)
    out = np.full(k, -1, dtype=np.int64)
    m = sel >= 0
    out[m] = cand[sel[m]]
    return out, s


def block_max_scores(q_bits, key_bits, length: int, w=None, block: int = BLOCK) -> np.ndarray:
    """Max-pooled block scores [ceil(L/block)]: the largest token score of each block."""
    keys = key_bits if isinstance(key_bits, Fp8Keys) else np.asarray(key_bits)
    ts = index_scores(q_bits, keys[:length], w)
    nb = (length + block - 1) // block
    out = np.full(nb, -np.inf, dtype=np.float32)
    for t in range(block):                       # each block's present tokens
        rows = np.arange(nb) * block + t
        present = rows < length
        out[present] = np.maximum(out[present], ts[rows[present]])
    return out


def full_indexer(q_bits, key_bits, length: int, w=None, hierarchical: bool = True,
                 pool_blocks: int = POOL_BLOCKS, block: int = BLOCK, k: int = TOP_K,
                 pooling: str = "mean"):
    """Full layer: returns (pool block ids [pool_blocks] ascending, -1 padded;
    selected positions [k] ascending, -1 padded; info dict).  pooling: the
    block score of the hierarchy, "mean" (block keys) or "max" (token scores)."""
    nb = (length + block - 1) // block
    info = {}
    if hierarchical and nb > pool_blocks:
        if pooling == "mean":
            kb = block_keys(key_bits, length, block)
            bs = index_scores(q_bits, kb, w)
        elif pooling == "max":
            bs = block_max_scores(q_bits, key_bits, length, w, block)
        else:
            raise ValueError(pooling)
        pool = top_k(bs, np.ones(nb, dtype=bool), pool_blocks)
        info["block_scores"] = bs
    else:
        pool = np.full(pool_blocks if hierarchical else nb, -1, dtype=np.int64)
        pool[:nb] = np.arange(nb)
    cand = pool_tokens(pool, length, block)
    idx, ts = select_tokens(q_bits, key_bits, cand, w, k)
    info["candidates"] = cand
    info["token_scores"] = ts
    return pool, idx, info


def reindex_indexer(q_bits, key_bits, length: int, pool: np.ndarray, w=None,
                    block: int = BLOCK, k: int = TOP_K):
    """Reindex layer: rank the Full layer's pool with this layer's own query."""
    cand = pool_tokens(pool, length, block)
    idx, ts = select_tokens(q_bits, key_bits, cand, w, k)
    return idx, {"candidates": cand, "token_scores": ts}


def flat_indexer(q_bits, key_bits, visible: int, w=None, k: int = TOP_K):
    """Encoder Full layer (no hierarchy): top-k over positions [0, visible)."""
    idx, ts = select_tokens(q_bits, key_bits, np.arange(visible), w, k)
    return idx, {"candidates": np.arange(visible), "token_scores": ts}
