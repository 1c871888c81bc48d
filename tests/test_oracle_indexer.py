"""Pins for the indexer oracle: closed-form scores, fp64 library cross-check, block-key
identities, brute-force top-k and a brute-force hierarchy on shrunken sizes."""
import json
import os

import numpy as np
import pytest

from oracle import formats, indexer

CONST = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_constants.json")))


def _bf16(x):
    return formats.f32_to_bf16(np.asarray(x, dtype=np.float32))


def test_constants_from_pages():
    assert indexer.TOP_K == CONST["top_k"]["value"]
    assert indexer.POOL_BLOCKS == CONST["pool_blocks"]["value"]
    assert indexer.BLOCK == CONST["block_tokens"]["value"]
    assert indexer.POOL_BLOCKS * indexer.BLOCK == CONST["pool_positions"]["value"]


def test_scores_against_fp64_einsum():
    rng = np.random.default_rng(0)
    q = _bf16(rng.standard_normal((4, 64)))
    k = _bf16(rng.standard_normal((5000, 64)))
    w = np.array([1.0, 0.5, 2.0, 0.25], dtype=np.float32)
    ours = indexer.index_scores(q, k, w).astype(np.float64)
    qf, kf = formats.bf16_to_f64(q), formats.bf16_to_f64(k)
    dots = np.einsum("hd,nd->nh", qf, kf)
    ref = (np.maximum(dots, 0.0) * w.astype(np.float64)).sum(axis=1)
    bound = 1e-5 * (np.abs(np.einsum("hd,nd->nh", np.abs(qf), np.abs(kf))) * w).sum(axis=1)
    assert np.all(np.abs(ours - ref) <= bound + 1e-30)
    # a head whose dot products are all negative contributes nothing
    assert np.sum(ref == 0.0) == np.sum(ours == 0.0)


def test_scores_closed_forms():
    rng = np.random.default_rng(1)
    k = _bf16(rng.standard_normal((300, 64)))
    kf = formats.bf16_to_f32(k)
    for d in (0, 17, 63):
        q = np.zeros((4, 64), dtype=np.uint16)
        q[0, d] = 0x3F80                                  # 1.0 in head 0 only
        s = indexer.index_scores(q, k)
        np.testing.assert_array_equal(s, np.maximum(kf[:, d], 0.0))
        q2 = q.copy()
        q2[0, d] = 0xBF80                                 # -1.0
        np.testing.assert_array_equal(indexer.index_scores(q2, k), np.maximum(-kf[:, d], 0.0))
        q3 = np.zeros((4, 64), dtype=np.uint16)
        q3[2, d] = 0x3F80
        w = np.array([0, 0, 3.0, 0], dtype=np.float32)
        np.testing.assert_array_equal(indexer.index_scores(q3, k, w),
                                      (np.float32(3.0) * np.maximum(kf[:, d], 0)).astype(np.float32))


def test_block_key_identities():
    rng = np.random.default_rng(2)
    k = _bf16(rng.standard_normal((40, 64)))
    # a single present token: the key is that token
    np.testing.assert_array_equal(indexer.block_keys(k, 1), k[:1])
    # eight identical tokens: the mean is the token itself
    same = np.repeat(k[:1], 8, axis=0)
    np.testing.assert_array_equal(indexer.block_keys(same, 8), k[:1])
    # partial last block of three tokens with values 1, 2, 3 -> 2
    t = np.zeros((11, 64), dtype=np.uint16)
    t[8:11] = _bf16(np.array([1.0, 2.0, 3.0]))[:, None]
    kb = indexer.block_keys(t, 11)
    assert kb.shape == (2, 64)
    np.testing.assert_array_equal(formats.bf16_to_f64(kb[1]), 2.0)
    # sign symmetry
    np.testing.assert_array_equal(indexer.block_keys(k ^ np.uint16(0x8000), 40),
                                  indexer.block_keys(k, 40) ^ np.uint16(0x8000))
    # means of small integers are exact
    ints = _bf16(np.arange(16, dtype=np.float32)[:, None] * np.ones((1, 64)))
    kb = formats.bf16_to_f64(indexer.block_keys(ints, 16))
    np.testing.assert_array_equal(kb[:, 0], [3.5, 11.5])


def _brute_topk(scores, valid, k):
    items = [(-float(scores[i]), i) for i in range(len(scores)) if valid[i]]
    items.sort()
    chosen = sorted(i for _, i in items[:k])
    return chosen + [-1] * (k - len(chosen))


def test_topk_against_brute_force_loops():
    rng = np.random.default_rng(3)
    for trial in range(200):
        n = int(rng.integers(0, 60))
        k = int(rng.integers(1, 20))
        s = rng.integers(-3, 4, n).astype(np.float32) * np.float32(0.5)   # many ties
        valid = rng.random(n) < 0.8
        assert list(indexer.top_k(s, valid, k)) == _brute_topk(s, valid, k)


def test_topk_tie_break_and_padding():
    s = np.full(2000, 7.0, dtype=np.float32)
    np.testing.assert_array_equal(indexer.top_k(s, np.ones(2000, bool), 512), np.arange(512))
    out = indexer.top_k(np.arange(10, dtype=np.float32), np.ones(10, bool), 16)
    assert list(out[:10]) == list(range(10)) and np.all(out[10:] == -1)
    v = np.ones(10, bool)
    v[9] = False
    assert 9 not in indexer.top_k(np.arange(10, dtype=np.float32), v, 3)


def test_hierarchy_equals_flat_up_to_16384_tokens():
    rng = np.random.default_rng(4)
    q = _bf16(rng.standard_normal((4, 64)))
    for L in (1, 7, 600, 4096, 16384):
        k = _bf16(rng.standard_normal((L, 64)))
        pool, idx, _ = indexer.full_indexer(q, k, L)
        flat, _ = indexer.flat_indexer(q, k, L)
        np.testing.assert_array_equal(idx, flat)
        nb = (L + 7) // 8
        np.testing.assert_array_equal(pool[:nb], np.arange(nb))
        assert np.all(pool[nb:] == -1)


def test_hierarchy_brute_force_on_shrunken_sizes():
    rng = np.random.default_rng(5)
    P, B, K = 4, 8, 8                  # pool of 4 blocks of 8, select 8
    for L in (33, 60, 100, 161):
        q = _bf16(rng.standard_normal((4, 64)))
        k = _bf16(rng.standard_normal((L, 64)))
        pool, idx, _ = indexer.full_indexer(q, k, L, pool_blocks=P, block=B, k=K)
        qf = formats.bf16_to_f32(q)
        kf = formats.bf16_to_f32(k)

        def score(vec):
            tot = np.float32(0)
            for h in range(4):
                dot = np.float32(0)
                for d in range(64):
                    dot = np.float32(dot + np.float32(qf[h, d] * vec[d]))
                tot = np.float32(tot + max(dot, np.float32(0)))
            return tot

        nb = (L + B - 1) // B
        keys = []
        for j in range(nb):
            acc = np.zeros(64, dtype=np.float32)
            n = 0
            for t in range(j * B, min(j * B + B, L)):
                acc = (acc + kf[t]).astype(np.float32)
                n += 1
            keys.append(formats.bf16_to_f32(formats.f32_to_bf16(acc / np.float32(n))))
        blocks = sorted(range(nb), key=lambda j: (-float(score(keys[j])), j))[:P]
        assert list(pool) == sorted(blocks)
        cand = [t for j in sorted(blocks) for t in range(j * B, min(j * B + B, L))]
        toks = sorted(cand, key=lambda t: (-float(score(kf[t])), t))[:K]
        assert list(idx[:len(toks)]) == sorted(toks)


def test_reindex_with_full_query_reproduces_full_set():
    rng = np.random.default_rng(6)
    L = 20000                             # > 16,384: hierarchical
    q = _bf16(rng.standard_normal((4, 64)))
    k = _bf16(rng.standard_normal((L, 64)))
    pool, idx, _ = indexer.full_indexer(q, k, L)
    assert (pool >= 0).sum() == 2048 and np.all(np.diff(pool) > 0)
    again, _ = indexer.reindex_indexer(q, k, L, pool)
    np.testing.assert_array_equal(again, idx)
    q2 = _bf16(rng.standard_normal((4, 64)))
    other, info = indexer.reindex_indexer(q2, k, L, pool)
    assert set(other.tolist()) <= set(info["candidates"].tolist())
    assert not np.array_equal(other, idx)


def _keys_of(kind, rng, L):
    if kind == "random":
        return _bf16(rng.standard_normal((L, 64)))
    if kind == "zero":
        return np.zeros((L, 64), np.uint16)
    base = _bf16(rng.standard_normal((5, 64)))          # few distinct keys: heavy ties
    return base[rng.integers(0, 5, L)]


@pytest.mark.parametrize("kind", ["random", "zero", "few"])
@pytest.mark.parametrize("L", [20000, 16391, 40960])
def test_max_pooled_hierarchy_is_lossless(kind, L):
    """With max-pooled block scores the pool's top-512 equals the flat top-512
    (the block-beating argument), ties included."""
    rng = np.random.default_rng(L)
    k = _keys_of(kind, rng, L)
    q = _bf16(rng.standard_normal((4, 64)))
    w = np.array([1.0, -0.5, 2.0, 0.25], np.float32)
    pool, idx, info = indexer.full_indexer(q, k, L, w, pooling="max")
    _, flat, _ = indexer.full_indexer(q, k, L, w, hierarchical=False)
    np.testing.assert_array_equal(idx, flat)
    assert pool[pool >= 0].size == 2048 and np.all(np.diff(pool[pool >= 0]) > 0)
    # the pool is the top-2048 of the block maxima, computed here by brute force
    ts = indexer.index_scores(q, k, w).astype(np.float64)
    nb = (L + 7) // 8
    bmax = np.array([ts[8 * b: min(8 * b + 8, L)].max() for b in range(nb)])
    order = sorted(range(nb), key=lambda b: (-bmax[b], b))[:2048]
    np.testing.assert_array_equal(pool[pool >= 0], np.sort(order))


def test_max_pooled_hierarchy_brute_force_on_shrunken_sizes():
    """Pools of 3 blocks of 4 tokens and k = 2: every pool and selection by loops."""
    rng = np.random.default_rng(9)
    for trial in range(40):
        L = int(rng.integers(13, 40))
        k = _bf16(rng.integers(-3, 4, (L, 64)).astype(np.float32))   # small integers: many ties
        q = _bf16(rng.integers(-2, 3, (4, 64)).astype(np.float32))
        pool, idx, _ = indexer.full_indexer(q, k, L, pool_blocks=3, block=4, k=2, pooling="max")
        ts = [float(indexer.index_scores(q, k[i:i + 1])[0]) for i in range(L)]
        blocks = [(-max(ts[4 * b: min(4 * b + 4, L)]), b) for b in range((L + 3) // 4)]
        want_pool = sorted(b for _, b in sorted(blocks)[:3])
        assert list(pool[pool >= 0]) == want_pool
        cand = [t for b in want_pool for t in range(4 * b, min(4 * b + 4, L))]
        want = sorted(sorted(cand, key=lambda t: (-ts[t], t))[:2])
        assert list(idx[idx >= 0]) == want
        flat = sorted(sorted(range(L), key=lambda t: (-ts[t], t))[:2])
        assert want == flat


def test_pool_tokens_expansion_and_clipping():
    """Pool blocks expand to their 8 positions each, ascending in pool order,
    -1 entries dropped, positions at or past the context length removed."""
    got = indexer.pool_tokens(np.array([0, 3, 5, -1, -1]), length=44)
    want = list(range(0, 8)) + list(range(24, 32)) + list(range(40, 44))
    np.testing.assert_array_equal(got, want)
    assert indexer.pool_tokens(np.array([-1, -1]), length=100).size == 0
    # a block wholly past the end contributes nothing
    np.testing.assert_array_equal(indexer.pool_tokens(np.array([1, 9]), length=16), np.arange(8, 16))


def test_select_tokens_brute_force():
    """select_tokens = the k best candidates by (score desc, position asc), as
    positions in ascending order, padded with -1; scores returned per candidate."""
    rng = np.random.default_rng(7)
    k = _bf16(rng.standard_normal((200, 64)))
    q = _bf16(rng.standard_normal((4, 64)))
    # ties: copy a few keys so that equal scores occur at different positions
    k[50] = k[10]
    k[120] = k[10]
    cand = np.array(sorted(rng.choice(200, size=60, replace=False).tolist() + [10, 50, 120]))
    cand = np.unique(cand)
    for kk in (5, 17, len(cand), len(cand) + 9):
        sel, s = indexer.select_tokens(q, k, cand, k=kk)
        kf = formats.bf16_to_f32(k)
        qf = formats.bf16_to_f32(q)
        scores = {}
        for p in cand:                               # brute force, same fp32 order as the oracle
            tot = np.float32(0)
            for h in range(4):
                dot = np.float32(0)
                for d in range(64):
                    dot = np.float32(dot + np.float32(qf[h, d] * kf[p, d]))
                tot = np.float32(tot + max(dot, np.float32(0)))
            scores[int(p)] = tot
        np.testing.assert_array_equal(s, np.array([scores[int(p)] for p in cand], dtype=np.float32))
        best = sorted(scores, key=lambda p: (-scores[p], p))[:kk]
        want = sorted(best) + [-1] * (kk - len(best))
        np.testing.assert_array_equal(sel, want)


def test_block_max_scores_brute_force():
    """Each block's max-pooled score is the largest score among its present
    tokens; a ragged last block uses only the tokens below the length."""
    rng = np.random.default_rng(8)
    k = _bf16(rng.standard_normal((77, 64)))
    q = _bf16(rng.standard_normal((4, 64)))
    for L in (1, 8, 9, 77):
        ts = indexer.index_scores(q, k[:L])
        got = indexer.block_max_scores(q, k, L)
        want = [max(ts[8 * b: min(8 * b + 8, L)]) for b in range((L + 7) // 8)]
        np.testing.assert_array_equal(got, np.array(want, dtype=np.float32))
