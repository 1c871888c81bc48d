"""GPU parity of the indexer's top-k on score distributions chosen to stress the
selection rather than the scoring: every score equal (all-zero indexer keys),
heavy ties (keys drawn from five distinct vectors), and scores of both signs
(head weights of mixed sign).  Hierarchical (20,000 and 16,400 tokens) and flat
(3,000 tokens) sequences; the expected sets come from the oracle on the same
key bits."""
import numpy as np
import pytest
import torch

import workload as wl
from oracle import indexer as oidx
from tests import parity
from tests.gpu_util import small_workload

pytestmark = pytest.mark.gpu

LENGTHS = [20000, 20000, 3000, 16400, 20000, 20000]
CASES = ["zero", "few", "few", "random", "random", "two"]
HEAD_W = [[1.0, 1.0, 1.0, 1.0], [1.0, 1.0, 1.0, 1.0], [1.0, 0.5, 2.0, 1.0],
          [1.0, -1.0, 0.5, -2.0], [-1.0, -0.25, -3.0, -0.5], [1.0, 1.0, 1.0, 1.0]]


def _keys(case: str, seed: int, seq: int, L: int) -> np.ndarray:
    if case == "zero":
        return np.zeros((L, 64), dtype=np.uint16)
    if case in ("few", "two"):   # keys drawn from 5 (or 2: thousands of equal scores) vectors
        m = 5 if case == "few" else 2
        base = wl.idxk_rows(seed + 1, seq, 0, m)
        pick = (np.arange(L, dtype=np.uint64) * np.uint64(2654435761) >> np.uint64(7)) % np.uint64(m)
        return base[pick.astype(np.int64)]
    return wl.idxk_rows(seed, seq, 0, L)


@pytest.fixture(scope="module")
def crafted(csa2_lib):
    import workload
    workload.build_cuda()
    from fp4_kv_cache_decode_b200 import synthetic as syn
    w = small_workload(LENGTHS, seed=23, heads=16)
    cache = syn.new_cache(w)
    syn.fill_decode_cache(w, cache)
    keys = []
    for b, (L, case) in enumerate(zip(LENGTHS, CASES)):
        k = _keys(case, w.seed, b, L)
        keys.append(k)
        kv = torch.zeros((L, 512), dtype=torch.bfloat16, device="cuda")
        idxk = torch.from_numpy(k.view(np.int16)).cuda().view(torch.bfloat16)
        seqs = torch.full((L,), b, dtype=torch.int32, device="cuda")
        pos = torch.arange(L, dtype=torch.int32, device="cuda")
        csa2_lib.csa2_kv_quant_append(cache, kv, idxk, seqs, pos)
    torch.cuda.synchronize()
    assert csa2_lib.csa2_check_device_error(cache) == 0
    return csa2_lib, w, cache, keys


def test_topk_on_ties_equal_and_signed_scores(crafted):
    csa2, w, cache, keys = crafted
    B = len(LENGTHS)
    iq = np.stack([wl.idxq_rows(w.seed, 0, b) for b in range(B)])
    idxq = torch.from_numpy(iq.view(np.int16)).cuda().view(torch.bfloat16)
    hw = np.asarray(HEAD_W, dtype=np.float32)
    head_w = torch.from_numpy(hw).cuda()
    qs = torch.arange(B, dtype=torch.int32, device="cuda")
    ws = torch.empty(csa2.csa2_workspace_bytes(csa2.OP_INDEXER, B, 0, max(LENGTHS), True),
                     dtype=torch.uint8, device="cuda")
    iset = csa2.IndexSet(B)
    csa2.csa2_indexer_score_topk(cache, idxq, qs, csa2.FULL, 0, iset, ws, max(LENGTHS), head_w=head_w)
    assert csa2.csa2_check_device_error(cache) == 0
    gpool = iset.pool_blocks.cpu().numpy()
    gidx = iset.idx.cpu().numpy()
    for b, L in enumerate(LENGTHS):
        k = keys[b]
        pool, idx, _ = oidx.full_indexer(iq[b], k, L, w=hw[b])
        if CASES[b] == "zero":   # every score is 0: the lowest blocks and positions win
            nb = (L + 7) // 8
            assert np.array_equal(gpool[b][: min(nb, 2048)], np.arange(min(nb, 2048)))
            assert np.array_equal(gidx[b], np.arange(512))
        kb = oidx.block_keys(k, L)
        parity.check_index_set(gpool[b], pool, lambda x: oidx.index_scores(iq[b], kb[np.asarray(x)], hw[b]),
                               f"blocks {CASES[b]} L={L}")
        if np.array_equal(gpool[b], pool):
            parity.check_index_set(gidx[b], idx, lambda x: oidx.index_scores(iq[b], k[np.asarray(x)], hw[b]),
                                   f"tokens {CASES[b]} L={L}")
        else:   # an allowed block swap: the tokens must be a valid top-512 of the GPU's pool
            alt, _ = oidx.reindex_indexer(iq[b], k, L, gpool[b], w=hw[b])
            parity.check_index_set(gidx[b], alt, lambda x: oidx.index_scores(iq[b], k[np.asarray(x)], hw[b]),
                                   f"tokens* {CASES[b]} L={L}")

    # flat (encoder) selection over the same keys: every visible entry is a candidate
    # (above 16,384 entries the top-k streams the scores from the workspace)
    iset2 = csa2.IndexSet(B)
    ws2 = torch.empty(csa2.csa2_workspace_bytes(csa2.OP_INDEXER, B, 0, max(LENGTHS), False),
                      dtype=torch.uint8, device="cuda")
    csa2.csa2_indexer_score_topk(cache, idxq, qs, csa2.FULL, 0, iset2, ws2, max(LENGTHS), head_w=head_w,
                                 hierarchical=False)
    assert csa2.csa2_check_device_error(cache) == 0
    gflat = iset2.idx.cpu().numpy()
    for b, L in enumerate(LENGTHS):
        _, idx, _ = oidx.full_indexer(iq[b], keys[b], L, w=hw[b], hierarchical=False)
        parity.check_index_set(gflat[b], idx, lambda x: oidx.index_scores(iq[b], keys[b][np.asarray(x)], hw[b]),
                               f"flat {CASES[b]} L={L}")


def test_flat_query_groups_uniform_and_mixed(csa2_lib):
    """Flat (encoder) selection with 48 queries, scored in groups of 16 that share
    their keys when a group's queries are of one sequence: a group on one sequence
    with staggered visible lengths, a group interleaving five sequences (scored
    query by query), and a ragged last group crossing into another sequence."""
    import workload
    workload.build_cuda()
    from fp4_kv_cache_decode_b200 import synthetic as syn
    from workload import device as wdev
    csa2 = csa2_lib
    lens = [20000, 3000, 16400, 9000, 700]
    w = small_workload(lens, seed=29, heads=16)
    cache = syn.new_cache(w)
    syn.fill_decode_cache(w, cache)
    seqs = [0] * 16 + [r % 5 for r in range(16)] + [3] * 10 + [4] * 6
    vis = ([19000 + 7 * r for r in range(16)] + [lens[s] for s in seqs[16:32]] +
           [9000 - 13 * r for r in range(10)] + [700, 1, 0, 8, 9, 511])
    nq = len(seqs)
    q_seq = torch.tensor(seqs, dtype=torch.int32, device="cuda")
    q_vis = torch.tensor(vis, dtype=torch.int32, device="cuda")
    idxq = torch.cat([wdev.idxq_batch(w.seed, 9, r, 1) for r in range(nq)])
    iset = csa2.IndexSet(nq)
    ws = torch.empty(csa2.csa2_workspace_bytes(csa2.OP_INDEXER, nq, 0, max(vis), 0), dtype=torch.uint8,
                     device="cuda")
    csa2.csa2_indexer_score_topk(cache, idxq, q_seq, csa2.FULL, 0, iset, ws, max(vis), q_visible=q_vis,
                                 hierarchical=False)
    assert csa2.csa2_check_device_error(cache) == 0
    gidx = iset.idx.cpu().numpy()
    keys = {s: parity.OracleSeq(w, s, lens[s]).keys for s in set(seqs)}
    for r in range(nq):
        iq = wl.idxq_rows(w.seed, 9, r)
        k = keys[seqs[r]]
        _, idx, _ = oidx.full_indexer(iq, k, vis[r], hierarchical=False)
        parity.check_index_set(gidx[r], idx, lambda x: oidx.index_scores(iq, k[np.asarray(x)]),
                               f"query {r} seq {seqs[r]} v={vis[r]}")
