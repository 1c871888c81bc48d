"""GPU parity of the indexer (flat and hierarchical Full, Reindex) and of sparse
attention (Full / Reindex / Reuse) on a ragged batch that spans the edge cases:
empty, single-token, block and window boundaries, the flat/hierarchical switch at
16,384 tokens and ragged tails."""
import numpy as np
import pytest
import torch

import workload as wl
from oracle import indexer as oidx
from tests import parity
from tests.gpu_util import bits, small_workload

pytestmark = pytest.mark.gpu

LENGTHS = [0, 1, 7, 8, 9, 127, 128, 129, 511, 512, 513, 640, 4096, 16384, 16385, 20000, 33333]


@pytest.fixture(scope="module")
def ragged(csa2_lib):
    import workload
    workload.build_cuda()
    from fp4_kv_cache_decode_b200 import synthetic as syn
    w = small_workload(LENGTHS, seed=11, heads=64)
    cache = syn.new_cache(w)
    syn.fill_decode_cache(w, cache)
    assert csa2_lib.csa2_check_device_error(cache) == 0
    oseqs = [parity.OracleSeq(w, b, L) for b, L in enumerate(LENGTHS)]
    return csa2_lib, syn, w, cache, oseqs


def _run_indexer(csa2, cache, w, mode, layer, iset, nq, max_vis, hierarchical=True):
    from workload import device as wdev
    idxq = wdev.idxq_batch(w.seed, layer, 0, nq)
    qs = torch.arange(nq, dtype=torch.int32, device="cuda")
    ws = torch.empty(csa2.csa2_workspace_bytes(csa2.OP_INDEXER, nq, 0, max_vis, hierarchical),
                     dtype=torch.uint8, device="cuda")
    csa2.csa2_indexer_score_topk(cache, idxq, qs, mode, layer, iset, ws, max_vis, hierarchical=hierarchical)
    return qs


def test_full_and_reindex_sets(ragged):
    csa2, syn, w, cache, oseqs = ragged
    B = len(LENGTHS)
    iset = csa2.IndexSet(B)
    _run_indexer(csa2, cache, w, csa2.FULL, 0, iset, B, max(LENGTHS))
    assert csa2.csa2_check_device_error(cache) == 0
    gpool = iset.pool_blocks.cpu().numpy()
    gidx = iset.idx.cpu().numpy()
    swaps = 0
    same_pool = {}
    for b, L in enumerate(LENGTHS):
        o = oseqs[b]
        iq = wl.idxq_rows(w.seed, 0, b)
        pool, idx, info = oidx.full_indexer(iq, o.keys, L)
        nb = (L + 7) // 8
        if nb <= 2048:
            np.testing.assert_array_equal(gpool[b], pool, err_msg=f"flat pool, L={L}")
        else:
            swaps += parity.check_index_set(gpool[b], pool, parity.block_scorer(o, iq, L), f"blocks L={L}")
        same_pool[b] = np.array_equal(gpool[b], pool)
        if same_pool[b]:
            swaps += parity.check_index_set(gidx[b], idx, parity.token_scorer(o, iq), f"tokens L={L}")
        else:   # an allowed block swap: the GPU's tokens must be a valid top-512 of the GPU's pool
            alt, _ = oidx.reindex_indexer(iq, o.keys, L, gpool[b])
            swaps += parity.check_index_set(gidx[b], alt, parity.token_scorer(o, iq), f"tokens* L={L}")
    # Reindex (layer 4) ranks the same pools with its own query
    _run_indexer(csa2, cache, w, csa2.REINDEX, 4, iset, B, max(LENGTHS))
    gri = iset.idx.cpu().numpy()
    for b, L in enumerate(LENGTHS):
        o = oseqs[b]
        iq = wl.idxq_rows(w.seed, 4, b)
        want, _ = oidx.reindex_indexer(iq, o.keys, L, gpool[b] if not same_pool[b] else
                                       oidx.full_indexer(wl.idxq_rows(w.seed, 0, b), o.keys, L)[0])
        swaps += parity.check_index_set(gri[b], want, parity.token_scorer(o, iq), f"reindex L={L}")
    print(f"allowed boundary swaps: {swaps}")


@pytest.mark.parametrize("heads", [64, 48, 32, 16])
def test_attention_on_oracle_sets(ragged, heads):
    """Attention alone: the oracle's index sets are loaded into the GPU set, so any
    difference is the attention kernel's."""
    csa2, syn, w, cache, oseqs = ragged
    from workload import device as wdev
    B = len(LENGTHS)
    iset = csa2.IndexSet(B)
    qs = _run_indexer(csa2, cache, w, csa2.FULL, 0, iset, B, max(LENGTHS))
    want_idx = np.full((B, 512), -1, dtype=np.int32)
    for b, L in enumerate(LENGTHS):
        _, idx, _ = oidx.full_indexer(wl.idxq_rows(w.seed, 0, b), oseqs[b].keys, L)
        want_idx[b] = idx
    iset.idx.copy_(torch.from_numpy(want_idx))
    ws = torch.empty(csa2.csa2_workspace_bytes(csa2.OP_ATTENTION, B, heads), dtype=torch.uint8, device="cuda")
    for layer, mode in ((0, csa2.FULL), (1, csa2.REUSE), (3, csa2.REUSE)):
        q = wdev.q_batch(w.seed, layer, 0, B, heads)
        out = torch.empty((B, heads, 512), dtype=torch.bfloat16, device="cuda")
        csa2.csa2_sparse_attn(cache, q, qs, mode, layer, iset, out, ws, 1.0)
        assert csa2.csa2_check_device_error(cache) == 0
        g = bits(out)
        for b, L in enumerate(LENGTHS):
            ref = parity.oracle_attention(oseqs[b], want_idx[b], wl.q_rows(w.seed, layer, b, heads), L)
            err, bound = parity.attention_error(g[b], ref)
            assert err <= bound, f"L={L} layer={layer}: err {err} > {bound}"
            if L == 0:
                assert np.all(g[b] == 0)


@pytest.mark.parametrize("nq,heads", [(1, 64), (2, 64), (3, 48), (2, 32), (5, 64), (1, 16)])
def test_attention_small_batches_split_heads(ragged, nq, heads):
    """Small batches split each query's heads over several clusters (4 groups of 16 at
    one or two queries of 64 heads, 3 of 16 at 48 heads, 2 of 16 or 32 at five queries
    or 32 heads) beside the row ranges: Full and Reuse outputs match the oracle on its
    own sets."""
    csa2, syn, w, cache, oseqs = ragged
    from workload import device as wdev
    seqs = [16, 15, 14, 13, 12][:nq]      # 33,333 / 20,000 / 16,385 / 16,384 / 4,096 tokens
    qs = torch.tensor(seqs, dtype=torch.int32, device="cuda")
    iset = csa2.IndexSet(nq)
    idxq = torch.cat([wdev.idxq_batch(w.seed, 0, s, 1) for s in seqs])
    ws_i = torch.empty(csa2.csa2_workspace_bytes(csa2.OP_INDEXER, nq, 0, 33333, True), dtype=torch.uint8,
                       device="cuda")
    csa2.csa2_indexer_score_topk(cache, idxq, qs, csa2.FULL, 0, iset, ws_i, 33333)
    want = np.full((nq, 512), -1, dtype=np.int32)
    for j, s in enumerate(seqs):
        _, idx, _ = oidx.full_indexer(wl.idxq_rows(w.seed, 0, s), oseqs[s].keys, LENGTHS[s])
        want[j] = idx
    iset.idx.copy_(torch.from_numpy(want))
    ws = torch.empty(csa2.csa2_workspace_bytes(csa2.OP_ATTENTION, nq, heads), dtype=torch.uint8, device="cuda")
    for layer, mode in ((0, csa2.FULL), (2, csa2.REUSE)):
        q = torch.cat([wdev.q_batch(w.seed, layer, s, 1, heads) for s in seqs])
        out = torch.empty((nq, heads, 512), dtype=torch.bfloat16, device="cuda")
        csa2.csa2_sparse_attn(cache, q, qs, mode, layer, iset, out, ws, 1.0)
        assert csa2.csa2_check_device_error(cache) == 0
        g = bits(out)
        for j, s in enumerate(seqs):
            ref = parity.oracle_attention(oseqs[s], want[j], wl.q_rows(w.seed, layer, s, heads), LENGTHS[s])
            err, bound = parity.attention_error(g[j], ref)
            assert err <= bound, f"nq={nq} H={heads} seq {s} layer={layer}: err {err} > {bound}"


def test_reuse_with_full_query_reproduces_full_output(ragged):
    csa2, syn, w, cache, oseqs = ragged
    from workload import device as wdev
    B = len(LENGTHS)
    iset = csa2.IndexSet(B)
    qs = _run_indexer(csa2, cache, w, csa2.FULL, 0, iset, B, max(LENGTHS))
    ws = torch.empty(csa2.csa2_workspace_bytes(csa2.OP_ATTENTION, B, 64), dtype=torch.uint8, device="cuda")
    q = wdev.q_batch(w.seed, 0, 0, B, 64)
    o1 = torch.empty((B, 64, 512), dtype=torch.bfloat16, device="cuda")
    o2 = torch.empty_like(o1)
    csa2.csa2_sparse_attn(cache, q, qs, csa2.FULL, 0, iset, o1, ws)
    csa2.csa2_sparse_attn(cache, q, qs, csa2.REUSE, 2, iset, o2, ws)
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))


def test_mode_errors_through_binding(ragged):
    csa2, syn, w, cache, oseqs = ragged
    iset = csa2.IndexSet(2)
    qs = torch.arange(2, dtype=torch.int32, device="cuda")
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    q = torch.zeros((2, 64, 512), dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q)
    with pytest.raises(csa2.Csa2Error) as e:
        csa2.csa2_sparse_attn(cache, q, qs, csa2.REUSE, 1, iset, out, ws)
    assert e.value.status == 4


def test_row_cache_changes_no_result(ragged):
    """Reuse layers read the rows the Full attention call resolved (row cache) or
    resolve them again (no cache): the outputs are the same bits either way, and an
    indexer call on the set discards the cached rows."""
    csa2, syn, w, cache, oseqs = ragged
    from workload import device as wdev
    B = len(LENGTHS)
    sets = {"cached": csa2.IndexSet(B), "plain": csa2.IndexSet(B, row_cache=False)}
    ws = torch.empty(csa2.csa2_workspace_bytes(csa2.OP_ATTENTION, B, 64), dtype=torch.uint8, device="cuda")
    outs = {}
    for name, s in sets.items():
        qs = _run_indexer(csa2, cache, w, csa2.FULL, 0, s, B, max(LENGTHS))
        outs[name] = []
        for layer, mode in ((0, csa2.FULL), (2, csa2.REUSE), (3, csa2.REUSE)):
            o = torch.empty((B, 64, 512), dtype=torch.bfloat16, device="cuda")
            csa2.csa2_sparse_attn(cache, wdev.q_batch(w.seed, layer, 0, B, 64), qs, mode, layer, s, o, ws)
            outs[name].append(o)
        assert csa2.csa2_check_device_error(cache) == 0
    for a, b in zip(outs["cached"], outs["plain"]):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    st = sets["cached"].struct
    assert st.rows_layer == 0 and st.rows_nq == B and st.rows_split in (1, 2, 4, 8)
    assert sets["plain"].struct.rows_layer == -1
    _run_indexer(csa2, cache, w, csa2.REINDEX, 4, sets["cached"], B, max(LENGTHS))
    assert sets["cached"].struct.rows_layer == -1
