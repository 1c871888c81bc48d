"""GPU parity of the max-pooled hierarchy (block score = the largest score of the
block's present tokens): the pool against the oracle's top-2048 block maxima, the
tokens against the oracle's pool-then-select result (which equals the flat top-512),
the Reindex layer that ranks that pool with its own query, with bf16 and FP8 keys,
and the all-equal case where ties decide everything."""
import numpy as np
import pytest
import torch

import workload as wl
from oracle import idxk_fp8 as ofp8
from oracle import indexer as oidx
from tests import parity
from tests.gpu_util import small_workload

pytestmark = pytest.mark.gpu

LENGTHS = [1, 9, 4096, 16384, 16391, 20000, 33333, 65536]


def _run(csa2, cache, w, mode, layer, iset, hierarchical):
    from workload import device as wdev
    B = len(LENGTHS)
    qs = torch.arange(B, dtype=torch.int32, device="cuda")
    ws = torch.empty(csa2.csa2_workspace_bytes(csa2.OP_INDEXER, B, 0, max(LENGTHS),
                                               hierarchical if mode == csa2.FULL else csa2.HIER_MEAN),
                     dtype=torch.uint8, device="cuda")
    csa2.csa2_indexer_score_topk(cache, wdev.idxq_batch(w.seed, layer, 0, B), qs, mode, layer, iset, ws,
                                 max(LENGTHS), hierarchical=hierarchical)
    assert csa2.csa2_check_device_error(cache) == 0


@pytest.mark.parametrize("fmt", ["bf16", "fp8"])
def test_max_pooled_full_and_reindex(csa2_lib, fmt):
    import workload
    workload.build_cuda()
    from fp4_kv_cache_decode_b200 import synthetic as syn
    csa2 = csa2_lib
    w = small_workload(LENGTHS, seed=51 if fmt == "bf16" else 52, heads=16)
    cache = syn.new_cache(w, idxk_format=csa2.IDXK_FP8 if fmt == "fp8" else csa2.IDXK_BF16)
    syn.fill_decode_cache(w, cache)
    keys = []
    for b, L in enumerate(LENGTHS):
        k = parity.OracleSeq(w, b, L).keys
        keys.append(ofp8.Fp8Keys.from_bf16(k) if fmt == "fp8" else k)
    B = len(LENGTHS)
    iset = csa2.IndexSet(B)
    _run(csa2, cache, w, csa2.FULL, 0, iset, csa2.HIER_MAX)
    assert iset.struct.pool_layer == 0
    gpool = iset.pool_blocks.cpu().numpy()
    gidx = iset.idx.cpu().numpy()
    swaps = 0
    for b, L in enumerate(LENGTHS):
        iq = wl.idxq_rows(w.seed, 0, b)
        pool, idx, _ = oidx.full_indexer(iq, keys[b], L, pooling="max")
        bmax = oidx.block_max_scores(iq, keys[b], L)
        swaps += parity.check_index_set(gpool[b], pool, lambda x: bmax[np.asarray(x)], f"pool L={L}")
        swaps += parity.check_index_set(gidx[b], idx, lambda x: oidx.index_scores(iq, keys[b][np.asarray(x)]),
                                        f"tokens L={L}")
        # the selected tokens lie in the GPU's pool
        sel = gidx[b][gidx[b] >= 0]
        assert np.all(np.isin(sel // 8, gpool[b]))
    _run(csa2, cache, w, csa2.REINDEX, 3, iset, csa2.HIER_MEAN)
    gri = iset.idx.cpu().numpy()
    for b, L in enumerate(LENGTHS):
        iq = wl.idxq_rows(w.seed, 3, b)
        want, _ = oidx.reindex_indexer(iq, keys[b], L, gpool[b])
        swaps += parity.check_index_set(gri[b], want, lambda x: oidx.index_scores(iq, keys[b][np.asarray(x)]),
                                        f"reindex L={L}")
    print(f"allowed boundary swaps: {swaps}")


def test_max_pooled_ties(csa2_lib):
    """All-zero keys: every score is 0, so the pool is the first 2,048 blocks (or
    all of them) and the tokens are positions 0..511."""
    import workload
    workload.build_cuda()
    from fp4_kv_cache_decode_b200 import synthetic as syn
    csa2 = csa2_lib
    w = small_workload(LENGTHS, seed=53, heads=16)
    cache = syn.new_cache(w)
    for b, L in enumerate(LENGTHS):
        z = torch.zeros((L, 512), dtype=torch.bfloat16, device="cuda")
        zk = torch.zeros((L, 64), dtype=torch.bfloat16, device="cuda")
        csa2.csa2_kv_quant_append(cache, z, zk, torch.full((L,), b, dtype=torch.int32, device="cuda"),
                                  torch.arange(L, dtype=torch.int32, device="cuda"))
    iset = csa2.IndexSet(len(LENGTHS))
    _run(csa2, cache, w, csa2.FULL, 0, iset, csa2.HIER_MAX)
    gpool = iset.pool_blocks.cpu().numpy()
    gidx = iset.idx.cpu().numpy()
    for b, L in enumerate(LENGTHS):
        nb = (L + 7) // 8
        n = min(nb, 2048)
        np.testing.assert_array_equal(gpool[b][:n], np.arange(n))
        assert np.all(gpool[b][n:] == -1)
        m = min(L, 512)
        np.testing.assert_array_equal(gidx[b][:m], np.arange(m))
        assert np.all(gidx[b][m:] == -1)
