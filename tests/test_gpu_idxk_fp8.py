"""GPU parity of the FP8 indexer-key format (64 E4M3 codes + one fp32 scale per
token): the stored codes, scales and block keys are byte-exact with the oracle at
compression ratios 1 and 2; Full (hierarchical and flat) and Reindex index sets
match the oracle's FP8 scores under the index-set rule; replay restores poisoned
keys; a whole decode step runs on an FP8-key cache."""
import numpy as np
import pytest
import torch

import workload as wl
from oracle import codec as ocodec
from oracle import idxk_fp8 as ofp8
from oracle import indexer as oidx
from oracle import modes as omodes
from tests import parity
from tests.gpu_util import bits, cache_block_keys, cache_keys_fp8, small_workload

pytestmark = pytest.mark.gpu

LENGTHS = [1, 7, 8, 9, 129, 640, 4096, 16384, 16385, 20000, 33333]


@pytest.fixture(scope="module")
def fp8(csa2_lib):
    import workload
    workload.build_cuda()
    from fp4_kv_cache_decode_b200 import synthetic as syn
    w = small_workload(LENGTHS, seed=41, heads=16)
    cache = syn.new_cache(w, idxk_format=csa2_lib.IDXK_FP8)
    syn.fill_decode_cache(w, cache)
    assert csa2_lib.csa2_check_device_error(cache) == 0
    keys = [ofp8.Fp8Keys.from_bf16(parity.OracleSeq(w, b, L).keys) for b, L in enumerate(LENGTHS)]
    return csa2_lib, syn, w, cache, keys


def _fp8_scorer(keys, iq):
    return lambda p: oidx.index_scores(iq, keys[np.asarray(p, dtype=np.int64)])


def test_append_stores_exact_codes_scales_and_block_keys(fp8):
    csa2, syn, w, cache, keys = fp8
    for b, L in enumerate(LENGTHS):
        codes, scales = cache_keys_fp8(cache, b, np.arange(L))
        np.testing.assert_array_equal(codes, keys[b].codes, err_msg=f"codes L={L}")
        np.testing.assert_array_equal(scales.view(np.uint32), keys[b].scales.view(np.uint32),
                                      err_msg=f"scales L={L}")
        np.testing.assert_array_equal(cache_block_keys(cache, b, np.arange((L + 7) // 8)),
                                      oidx.block_keys(keys[b], L), err_msg=f"block keys L={L}")


def test_ratio2_append_quantises_the_pair_mean_key(csa2_lib):
    import workload
    workload.build_cuda()
    from fp4_kv_cache_decode_b200 import synthetic as syn
    lens = [300, 64, 1]
    w = small_workload(lens, seed=42)
    cache = syn.new_cache(w, idxk_format=csa2_lib.IDXK_FP8)
    for b, L in enumerate(lens):
        raw = wl.kv_rows(w.seed, b, 0, 2 * L)
        rawk = wl.idxk_rows(w.seed, b, 0, 2 * L)
        dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()
        csa2_lib.csa2_kv_quant_append(cache, dev(raw), dev(rawk), torch.full((L,), b, dtype=torch.int32,
                                      device="cuda"), torch.arange(L, dtype=torch.int32, device="cuda"), 2)
        want = ofp8.Fp8Keys.from_bf16(ocodec.idxk_entries(rawk, 2))
        codes, scales = cache_keys_fp8(cache, b, np.arange(L))
        np.testing.assert_array_equal(codes, want.codes)
        np.testing.assert_array_equal(scales, want.scales)
        np.testing.assert_array_equal(cache_block_keys(cache, b, np.arange((L + 7) // 8)),
                                      oidx.block_keys(want, L))
    assert csa2_lib.csa2_check_device_error(cache) == 0


def _indexer(csa2, cache, w, mode, layer, iset, hierarchical=True):
    from workload import device as wdev
    B = len(LENGTHS)
    qs = torch.arange(B, dtype=torch.int32, device="cuda")
    ws = torch.empty(csa2.csa2_workspace_bytes(csa2.OP_INDEXER, B, 0, max(LENGTHS), hierarchical),
                     dtype=torch.uint8, device="cuda")
    csa2.csa2_indexer_score_topk(cache, wdev.idxq_batch(w.seed, layer, 0, B), qs, mode, layer, iset, ws,
                                 max(LENGTHS), hierarchical=hierarchical)
    assert csa2.csa2_check_device_error(cache) == 0
    return qs


def test_full_reindex_and_flat_sets_on_fp8_keys(fp8):
    csa2, syn, w, cache, keys = fp8
    B = len(LENGTHS)
    iset = csa2.IndexSet(B)
    _indexer(csa2, cache, w, csa2.FULL, 0, iset)
    gpool = iset.pool_blocks.cpu().numpy()
    gidx = iset.idx.cpu().numpy()
    swaps = 0
    pools = {}
    for b, L in enumerate(LENGTHS):
        iq = wl.idxq_rows(w.seed, 0, b)
        pool, idx, _ = oidx.full_indexer(iq, keys[b], L)
        kb = oidx.block_keys(keys[b], L)
        swaps += parity.check_index_set(gpool[b], pool, lambda x: oidx.index_scores(iq, kb[np.asarray(x)]),
                                        f"blocks L={L}")
        pools[b] = gpool[b]
        want = idx if np.array_equal(gpool[b], pool) else oidx.reindex_indexer(iq, keys[b], L, gpool[b])[0]
        swaps += parity.check_index_set(gidx[b], want, _fp8_scorer(keys[b], iq), f"tokens L={L}")
    _indexer(csa2, cache, w, csa2.REINDEX, 4, iset)
    gri = iset.idx.cpu().numpy()
    for b, L in enumerate(LENGTHS):
        iq = wl.idxq_rows(w.seed, 4, b)
        want, _ = oidx.reindex_indexer(iq, keys[b], L, pools[b])
        swaps += parity.check_index_set(gri[b], want, _fp8_scorer(keys[b], iq), f"reindex L={L}")
    flat = csa2.IndexSet(B)
    _indexer(csa2, cache, w, csa2.FULL, 6, flat, hierarchical=False)
    gflat = flat.idx.cpu().numpy()
    for b, L in enumerate(LENGTHS):
        iq = wl.idxq_rows(w.seed, 6, b)
        _, idx, _ = oidx.full_indexer(iq, keys[b], L, hierarchical=False)
        swaps += parity.check_index_set(gflat[b], idx, _fp8_scorer(keys[b], iq), f"flat L={L}")
    print(f"allowed boundary swaps: {swaps}")


def test_replay_restores_poisoned_fp8_keys(csa2_lib):
    import workload
    workload.build_cuda()
    from fp4_kv_cache_decode_b200 import synthetic as syn
    lens = [300, 50, 1000, 129]
    w = small_workload(lens, seed=43)
    miss = np.array([True, True, False, True])
    cache = syn.new_cache(w, idxk_format=csa2_lib.IDXK_FP8)
    syn.fill_decode_cache(w, cache)
    pt = cache.page_table.cpu().numpy()
    for b, L in enumerate(lens):
        for p in range(max(0, L - 128), L):
            pg = int(pt[b, p >> 6])
            cache.idxk_pool[pg * 4352 + (p & 63) * 64: pg * 4352 + (p & 63) * 64 + 64] = 0x55
            cache.idxk_pool[pg * 4352 + 4096 + (p & 63) * 4: pg * 4352 + 4096 + (p & 63) * 4 + 4] = 0x7F
    kv_last = torch.zeros((len(lens), 128, 512), dtype=torch.int16, device="cuda")
    k_last = torch.zeros((len(lens), 128, 64), dtype=torch.int16, device="cuda")
    for b, L in enumerate(lens):
        n = min(128, L)
        kv_last[b, 128 - n:] = torch.from_numpy(wl.kv_rows(w.seed, b, L - n, n).view(np.int16))
        k_last[b, 128 - n:] = torch.from_numpy(wl.idxk_rows(w.seed, b, L - n, n).view(np.int16))
    csa2_lib.csa2_swa_replay(cache, kv_last, k_last, torch.from_numpy(miss.astype(np.uint8)).cuda())
    assert csa2_lib.csa2_check_device_error(cache) == 0
    for b, L in enumerate(lens):
        want = ofp8.Fp8Keys.from_bf16(wl.idxk_rows(w.seed, b, 0, L))
        pos, _ = omodes.replay_positions(L, bool(miss[b]))
        codes, scales = cache_keys_fp8(cache, b, pos)
        np.testing.assert_array_equal(codes, want.codes[pos])
        np.testing.assert_array_equal(scales, want.scales[pos])
        if miss[b]:
            np.testing.assert_array_equal(cache_block_keys(cache, b, np.arange((L + 7) // 8)),
                                          oidx.block_keys(want, L))


def test_decode_step_on_fp8_keys(fp8):
    """Full layer then Reuse layers over an FP8-key cache: attention over the GPU's
    own sets follows the oracle (the main KV is unchanged by the key format)."""
    csa2, syn, w, cache, keys = fp8
    w.layers = ["F", "R"]
    step = syn.DecodeStep(w, cache)
    step.run(append=True)
    assert csa2.csa2_check_device_error(cache) == 0
    gidx = step.iset.idx.cpu().numpy()
    for i in range(2):
        g = bits(step.out[i])
        for b, L in enumerate(LENGTHS):
            ref = parity.oracle_attention(parity.OracleSeq(w, b, L), gidx[b], wl.q_rows(w.seed, i, b, 16), L)
            err, bound = parity.attention_error(g[b], ref)
            assert err <= bound, f"layer {i} L={L}: err {err} > {bound}"
