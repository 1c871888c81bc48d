"""GPU parity of the position-sharded Full layer, all shards emulated on one GPU
(shard s of sequence b is sequence b * S + s of one cache): the merged pool and
index set equal the unsharded call's exactly (same kernels, same scores) and the
oracle's under the index-set rule, and the log-sum-exp combination of the shards'
attention follows the oracle over the whole sequence -- with 2 and 4 shards, a
window split across two shards, and a shard that holds none of the set."""
import numpy as np
import pytest
import torch

import workload as wl
from oracle import indexer as oidx
from oracle.formats import bf16_to_f64
from tests import parity
from tests.gpu_util import bits, small_workload

pytestmark = pytest.mark.gpu

LENGTHS = [40000, 20011, 3000]
HEADS = 16


def _plans():
    from fp4_kv_cache_decode_b200.sharded import shard_bounds
    yield "2 shards", [shard_bounds(L, 2) for L in LENGTHS]
    yield "4 shards", [shard_bounds(L, 4) for L in LENGTHS]
    # the window [L - 128, L) split across the last two shards; a shard of 8 entries
    yield "split window", [[(0, 39936), (39936, 39992), (39992, 40000)],
                           [(0, 19920), (19920, 19992), (19992, 20011)],
                           [(0, 8), (8, 2920), (2920, 3000)]]


@pytest.fixture(scope="module")
def unsharded(csa2_lib):
    import workload
    workload.build_cuda()
    from fp4_kv_cache_decode_b200 import synthetic as syn
    from workload import device as wdev
    csa2 = csa2_lib
    w = small_workload(LENGTHS, seed=61, heads=HEADS, spare_pages=64)
    cache = syn.new_cache(w)
    syn.fill_decode_cache(w, cache)
    B = len(LENGTHS)
    qs = torch.arange(B, dtype=torch.int32, device="cuda")
    iset = csa2.IndexSet(B)
    ws = torch.empty(csa2.csa2_workspace_bytes(csa2.OP_INDEXER, B, 0, max(LENGTHS), 1), dtype=torch.uint8,
                     device="cuda")
    csa2.csa2_indexer_score_topk(cache, wdev.idxq_batch(w.seed, 0, 0, B), qs, csa2.FULL, 0, iset, ws, max(LENGTHS))
    out = torch.empty((B, HEADS, 512), dtype=torch.bfloat16, device="cuda")
    wsa = torch.empty(max(256, csa2.csa2_workspace_bytes(csa2.OP_ATTENTION, B, HEADS)), dtype=torch.uint8,
                      device="cuda")
    csa2.csa2_sparse_attn(cache, wdev.q_batch(w.seed, 0, 0, B, HEADS), qs, csa2.FULL, 0, iset, out, wsa)
    assert csa2.csa2_check_device_error(cache) == 0
    return w, iset.pool_blocks.cpu().numpy(), iset.idx.cpu().numpy(), out


@pytest.mark.parametrize("plan", list(_plans()), ids=lambda p: p[0])
def test_sharded_full_layer_equals_unsharded(csa2_lib, unsharded, plan):
    from fp4_kv_cache_decode_b200 import synthetic as syn
    from fp4_kv_cache_decode_b200.sharded import emulate_full_layer
    from workload import device as wdev
    csa2 = csa2_lib
    w, upool, uidx, uout = unsharded
    name, bounds = plan
    S = len(bounds[0])
    lens = [hi - lo for shards in bounds for lo, hi in shards]
    ws = small_workload(lens, seed=w.seed, heads=HEADS, spare_pages=64)
    cache = syn.new_cache(ws, lengths=lens)
    syn.fill_sharded_cache(w, cache, bounds)
    B = len(LENGTHS)
    off = torch.tensor([lo for shards in bounds for lo, _ in shards], dtype=torch.int32, device="cuda")
    wstart = torch.tensor([max(0, L - 128) for L in LENGTHS], dtype=torch.int32, device="cuda")
    pool, idx, out, lse2 = emulate_full_layer(cache, S, off, wstart, wdev.idxq_batch(w.seed, 0, 0, B),
                                              wdev.q_batch(w.seed, 0, 0, B, HEADS), max(lens))
    torch.cuda.synchronize()
    assert csa2.csa2_check_device_error(cache) == 0
    gpool, gidx = pool.cpu().numpy(), idx.cpu().numpy()
    np.testing.assert_array_equal(gpool, upool, err_msg=name)
    np.testing.assert_array_equal(gidx, uidx, err_msg=name)
    g = bits(out)
    ug = bits(uout)
    for b, L in enumerate(LENGTHS):
        o = parity.OracleSeq(w, b, L)
        iq = wl.idxq_rows(w.seed, 0, b)
        opool, oidx_, _ = oidx.full_indexer(iq, o.keys, L)
        parity.check_index_set(gpool[b], opool, lambda x: oidx.index_scores(iq, oidx.block_keys(o.keys, L)[
            np.asarray(x)]), f"{name} pool L={L}")
        if np.array_equal(gpool[b], opool):
            parity.check_index_set(gidx[b], oidx_, parity.token_scorer(o, iq), f"{name} tokens L={L}")
        ref = parity.oracle_attention(o, gidx[b], wl.q_rows(w.seed, 0, b, HEADS), L)
        err, bound = parity.attention_error(g[b], ref)
        assert err <= bound, f"{name} L={L}: err {err} > {bound}"
        err_u = float(np.max(np.abs(bf16_to_f64(g[b]) - bf16_to_f64(ug[b]))))
        assert err_u <= bound, f"{name} L={L}: sharded vs unsharded {err_u}"
    # a shard holding none of the set reports -inf and adds nothing
    l2 = lse2.view(B, S, HEADS).cpu().numpy()
    assert np.all(np.isfinite(l2) | (l2 == -np.inf))


def test_emulated_decoder_layers_equal_unsharded(csa2_lib):
    """Full, Reuse, Reindex, Reuse through the emulated sharded decoder (the
    bench's 1M leg): index sets equal the unsharded calls', outputs within the
    parity bound of the unsharded outputs."""
    import workload
    workload.build_cuda()
    from fp4_kv_cache_decode_b200 import synthetic as syn
    from fp4_kv_cache_decode_b200.sharded import EmulatedDecoder, shard_bounds
    from workload import device as wdev
    csa2 = csa2_lib
    layers = ["F", "R", "RI", "R"]
    w = small_workload(LENGTHS, seed=67, heads=HEADS, spare_pages=64)
    w.layers = list(layers)
    cache = syn.new_cache(w)
    syn.fill_decode_cache(w, cache)
    full = syn.DecodeStep(w, cache, layers=["F"])
    full.run(append=False)
    step = syn.DecodeStep(w, cache)
    step.run(append=False)
    S = 3
    bounds = [shard_bounds(L, S) for L in LENGTHS]
    lens = [hi - lo for sh in bounds for lo, hi in sh]
    cs = syn.new_cache(small_workload(lens, seed=w.seed, heads=HEADS, spare_pages=64), lengths=lens)
    syn.fill_sharded_cache(w, cs, bounds)
    B = len(LENGTHS)
    off = torch.tensor([lo for sh in bounds for lo, _ in sh], dtype=torch.int32, device="cuda")
    wstart = torch.tensor([max(0, L - 128) for L in LENGTHS], dtype=torch.int32, device="cuda")
    dec = EmulatedDecoder(cs, S, off, wstart, HEADS, max(lens))
    for l, m in enumerate(layers):
        q = wdev.q_batch(w.seed, l, 0, B, HEADS)
        if m == "F":
            o = dec.full(wdev.idxq_batch(w.seed, l, 0, B), q)
            np.testing.assert_array_equal(dec.buf.pool.cpu().numpy(), full.iset.pool_blocks.cpu().numpy())
            np.testing.assert_array_equal(dec.buf.idx.cpu().numpy(), full.iset.idx.cpu().numpy())
        elif m == "RI":
            o = dec.reindex(wdev.idxq_batch(w.seed, l, 0, B), q)
            np.testing.assert_array_equal(dec.buf.idx.cpu().numpy(), step.iset.idx.cpu().numpy())
        else:
            o = dec.reuse(q)
        got, want = bits(o), bits(step.out[l])
        for b in range(B):
            ref = bf16_to_f64(want[b])
            bound = 1e-2 * float(np.abs(ref).max()) + 1e-3
            assert float(np.max(np.abs(bf16_to_f64(got[b]) - ref))) <= bound, f"layer {l} seq {b}"
    torch.cuda.synchronize()
    assert csa2.csa2_check_device_error(cs) == 0 and csa2.csa2_check_device_error(cache) == 0
