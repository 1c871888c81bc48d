"""GPU parity at the five workloads' full sizes, in the launch configuration the
benchmark times, checked on sampled sequences / queries that the oracle computes
one by one from the seeded inputs."""
import numpy as np
import pytest
import torch

import workload as wl
from oracle import indexer as oidx
from oracle import modes as omodes
from tests import parity
from tests.gpu_util import bits, cache_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def env(csa2_lib):
    import workload
    workload.build_cuda()
    from fp4_kv_cache_decode_b200 import synthetic
    return csa2_lib, synthetic


def _check_decode(w, step, sample, layers, gpu_sets):
    """Oracle replay of the layer schedule for sampled sequences of a DecodeStep.

    gpu_sets[i] = (idx rows, pool rows) that the GPU produced at Full / Reindex
    layer i.  The GPU's pool is compared with the oracle's under the
    boundary-swap rule; its token set with the oracle's selection over the
    GPU's own pool (the same rule), so a swap in the pool does not hide the
    token level; and every layer's attention is compared with the oracle's
    attention over the GPU's own index set.  Returns (attention comparisons,
    boundary swaps)."""
    outs = [bits(o) for o in step.out]
    compared = swaps = 0
    for j in sample:
        seq = step.seqs[j]
        L = w.lengths[seq]
        o = parity.OracleSeq(w, seq, L)
        gpool = gset = None
        for i, mode in enumerate(layers):
            l = step.layer0 + i
            if mode in ("F", "RI"):
                iq = wl.idxq_rows(w.seed, l, seq)
                gidx, gpools = gpu_sets[i]
                if mode == "F":
                    pool, _, _ = oidx.full_indexer(iq, o.keys, L)
                    gpool = gpools[j]
                    if (L + 7) // 8 > 2048:
                        swaps += parity.check_index_set(gpool, pool, parity.block_scorer(o, iq, L),
                                                        f"blocks seq {seq}")
                    else:
                        np.testing.assert_array_equal(gpool, pool)
                # the oracle's token selection over the GPU's pool
                want, _ = oidx.reindex_indexer(iq, o.keys, L, gpool)
                swaps += parity.check_index_set(gidx[j], want, parity.token_scorer(o, iq),
                                                f"tokens seq {seq} layer {l}")
                gset = gidx[j]
            ref = parity.oracle_attention(o, gset, wl.q_rows(w.seed, l, seq, w.heads), L)
            err, bound = parity.attention_error(outs[i][j], ref)
            assert err <= bound, f"seq {seq} layer {l} ({mode}): err {err} > {bound}"
            compared += 1
    return compared, swaps


def _sets(iset):
    return iset.idx.cpu().numpy(), iset.pool_blocks.cpu().numpy()


def test_config0_tiny_decode(env):
    csa2, syn = env
    w = wl.workload(0)
    cache = syn.new_cache(w)
    syn.fill_decode_cache(w, cache)
    step = syn.DecodeStep(w, cache)
    step.run()
    assert csa2.csa2_check_device_error(cache) == 0
    o = parity.OracleSeq(w, 0, 4096)
    iq = wl.idxq_rows(w.seed, 0, 0)
    pool, idx, _ = oidx.full_indexer(iq, o.keys, 4096)
    n = parity.check_index_set(step.iset.idx[0].cpu().numpy(), idx, parity.token_scorer(o, iq), "config 0")
    ref = parity.oracle_attention(o, idx, wl.q_rows(w.seed, 0, 0, 16), 4096)
    err, bound = parity.attention_error(bits(step.out[0])[0], ref)
    assert err <= bound and n == 0


def test_config1_decode_sampled(env):
    csa2, syn = env
    w = wl.workload(1)
    cache = syn.new_cache(w)
    syn.fill_decode_cache(w, cache)
    step = syn.DecodeStep(w, cache)
    step.run()
    torch.cuda.synchronize()
    assert csa2.csa2_check_device_error(cache) == 0
    # the Full set of layer 0 comes from a separate Full-only run (same inputs);
    # the step's own set holds the Reindex layer's result
    full = syn.DecodeStep(w, cache, layers=["F"])
    full.run(append=False)
    sample = [0, 5, 13, 22, 31]
    n, swaps = _check_decode(w, step, sample, w.layers, {0: _sets(full.iset), 4: _sets(step.iset)})
    assert n == len(sample) * len(w.layers)
    assert swaps <= 2 * len(sample), f"{swaps} boundary swaps"   # near-ties are rare
    # the appended token wrote the same row the setup wrote
    np.testing.assert_array_equal(cache_rows(cache, 5, [65535]),
                                  parity.OracleSeq(w, 5, 65536).encoded_rows([65535]))


def test_config2_long_context_sampled(env):
    csa2, syn = env
    w = wl.workload(2)
    cache = syn.new_cache(w)
    syn.fill_decode_cache(w, cache)
    step = syn.DecodeStep(w, cache)
    step.run()
    assert csa2.csa2_check_device_error(cache) == 0
    # oracle over the first two groups (Full + 3 Reuse, Reindex + 3 Reuse) of sequence 2
    sub = syn.DecodeStep(w, cache, layers=w.layers[:8], seqs=[2])
    sub.run(append=False)
    full = syn.DecodeStep(w, cache, layers=["F"], seqs=[2])
    full.run(append=False)
    n, swaps = _check_decode(w, sub, [0], w.layers[:8], {0: _sets(full.iset), 4: _sets(sub.iset)})
    assert n == 8 and swaps <= 4, (n, swaps)
    # the full 20-layer run agrees with the 8-layer sub-run on those layers
    for i in range(8):
        assert torch.equal(step.out[i][2].view(torch.int16), sub.out[i][0].view(torch.int16))


def test_config3_prefill_sampled(env):
    csa2, syn = env
    w = wl.workload(3)
    cache = syn.new_cache(w)
    for c in range(w.raw_tokens // w.chunk):
        syn.fill_prefill_chunk(w, cache, c)
    assert csa2.csa2_check_device_error(cache) == 0
    # a whole chunk through the bench's launch shape, then sampled queries
    ch = syn.PrefillChunk(w, cache, 15)
    ch.indexer()
    outs = {layer: bits(ch.attention(layer)) for layer in (0, 5)}
    assert csa2.csa2_check_device_error(cache) == 0
    keys_o = parity.OracleSeq(w, 0, 65536, compress=2)
    gidx = ch.iset.idx.cpu().numpy()
    swaps = 0
    for qi in (0, 1, 1000, 2048, 4095, 6000, 7777, 8191):
        P = int(ch.qpos[qi])
        v = (P + 1) // 2
        iq = wl.idxq_rows(w.seed, 0, P)
        idx, _ = oidx.flat_indexer(iq, keys_o.keys, v)
        swaps += parity.check_index_set(gidx[qi], idx, parity.token_scorer(keys_o, iq), f"prefill P={P}")
        for layer in (0, 5):   # attention over the GPU's own (checked) set
            ref = parity.oracle_attention(keys_o, gidx[qi], wl.q_rows(w.seed, layer, P, 64), v)
            err, bound = parity.attention_error(outs[layer][qi], ref)
            assert err <= bound, f"P={P} layer={layer}: {err} > {bound}"
    assert swaps <= 8, f"{swaps} boundary swaps"
    # early queries of the first chunk: tiny and empty visible sets
    early = syn.PrefillChunk(w, cache, 0, queries=[0, 1, 2, 3, 255, 1023, 1024, 1025, 2047])
    early.indexer()
    eo = bits(early.attention(0))
    eidx = early.iset.idx.cpu().numpy()
    for qi, P in enumerate(early.qpos):
        v = (int(P) + 1) // 2
        iq = wl.idxq_rows(w.seed, 0, int(P))
        idx, _ = oidx.flat_indexer(iq, keys_o.keys, v)
        parity.check_index_set(eidx[qi], idx, parity.token_scorer(keys_o, iq), f"early P={P}")
        ref = parity.oracle_attention(keys_o, eidx[qi], wl.q_rows(w.seed, 0, int(P), 64), v)
        err, bound = parity.attention_error(eo[qi], ref)
        assert err <= bound, f"early P={P}: {err} > {bound}"
        if v == 0:
            assert np.all(eo[qi] == 0)


def test_config4_ragged_replay_sampled(env):
    csa2, syn = env
    w = wl.workload(4)
    cache = syn.new_cache(w)
    syn.fill_decode_cache(w, cache)
    st = syn.RaggedStep(w, cache)
    st.setup()
    # poison the windows of the flagged sequences; replay must restore them
    pt = cache.page_table.cpu().numpy()
    misses = [int(b) for b in np.nonzero(w.miss_mask)[0]]
    for b in misses:
        L = w.lengths[b]
        for p in range(L - 128, L):
            pg = int(pt[b, p >> 6])
            cache.kv_pool[pg * 18432 + (p & 63) * 288: pg * 18432 + (p & 63) * 288 + 288] = 0xFF
    st.run()
    assert csa2.csa2_check_device_error(cache) == 0
    for b in misses[:3]:
        L = w.lengths[b]
        pos = np.arange(L - 128, L)
        np.testing.assert_array_equal(cache_rows(cache, b, pos), parity.OracleSeq(w, b, L).encoded_rows(pos))
    ri, ru = st.groups["ri"], st.groups["ru"]
    gri = ri["iset"].idx.cpu().numpy()
    gpool = ri["iset"].pool_blocks.cpu().numpy()
    out_ri, out_ru = bits(ri["out"]), bits(ru["out"])
    lens = np.array(w.lengths)
    # sampled: the longest and shortest Reindex and Reuse sequences, and a miss
    pick_ri = [int(np.argmax(lens[st.ri])), int(np.argmin(lens[st.ri]))]
    pick_ru = [int(np.argmax(lens[st.ru])), int(np.argmin(lens[st.ru]))]
    compared = swaps = 0
    for j in pick_ri:
        seq = st.ri[j]
        L = w.lengths[seq]
        o = parity.OracleSeq(w, seq, L)
        iq0 = wl.idxq_rows(w.seed, 0, seq)
        pool, _, _ = oidx.full_indexer(iq0, o.keys, L)
        if (L + 7) // 8 > 2048:
            swaps += parity.check_index_set(gpool[j], pool, parity.block_scorer(o, iq0, L), f"blocks seq {seq}")
        else:
            np.testing.assert_array_equal(gpool[j], pool)
        iq = wl.idxq_rows(w.seed, 1, seq)
        want, _ = oidx.reindex_indexer(iq, o.keys, L, gpool[j])   # over the GPU's own pool
        swaps += parity.check_index_set(gri[j], want, parity.token_scorer(o, iq), f"reindex seq {seq} L={L}")
        ref = parity.oracle_attention(o, gri[j], wl.q_rows(w.seed, 1, seq, 64), L)
        err, bound = parity.attention_error(out_ri[j], ref)
        assert err <= bound, f"reindex seq {seq}: {err} > {bound}"
        compared += 1
    gru = ru["iset"].idx.cpu().numpy()
    gpool_ru = ru["iset"].pool_blocks.cpu().numpy()
    for j in pick_ru:
        seq = st.ru[j]
        L = w.lengths[seq]
        o = parity.OracleSeq(w, seq, L)
        iq = wl.idxq_rows(w.seed, 0, seq)
        pool, _, _ = oidx.full_indexer(iq, o.keys, L)
        if (L + 7) // 8 > 2048:
            swaps += parity.check_index_set(gpool_ru[j], pool, parity.block_scorer(o, iq, L), f"blocks seq {seq}")
        else:
            np.testing.assert_array_equal(gpool_ru[j], pool)
        want, _ = oidx.reindex_indexer(iq, o.keys, L, gpool_ru[j])
        swaps += parity.check_index_set(gru[j], want, parity.token_scorer(o, iq), f"reuse seq {seq}")
        ref = parity.oracle_attention(o, gru[j], wl.q_rows(w.seed, 1, seq, 64), L)
        err, bound = parity.attention_error(out_ru[j], ref)
        assert err <= bound, f"reuse seq {seq}: {err} > {bound}"
        compared += 1
    assert compared == len(pick_ri) + len(pick_ru) and swaps <= 8, (compared, swaps)
