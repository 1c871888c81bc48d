"""GPU parity of the separate sliding-window store and of bounded replay at
compression ratio 2 (encoder).

* append writes each sequence's last 128 entries into the store, byte-exact
  with the oracle codec, and attention that reads the window from the store
  gives the same bits as attention that reads it from the global cache;
* after the store is lost, replay with freshly supplied rows rebuilds only the
  store (the global cache is untouched) and attention follows the oracle over
  the replayed window rows;
* ratio-2 replay, with and without a store, re-encodes the supplied raw row
  pairs byte-exact with the oracle."""
import numpy as np
import pytest
import torch

import workload as wl
from oracle import attention as oattn
from oracle import codec as ocodec
from oracle import indexer as oidx
from oracle import modes as omodes
from tests import parity
from tests.gpu_util import bits, cache_block_keys, cache_keys, cache_rows, small_workload

pytestmark = pytest.mark.gpu

LENGTHS = [3000, 200, 17000, 128, 129, 1, 127, 640]


@pytest.fixture(scope="module")
def gpu(csa2_lib):
    import workload
    workload.build_cuda()
    from fp4_kv_cache_decode_b200 import synthetic as syn
    return csa2_lib, syn


def _dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()


def _store_rows(cache, seq: int, slots) -> np.ndarray:
    return cache.swa_rows[seq].cpu().numpy()[np.asarray(slots, dtype=np.int64)]


def test_append_fills_the_store_and_attention_reads_it(gpu):
    csa2, syn = gpu
    w = small_workload(LENGTHS, seed=31, heads=64)
    w.layers = ["F", "R", "R"]
    plain = syn.new_cache(w, cache_id=1)
    store = syn.new_cache(w, cache_id=2, swa_store=True)
    for c in (plain, store):
        syn.fill_decode_cache(w, c)
        assert csa2.csa2_check_device_error(c) == 0
    for b, L in enumerate(LENGTHS):
        pos, slot = omodes.window_store_slots(L)
        np.testing.assert_array_equal(_store_rows(store, b, slot),
                                      parity.OracleSeq(w, b, L).encoded_rows(pos), err_msg=f"L={L}")
        empty = np.setdiff1d(np.arange(128), slot)
        assert np.all(_store_rows(store, b, empty) == 0)
    # the global cache is the same either way
    assert torch.equal(plain.kv_pool, store.kv_pool) and torch.equal(plain.idxk_pool, store.idxk_pool)
    outs = []
    for c in (plain, store):
        step = syn.DecodeStep(w, c)
        step.run(append=True)
        assert csa2.csa2_check_device_error(c) == 0
        outs.append(step.out)
    for a, b in zip(*outs):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_replay_rebuilds_a_lost_store_and_attention_follows(gpu):
    csa2, syn = gpu
    w = small_workload(LENGTHS, seed=32, heads=16)
    miss = np.array([True, True, True, False, True, True, False, True])
    cache = syn.new_cache(w, swa_store=True)
    syn.fill_decode_cache(w, cache)
    pools = [t.clone() for t in (cache.kv_pool, cache.idxk_pool, cache.bk_pool)]
    cache.swa_rows.fill_(0xFF)   # the store's content is gone
    # recomputed window rows: drawn from another seed so that every attended
    # window row shows where it was read from
    B = len(LENGTHS)
    fresh = np.zeros((B, 128, 512), np.uint16)
    for b, L in enumerate(LENGTHS):
        n = min(128, L)
        fresh[b, 128 - n:] = wl.kv_rows(w.seed + 1000, b, L - n, n)
    csa2.csa2_swa_replay(cache, _dev(fresh), None, torch.from_numpy(miss.astype(np.uint8)).cuda())
    assert csa2.csa2_check_device_error(cache) == 0
    for t, t0 in zip((cache.kv_pool, cache.idxk_pool, cache.bk_pool), pools):
        assert torch.equal(t, t0)
    for b, L in enumerate(LENGTHS):
        pos, rows = omodes.replay_entries(fresh[b], L, bool(miss[b]))
        np.testing.assert_array_equal(_store_rows(cache, b, pos % 128), rows, err_msg=f"L={L}")
        assert np.all(_store_rows(cache, b, np.setdiff1d(np.arange(128), pos % 128)) == 0xFF)
    # attention of the rebuilt sequences: the window from the store, the rest from the cache
    seqs = [b for b in range(B) if miss[b]]
    step = syn.DecodeStep(w, cache, seqs=seqs)
    step.run(append=False)
    assert csa2.csa2_check_device_error(cache) == 0
    g = bits(step.out[0])
    gidx = step.iset.idx.cpu().numpy()
    for j, b in enumerate(seqs):
        L = LENGTHS[b]
        o = parity.OracleSeq(w, b, L)
        pos = oattn.attended_positions(gidx[j], L)   # (index parity has its own tests)
        in_store = omodes.from_window_store(pos, L)
        rows = np.empty((pos.size, 512))
        rows[~in_store] = o.rows(pos[~in_store])
        rpos, rrows = omodes.replay_entries(fresh[b], L, True)
        lookup = dict(zip(rpos.tolist(), range(rpos.size)))
        rows[in_store] = ocodec.dequantize(*ocodec.unpack_rows(rrows[[lookup[p] for p in pos[in_store]]]))
        ref = oattn.attend(wl.q_rows(w.seed, 0, b, 16), rows)
        err, bound = parity.attention_error(g[j], ref)
        assert err <= bound, f"L={L}: err {err} > {bound}"


ENC_LENGTHS = [300, 50, 128, 1, 700, 129]


def _encoder_cache(csa2, syn, w, swa_store):
    """Entries [0, L) at compression ratio 2 from the seeded raw rows [0, 2L)."""
    cache = syn.new_cache(w, swa_store=swa_store)
    for b, L in enumerate(ENC_LENGTHS):
        raw = wl.kv_rows(w.seed, b, 0, 2 * L)
        rawk = wl.idxk_rows(w.seed, b, 0, 2 * L)
        seqs = torch.full((L,), b, dtype=torch.int32, device="cuda")
        pos = torch.arange(L, dtype=torch.int32, device="cuda")
        csa2.csa2_kv_quant_append(cache, _dev(raw), _dev(rawk), seqs, pos, 2)
    assert csa2.csa2_check_device_error(cache) == 0
    return cache


def _last_blocks(w, lens):
    """Raw rows behind each sequence's last 128 entries, [B, 256, 512] and [B, 256, 64]."""
    kv = np.zeros((len(lens), 256, 512), np.uint16)
    k = np.zeros((len(lens), 256, 64), np.uint16)
    for b, L in enumerate(lens):
        n = min(128, L)
        kv[b, 256 - 2 * n:] = wl.kv_rows(w.seed, b, 2 * (L - n), 2 * n)
        k[b, 256 - 2 * n:] = wl.idxk_rows(w.seed, b, 2 * (L - n), 2 * n)
    return kv, k


def test_ratio2_replay_restores_poisoned_entries(gpu):
    csa2, syn = gpu
    w = small_workload(ENC_LENGTHS, seed=33)
    miss = np.array([True, True, False, True, True, False])
    cache = _encoder_cache(csa2, syn, w, swa_store=False)
    before = {b: cache_rows(cache, b, np.arange(L)) for b, L in enumerate(ENC_LENGTHS)}
    pt = cache.page_table.cpu().numpy()
    for b, L in enumerate(ENC_LENGTHS):
        for p in range(max(0, L - 128), L):
            pg = int(pt[b, p >> 6])
            cache.kv_pool[pg * 18432 + (p & 63) * 288: pg * 18432 + (p & 63) * 288 + 288] = 0xFF
            cache.idxk_pool[pg * 8192 + (p & 63) * 128: pg * 8192 + (p & 63) * 128 + 128] = 0x7F
    kv, k = _last_blocks(w, ENC_LENGTHS)
    csa2.csa2_swa_replay(cache, _dev(kv), _dev(k), torch.from_numpy(miss.astype(np.uint8)).cuda(), compress=2)
    assert csa2.csa2_check_device_error(cache) == 0
    for b, L in enumerate(ENC_LENGTHS):
        pos, rows = omodes.replay_entries(kv[b], L, bool(miss[b]), compress=2)
        kpos, keys = omodes.replay_keys(k[b], L, bool(miss[b]), compress=2)
        after = cache_rows(cache, b, np.arange(L))
        np.testing.assert_array_equal(after[pos], rows, err_msg=f"L={L}")
        np.testing.assert_array_equal(after[pos], before[b][pos])   # the same as the append made
        np.testing.assert_array_equal(cache_keys(cache, b, kpos), keys)
        lo = max(0, L - 128)
        assert np.all(after[np.setdiff1d(np.arange(lo, L), pos)] == 0xFF)
        assert np.array_equal(after[:lo], before[b][:lo])
        if miss[b]:
            allk = ocodec.idxk_entries(wl.idxk_rows(w.seed, b, 0, 2 * L), 2)
            np.testing.assert_array_equal(cache_block_keys(cache, b, np.arange((L + 7) // 8)),
                                          oidx.block_keys(allk, L))


def test_ratio2_replay_into_the_store(gpu):
    csa2, syn = gpu
    w = small_workload(ENC_LENGTHS, seed=34)
    cache = _encoder_cache(csa2, syn, w, swa_store=True)
    for b, L in enumerate(ENC_LENGTHS):
        pos, slot = omodes.window_store_slots(L)
        want = ocodec.encode_entries(wl.kv_rows(w.seed, b, 2 * pos[0], 2 * pos.size), 2)
        np.testing.assert_array_equal(_store_rows(cache, b, slot), want, err_msg=f"L={L}")
    kv_pool = cache.kv_pool.clone()
    cache.swa_rows.fill_(0)
    kv, _ = _last_blocks(w, ENC_LENGTHS)
    miss = torch.ones(len(ENC_LENGTHS), dtype=torch.uint8, device="cuda")
    csa2.csa2_swa_replay(cache, _dev(kv), None, miss, compress=2)
    assert csa2.csa2_check_device_error(cache) == 0
    assert torch.equal(cache.kv_pool, kv_pool)
    for b, L in enumerate(ENC_LENGTHS):
        pos, rows = omodes.replay_entries(kv[b], L, True, compress=2)
        np.testing.assert_array_equal(_store_rows(cache, b, pos % 128), rows, err_msg=f"L={L}")
