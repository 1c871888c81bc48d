"""GPU parity of the encoder path: generator twin, exhaustive codec, ratio-2 compression,
indexer keys and block keys, bounded replay, and device-side bounds reporting."""
import numpy as np
import pytest
import torch

import workload as wl
from oracle import codec as ocodec
from oracle import formats as ofmt
from oracle import indexer as oidx
from oracle import modes as omodes
from oracle import idxk_fp8 as ofp8
from tests.gpu_util import bits, cache_block_keys, cache_keys, cache_keys_fp8, cache_rows, small_workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gpu(csa2_lib):
    import workload
    workload.build_cuda()
    assert torch.cuda.is_available()
    from fp4_kv_cache_decode_b200 import synthetic
    return csa2_lib, synthetic


def test_device_generator_matches_host(gpu):
    from workload import device as wdev
    for seed, seq, p0, n in [(0, 0, 0, 100), (1, 5, 65000, 600), (2, 3, 1048000, 576)]:
        np.testing.assert_array_equal(bits(wdev.kv_rows(seed, seq, p0, n)), wl.kv_rows(seed, seq, p0, n))
        np.testing.assert_array_equal(bits(wdev.idxk_rows(seed, seq, p0, n)), wl.idxk_rows(seed, seq, p0, n))
    q = bits(wdev.q_batch(3, 2, 7, 4, 64))
    for i in range(4):
        np.testing.assert_array_equal(q[i], wl.q_rows(3, 2, 7 + i, 64))
    iq = bits(wdev.idxq_batch(3, 4, 11, 3))
    for i in range(3):
        np.testing.assert_array_equal(iq[i], wl.idxq_rows(3, 4, 11 + i))


def _encode_on_gpu(csa2, kv_bits: np.ndarray, k_bits: np.ndarray, compress: int = 1):
    n_in = kv_bits.shape[0]
    n = n_in // compress
    pages = (n + 63) // 64
    cache = csa2.Cache(pages, 1, pages)
    cache.page_table[0] = torch.arange(pages, dtype=torch.int32)
    cache.seq_lens[0] = n
    kv = torch.from_numpy(kv_bits.view(np.int16)).cuda()
    k = torch.from_numpy(k_bits.view(np.int16)).cuda()
    eseq = torch.zeros(n, dtype=torch.int32, device="cuda")
    epos = torch.arange(n, dtype=torch.int32, device="cuda")
    csa2.csa2_kv_quant_append(cache, kv, k, eseq, epos, compress)
    assert csa2.csa2_check_device_error(cache) == 0
    rows = cache.kv_pool.view(-1, 288)[:n].cpu().numpy()
    keys = cache.idxk_pool.view(-1, 128)[:n].cpu().numpy().view(np.uint16)
    nb = (n + 7) // 8
    bk = cache.bk_pool.view(-1, 128)[:nb].cpu().numpy().view(np.uint16)
    return rows, keys, bk


def _exhaustive_rows():
    """Rows whose 16-value groups cover, for every positive E4M3 scale, every
    finite bf16 value up to the group maximum that selects that scale, plus
    zero, underflowing and saturating groups."""
    allb = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    v = ofmt.bf16_to_f64(allb)
    fin = np.isfinite(v)
    allb, v = allb[fin], v[fin]
    groups = []
    for sc in range(1, 127):
        A = 6.0 * ocodec.E4M3_GRID[sc]                  # amax that selects scale code sc
        a_bits = ofmt.f32_to_bf16(np.float32(A))
        assert ofmt.bf16_to_f64(a_bits) == A
        vals = allb[np.abs(v) <= A]
        pad = (-vals.size) % 15
        vals = np.concatenate([vals, np.zeros(pad, dtype=np.uint16)]).reshape(-1, 15)
        lead = np.full((vals.shape[0], 1), a_bits, dtype=np.uint16)
        lead[1::2] ^= np.uint16(0x8000)
        groups.append(np.concatenate([lead, vals], axis=1))
    special = np.zeros((4, 16), dtype=np.uint16)
    special[1] = ofmt.f32_to_bf16(np.full(16, 2.0 ** -20, np.float32))     # scale underflows to 0
    special[2] = ofmt.f32_to_bf16(np.linspace(-3e4, 3e4, 16).astype(np.float32))   # saturating scale
    special[3, ::2] = 0x8000                                                # negative zeros
    g = np.concatenate(groups + [special])
    g = np.concatenate([g, np.zeros(((-g.shape[0]) % 32, 16), np.uint16)])
    return g.reshape(-1, 512)


def test_codec_exhaustive_bit_exact(gpu):
    csa2, _ = gpu
    rows = _exhaustive_rows()
    rng = np.random.default_rng(0)
    keys = ofmt.f32_to_bf16(rng.standard_normal((rows.shape[0], 64)).astype(np.float32))
    got, gk, gbk = _encode_on_gpu(csa2, rows, keys)
    want = ocodec.encode_bf16_rows(rows)
    mism = np.nonzero(np.any(got != want, axis=1))[0]
    assert mism.size == 0, f"{mism.size} of {rows.shape[0]} rows differ; first {mism[:5]}"
    np.testing.assert_array_equal(gk, keys)
    np.testing.assert_array_equal(gbk, oidx.block_keys(keys, keys.shape[0]))


def test_ratio2_compression_bit_exact(gpu):
    csa2, _ = gpu
    rng = np.random.default_rng(1)
    x = (rng.standard_normal((4096, 512)) * np.exp(rng.uniform(-8, 8, (4096, 1)))).astype(np.float32)
    kv = ofmt.f32_to_bf16(x)
    keys = ofmt.f32_to_bf16(rng.standard_normal((4096, 64)).astype(np.float32))
    got, gk, gbk = _encode_on_gpu(csa2, kv, keys, compress=2)
    np.testing.assert_array_equal(got, ocodec.encode_entries(kv, 2))
    want_k = ocodec.idxk_entries(keys, 2)
    np.testing.assert_array_equal(gk, want_k)
    np.testing.assert_array_equal(gbk, oidx.block_keys(want_k, want_k.shape[0]))


def test_seeded_cache_pages_bit_exact(gpu):
    """Config-0-shaped cache (4,096 tokens, scattered pages) plus ragged lengths."""
    csa2, syn = gpu
    w = small_workload([4096, 1, 7, 8, 9, 129, 1000], seed=0)
    cache = syn.new_cache(w)
    syn.fill_decode_cache(w, cache, chunk=1024)
    assert csa2.csa2_check_device_error(cache) == 0
    for b, L in enumerate(w.lengths):
        pos = np.arange(L)
        np.testing.assert_array_equal(cache_rows(cache, b, pos),
                                      ocodec.encode_bf16_rows(wl.kv_rows(w.seed, b, 0, L)))
        keys = wl.idxk_rows(w.seed, b, 0, L)
        np.testing.assert_array_equal(cache_keys(cache, b, pos), keys)
        np.testing.assert_array_equal(cache_block_keys(cache, b, np.arange((L + 7) // 8)),
                                      oidx.block_keys(keys, L))


@pytest.mark.parametrize("fmt", ["bf16", "fp8"])
def test_small_appends_in_any_order_bit_exact(gpu, fmt):
    """Small append calls (64, 50 and 23 entries, as a decode step's): entries of two
    sequences in shuffled order, several of one block in one call (not contiguous)
    and one block's entries spread over calls, pages in reverse order -- rows, keys
    and block keys equal the oracle's."""
    csa2, _ = gpu
    lengths = [100, 37]
    pages = [(L + 63) // 64 for L in lengths]
    fmt_id = csa2.IDXK_FP8 if fmt == "fp8" else csa2.IDXK_BF16
    cache = csa2.Cache(sum(pages), 2, max(pages), idxk_format=fmt_id)
    order_pages = list(range(sum(pages)))[::-1]
    cache.page_table[0, :pages[0]] = torch.tensor(order_pages[:pages[0]], dtype=torch.int32)
    cache.page_table[1, :pages[1]] = torch.tensor(order_pages[pages[0]:], dtype=torch.int32)
    cache.seq_lens[:] = torch.tensor(lengths, dtype=torch.int32)
    rng = np.random.default_rng(11)
    kv = [ofmt.f32_to_bf16(rng.standard_normal((L, 512)).astype(np.float32)) for L in lengths]
    keys = [ofmt.f32_to_bf16(rng.standard_normal((L, 64)).astype(np.float32)) for L in lengths]
    entries = [(b, p) for b, L in enumerate(lengths) for p in range(L)]
    order = rng.permutation(len(entries))
    for call in np.split(order, [64, 114]):   # 64, 50 and 23 entries
        es = np.array([entries[i][0] for i in call], dtype=np.int32)
        ep = np.array([entries[i][1] for i in call], dtype=np.int32)
        kv_t = torch.from_numpy(np.stack([kv[b][p] for b, p in zip(es, ep)]).view(np.int16)).cuda()
        k_t = torch.from_numpy(np.stack([keys[b][p] for b, p in zip(es, ep)]).view(np.int16)).cuda()
        csa2.csa2_kv_quant_append(cache, kv_t, k_t, torch.from_numpy(es).cuda(), torch.from_numpy(ep).cuda())
    assert csa2.csa2_check_device_error(cache) == 0
    for b, L in enumerate(lengths):
        pos = np.arange(L)
        np.testing.assert_array_equal(cache_rows(cache, b, pos), ocodec.encode_bf16_rows(kv[b]))
        if fmt == "fp8":
            want = ofp8.Fp8Keys.from_bf16(keys[b])
            codes, scales = cache_keys_fp8(cache, b, pos)
            np.testing.assert_array_equal(codes, want.codes)
            np.testing.assert_array_equal(scales.view(np.uint32), want.scales.astype(np.float32).view(np.uint32))
        else:
            want = keys[b]
            np.testing.assert_array_equal(cache_keys(cache, b, pos), want)
        np.testing.assert_array_equal(cache_block_keys(cache, b, np.arange((L + 7) // 8)),
                                      oidx.block_keys(want, L))


def test_replay_restores_poisoned_rows(gpu):
    csa2, syn = gpu
    lens = [300, 50, 1000, 128, 129, 1]
    w = small_workload(lens, seed=5)
    w.miss_mask = np.array([True, True, False, True, False, True])
    cache = syn.new_cache(w)
    syn.fill_decode_cache(w, cache)
    before = {b: cache_rows(cache, b, np.arange(L)) for b, L in enumerate(lens)}
    # poison the last 128 rows (and keys) of every sequence
    pt = cache.page_table.cpu().numpy()
    for b, L in enumerate(lens):
        lo = max(0, L - 128)
        for p in range(lo, L):
            pg = int(pt[b, p >> 6])
            cache.kv_pool[pg * 18432 + (p & 63) * 288: pg * 18432 + (p & 63) * 288 + 288] = 0xFF
            cache.idxk_pool[pg * 8192 + (p & 63) * 128: pg * 8192 + (p & 63) * 128 + 128] = 0x7F
    kv_last = torch.zeros((len(lens), 128, 512), dtype=torch.int16, device="cuda")
    k_last = torch.zeros((len(lens), 128, 64), dtype=torch.int16, device="cuda")
    for b, L in enumerate(lens):
        n = min(128, L)
        kv_last[b, 128 - n:] = torch.from_numpy(wl.kv_rows(w.seed, b, L - n, n).view(np.int16))
        k_last[b, 128 - n:] = torch.from_numpy(wl.idxk_rows(w.seed, b, L - n, n).view(np.int16))
    miss = torch.from_numpy(w.miss_mask.astype(np.uint8)).cuda()
    csa2.csa2_swa_replay(cache, kv_last, k_last, miss)
    assert csa2.csa2_check_device_error(cache) == 0
    for b, L in enumerate(lens):
        after = cache_rows(cache, b, np.arange(L))
        rewritten, _ = omodes.replay_positions(L, bool(w.miss_mask[b]))
        untouched = np.setdiff1d(np.arange(max(0, L - 128), L), rewritten)
        np.testing.assert_array_equal(after[rewritten], before[b][rewritten])
        assert np.all(after[untouched] == 0xFF)
        assert np.array_equal(after[:max(0, L - 128)], before[b][:max(0, L - 128)])
        if w.miss_mask[b]:
            keys = wl.idxk_rows(w.seed, b, 0, L)
            np.testing.assert_array_equal(cache_block_keys(cache, b, np.arange((L + 7) // 8)),
                                          oidx.block_keys(keys, L))


def test_device_bounds_are_reported_not_faulted(gpu):
    csa2, syn = gpu
    w = small_workload([200, 200], seed=6)
    cache = syn.new_cache(w)
    syn.fill_decode_cache(w, cache)
    assert csa2.csa2_check_device_error(cache) == 0
    # a page-table entry beyond the pool: the row is skipped and reported
    cache.page_table[1, 0] = w.n_pages_pool + 5
    kv = torch.zeros((1, 512), dtype=torch.int16, device="cuda")
    k = torch.zeros((1, 64), dtype=torch.int16, device="cuda")
    csa2.csa2_kv_quant_append(cache, kv, k, torch.tensor([1], dtype=torch.int32, device="cuda"),
                              torch.tensor([3], dtype=torch.int32, device="cuda"))
    assert csa2.csa2_check_device_error(cache) & csa2.DEVERR_PAGE
    # a position beyond the sequence length and a bad sequence id
    csa2.csa2_kv_quant_append(cache, kv, k, torch.tensor([0], dtype=torch.int32, device="cuda"),
                              torch.tensor([250], dtype=torch.int32, device="cuda"))
    assert csa2.csa2_check_device_error(cache) & csa2.DEVERR_POS
    csa2.csa2_kv_quant_append(cache, kv, k, torch.tensor([9], dtype=torch.int32, device="cuda"),
                              torch.tensor([0], dtype=torch.int32, device="cuda"))
    assert csa2.csa2_check_device_error(cache) & csa2.DEVERR_SEQ
    # attention over an index set holding a position past the context
    iset = csa2.IndexSet(1)
    ws = torch.empty(csa2.csa2_workspace_bytes(csa2.OP_INDEXER, 1, 0, 200, True), dtype=torch.uint8,
                     device="cuda")
    iq = torch.zeros((1, 4, 64), dtype=torch.int16, device="cuda")
    qs = torch.tensor([0], dtype=torch.int32, device="cuda")
    csa2.csa2_indexer_score_topk(cache, iq, qs, csa2.FULL, 0, iset, ws, 200)
    iset.idx[0, 0] = 5000
    wa = torch.empty(csa2.csa2_workspace_bytes(csa2.OP_ATTENTION, 1, 16), dtype=torch.uint8, device="cuda")
    out = torch.empty((1, 16, 512), dtype=torch.bfloat16, device="cuda")
    q = torch.zeros((1, 16, 512), dtype=torch.bfloat16, device="cuda")
    csa2.csa2_sparse_attn(cache, q, qs, csa2.FULL, 0, iset, out, wa)
    assert csa2.csa2_check_device_error(cache) & csa2.DEVERR_POS
    assert csa2.csa2_check_device_error(cache) == 0   # cleared by the read
