"""Host-side tests of the C ABI (no GPU): the library loads, exports every symbol the
headers declare, and rejects bad arguments and out-of-order layer modes on the host
before anything is launched."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared(header):
    text = open(os.path.join(ROOT, "include", header)).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b((?:csa2|wl|wl_cuda)_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol(csa2_lib):
    lib = csa2_lib.lib()
    names = _declared("csa2.h")
    assert "csa2_sparse_attn" in names and len(names) >= 9
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(csa2_lib.SIGNATURES)


def test_workload_libraries_export_declared_symbols(host_gen):
    import workload
    host = ctypes.CDLL(workload.build_host())
    dev = ctypes.CDLL(workload.build_cuda())
    for n in _declared("csa2_workload.h"):
        target = dev if n.startswith("wl_cuda_") else host
        assert hasattr(target, n), n


def test_status_strings_and_version(csa2_lib):
    for code in range(8):
        assert csa2_lib.status_string(code)
    assert csa2_lib.status_string(99) == "unknown status"
    assert csa2_lib.lib().csa2_version() >= 100


def test_workspace_sizes(csa2_lib):
    ws = csa2_lib.csa2_workspace_bytes
    # hierarchical decode at 64K: max(8192 block scores, 16384 pool scores) per query
    assert ws(1, 32, 0, 65536, True) == 32 * 16384 * 4 + 256
    # 1M: 131072 block scores per query dominate; the block top-2048 runs in 8
    # segments of 16384 whose candidates (8 x 2048 x 8 B per query) follow the scores
    assert ws(1, 4, 0, 1048576, True) == 4 * 131072 * 4 + 4 * 8 * 2048 * 8 + 256
    # flat encoder chunk: 8192 queries x 65536 entries (enough rows to fill the GPU:
    # one streaming top-k per row, no segments); 32 queries: 4 segments each
    assert ws(1, 8192, 0, 65536, False) == 8192 * 65536 * 4 + 256
    assert ws(1, 32, 0, 65536, False) == 32 * 65536 * 4 + 32 * 4 * 512 * 8 + 256
    # attention: 32 queries split 4 ways (4 x 32 <= 148 SMs) exchange f16 partials
    # [4][64][512]; 148 queries are not split
    assert ws(2, 32, 64, 0, False) == 32 * 4 * 64 * 512 * 2 + 256
    assert ws(2, 16, 32, 0, False) == 16 * 8 * 32 * 512 * 2 + 256
    assert ws(2, 148, 64, 0, False) == 0
    assert ws(2, 32, 20, 0, False) == 0          # unsupported head count
    assert ws(7, 1, 64, 0, False) == 0
    # max-pooled hierarchy: every token's score, then the 8,192 block maxima
    assert ws(1, 32, 0, 65536, 2) == 32 * (65536 + 8192) * 4 + 32 * 4 * 512 * 8 + 256
    assert ws(1, 3, 0, 100, 2) == 3 * (104 + 16) * 4 + 256
    assert ws(1, 32, 0, 65536, 3) == 0


class _Fake:
    """Host buffers whose addresses stand in for device pointers; the host-side
    checks under test never dereference them."""

    def __init__(self):
        self.buf = (ctypes.c_uint8 * 4096)()
        base = ctypes.addressof(self.buf)
        self.aligned = (base + 255) & ~255

    def p(self, off=0):
        return self.aligned + off


def _cache(csa2, f, **kw):
    c = csa2.CacheStruct()
    c.kv_pool = f.p(0)
    c.idxk_pool = f.p(256)
    c.blockkey_pool = f.p(512)
    c.n_pages = 4
    c.page_table = f.p(768)
    c.max_pages = 2
    c.batch = 2
    c.seq_lens = f.p(1024)
    c.error_word = f.p(1280)
    c.cache_id = 7
    for k, v in kw.items():
        setattr(c, k, v)
    return c


def _iset(csa2, f, rows=2):
    s = csa2.IndexSetStruct()
    csa2.lib().csa2_indexset_init(ctypes.byref(s), f.p(1536), f.p(2048), rows)
    return s


def test_append_argument_checks(csa2_lib):
    L = csa2_lib.lib()
    f = _Fake()
    c = _cache(csa2_lib, f)
    B = ctypes.byref
    assert L.csa2_kv_quant_append(None, f.p(), f.p(), f.p(), f.p(), 1, 1, None) == 1
    assert L.csa2_kv_quant_append(B(_cache(csa2_lib, f, kv_pool=None)), f.p(), f.p(), f.p(), f.p(), 1, 1, None) == 1
    assert L.csa2_kv_quant_append(B(_cache(csa2_lib, f, kv_pool=f.p(8))), f.p(), f.p(), f.p(), f.p(), 1, 1, None) == 3
    assert L.csa2_kv_quant_append(B(_cache(csa2_lib, f, batch=0)), f.p(), f.p(), f.p(), f.p(), 1, 1, None) == 2
    assert L.csa2_kv_quant_append(B(c), f.p(), f.p(), f.p(), f.p(), 1, 3, None) == 2
    assert L.csa2_kv_quant_append(B(c), f.p(), f.p(), f.p(), f.p(), -1, 1, None) == 1
    assert L.csa2_kv_quant_append(B(c), f.p(8), f.p(), f.p(), f.p(), 1, 1, None) == 3
    assert L.csa2_kv_quant_append(B(c), None, f.p(), f.p(), f.p(), 1, 1, None) == 1
    assert L.csa2_kv_quant_append(B(c), f.p(), f.p(), f.p(), f.p(), 0, 1, None) == 0


def test_mode_order_state_machine(csa2_lib):
    """Full -> Reuse -> Reindex -> Reuse ordering, exercised with zero-query calls
    (which update the host tags without launching anything)."""
    L = csa2_lib.lib()
    f = _Fake()
    c = _cache(csa2_lib, f)
    s = _iset(csa2_lib, f)
    B = ctypes.byref
    FULL, REINDEX, REUSE = 0, 1, 2
    attn = lambda mode, layer, heads=64, st=s: L.csa2_sparse_attn(
        B(c), f.p(), heads, 1.0, f.p(), None, 0, mode, layer, B(st), f.p(), f.p(), 1 << 20, None)
    idx = lambda mode, layer, hier=1, nq=0: L.csa2_indexer_score_topk(
        B(c), f.p(), None, f.p(), None, nq, 65536, mode, hier, layer, B(s), f.p(), 1 << 30, None)
    # nothing selected yet: Reuse and Reindex are out of order
    assert attn(REUSE, 1) == 4
    assert idx(REINDEX, 1) == 4
    # Full at layer 0 writes a pool and a set
    assert idx(FULL, 0) == 0
    assert s.layer == 0 and s.mode == FULL and s.pool_layer == 0 and s.cache_id == 7
    assert attn(FULL, 0) == 0
    assert attn(REINDEX, 0) == 4           # the set was made by a Full call
    assert attn(FULL, 1) == 4              # a Full layer attends over its own fresh set
    for layer in (1, 2, 3):
        assert attn(REUSE, layer) == 0
    assert attn(REUSE, 0) == 4             # Reuse needs an earlier layer's set
    assert attn(REUSE, 1, heads=20) == 2
    # Reindex at layer 4 ranks the layer-0 pool
    assert idx(REINDEX, 4) == 0
    assert s.layer == 4 and s.mode == REINDEX and s.pool_layer == 0
    assert attn(REINDEX, 4) == 0
    assert attn(REUSE, 3) == 4
    assert attn(REUSE, 5) == 0
    # a set computed on another cache is rejected
    c2 = _cache(csa2_lib, f, cache_id=8)
    assert L.csa2_sparse_attn(B(c2), f.p(), 64, 1.0, f.p(), None, 0, REUSE, 5, B(s), f.p(), f.p(),
                              1 << 20, None) == 4
    # a flat (encoder) Full call leaves no pool for a Reindex layer
    assert idx(FULL, 6, hier=0) == 0
    assert s.pool_layer == -1
    assert idx(REINDEX, 7) == 4
    # a max-pooled Full call leaves a pool for Reindex; an unknown block score is refused
    assert idx(FULL, 6, hier=2) == 0 and s.pool_layer == 6
    assert idx(REINDEX, 7) == 0
    assert idx(FULL, 8, hier=3) == 1
    # more queries than the set has rows
    assert idx(FULL, 8, nq=3) == 2
    # workspace too small
    assert L.csa2_indexer_score_topk(B(c), f.p(), None, f.p(), None, 2, 65536, FULL, 1, 9, B(s),
                                     f.p(), 16, None) == 5
    assert L.csa2_indexer_score_topk(B(c), f.p(8), None, f.p(), None, 2, 65536, FULL, 1, 9, B(s),
                                     f.p(), 1 << 30, None) == 3


def test_noalloc_checks_arguments_before_size(csa2_lib):
    """The entry point without a workspace reports argument and mode-order errors
    like the regular call, and refuses a valid request larger than its static
    array with CSA2_ERR_WORKSPACE; none of these launches anything."""
    L = csa2_lib.lib()
    f = _Fake()
    c = _cache(csa2_lib, f)
    s = _iset(csa2_lib, f, rows=64)
    B = ctypes.byref
    FULL, REINDEX = 0, 1
    big = 1 << 20                                  # 64 queries at 1M: far above 16 MiB
    assert csa2_lib.csa2_workspace_bytes(1, 64, 0, big, True) > csa2_lib.NOALLOC_SCRATCH_BYTES
    na = lambda mode, hier=1, cache=c, q=f.p(): L.csa2_indexer_score_topk_noalloc(
        B(cache), q, None, f.p(), None, 64, big, mode, hier, 3, B(s), None)
    assert na(REINDEX) == 4                        # no Full pool yet: mode order first
    assert na(FULL, hier=3) == 1                   # unknown block score
    assert na(FULL, q=f.p(8)) == 3                 # misaligned query
    assert na(FULL, cache=_cache(csa2_lib, f, batch=0)) == 2
    assert na(FULL) == 5                           # valid, but larger than the array
    assert s.layer == -1                           # nothing was recorded


def test_replay_and_cache_argument_checks(csa2_lib):
    L = csa2_lib.lib()
    f = _Fake()
    c = _cache(csa2_lib, f)
    B = ctypes.byref
    rep = lambda cache, kv, k, miss, comp: L.csa2_swa_replay(B(cache), kv, k, miss, comp, None)
    assert rep(c, f.p(), f.p(), f.p(), 3) == 2                 # compression ratio 1 or 2
    assert rep(c, f.p(), f.p(), f.p(), 0) == 2
    assert rep(c, f.p(), None, f.p(), 1) == 1                  # keys needed without a window store
    assert rep(c, None, f.p(), f.p(), 1) == 1
    assert rep(c, f.p(8), f.p(), f.p(), 2) == 3
    assert rep(_cache(csa2_lib, f, swa_rows=f.p(8)), f.p(), None, f.p(), 1) == 3   # store 16-B aligned
    # attention names rows by 31-bit ids: the pool and batch limits
    assert rep(_cache(csa2_lib, f, n_pages=(1 << 25) + 1), f.p(), f.p(), f.p(), 1) == 2
    assert rep(_cache(csa2_lib, f, batch=(1 << 23) + 1), f.p(), f.p(), f.p(), 1) == 2


def test_indexer_key_format_is_checked(csa2_lib):
    L = csa2_lib.lib()
    f = _Fake()
    B = ctypes.byref
    rep = lambda cache: L.csa2_swa_replay(B(cache), f.p(), f.p(), f.p(), 1, None)
    assert rep(_cache(csa2_lib, f, idxk_format=2)) == 1
    assert rep(_cache(csa2_lib, f, idxk_format=-1)) == 1
    assert L.csa2_kv_quant_append(B(_cache(csa2_lib, f, idxk_format=7)), f.p(), f.p(), f.p(), f.p(), 1, 1,
                                  None) == 1


def test_sharded_call_argument_checks(csa2_lib):
    L = csa2_lib.lib()
    f = _Fake()
    c = _cache(csa2_lib, f)
    B = ctypes.byref
    ws = csa2_lib.csa2_workspace_bytes
    assert ws(3, 4, 0, 40000, 0) == 4 * (16384 + 2048) * 4 + 256
    assert ws(4, 4, 8, 2048, 0) == 4 * 8 * 2048 * 8 + 256
    assert ws(4, 4, 8, 12, 0) == 0                      # candidates per shard: a multiple of 8
    assert ws(5, 4, 20, 0, 0) == 0
    cand = lambda stage, pool=None, wsz=1 << 30: L.csa2_shard_indexer_candidates(
        B(c), f.p(), None, f.p(), f.p(), 2, 40000, stage, pool, f.p(), f.p(), f.p(), wsz, None)
    assert cand(2) == 1                                 # unknown stage
    assert cand(1) == 1                                 # the token stage needs the pool
    assert cand(0, wsz=16) == 5
    merge = lambda nshard, n, k, wsz=1 << 30: L.csa2_shard_merge_topk(
        f.p(), f.p(), nshard, 2, n, 1, 2, k, f.p(), None, f.p(), wsz, None)
    assert merge(0, 2048, 2048) == 1
    assert merge(2, 12, 8) == 1
    assert merge(2, 2048, 0) == 1
    assert merge(2, 2048, 2048, wsz=100) == 5
    attn = lambda heads, wsz=1 << 30: L.csa2_sparse_attn_shard(
        B(c), f.p(), heads, ctypes.c_float(1.0), f.p(), f.p(), f.p(), f.p(), 2, f.p(), f.p(), f.p(), wsz, None)
    assert attn(20) == 2
    assert attn(64, wsz=0) == 5
    assert L.csa2_shard_combine(f.p(), f.p(), 0, 2, 64, 1, 2, f.p(), None) == 1
    assert L.csa2_shard_combine(f.p(), f.p(), 2, 2, 24, 1, 2, f.p(), None) == 2
    assert L.csa2_shard_combine(f.p(8), f.p(), 2, 2, 64, 1, 2, f.p(), None) == 3
