"""Thin Python binding of the CSA2 C ABI (``include/csa2.h``, ``lib/libcsa2.so``).

Argument marshalling only: every function below checks tensor dtypes/devices,
passes raw device pointers and the current torch CUDA stream to the C entry
point of the same name, and raises :class:`Csa2Error` on a non-zero status.
All computation happens in the library's CUDA kernels; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

from . import _build

FULL, REINDEX, REUSE = 0, 1, 2
OP_INDEXER, OP_ATTENTION = 1, 2
OP_SHARD_INDEXER, OP_SHARD_MERGE, OP_SHARD_ATTENTION = 3, 4, 5
SHARD_BLOCKS, SHARD_TOKENS = 0, 1
LATENT_DIM = 512
ROW_BYTES = 288
PAGE_TOKENS = 64
PAGE_BYTES = ROW_BYTES * PAGE_TOKENS
IDX_PAGE_BYTES = 64 * 128
IDX8_PAGE_BYTES = 64 * 64 + 64 * 4   # FP8 indexer keys: codes, then fp32 scales
IDXK_BF16, IDXK_FP8 = 0, 1
HIER_FLAT, HIER_MEAN, HIER_MAX = 0, 1, 2   # indexer candidate sets (hierarchical argument)
BK_PAGE_BYTES = 8 * 128
TOP_K = 512
POOL_BLOCKS = 2048
WINDOW = 128
REPLAY = 128          # entries rewritten by bounded replay; slots of the sliding-window store

DEVERR_PAGE, DEVERR_POS, DEVERR_SEQ = 1, 2, 4


class Csa2Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


class CacheStruct(ctypes.Structure):
    _fields_ = [
        ("kv_pool", ctypes.c_void_p),
        ("idxk_pool", ctypes.c_void_p),
        ("blockkey_pool", ctypes.c_void_p),
        ("n_pages", ctypes.c_int64),
        ("page_table", ctypes.c_void_p),
        ("max_pages", ctypes.c_int32),
        ("batch", ctypes.c_int32),
        ("seq_lens", ctypes.c_void_p),
        ("error_word", ctypes.c_void_p),
        ("cache_id", ctypes.c_uint64),
        ("swa_rows", ctypes.c_void_p),
        ("idxk_format", ctypes.c_int32),
    ]


class IndexSetStruct(ctypes.Structure):
    _fields_ = [
        ("idx", ctypes.c_void_p),
        ("pool_blocks", ctypes.c_void_p),
        ("rows", ctypes.c_int32),
        ("layer", ctypes.c_int32),
        ("mode", ctypes.c_int32),
        ("pool_layer", ctypes.c_int32),
        ("cache_id", ctypes.c_uint64),
        ("nq", ctypes.c_int32),
        ("attn_rows", ctypes.c_void_p),
        ("rows_layer", ctypes.c_int32),
        ("rows_split", ctypes.c_int32),
        ("rows_nq", ctypes.c_int32),
    ]


ATTN_ROWS_INTS = 648


# every entry point declared in include/csa2.h, with its ctypes signature
_VP, _I32, _I64, _F32, _SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
SIGNATURES = {
    "csa2_indexset_init": (None, [_VP, _VP, _VP, _I32]),
    "csa2_indexset_attach_rows": (None, [_VP, _VP]),
    "csa2_kv_quant_append": (ctypes.c_int, [_VP, _VP, _VP, _VP, _VP, _I32, _I32, _VP]),
    "csa2_indexer_score_topk": (ctypes.c_int, [_VP, _VP, _VP, _VP, _VP, _I32, _I64, _I32, _I32, _I32,
                                               _VP, _VP, _SZ, _VP]),
    "csa2_sparse_attn": (ctypes.c_int, [_VP, _VP, _I32, _F32, _VP, _VP, _I32, _I32, _I32, _VP, _VP,
                                        _VP, _SZ, _VP]),
    "csa2_indexer_score_topk_noalloc": (ctypes.c_int, [_VP, _VP, _VP, _VP, _VP, _I32, _I64, _I32, _I32,
                                                       _I32, _VP, _VP]),
    "csa2_swa_replay": (ctypes.c_int, [_VP, _VP, _VP, _VP, ctypes.c_int32, _VP]),
    "csa2_shard_indexer_candidates": (ctypes.c_int, [_VP, _VP, _VP, _VP, _VP, _I32, _I64, _I32, _VP, _VP,
                                                     _VP, _VP, _SZ, _VP]),
    "csa2_shard_merge_topk": (ctypes.c_int, [_VP, _VP, _I32, _I32, _I32, _I64, _I64, _I32, _VP, _VP, _VP,
                                             _SZ, _VP]),
    "csa2_sparse_attn_shard": (ctypes.c_int, [_VP, _VP, _I32, _F32, _VP, _VP, _VP, _VP, _I32, _VP, _VP,
                                              _VP, _SZ, _VP]),
    "csa2_shard_combine": (ctypes.c_int, [_VP, _VP, _I32, _I32, _I32, _I64, _I64, _VP, _VP]),
    "csa2_workspace_bytes": (_SZ, [_I32, _I32, _I32, _I64, _I32]),
    "csa2_check_device_error": (ctypes.c_int, [_VP, _VP, ctypes.POINTER(ctypes.c_uint32)]),
    "csa2_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "csa2_version": (ctypes.c_int, []),
}

_lib = None


def lib():
    """The loaded library.  Raises if it has not been built (no fallback path)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_build.LIB):
            raise RuntimeError(f"CSA2 CUDA library missing at {_build.LIB}: run "
                               "__graft_entry__.build() (nvcc, sm_100a) first")
        l = ctypes.CDLL(_build.LIB)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(l, name)
            f.restype = res
            f.argtypes = args
        _lib = l
    return _lib


def status_string(status: int) -> str:
    return lib().csa2_status_string(status).decode()


def _check(status: int, where: str):
    if status != 0:
        raise Csa2Error(status, where)


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t: torch.Tensor | None, dtypes, name: str, numel: int | None = None) -> int | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype not in dtypes:
        raise ValueError(f"{name}: dtype {t.dtype} not in {dtypes}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if numel is not None and t.numel() < numel:
        raise ValueError(f"{name}: {t.numel()} elements, need {numel}")
    return t.data_ptr()


_BF16 = (torch.bfloat16, torch.int16, torch.uint16)
_I32T = (torch.int32,)


class Cache:
    """Paged FP4 cache: three page pools, page table, lengths, error word,
    (swa_store=True) a separate sliding-window store [batch, 128, 288] bytes, and
    the indexer-key format (IDXK_BF16 or IDXK_FP8)."""

    def __init__(self, n_pages: int, batch: int, max_pages: int, device="cuda", cache_id: int = 1,
                 swa_store: bool = False, idxk_format: int = IDXK_BF16):
        dev = torch.device(device)
        self.n_pages, self.batch, self.max_pages = n_pages, batch, max_pages
        self.kv_pool = torch.zeros(n_pages * PAGE_BYTES, dtype=torch.uint8, device=dev)
        self.idxk_format = idxk_format
        kpage = IDX8_PAGE_BYTES if idxk_format == IDXK_FP8 else IDX_PAGE_BYTES
        self.idxk_pool = torch.zeros(n_pages * kpage, dtype=torch.uint8, device=dev)
        self.bk_pool = torch.zeros(n_pages * BK_PAGE_BYTES, dtype=torch.uint8, device=dev)
        self.page_table = torch.full((batch, max_pages), -1, dtype=torch.int32, device=dev)
        self.seq_lens = torch.zeros(batch, dtype=torch.int32, device=dev)
        self.error_word = torch.zeros(1, dtype=torch.int32, device=dev)
        self.cache_id = cache_id
        self.swa_rows = (torch.zeros((batch, REPLAY, ROW_BYTES), dtype=torch.uint8, device=dev)
                         if swa_store else None)
        self.struct = CacheStruct()
        self.refresh()

    def refresh(self):
        s = self.struct
        s.kv_pool = self.kv_pool.data_ptr()
        s.idxk_pool = self.idxk_pool.data_ptr()
        s.blockkey_pool = self.bk_pool.data_ptr()
        s.n_pages = self.n_pages
        s.page_table = self.page_table.data_ptr()
        s.max_pages = self.max_pages
        s.batch = self.batch
        s.seq_lens = self.seq_lens.data_ptr()
        s.error_word = self.error_word.data_ptr()
        s.cache_id = self.cache_id
        s.swa_rows = None if self.swa_rows is None else self.swa_rows.data_ptr()
        s.idxk_format = self.idxk_format

    def ref(self):
        return ctypes.byref(self.struct)


class IndexSet:
    """Device index rows [rows, 512] + pool rows [rows, 2048], the attention row
    cache [rows, ATTN_ROWS_INTS] (row_cache=False leaves it out) and the mode tags."""

    def __init__(self, rows: int, device="cuda", row_cache: bool = True):
        dev = torch.device(device)
        self.idx = torch.full((rows, TOP_K), -1, dtype=torch.int32, device=dev)
        self.pool_blocks = torch.full((rows, POOL_BLOCKS), -1, dtype=torch.int32, device=dev)
        self.struct = IndexSetStruct()
        lib().csa2_indexset_init(ctypes.byref(self.struct), self.idx.data_ptr(),
                                 self.pool_blocks.data_ptr(), rows)
        self.attn_rows = None
        if row_cache:
            self.attn_rows = torch.zeros((rows, ATTN_ROWS_INTS), dtype=torch.int32, device=dev)
            lib().csa2_indexset_attach_rows(ctypes.byref(self.struct), self.attn_rows.data_ptr())

    def detach_rows(self):
        lib().csa2_indexset_attach_rows(ctypes.byref(self.struct), None)
        self.attn_rows = None

    def ref(self):
        return ctypes.byref(self.struct)

    @property
    def layer(self):
        return self.struct.layer

    @property
    def mode(self):
        return self.struct.mode


def csa2_workspace_bytes(op: int, nq: int, heads: int = 0, max_visible: int = 0,
                         hierarchical: bool = True) -> int:
    return int(lib().csa2_workspace_bytes(op, nq, heads, max_visible, int(hierarchical)))


def csa2_kv_quant_append(cache: Cache, kv: torch.Tensor, idxk: torch.Tensor, entry_seq: torch.Tensor,
                         entry_pos: torch.Tensor, compress: int = 1, stream=None):
    n = entry_seq.numel()
    if entry_pos.numel() != n:
        raise ValueError("entry_seq and entry_pos differ in length")
    st = lib().csa2_kv_quant_append(
        cache.ref(), _ptr(kv, _BF16, "kv", n * compress * LATENT_DIM),
        _ptr(idxk, _BF16, "idxk", n * compress * 64), _ptr(entry_seq, _I32T, "entry_seq"),
        _ptr(entry_pos, _I32T, "entry_pos"), n, compress, _stream(stream))
    _check(st, "csa2_kv_quant_append")


def csa2_indexer_score_topk(cache: Cache, idx_q: torch.Tensor, q_seq: torch.Tensor, mode: int,
                            layer: int, indexset: IndexSet, workspace: torch.Tensor, max_visible: int,
                            q_visible: torch.Tensor | None = None, head_w: torch.Tensor | None = None,
                            hierarchical: bool = True, stream=None):
    nq = q_seq.numel()
    st = lib().csa2_indexer_score_topk(
        cache.ref(), _ptr(idx_q, _BF16, "idx_q", nq * 256),
        _ptr(head_w, (torch.float32,), "head_w", nq * 4), _ptr(q_seq, _I32T, "q_seq"),
        _ptr(q_visible, _I32T, "q_visible", nq), nq, int(max_visible), mode, int(hierarchical),
        layer, indexset.ref(), _ptr(workspace, (torch.uint8,), "workspace"),
        workspace.numel(), _stream(stream))
    _check(st, "csa2_indexer_score_topk")


NOALLOC_SCRATCH_BYTES = 16 << 20


def csa2_indexer_score_topk_noalloc(cache: Cache, idx_q: torch.Tensor, q_seq: torch.Tensor, mode: int,
                                    layer: int, indexset: IndexSet, max_visible: int,
                                    q_visible: torch.Tensor | None = None,
                                    head_w: torch.Tensor | None = None, hierarchical: bool = True,
                                    stream=None):
    """csa2_indexer_score_topk for callers that cannot allocate: the score buffer is
    the library's own static device array (NOALLOC_SCRATCH_BYTES); calls that
    overlap on the GPU share it and race."""
    nq = q_seq.numel()
    st = lib().csa2_indexer_score_topk_noalloc(
        cache.ref(), _ptr(idx_q, _BF16, "idx_q", nq * 256),
        _ptr(head_w, (torch.float32,), "head_w", nq * 4), _ptr(q_seq, _I32T, "q_seq"),
        _ptr(q_visible, _I32T, "q_visible", nq), nq, int(max_visible), mode, int(hierarchical),
        layer, indexset.ref(), _stream(stream))
    _check(st, "csa2_indexer_score_topk_noalloc")


def csa2_sparse_attn(cache: Cache, q: torch.Tensor, q_seq: torch.Tensor, mode: int, layer: int,
                     indexset: IndexSet, out: torch.Tensor, workspace: torch.Tensor,
                     sm_scale: float = 1.0, q_visible: torch.Tensor | None = None, stream=None):
    nq = q_seq.numel()
    heads = q.shape[-2]
    st = lib().csa2_sparse_attn(
        cache.ref(), _ptr(q, _BF16, "q", nq * heads * LATENT_DIM), heads, float(sm_scale),
        _ptr(q_seq, _I32T, "q_seq"), _ptr(q_visible, _I32T, "q_visible", nq), nq, mode, layer,
        indexset.ref(), _ptr(out, _BF16, "out", nq * heads * LATENT_DIM),
        _ptr(workspace, (torch.uint8,), "workspace"), workspace.numel(), _stream(stream))
    _check(st, "csa2_sparse_attn")


def csa2_swa_replay(cache: Cache, kv_last: torch.Tensor, idxk_last: torch.Tensor | None, miss: torch.Tensor,
                    compress: int = 1, stream=None):
    b = cache.batch
    st = lib().csa2_swa_replay(
        cache.ref(), _ptr(kv_last, _BF16, "kv_last", b * REPLAY * compress * LATENT_DIM),
        _ptr(idxk_last, _BF16, "idxk_last", b * REPLAY * compress * 64),
        _ptr(miss, (torch.uint8, torch.bool), "miss", b), compress, _stream(stream))
    _check(st, "csa2_swa_replay")


def csa2_shard_indexer_candidates(cache: Cache, idx_q: torch.Tensor, q_seq: torch.Tensor,
                                  shard_offset: torch.Tensor, stage: int, cand_score: torch.Tensor,
                                  cand_id: torch.Tensor, workspace: torch.Tensor, max_visible: int,
                                  global_pool: torch.Tensor | None = None, head_w: torch.Tensor | None = None,
                                  stream=None):
    nq = q_seq.numel()
    k = POOL_BLOCKS if stage == SHARD_BLOCKS else TOP_K
    st = lib().csa2_shard_indexer_candidates(
        cache.ref(), _ptr(idx_q, _BF16, "idx_q", nq * 4 * 64), _ptr(head_w, (torch.float32,), "head_w", nq * 4),
        _ptr(q_seq, _I32T, "q_seq"), _ptr(shard_offset, _I32T, "shard_offset", nq), nq, int(max_visible),
        stage, _ptr(global_pool, _I32T, "global_pool", nq * POOL_BLOCKS),
        _ptr(cand_score, (torch.float32,), "cand_score", nq * k), _ptr(cand_id, _I32T, "cand_id", nq * k),
        _ptr(workspace, (torch.uint8,), "workspace"), workspace.numel(), _stream(stream))
    _check(st, "csa2_shard_indexer_candidates")


def csa2_shard_merge_topk(cand_score: torch.Tensor, cand_id: torch.Tensor, nshard: int, nq: int, n: int,
                          query_stride: int, shard_stride: int, k: int, out_id: torch.Tensor,
                          workspace: torch.Tensor, out_score: torch.Tensor | None = None, stream=None):
    st = lib().csa2_shard_merge_topk(
        _ptr(cand_score, (torch.float32,), "cand_score"), _ptr(cand_id, _I32T, "cand_id"), nshard, nq, n,
        query_stride, shard_stride, k, _ptr(out_id, _I32T, "out_id", nq * k),
        _ptr(out_score, (torch.float32,), "out_score", nq * k), _ptr(workspace, (torch.uint8,), "workspace"),
        workspace.numel(), _stream(stream))
    _check(st, "csa2_shard_merge_topk")


def csa2_sparse_attn_shard(cache: Cache, q: torch.Tensor, q_seq: torch.Tensor, shard_offset: torch.Tensor,
                           global_idx: torch.Tensor, window_start: torch.Tensor, out: torch.Tensor,
                           lse2: torch.Tensor, workspace: torch.Tensor, sm_scale: float = 1.0, stream=None):
    nq, heads = q.shape[0], q.shape[1]
    st = lib().csa2_sparse_attn_shard(
        cache.ref(), _ptr(q, _BF16, "q", nq * heads * LATENT_DIM), heads, float(sm_scale),
        _ptr(q_seq, _I32T, "q_seq", nq), _ptr(shard_offset, _I32T, "shard_offset", nq),
        _ptr(global_idx, _I32T, "global_idx", nq * TOP_K), _ptr(window_start, _I32T, "window_start", nq), nq,
        _ptr(out, _BF16, "out", nq * heads * LATENT_DIM), _ptr(lse2, (torch.float32,), "lse2", nq * heads),
        _ptr(workspace, (torch.uint8,), "workspace"), workspace.numel(), _stream(stream))
    _check(st, "csa2_sparse_attn_shard")


def csa2_shard_combine(part: torch.Tensor, lse2: torch.Tensor, nshard: int, nq: int, heads: int,
                       query_stride: int, shard_stride: int, out: torch.Tensor, stream=None):
    st = lib().csa2_shard_combine(
        _ptr(part, _BF16, "part"), _ptr(lse2, (torch.float32,), "lse2"), nshard, nq, heads, query_stride,
        shard_stride, _ptr(out, _BF16, "out", nq * heads * LATENT_DIM), _stream(stream))
    _check(st, "csa2_shard_combine")


def csa2_check_device_error(cache: Cache, stream=None) -> int:
    """Synchronise, read and clear the cache's device error word; returns its bits."""
    bits = ctypes.c_uint32(0)
    st = lib().csa2_check_device_error(cache.ref(), _stream(stream), ctypes.byref(bits))
    if st not in (0, 7):
        raise Csa2Error(st, "csa2_check_device_error")
    return int(bits.value)
