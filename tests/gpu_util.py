"""GPU-test helpers: read cache bytes back through the page table, build small caches."""
from __future__ import annotations

import numpy as np
import torch

import workload as wl


def bits(t: torch.Tensor) -> np.ndarray:
    """bf16 / int16 CUDA tensor -> host uint16 bit patterns."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _byte_index(pt_row: np.ndarray, positions, page_bytes: int, row_bytes: int) -> np.ndarray:
    pos = np.asarray(positions, dtype=np.int64)
    pages = pt_row[pos >> 6].astype(np.int64)
    base = pages * page_bytes + (pos & 63) * row_bytes
    return base[:, None] + np.arange(row_bytes)[None, :]


def cache_rows(cache, seq: int, positions) -> np.ndarray:
    """The 288-B FP4 rows of the given positions, read from the GPU pool."""
    pt = cache.page_table[seq].cpu().numpy()
    idx = torch.from_numpy(_byte_index(pt, positions, 18432, 288)).cuda()
    return cache.kv_pool[idx].cpu().numpy()


def cache_keys(cache, seq: int, positions) -> np.ndarray:
    pt = cache.page_table[seq].cpu().numpy()
    idx = torch.from_numpy(_byte_index(pt, positions, 8192, 128)).cuda()
    return cache.idxk_pool[idx].cpu().numpy().view(np.uint16).reshape(-1, 64)


def cache_keys_fp8(cache, seq: int, positions) -> tuple[np.ndarray, np.ndarray]:
    """(E4M3 codes [n, 64], fp32 scales [n]) of the given positions of an FP8 key cache."""
    pt = cache.page_table[seq].cpu().numpy()
    pos = np.asarray(positions, dtype=np.int64)
    pages = pt[pos >> 6].astype(np.int64)
    cidx = (pages * 4352 + (pos & 63) * 64)[:, None] + np.arange(64)[None, :]
    sidx = (pages * 4352 + 4096 + (pos & 63) * 4)[:, None] + np.arange(4)[None, :]
    pool = cache.idxk_pool
    codes = pool[torch.from_numpy(cidx).cuda()].cpu().numpy()
    scales = pool[torch.from_numpy(sidx).cuda()].cpu().numpy().copy().view(np.float32).reshape(-1)
    return codes, scales


def cache_block_keys(cache, seq: int, blocks) -> np.ndarray:
    pt = cache.page_table[seq].cpu().numpy()
    blk = np.asarray(blocks, dtype=np.int64)
    pages = pt[blk >> 3].astype(np.int64)
    base = pages * 1024 + (blk & 7) * 128
    idx = torch.from_numpy(base[:, None] + np.arange(128)[None, :]).cuda()
    return cache.bk_pool[idx].cpu().numpy().view(np.uint16).reshape(-1, 64)


def small_workload(lengths, seed=10, heads=64, spare_pages=16) -> wl.Workload:
    pages = sum((L + 63) // 64 for L in lengths)
    return wl.Workload(cid=-1, name="test", seed=seed, batch=len(lengths), heads=heads, layers=["F"],
                       lengths=list(lengths), n_pages_pool=max(1, pages + spare_pages))
