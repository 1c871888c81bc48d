"""Seeded synthetic inputs shared by the parity tests, the benchmark and the oracle.

This package holds no CSA2 arithmetic.  It draws every input of the five
workloads from one counter-based SplitMix64 stream (definition in
``include/csa2_workload.h``), so that any single row can be regenerated on its
own, on the host (``gen.c``, through ctypes here) or on the GPU
(``gen_device.cu``, see :mod:`workload.device`), with identical bits.

Value recipe (the distributions the workloads name):

* KV latent rows: N(0,1) per element, rounded to bf16; five seeded channels
  (1 % of 512) are multiplied by 8 before rounding (outlier channels).
* Indexer keys and indexer queries: N(0,1) bf16, 4 query heads x 64, one
  shared 64-d key per token.
* Attention queries: N(0,1) * fp32(1/sqrt(512)), rounded to bf16.
* Page tables: a seeded permutation of the page pool.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
HOST_LIB = os.path.join(_HERE, "libcsa2_workload_host.so")
CUDA_LIB = os.path.join(_HERE, "libcsa2_workload_cuda.so")

D_LATENT = 512
IDX_HEADS = 4
IDX_DIM = 64
PAGE_TOKENS = 64

# stream tags: stream id = tag << 56 | layer << 40 | index
TAG_KV = 1
TAG_IDXK = 2
TAG_Q = 3
TAG_IDXQ = 4
TAG_OUTLIER = 5
TAG_PAGES = 6
TAG_LENS = 7
TAG_MISS = 8
TAG_MODES = 9

Q_SCALE = float(np.float32(1.0 / math.sqrt(512.0)))


def stream_id(tag: int, layer: int = 0, index: int = 0) -> int:
    assert 0 <= tag < 256 and 0 <= layer < (1 << 16) and 0 <= index < (1 << 40)
    return (tag << 56) | (layer << 40) | index


def build_host(force: bool = False) -> str:
    """Compile gen.c into the host generator library (gcc, a second or so)."""
    src = os.path.join(_HERE, "gen.c")
    if force or not os.path.exists(HOST_LIB) or os.path.getmtime(HOST_LIB) < os.path.getmtime(src):
        tmp = HOST_LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
                               "-ffp-contract=off", src, "-o", tmp])
        os.replace(tmp, HOST_LIB)
    return HOST_LIB


def build_cuda(force: bool = False) -> str:
    """Compile gen_device.cu into the device generator library (nvcc, sm_100a)."""
    src = os.path.join(_HERE, "gen_device.cu")
    hdr = os.path.join(_HERE, "..", "include", "csa2_workload.h")
    newest = max(os.path.getmtime(src), os.path.getmtime(hdr))
    if force or not os.path.exists(CUDA_LIB) or os.path.getmtime(CUDA_LIB) < newest:
        tmp = CUDA_LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["nvcc", "-O3", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
                               "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
                               "-fmad=false", src, "-o", tmp])
        os.replace(tmp, CUDA_LIB)
    return CUDA_LIB


_lib = None


def host_lib():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build_host())
        u64, f32, i64, u32 = ctypes.c_uint64, ctypes.c_float, ctypes.c_int64, ctypes.c_uint32
        vp = ctypes.c_void_p
        lib.wl_key.argtypes = [u64, u64]
        lib.wl_key.restype = u64
        lib.wl_u64.argtypes = [u64, u64]
        lib.wl_u64.restype = u64
        lib.wl_splitmix64_next.argtypes = [ctypes.POINTER(u64)]
        lib.wl_splitmix64_next.restype = u64
        lib.wl_normal.argtypes = [u64, u64]
        lib.wl_normal.restype = f32
        lib.wl_bf16.argtypes = [f32]
        lib.wl_bf16.restype = ctypes.c_uint16
        lib.wl_fill_normal_bf16.argtypes = [u64, u64, u64, u64, f32, vp, u32, vp, ctypes.c_int]
        lib.wl_fill_normal_bf16.restype = None
        lib.wl_fill_normal_f32.argtypes = [u64, u64, u64, u64, vp]
        lib.wl_fill_normal_f32.restype = None
        lib.wl_fill_u32.argtypes = [u64, u64, u64, u64, vp]
        lib.wl_fill_u32.restype = None
        lib.wl_permutation.argtypes = [u64, u64, i64, vp]
        lib.wl_permutation.restype = None
        _lib = lib
    return _lib


def _nthreads() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def normal_bf16(seed: int, stream: int, start: int, n: int, scale: float = 1.0,
                col_scale: np.ndarray | None = None) -> np.ndarray:
    """bf16 bit patterns (uint16) of n consecutive normal draws of one stream."""
    out = np.empty(n, dtype=np.uint16)
    cs = None
    ncols = 0
    if col_scale is not None:
        cs = np.ascontiguousarray(col_scale, dtype=np.float32)
        ncols = cs.size
    host_lib().wl_fill_normal_bf16(seed, stream, start, n, scale,
                                   None if cs is None else cs.ctypes.data, ncols,
                                   out.ctypes.data, _nthreads())
    return out


def normal_f32(seed: int, stream: int, start: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.float32)
    host_lib().wl_fill_normal_f32(seed, stream, start, n, out.ctypes.data)
    return out


def uniform_u32(seed: int, stream: int, start: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.uint32)
    host_lib().wl_fill_u32(seed, stream, start, n, out.ctypes.data)
    return out


def permutation(seed: int, stream: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.int32)
    host_lib().wl_permutation(seed, stream, n, out.ctypes.data)
    return out


# ---------------------------------------------------------------------------
# per-tensor recipes
# ---------------------------------------------------------------------------

def outlier_channels(seed: int) -> np.ndarray:
    """The five outlier channels (1 % of 512) of a workload, ascending."""
    perm = permutation(seed, stream_id(TAG_OUTLIER), D_LATENT)
    return np.sort(perm[:5]).astype(np.int64)


def kv_col_scale(seed: int) -> np.ndarray:
    s = np.ones(D_LATENT, dtype=np.float32)
    s[outlier_channels(seed)] = 8.0
    return s


def kv_rows(seed: int, seq: int, pos0: int, n: int) -> np.ndarray:
    """bf16 bits [n, 512] of the KV latent of sequence `seq`, positions pos0..pos0+n-1
    (raw, uncompressed token coordinates)."""
    flat = normal_bf16(seed, stream_id(TAG_KV, 0, seq), pos0 * D_LATENT, n * D_LATENT,
                       1.0, kv_col_scale(seed))
    return flat.reshape(n, D_LATENT)


def idxk_rows(seed: int, seq: int, pos0: int, n: int) -> np.ndarray:
    """bf16 bits [n, 64] of the indexer key of sequence `seq` (raw token coordinates)."""
    flat = normal_bf16(seed, stream_id(TAG_IDXK, 0, seq), pos0 * IDX_DIM, n * IDX_DIM)
    return flat.reshape(n, IDX_DIM)


def q_rows(seed: int, layer: int, query: int, heads: int) -> np.ndarray:
    """bf16 bits [heads, 512] of the attention query of (layer, query)."""
    flat = normal_bf16(seed, stream_id(TAG_Q, layer, query), 0, heads * D_LATENT, Q_SCALE)
    return flat.reshape(heads, D_LATENT)


def idxq_rows(seed: int, layer: int, query: int) -> np.ndarray:
    """bf16 bits [4, 64] of the indexer query of (layer, query)."""
    flat = normal_bf16(seed, stream_id(TAG_IDXQ, layer, query), 0, IDX_HEADS * IDX_DIM)
    return flat.reshape(IDX_HEADS, IDX_DIM)


def page_table(seed: int, n_pages_pool: int, pages_per_seq: list[int], max_pages: int) -> np.ndarray:
    """[B, max_pages] int32 page ids drawn without replacement from a seeded
    permutation of the pool; unused slots are -1."""
    need = int(sum(pages_per_seq))
    if need > n_pages_pool:
        raise ValueError(f"pool of {n_pages_pool} pages cannot hold {need}")
    perm = permutation(seed, stream_id(TAG_PAGES), n_pages_pool)
    pt = np.full((len(pages_per_seq), max_pages), -1, dtype=np.int32)
    off = 0
    for b, n in enumerate(pages_per_seq):
        pt[b, :n] = perm[off:off + n]
        off += n
    return pt


def log_uniform_lengths(seed: int, n: int, lo: int, hi: int) -> np.ndarray:
    """Context lengths log-uniform on [lo, hi] (host only; integers are passed
    to both sides)."""
    u = uniform_u32(seed, stream_id(TAG_LENS), 0, n).astype(np.float64) / 2.0 ** 32
    lens = np.floor(np.exp(math.log(lo) + u * (math.log(hi) - math.log(lo)))).astype(np.int64)
    return np.clip(lens, lo, hi)


def seeded_subset(seed: int, tag: int, n: int, count: int) -> np.ndarray:
    """Boolean mask of `count` of n items chosen by a seeded permutation."""
    perm = permutation(seed, stream_id(tag), n)
    mask = np.zeros(n, dtype=bool)
    mask[perm[:count]] = True
    return mask


# ---------------------------------------------------------------------------
# the five workloads
# ---------------------------------------------------------------------------

POOL_BYTES_4G = 4 * 1024 ** 3
ROW_BYTES = 288
PAGE_BYTES = ROW_BYTES * PAGE_TOKENS


@dataclass
class Workload:
    cid: int
    name: str
    seed: int
    batch: int
    heads: int
    layers: list[str]              # per-layer mode: "F" Full, "RI" Reindex, "R" Reuse
    lengths: list[int] = field(default_factory=list)  # per-sequence context (entries)
    n_pages_pool: int = 0
    hierarchical: bool = True
    compress: int = 1
    chunk: int = 0                 # prefill query chunk (raw tokens), 0 = decode
    raw_tokens: int = 0            # prefill: raw tokens per sequence
    reindex_mask: np.ndarray | None = None   # config 4: which sequences are in Reindex
    miss_mask: np.ndarray | None = None      # config 4: replay cache misses

    @property
    def max_pages(self) -> int:
        return max((l + PAGE_TOKENS - 1) // PAGE_TOKENS for l in self.lengths)


def workload(cid: int) -> Workload:
    """The five seeded synthetic workloads (shapes and distributions as named
    for the CSA2 decode/prefill step; seeds 0..4)."""
    n_pool_4g = POOL_BYTES_4G // PAGE_BYTES          # 233,016 pages of 18,432 B
    if cid == 0:
        return Workload(0, "tiny decode: B=1, L=4096, H=16, one Full layer", 0, 1, 16, ["F"],
                        [4096], 256)
    if cid == 1:
        return Workload(1, "decode: B=32, L=65536, H=64, layers F,R,R,R,RI,R,R,R, 4 GiB paged pool",
                        1, 32, 64, ["F", "R", "R", "R", "RI", "R", "R", "R"], [65536] * 32,
                        n_pool_4g)
    if cid == 2:
        layers = ["F", "R", "R", "R"] + ["RI", "R", "R", "R"] * 4
        return Workload(2, "long decode: B=4, L=1048576, H=64, 20 layers", 2, 4, 64, layers,
                        [1048576] * 4, n_pool_4g)
    if cid == 3:
        return Workload(3, "chunked prefill: 131072 tokens at ratio 2, 8192-token chunks, F+5R",
                        3, 1, 64, ["F", "R", "R", "R", "R", "R"], [65536], n_pool_4g,
                        hierarchical=False, compress=2, chunk=8192, raw_tokens=131072)
    if cid == 4:
        lens = [int(x) for x in log_uniform_lengths(4, 64, 4096, 1048576)]
        need = sum((l + PAGE_TOKENS - 1) // PAGE_TOKENS for l in lens)
        return Workload(4, "ragged decode: B=64, L log-uniform 4K..1M, 16 Reindex + 48 Reuse, "
                        "replay with 6 misses", 4, 64, 64, ["RI/R"], lens, max(n_pool_4g, need),
                        reindex_mask=seeded_subset(4, TAG_MODES, 64, 16),
                        miss_mask=seeded_subset(4, TAG_MISS, 64, 6))
    raise ValueError(cid)
