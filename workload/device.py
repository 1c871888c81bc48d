"""GPU twin of the host generator (``gen_device.cu``): fills torch CUDA tensors with
the same seeded bf16 values that :mod:`workload` produces on the host."""
from __future__ import annotations

import ctypes
import os

import torch

from . import CUDA_LIB, D_LATENT, IDX_DIM, IDX_HEADS, Q_SCALE, TAG_IDXK, TAG_IDXQ, TAG_KV, TAG_Q
from . import kv_col_scale, stream_id

_lib = None


def cuda_lib():
    global _lib
    if _lib is None:
        if not os.path.exists(CUDA_LIB):
            raise RuntimeError(f"device generator library missing at {CUDA_LIB}: run "
                               "__graft_entry__.build() first")
        l = ctypes.CDLL(CUDA_LIB)
        l.wl_cuda_fill_normal_bf16.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64,
                                               ctypes.c_int64, ctypes.c_uint64, ctypes.c_uint64,
                                               ctypes.c_float, ctypes.c_void_p, ctypes.c_uint32,
                                               ctypes.c_void_p, ctypes.c_void_p]
        l.wl_cuda_fill_normal_bf16.restype = ctypes.c_int
        _lib = l
    return _lib


def fill_normal_bf16(out: torch.Tensor, seed: int, stream0: int, nbatch: int, per_batch: int,
                     start: int = 0, scale: float = 1.0, col_scale: torch.Tensor | None = None,
                     stream_stride: int = 1):
    assert out.is_cuda and out.is_contiguous() and out.element_size() == 2
    assert out.numel() >= nbatch * per_batch
    cs = None
    ncols = 0
    if col_scale is not None:
        assert col_scale.is_cuda and col_scale.dtype == torch.float32
        cs = col_scale.data_ptr()
        ncols = col_scale.numel()
    st = cuda_lib().wl_cuda_fill_normal_bf16(seed, stream0, stream_stride, nbatch, per_batch, start,
                                             scale, cs, ncols, out.data_ptr(),
                                             torch.cuda.current_stream().cuda_stream)
    if st != 0:
        raise RuntimeError(f"wl_cuda_fill_normal_bf16 failed with {st}")


def kv_rows(seed: int, seq: int, pos0: int, n: int, out: torch.Tensor | None = None,
            col_scale: torch.Tensor | None = None) -> torch.Tensor:
    """Device bf16 [n, 512] of the KV latent of one sequence (raw positions)."""
    if out is None:
        out = torch.empty((n, D_LATENT), dtype=torch.bfloat16, device="cuda")
    if col_scale is None:
        col_scale = torch.from_numpy(kv_col_scale(seed)).cuda()
    fill_normal_bf16(out, seed, stream_id(TAG_KV, 0, seq), 1, n * D_LATENT, pos0 * D_LATENT, 1.0,
                     col_scale)
    return out


def idxk_rows(seed: int, seq: int, pos0: int, n: int, out: torch.Tensor | None = None) -> torch.Tensor:
    if out is None:
        out = torch.empty((n, IDX_DIM), dtype=torch.bfloat16, device="cuda")
    fill_normal_bf16(out, seed, stream_id(TAG_IDXK, 0, seq), 1, n * IDX_DIM, pos0 * IDX_DIM)
    return out


def q_batch(seed: int, layer: int, query0: int, nq: int, heads: int,
            out: torch.Tensor | None = None) -> torch.Tensor:
    """Device bf16 [nq, heads, 512] attention queries of queries query0..query0+nq-1."""
    if out is None:
        out = torch.empty((nq, heads, D_LATENT), dtype=torch.bfloat16, device="cuda")
    fill_normal_bf16(out, seed, stream_id(TAG_Q, layer, query0), nq, heads * D_LATENT, 0, Q_SCALE)
    return out


def idxq_batch(seed: int, layer: int, query0: int, nq: int, out: torch.Tensor | None = None) -> torch.Tensor:
    """Device bf16 [nq, 4, 64] indexer queries."""
    if out is None:
        out = torch.empty((nq, IDX_HEADS, IDX_DIM), dtype=torch.bfloat16, device="cuda")
    fill_normal_bf16(out, seed, stream_id(TAG_IDXQ, layer, query0), nq, IDX_HEADS * IDX_DIM)
    return out
