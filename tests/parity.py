"""Parity helpers shared by the GPU tests: oracle-side views of a seeded workload
(generated on the host, never read back from the GPU) and the comparison rules.

Rules (fixed for the CSA2 step):
* FP4 codes, scale bytes, stored indexer keys and block keys: bit-exact;
* index sets: exact, except boundary swaps whose oracle scores lie within
  1e-4 * |k-th score| of the k-th best score (counted and returned);
* attention output (bf16): max |gpu - oracle| <= 1e-2 * max |oracle| + 1e-3.
"""
from __future__ import annotations

import numpy as np

import workload as wl
from oracle import attention as oattn
from oracle import codec as ocodec
from oracle import indexer as oidx

REL_TIE = 1e-4


class OracleSeq:
    """Host-generated view of one sequence of a workload, in entry coordinates."""

    def __init__(self, w: wl.Workload, seq: int, length: int, compress: int = 1):
        self.w, self.seq, self.length, self.compress = w, seq, length, compress
        self._keys = None

    @property
    def keys(self) -> np.ndarray:
        if self._keys is None:
            raw = wl.idxk_rows(self.w.seed, self.seq, 0, self.length * self.compress)
            self._keys = ocodec.idxk_entries(raw, self.compress)
        return self._keys

    def encoded_rows(self, positions) -> np.ndarray:
        """288-B cache rows (oracle codec) of the given entry positions."""
        pos = np.asarray(positions, dtype=np.int64)
        out = np.empty((pos.size, ocodec.ROW_BYTES), dtype=np.uint8)
        # group contiguous runs to keep the generator calls few
        i = 0
        while i < pos.size:
            j = i
            while j + 1 < pos.size and pos[j + 1] == pos[j] + 1:
                j += 1
            n = j - i + 1
            raw = wl.kv_rows(self.w.seed, self.seq, int(pos[i]) * self.compress, n * self.compress)
            out[i:j + 1] = ocodec.encode_entries(raw, self.compress)
            i = j + 1
        return out

    def rows(self, positions) -> np.ndarray:
        codes, scales = ocodec.unpack_rows(self.encoded_rows(positions))
        return ocodec.dequantize(codes, scales)


def check_index_set(gpu_idx, oracle_idx, score_of, what="index set") -> int:
    """Compare a GPU index set with the oracle's.  score_of(positions) returns the
    oracle's fp32 scores.  Returns the number of allowed boundary swaps."""
    g = np.asarray(gpu_idx, dtype=np.int64)
    o = np.asarray(oracle_idx, dtype=np.int64)
    gs = g[g >= 0]
    os_ = o[o >= 0]
    assert gs.size == os_.size, f"{what}: {gs.size} selected vs oracle {os_.size}"
    assert np.all(np.diff(gs) > 0), f"{what}: not strictly ascending"
    assert np.all(g[gs.size:] == -1), f"{what}: padding is not -1"
    if np.array_equal(gs, os_):
        return 0
    diff = np.setxor1d(gs, os_)
    kth = float(np.min(score_of(os_)))
    sc = score_of(diff).astype(np.float64)
    bad = np.abs(sc - kth) > REL_TIE * abs(kth)
    assert not np.any(bad), (f"{what}: {int(bad.sum())} of {diff.size} differing positions are not "
                             f"near-ties of the k-th score {kth}: {diff[bad][:8]} {sc[bad][:8]}")
    return int(np.setdiff1d(gs, os_).size)


def attention_error(gpu_bf16_bits: np.ndarray, oracle: np.ndarray) -> tuple[float, float]:
    """(max |gpu - oracle|, allowed bound) for one query's [H, 512] output."""
    from oracle.formats import bf16_to_f64
    g = bf16_to_f64(gpu_bf16_bits)
    err = float(np.max(np.abs(g - oracle))) if oracle.size else 0.0
    bound = 1e-2 * float(np.max(np.abs(oracle))) + 1e-3
    return err, bound


def oracle_full(oseq: OracleSeq, idxq_bits, visible: int, hierarchical: bool = True):
    """Oracle Full indexer for one query (decoder hierarchical or encoder flat)."""
    if hierarchical:
        return oidx.full_indexer(idxq_bits, oseq.keys, visible, hierarchical=True)
    idx, info = oidx.flat_indexer(idxq_bits, oseq.keys, visible)
    return None, idx, info


def oracle_attention(oseq: OracleSeq, idx, q_bits, visible: int, sm_scale: float = 1.0):
    pos = oattn.attended_positions(idx, visible)
    return oattn.attend(q_bits, oseq.rows(pos), sm_scale)


def token_scorer(oseq: OracleSeq, idxq_bits):
    """score_of(positions) with the oracle's fp32 indexer score."""
    return lambda p: oidx.index_scores(idxq_bits, oseq.keys[np.asarray(p, dtype=np.int64)])


def block_scorer(oseq: OracleSeq, idxq_bits, visible: int):
    kb = oidx.block_keys(oseq.keys, visible)
    return lambda b: oidx.index_scores(idxq_bits, kb[np.asarray(b, dtype=np.int64)])
