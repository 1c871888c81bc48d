"""The C restatement of the CSA2 decode oracle (``oracle/c/csa2_oracle.c``),
through ctypes -- TEST INFRASTRUCTURE ONLY.

A second CPU oracle, written in plain C independently of this package's
numpy functions (it shares no code with them or with the CUDA path): the FP4
codec, block keys, fp32 indexer scores, the lowest-position top-k, the
hierarchical Full and the Reindex selection, the attended set and fp64
softmax attention, ratio-2 entries and the flat causal indexer, and drivers
that run whole decode steps, sampled prefill queries (with the whole append)
and ragged steps with bounded replay on host threads (the benchmark's CPU
baselines).  Its roundings are
brute-force nearest-grid searches rather than the numpy oracle's midpoint
counts; ``tests/test_oracle_c.py`` pins it to the pages' value tables, closed
forms and brute force, and checks it against the numpy oracle.

Scope: bf16 indexer keys -- the decode path, the encoder prefill at 2:1
compression (entry encoding, stored keys, the flat causal indexer) and the
ragged decode with bounded replay (FP8 keys and the sliding-window store are
the numpy oracle's only).

Only ``tests/``, ``__graft_entry__`` (build) and ``bench.py`` (CPU baseline)
use it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(_HERE, "c", "csa2_oracle.c")
LIB = os.path.join(_HERE, "c", "libcsa2_oracle.so")
CFLAGS = ["-std=c11", "-O2", "-ffp-contract=off", "-fPIC", "-shared", "-pthread"]

TOP_K = 512
POOL_BLOCKS = 2048
WINDOW = 128
D = 512

_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (no contraction of multiply-adds)."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        tmp = LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, SRC, "-lm"])
        os.replace(tmp, LIB)
    return LIB


class Schedule(ctypes.Structure):
    _fields_ = [("nlayers", ctypes.c_int), ("modes", ctypes.c_char_p), ("heads", ctypes.c_int),
                ("sm_scale", ctypes.c_double), ("seed", ctypes.c_uint64), ("kv_col_scale", ctypes.c_void_p),
                ("gen", ctypes.c_void_p)]


class Sequence(ctypes.Structure):
    _fields_ = [("L", ctypes.c_int64), ("keys", ctypes.c_void_p), ("idxq", ctypes.c_void_p),
                ("q", ctypes.c_void_p), ("new_row", ctypes.c_void_p), ("kv_stream", ctypes.c_uint64),
                ("row_cache", ctypes.c_void_p), ("drawn", ctypes.c_void_p), ("idx", ctypes.c_void_p),
                ("out", ctypes.c_void_p), ("status", ctypes.c_int)]


class Prefill(ctypes.Structure):
    _fields_ = [("nlayers", ctypes.c_int), ("heads", ctypes.c_int), ("sm_scale", ctypes.c_double),
                ("compress", ctypes.c_int), ("n_entries", ctypes.c_int64), ("keys", ctypes.c_void_p),
                ("raw_kv", ctypes.c_void_p)]


class PrefillQuery(ctypes.Structure):
    _fields_ = [("P", ctypes.c_int64), ("iq", ctypes.c_void_p), ("q", ctypes.c_void_p), ("idx", ctypes.c_void_p),
                ("out", ctypes.c_void_p)]


class RaggedSequence(ctypes.Structure):
    _fields_ = [("L", ctypes.c_int64), ("reindex", ctypes.c_int), ("miss", ctypes.c_int),
                ("kv_last", ctypes.c_void_p), ("keys", ctypes.c_void_p), ("pool", ctypes.c_void_p),
                ("set", ctypes.c_void_p), ("iq", ctypes.c_void_p), ("q", ctypes.c_void_p),
                ("kv_stream", ctypes.c_uint64), ("row_cache", ctypes.c_void_p), ("drawn", ctypes.c_void_p),
                ("idx", ctypes.c_void_p), ("out", ctypes.c_void_p), ("replayed", ctypes.c_void_p),
                ("nreplayed", ctypes.c_int64)]


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        vp, i64, i32, f64 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_double
        sig = {
            "csa2o_e2m1_value": (f64, [i32]),
            "csa2o_e4m3_value": (f64, [i32]),
            "csa2o_encode_rows": (None, [vp, i64, vp]),
            "csa2o_decode_rows": (None, [vp, i64, vp]),
            "csa2o_block_keys": (None, [vp, i64, vp]),
            "csa2o_scores": (None, [vp, vp, vp, i64, vp]),
            "csa2o_topk": (i64, [vp, i64, i64, vp]),
            "csa2o_full_indexer": (None, [vp, vp, vp, i64, vp, vp]),
            "csa2o_reindex_indexer": (None, [vp, vp, vp, i64, vp, vp]),
            "csa2o_attended_positions": (i64, [vp, i64, vp]),
            "csa2o_attend": (None, [vp, i32, vp, i64, f64, vp]),
            "csa2o_decode_steps": (i32, [ctypes.POINTER(Schedule), ctypes.POINTER(Sequence), i32, i32]),
            "csa2o_encode_entries": (None, [vp, i64, i32, vp]),
            "csa2o_key_entries": (None, [vp, i64, i32, vp]),
            "csa2o_flat_indexer": (None, [vp, vp, vp, i64, vp]),
            "csa2o_prefill_queries": (None, [ctypes.POINTER(Prefill), ctypes.POINTER(PrefillQuery), i32, i32]),
            "csa2o_prefill_append": (None, [ctypes.POINTER(Prefill), vp, vp, vp, i32]),
            "csa2o_ragged_steps": (None, [ctypes.POINTER(Schedule), ctypes.POINTER(RaggedSequence), i32, i32]),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype, f.argtypes = res, args
        _lib = L
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


def e2m1_value(code: int) -> float:
    return lib().csa2o_e2m1_value(int(code))


def e4m3_value(byte: int) -> float:
    return lib().csa2o_e4m3_value(int(byte))


def encode_rows(kv_bits) -> np.ndarray:
    """bf16 rows [n, 512] -> 288-byte cache rows [n, 288]."""
    kv = _c(kv_bits, np.uint16).reshape(-1, D)
    out = np.zeros((kv.shape[0], 288), np.uint8)
    lib().csa2o_encode_rows(_p(kv), kv.shape[0], _p(out))
    return out


def encode_entries(raw_bits, compress: int) -> np.ndarray:
    """Raw bf16 rows [compress x n, 512] -> n cache rows (ratio 2: pair means)."""
    raw = _c(raw_bits, np.uint16).reshape(-1, D)
    n = raw.shape[0] // compress
    out = np.zeros((n, 288), np.uint8)
    lib().csa2o_encode_entries(_p(raw), n, int(compress), _p(out))
    return out


def key_entries(raw_bits, compress: int) -> np.ndarray:
    """Raw bf16 indexer keys [compress x n, 64] -> n stored keys."""
    raw = _c(raw_bits, np.uint16).reshape(-1, 64)
    n = raw.shape[0] // compress
    out = np.zeros((n, 64), np.uint16)
    lib().csa2o_key_entries(_p(raw), n, int(compress), _p(out))
    return out


def decode_rows(rows) -> np.ndarray:
    """288-byte rows [n, 288] -> fp64 values [n, 512]."""
    r = _c(rows, np.uint8).reshape(-1, 288)
    out = np.zeros((r.shape[0], D), np.float64)
    lib().csa2o_decode_rows(_p(r), r.shape[0], _p(out))
    return out


def block_keys(key_bits, length: int) -> np.ndarray:
    k = _c(key_bits, np.uint16)
    nb = (length + 7) // 8
    out = np.zeros((nb, 64), np.uint16)
    lib().csa2o_block_keys(_p(k), length, _p(out))
    return out


def index_scores(q_bits, key_bits, w=None) -> np.ndarray:
    q = _c(q_bits, np.uint16)
    k = _c(key_bits, np.uint16).reshape(-1, 64)
    wv = None if w is None else _c(w, np.float32)
    out = np.zeros(k.shape[0], np.float32)
    lib().csa2o_scores(_p(q), None if wv is None else _p(wv), _p(k), k.shape[0], _p(out))
    return out


def top_k(scores, k: int) -> np.ndarray:
    s = _c(scores, np.float32)
    out = np.zeros(k, np.int64)
    lib().csa2o_topk(_p(s), s.size, k, _p(out))
    return out


def full_indexer(q_bits, key_bits, length: int):
    """(pool [2048] ascending block ids, -1 padded; selected positions [512])."""
    q, k = _c(q_bits, np.uint16), _c(key_bits, np.uint16)
    pool, idx = np.zeros(POOL_BLOCKS, np.int64), np.zeros(TOP_K, np.int64)
    lib().csa2o_full_indexer(_p(q), None, _p(k), length, _p(pool), _p(idx))
    return pool, idx


def reindex_indexer(q_bits, key_bits, length: int, pool) -> np.ndarray:
    q, k, pl = _c(q_bits, np.uint16), _c(key_bits, np.uint16), _c(pool, np.int64)
    idx = np.zeros(TOP_K, np.int64)
    lib().csa2o_reindex_indexer(_p(q), None, _p(k), length, _p(pl), _p(idx))
    return idx


def flat_indexer(q_bits, key_bits, visible: int) -> np.ndarray:
    """Top-512 positions among [0, visible), ascending, -1 padded."""
    q, k = _c(q_bits, np.uint16), _c(key_bits, np.uint16)
    idx = np.zeros(TOP_K, np.int64)
    lib().csa2o_flat_indexer(_p(q), None, _p(k), int(visible), _p(idx))
    return idx


def attended_positions(idx, length: int) -> np.ndarray:
    i = _c(idx, np.int64)
    pos = np.zeros(TOP_K + WINDOW, np.int64)
    n = lib().csa2o_attended_positions(_p(i), length, _p(pos))
    if n < 0:
        raise ValueError("selected position beyond the visible context")
    return pos[:n].copy()


def attend(q_bits, rows, sm_scale: float = 1.0) -> np.ndarray:
    q = _c(q_bits, np.uint16)
    r = _c(rows, np.float64).reshape(-1, D)
    out = np.zeros((q.shape[0], D), np.float64)
    lib().csa2o_attend(_p(q), q.shape[0], _p(r), r.shape[0], float(sm_scale), _p(out))
    return out


class DecodeSteps:
    """Decode steps of many sequences on host threads.

    seqs: per sequence a dict with ``L`` (context length), ``seq`` (its index,
    which names its generator stream), ``keys`` [L, 64], ``iq`` {layer: [4, 64]}
    and ``q`` {layer: [heads, 512]} bf16 bits, and ``new`` [1, 512] (the
    appended token's KV).  KV rows are drawn from the seeded generator the
    first time a set needs them and kept (input generation, not oracle work)."""

    MODE = {"F": b"F", "RI": b"I", "R": b"R"}

    def __init__(self, layers, heads: int, seed: int, seqs, sm_scale: float = 1.0):
        import workload as wl
        self.n = len(seqs)
        nl = len(layers)
        self._modes = b"".join(self.MODE[m] for m in layers)
        self._col = wl.kv_col_scale(seed).astype(np.float32)
        gen = ctypes.cast(wl.host_lib().wl_fill_normal_bf16, ctypes.c_void_p).value
        self.sched = Schedule(nl, self._modes, heads, sm_scale, seed, _p(self._col).value, gen)
        self._keep = []
        self.arr = (Sequence * self.n)()
        self.idx, self.out = [], []
        for i, s in enumerate(seqs):
            L = int(s["L"])
            keys = _c(s["keys"], np.uint16)
            iq = np.zeros((nl, 4, 64), np.uint16)
            for l, v in s["iq"].items():
                iq[l] = v
            q = np.stack([_c(s["q"][l], np.uint16) for l in range(nl)])
            new = _c(s["new"], np.uint16)
            cache = np.zeros((L, D), np.uint16)       # pages touched only where drawn
            drawn = np.zeros(L, np.uint8)
            idx = np.zeros((nl, TOP_K), np.int64)
            out = np.zeros((nl, heads, D), np.float64)
            self._keep += [keys, iq, q, new, cache, drawn]
            self.idx.append(idx)
            self.out.append(out)
            self.arr[i] = Sequence(L, _p(keys).value, _p(iq).value, _p(q).value, _p(new).value,
                                   wl.stream_id(wl.TAG_KV, 0, int(s["seq"])), _p(cache).value,
                                   _p(drawn).value, _p(idx).value, _p(out).value, 0)

    def step(self, threads: int) -> None:
        if lib().csa2o_decode_steps(ctypes.byref(self.sched), self.arr, self.n, int(threads)) != 0:
            raise ValueError("decode step failed (schedule or position)")


class PrefillQueries:
    """Sampled queries of an encoder prefill on host threads, and the whole append.

    keys: stored keys [n_entries, 64]; raw_kv / raw_k: the sequence's raw bf16 rows
    [compress x n_entries, 512 / 64]; queries: per sampled raw position P a dict
    with ``P``, ``iq`` [4, 64] and ``q`` [nlayers, heads, 512]."""

    def __init__(self, nlayers: int, heads: int, compress: int, keys, raw_kv, raw_k, queries,
                 sm_scale: float = 1.0):
        self._keys, self._kv, self._k = _c(keys, np.uint16), _c(raw_kv, np.uint16), _c(raw_k, np.uint16)
        n_e = self._keys.shape[0]
        self.pf = Prefill(nlayers, heads, sm_scale, compress, n_e, _p(self._keys).value, _p(self._kv).value)
        self.rows_out = np.zeros((n_e, 288), np.uint8)
        self.keys_out = np.zeros((n_e, 64), np.uint16)
        self._keep, self.idx, self.out = [], [], []
        self.arr = (PrefillQuery * len(queries))()
        for i, qq in enumerate(queries):
            iq, q = _c(qq["iq"], np.uint16), _c(qq["q"], np.uint16)
            idx, out = np.zeros(TOP_K, np.int64), np.zeros((nlayers, heads, D), np.float64)
            self._keep += [iq, q]
            self.idx.append(idx)
            self.out.append(out)
            self.arr[i] = PrefillQuery(int(qq["P"]), _p(iq).value, _p(q).value, _p(idx).value, _p(out).value)

    def queries(self, threads: int) -> None:
        lib().csa2o_prefill_queries(ctypes.byref(self.pf), self.arr, len(self.arr), int(threads))

    def append(self, threads: int) -> None:
        lib().csa2o_prefill_append(ctypes.byref(self.pf), _p(self._k), _p(self.rows_out), _p(self.keys_out),
                                   int(threads))


class RaggedSteps:
    """Ragged decode steps with bounded replay on host threads: per sequence a dict
    with ``L``, ``seq``, ``ri`` (Reindex, else Reuse), ``miss``, ``kv_last`` [128, 512],
    ``keys`` [L, 64], the Full layer's ``pool`` [2048] and ``set`` [512], ``iq`` [4, 64]
    and ``q`` [heads, 512]."""

    def __init__(self, heads: int, seed: int, seqs, sm_scale: float = 1.0):
        import workload as wl
        self.n = len(seqs)
        self._col = wl.kv_col_scale(seed).astype(np.float32)
        gen = ctypes.cast(wl.host_lib().wl_fill_normal_bf16, ctypes.c_void_p).value
        self.sched = Schedule(0, b"", heads, sm_scale, seed, _p(self._col).value, gen)
        self._keep, self.idx, self.out, self.replayed = [], [], [], []
        self.arr = (RaggedSequence * self.n)()
        for i, s in enumerate(seqs):
            L = int(s["L"])
            parts = [_c(s["kv_last"], np.uint16), _c(s["keys"], np.uint16), _c(s["pool"], np.int64),
                     _c(s["set"], np.int64), _c(s["iq"], np.uint16), _c(s["q"], np.uint16),
                     np.zeros((max(L, 1), D), np.uint16), np.zeros(max(L, 1), np.uint8)]
            idx, out = np.zeros(TOP_K, np.int64), np.zeros((heads, D), np.float64)
            rep = np.zeros((WINDOW, 288), np.uint8)
            self._keep += parts
            self.idx.append(idx)
            self.out.append(out)
            self.replayed.append(rep)
            self.arr[i] = RaggedSequence(L, int(bool(s["ri"])), int(bool(s["miss"])),
                                         *[_p(x).value for x in parts[:6]],
                                         wl.stream_id(wl.TAG_KV, 0, int(s["seq"])),
                                         _p(parts[6]).value, _p(parts[7]).value, _p(idx).value, _p(out).value,
                                         _p(rep).value, 0)

    def replayed_rows(self, i: int) -> np.ndarray:
        """The entries sequence i re-encoded in the last step (oldest first)."""
        return self.replayed[i][:self.arr[i].nreplayed].copy()

    def step(self, threads: int) -> None:
        lib().csa2o_ragged_steps(ctypes.byref(self.sched), self.arr, self.n, int(threads))
