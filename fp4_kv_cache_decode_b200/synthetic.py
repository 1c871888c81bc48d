"""Seeded synthetic CSA2 workloads on the GPU, driven through the C ABI.

Builds the paged FP4 cache of a workload by generating its bf16 KV rows and
indexer keys on the device (:mod:`workload.device`) and encoding them with
``csa2_kv_quant_append``; runs decode steps (append one token per sequence,
then the layer schedule: Full / Reindex indexer + attention, Reuse attention)
and prefill chunks.  Used by ``bench.py`` and the GPU tests.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import workload as wl
from workload import device as wdev

from . import csa2

SM_SCALE = 1.0   # queries are drawn pre-scaled by 1/sqrt(512)


def _pages(n_entries: int) -> int:
    return (n_entries + csa2.PAGE_TOKENS - 1) // csa2.PAGE_TOKENS


def new_cache(w: wl.Workload, lengths=None, cache_id: int = 1, swa_store: bool = False,
              idxk_format: int = csa2.IDXK_BF16) -> csa2.Cache:
    lens = list(lengths if lengths is not None else w.lengths)
    pages = [_pages(L) for L in lens]
    max_pages = max(pages)
    pt = wl.page_table(w.seed, w.n_pages_pool, pages, max_pages)
    cache = csa2.Cache(w.n_pages_pool, len(lens), max_pages, cache_id=cache_id, swa_store=swa_store,
                       idxk_format=idxk_format)
    cache.page_table.copy_(torch.from_numpy(pt))
    cache.seq_lens.copy_(torch.tensor(lens, dtype=torch.int32))
    return cache


def fill_decode_cache(w: wl.Workload, cache: csa2.Cache, lengths=None, chunk: int = 65536):
    """Encode positions [0, L_b) of every sequence (ratio 1)."""
    lens = list(lengths if lengths is not None else w.lengths)
    col = torch.from_numpy(wl.kv_col_scale(w.seed)).cuda()
    kvbuf = torch.empty((chunk, 512), dtype=torch.bfloat16, device="cuda")
    kbuf = torch.empty((chunk, 64), dtype=torch.bfloat16, device="cuda")
    for b, L in enumerate(lens):
        for p0 in range(0, L, chunk):
            n = min(chunk, L - p0)
            wdev.kv_rows(w.seed, b, p0, n, out=kvbuf[:n], col_scale=col)
            wdev.idxk_rows(w.seed, b, p0, n, out=kbuf[:n])
            eseq = torch.full((n,), b, dtype=torch.int32, device="cuda")
            epos = torch.arange(p0, p0 + n, dtype=torch.int32, device="cuda")
            csa2.csa2_kv_quant_append(cache, kvbuf[:n], kbuf[:n], eseq, epos, 1)


def fill_sharded_cache(w: wl.Workload, cache: csa2.Cache, bounds, chunk: int = 65536):
    """Shard caches of position-sharded sequences: sequence b * S + s of `cache`
    holds positions [start, end) = bounds[b][s] of sequence b of the workload
    as its entries 0 .. end - start - 1 (ratio 1)."""
    col = torch.from_numpy(wl.kv_col_scale(w.seed)).cuda()
    kvbuf = torch.empty((chunk, 512), dtype=torch.bfloat16, device="cuda")
    kbuf = torch.empty((chunk, 64), dtype=torch.bfloat16, device="cuda")
    for b, shards in enumerate(bounds):
        for s, (lo, hi) in enumerate(shards):
            seq = b * len(shards) + s
            for p0 in range(lo, hi, chunk):
                n = min(chunk, hi - p0)
                wdev.kv_rows(w.seed, b, p0, n, out=kvbuf[:n], col_scale=col)
                wdev.idxk_rows(w.seed, b, p0, n, out=kbuf[:n])
                eseq = torch.full((n,), seq, dtype=torch.int32, device="cuda")
                epos = torch.arange(p0 - lo, p0 - lo + n, dtype=torch.int32, device="cuda")
                csa2.csa2_kv_quant_append(cache, kvbuf[:n], kbuf[:n], eseq, epos, 1)


def fill_prefill_chunk(w: wl.Workload, cache: csa2.Cache, chunk_index: int, seq: int = 0):
    """Encode the raw tokens of one prefill chunk at compression ratio w.compress."""
    r0 = chunk_index * w.chunk
    n_raw = w.chunk
    e0, n_e = r0 // w.compress, n_raw // w.compress
    col = torch.from_numpy(wl.kv_col_scale(w.seed)).cuda()
    kv = wdev.kv_rows(w.seed, seq, r0, n_raw, col_scale=col)
    k = wdev.idxk_rows(w.seed, seq, r0, n_raw)
    cache.seq_lens[seq] = e0 + n_e
    eseq = torch.full((n_e,), seq, dtype=torch.int32, device="cuda")
    epos = torch.arange(e0, e0 + n_e, dtype=torch.int32, device="cuda")
    csa2.csa2_kv_quant_append(cache, kv, k, eseq, epos, w.compress)


class DecodeStep:
    """One decode step of a workload: append the newest token of every
    sequence, then run the layer schedule through the C ABI."""

    def __init__(self, w: wl.Workload, cache: csa2.Cache, layers=None, seqs=None, lengths=None,
                 layer0: int = 0):
        self.w = w
        self.cache = cache
        self.layers = list(layers if layers is not None else w.layers)
        lens = list(lengths if lengths is not None else w.lengths)
        seqs = list(range(len(lens))) if seqs is None else list(seqs)
        self.seqs = seqs
        self.nq = len(seqs)
        self.heads = w.heads
        self.layer0 = layer0
        dev = "cuda"
        self.q_seq = torch.tensor(seqs, dtype=torch.int32, device=dev)
        self.max_visible = max(lens[s] for s in seqs)
        self.iset = csa2.IndexSet(self.nq)
        self.ws_idx = torch.empty(csa2.csa2_workspace_bytes(csa2.OP_INDEXER, self.nq, 0, self.max_visible,
                                                            w.hierarchical), dtype=torch.uint8, device=dev)
        self.ws_attn = torch.empty(csa2.csa2_workspace_bytes(csa2.OP_ATTENTION, self.nq, self.heads),
                                   dtype=torch.uint8, device=dev)
        # the step's inputs -- the new token's KV [nq, 512] and indexer key [nq, 64], the
        # Full/Reindex layers' indexer queries [nq, 4, 64] and every layer's attention
        # queries [nq, H, 512], bf16 -- are views of one byte buffer (`inputs`, parts at
        # 256-B offsets), so that a serving loop moves them to the device in one copy
        # (the four small copies beside the queries' measured 522 against 341 us per
        # pipelined step); the layers' outputs are views of one tensor (one copy back)
        nl = len(self.layers)
        iq_layers = [i for i, m in enumerate(self.layers) if m in ("F", "RI")]
        shapes = [(self.nq, 512), (self.nq, 64), (len(iq_layers), self.nq, 4, 64), (nl, self.nq, self.heads, 512)]
        offs, total = [], 0
        for shp in shapes:
            offs.append(total)
            total += (int(np.prod(shp)) * 2 + 255) // 256 * 256
        self.inputs = torch.zeros(total, dtype=torch.uint8, device=dev)
        parts = [self.inputs[o:o + int(np.prod(shp)) * 2].view(torch.bfloat16).view(shp)
                 for o, shp in zip(offs, shapes)]
        self.new_kv, self.new_k, iq_all, self.q_all = parts
        self.out_all = torch.empty((nl, self.nq, self.heads, 512), dtype=torch.bfloat16, device=dev)
        self.q = [self.q_all[i] for i in range(nl)]
        self.out = [self.out_all[i] for i in range(nl)]
        self.idxq = {i: iq_all[j] for j, i in enumerate(iq_layers)}
        for i, mode in enumerate(self.layers):
            l = layer0 + i
            self.q[i].copy_(_gather_rows(lambda s, n: wdev.q_batch(w.seed, l, s, n, self.heads), seqs))
            if mode in ("F", "RI"):
                self.idxq[i].copy_(_gather_rows(lambda s, n: wdev.idxq_batch(w.seed, l, s, n), seqs))
        # the step's new token: position L-1 of each sequence (its seeded value)
        col = torch.from_numpy(wl.kv_col_scale(w.seed)).cuda()
        for j, s in enumerate(seqs):
            wdev.kv_rows(w.seed, s, lens[s] - 1, 1, out=self.new_kv[j:j + 1], col_scale=col)
            wdev.idxk_rows(w.seed, s, lens[s] - 1, 1, out=self.new_k[j:j + 1])
        self.new_pos = torch.tensor([lens[s] - 1 for s in seqs], dtype=torch.int32, device=dev)

    def append(self):
        csa2.csa2_kv_quant_append(self.cache, self.new_kv, self.new_k, self.q_seq, self.new_pos, 1)

    def layer(self, i: int):
        mode = self.layers[i]
        l = self.layer0 + i
        c, s = self.cache, self.iset
        if mode == "F":
            csa2.csa2_indexer_score_topk(c, self.idxq[i], self.q_seq, csa2.FULL, l, s, self.ws_idx,
                                         self.max_visible, hierarchical=self.w.hierarchical)
            m = csa2.FULL
        elif mode == "RI":
            csa2.csa2_indexer_score_topk(c, self.idxq[i], self.q_seq, csa2.REINDEX, l, s, self.ws_idx,
                                         self.max_visible)
            m = csa2.REINDEX
        else:
            m = csa2.REUSE
        csa2.csa2_sparse_attn(c, self.q[i], self.q_seq, m, l, s, self.out[i], self.ws_attn, SM_SCALE)

    def run(self, append: bool = True):
        if append:
            self.append()
        for i in range(len(self.layers)):
            self.layer(i)


def _gather_rows(make, seqs):
    """Stack per-sequence rows made by make(first_query, count) for the listed
    sequences (contiguous runs generated in one call)."""
    parts = []
    i = 0
    while i < len(seqs):
        j = i
        while j + 1 < len(seqs) and seqs[j + 1] == seqs[j] + 1:
            j += 1
        parts.append(make(seqs[i], j - i + 1))
        i = j + 1
    return parts[0] if len(parts) == 1 else torch.cat(parts).contiguous()


class PrefillChunk:
    """Queries of one prefill chunk (encoder, flat indexer, causal visibility):
    Full indexer over [0, v(P)) per query, then the Full + Reuse attention layers."""

    def __init__(self, w: wl.Workload, cache: csa2.Cache, chunk_index: int, queries=None, ws_idx=None,
                 out=None):
        """ws_idx / out: an indexer workspace and an output buffer to use instead
        of allocating them (chunks run one after another can share them)."""
        self.w, self.cache = w, cache
        r0 = chunk_index * w.chunk
        qpos = np.arange(r0, r0 + w.chunk) if queries is None else np.asarray(queries)
        self.qpos = qpos
        self.nq = len(qpos)
        dev = "cuda"
        vis = (qpos + 1) // w.compress
        self.q_vis = torch.from_numpy(vis.astype(np.int32)).to(dev)
        self.q_seq = torch.zeros(self.nq, dtype=torch.int32, device=dev)
        self.max_visible = int(vis.max())
        self.iset = csa2.IndexSet(self.nq)
        need = csa2.csa2_workspace_bytes(csa2.OP_INDEXER, self.nq, 0, self.max_visible, False)
        if ws_idx is not None and ws_idx.numel() < need:
            raise ValueError("shared indexer workspace too small")
        self.ws_idx = ws_idx if ws_idx is not None else torch.empty(need, dtype=torch.uint8, device=dev)
        self.ws_attn = torch.empty(csa2.csa2_workspace_bytes(csa2.OP_ATTENTION, self.nq, w.heads),
                                   dtype=torch.uint8, device=dev)
        contiguous = queries is None
        self.idxq = (wdev.idxq_batch(w.seed, 0, int(qpos[0]), self.nq) if contiguous else
                     torch.cat([wdev.idxq_batch(w.seed, 0, int(p), 1) for p in qpos]))
        self.out = out if out is not None else torch.empty((self.nq, w.heads, 512), dtype=torch.bfloat16,
                                                           device=dev)
        self.q_buf = None

    def queries(self, layer: int):
        if len(self.qpos) and np.all(np.diff(self.qpos) == 1):
            if self.q_buf is None:
                self.q_buf = torch.empty((self.nq, self.w.heads, 512), dtype=torch.bfloat16, device="cuda")
            return wdev.q_batch(self.w.seed, layer, int(self.qpos[0]), self.nq, self.w.heads, out=self.q_buf)
        return torch.cat([wdev.q_batch(self.w.seed, layer, int(p), 1, self.w.heads) for p in self.qpos])

    def indexer(self):
        csa2.csa2_indexer_score_topk(self.cache, self.idxq, self.q_seq, csa2.FULL, 0, self.iset, self.ws_idx,
                                     self.max_visible, q_visible=self.q_vis, hierarchical=False)

    def attention(self, layer: int, q=None, out=None):
        mode = csa2.FULL if self.w.layers[layer] == "F" else csa2.REUSE
        q = self.queries(layer) if q is None else q
        out = self.out if out is None else out
        csa2.csa2_sparse_attn(self.cache, q, self.q_seq, mode, layer, self.iset, out, self.ws_attn, SM_SCALE,
                              q_visible=self.q_vis)
        return out


class RaggedStep:
    """Ragged mixed decode batch: every step runs SWA bounded replay for all
    sequences (flagged cache misses rewrite their last 128 entries, the others
    their newest one), then one layer in which the Reindex sequences rank the
    pool of an earlier Full layer with their own indexer query and attend, and
    the Reuse sequences attend over that Full layer's indices."""

    def __init__(self, w: wl.Workload, cache: csa2.Cache):
        self.w, self.cache = w, cache
        dev = "cuda"
        lens = list(w.lengths)
        self.ri = [int(i) for i in np.nonzero(w.reindex_mask)[0]]
        self.ru = [int(i) for i in np.nonzero(~w.reindex_mask)[0]]
        self.miss = torch.from_numpy(w.miss_mask.astype(np.uint8)).to(dev)
        B = w.batch
        col = torch.from_numpy(wl.kv_col_scale(w.seed)).cuda()
        self.kv_last = torch.zeros((B, 128, 512), dtype=torch.bfloat16, device=dev)
        self.k_last = torch.zeros((B, 128, 64), dtype=torch.bfloat16, device=dev)
        for b, L in enumerate(lens):
            n = min(128, L)
            wdev.kv_rows(w.seed, b, L - n, n, out=self.kv_last[b, 128 - n:], col_scale=col)
            wdev.idxk_rows(w.seed, b, L - n, n, out=self.k_last[b, 128 - n:])
        self.groups = {}
        for name, seqs in (("ri", self.ri), ("ru", self.ru)):
            g = {}
            g["q_seq"] = torch.tensor(seqs, dtype=torch.int32, device=dev)
            g["max_visible"] = max(lens[s] for s in seqs)
            g["iset"] = csa2.IndexSet(len(seqs))
            g["ws_idx"] = torch.empty(csa2.csa2_workspace_bytes(csa2.OP_INDEXER, len(seqs), 0,
                                                               g["max_visible"], True),
                                      dtype=torch.uint8, device=dev)
            g["ws_attn"] = torch.empty(csa2.csa2_workspace_bytes(csa2.OP_ATTENTION, len(seqs), w.heads),
                                       dtype=torch.uint8, device=dev)
            g["idxq0"] = _gather_rows(lambda s, n: wdev.idxq_batch(w.seed, 0, s, n), seqs)
            g["idxq1"] = _gather_rows(lambda s, n: wdev.idxq_batch(w.seed, 1, s, n), seqs)
            g["q1"] = _gather_rows(lambda s, n: wdev.q_batch(w.seed, 1, s, n, w.heads), seqs)
            g["out"] = torch.empty((len(seqs), w.heads, 512), dtype=torch.bfloat16, device=dev)
            self.groups[name] = g

    def setup(self):
        """The earlier Full layer (layer 0) of every sequence: pools and indices."""
        for g in self.groups.values():
            csa2.csa2_indexer_score_topk(self.cache, g["idxq0"], g["q_seq"], csa2.FULL, 0, g["iset"],
                                         g["ws_idx"], g["max_visible"], hierarchical=True)

    def replay(self):
        csa2.csa2_swa_replay(self.cache, self.kv_last, self.k_last, self.miss)

    def layer(self):
        ri, ru = self.groups["ri"], self.groups["ru"]
        csa2.csa2_indexer_score_topk(self.cache, ri["idxq1"], ri["q_seq"], csa2.REINDEX, 1, ri["iset"],
                                     ri["ws_idx"], ri["max_visible"])
        csa2.csa2_sparse_attn(self.cache, ri["q1"], ri["q_seq"], csa2.REINDEX, 1, ri["iset"], ri["out"],
                              ri["ws_attn"], SM_SCALE)
        csa2.csa2_sparse_attn(self.cache, ru["q1"], ru["q_seq"], csa2.REUSE, 1, ru["iset"], ru["out"],
                              ru["ws_attn"], SM_SCALE)

    def run(self):
        self.replay()
        self.layer()
