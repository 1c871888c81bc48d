"""Position-sharded decode of long sequences through the C ABI.

A sequence of L entries is split into contiguous shards (one per GPU, each
starting at a multiple of 8); every shard's cache holds its positions as the
entries 0 .. n-1 of its own sequence.  The layer modes then run as:

* Full (hierarchical): shard block candidates -> all-gather -> merge (the
  global pool) -> shard token candidates over the pool -> all-gather -> merge
  (the global index set) -> attention;
* Reindex: shard token candidates of the Full layer's global pool with the
  layer's own indexer query -> all-gather -> merge -> attention;
* Reuse: attention over the latest global index set;

where attention is: shard attention (normalised output + base-2
log-sum-exp) -> all-gather -> combine.  Every step is a library call; the
all-gathers are ``torch.distributed`` collectives (NCCL between GPUs; with
gloo they pass through host memory).

:class:`ShardedDecoder` runs the layers on one GPU per rank.
:func:`emulate_full_layer` runs the Full layer's calls for all shards of a
batch on a single GPU, the shards being separate sequences of one cache and
the gathered rows addressed through strides instead of being copied -- the
single-process form used by the GPU tests (ranks whose kernels wait on one
another never share a GPU here: the calls of different shards are
independent launches).
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import csa2


def shard_bounds(length: int, nshard: int, align: int = 64) -> list[tuple[int, int]]:
    """Contiguous [start, end) ranges of `length` positions over `nshard`
    shards, each start a multiple of `align` (a multiple of 8)."""
    assert align % 8 == 0 and nshard >= 1
    per = -(-length // nshard)
    per = max(align, -(-per // align) * align)
    return [(min(s * per, length), min((s + 1) * per, length)) for s in range(nshard)]


def gather_rows(local: torch.Tensor, world: int, group=None) -> torch.Tensor:
    """All-gather of every rank's rows: [world * rows, ...], rank-major (row
    r * rows + q is rank r's row q).  With one rank the tensor itself."""
    if world == 1:
        return local
    if dist.get_backend(group) == "nccl":
        out = torch.empty((world * local.shape[0],) + tuple(local.shape[1:]), dtype=local.dtype,
                          device=local.device)
        dist.all_gather_into_tensor(out, local.contiguous(), group=group)
        return out
    # gloo: the rows pass through host memory
    host = local.detach().cpu().contiguous()
    parts = [torch.empty_like(host) for _ in range(world)]
    dist.all_gather(parts, host, group=group)
    return torch.cat(parts, dim=0).to(local.device)


class _Buffers:
    def __init__(self, nq_shard: int, nq: int, nshard: int, heads: int, max_visible: int, dev):
        ws = lambda n: torch.empty(max(n, 256), dtype=torch.uint8, device=dev)
        self.ws_idx = ws(csa2.csa2_workspace_bytes(csa2.OP_SHARD_INDEXER, nq_shard, 0, max_visible, 0))
        self.ws_merge_b = ws(csa2.csa2_workspace_bytes(csa2.OP_SHARD_MERGE, nq, nshard, csa2.POOL_BLOCKS, 0))
        self.ws_merge_t = ws(csa2.csa2_workspace_bytes(csa2.OP_SHARD_MERGE, nq, nshard, csa2.TOP_K, 0))
        self.ws_attn = ws(csa2.csa2_workspace_bytes(csa2.OP_SHARD_ATTENTION, nq_shard, heads, 0, 0))
        f32, i32 = torch.float32, torch.int32
        self.bscore = torch.empty((nq_shard, csa2.POOL_BLOCKS), dtype=f32, device=dev)
        self.bid = torch.empty((nq_shard, csa2.POOL_BLOCKS), dtype=i32, device=dev)
        self.tscore = torch.empty((nq_shard, csa2.TOP_K), dtype=f32, device=dev)
        self.tid = torch.empty((nq_shard, csa2.TOP_K), dtype=i32, device=dev)
        self.pool = torch.empty((nq, csa2.POOL_BLOCKS), dtype=i32, device=dev)
        self.idx = torch.empty((nq, csa2.TOP_K), dtype=i32, device=dev)
        self.part = torch.empty((nq_shard, heads, csa2.LATENT_DIM), dtype=torch.bfloat16, device=dev)
        self.lse2 = torch.empty((nq_shard, heads), dtype=f32, device=dev)
        self.out = torch.empty((nq, heads, csa2.LATENT_DIM), dtype=torch.bfloat16, device=dev)


class ShardedDecoder:
    """The layer modes of B sequences on this rank's shards: full(), reindex()
    and reuse() run one layer each and return its output [B, H, 512] (the same
    on every rank); the global pool and index set persist between layers.

    cache: this rank's shard of each sequence (sequence b = shard of global
    sequence b); shard_offset: int32 [B] global position of each shard's entry
    0; window_start: int32 [B] = max(0, L_b - 128) of the global lengths."""

    def __init__(self, cache: csa2.Cache, shard_offset: torch.Tensor, window_start: torch.Tensor, heads: int,
                 max_visible: int, world: int, group=None):
        self.cache, self.world, self.group = cache, world, group
        self.B = shard_offset.numel()
        self.q_seq = torch.arange(self.B, dtype=torch.int32, device=shard_offset.device)
        self.shard_offset, self.window_start = shard_offset, window_start
        self.max_visible, self.heads = max_visible, heads
        self.buf = _Buffers(self.B, self.B, world, heads, max_visible, shard_offset.device)
        self.have_pool = self.have_set = False

    def _tokens(self, idx_q: torch.Tensor):
        """The global index set: shard token candidates of the global pool, merged."""
        b, B, W = self.buf, self.B, self.world
        csa2.csa2_shard_indexer_candidates(self.cache, idx_q, self.q_seq, self.shard_offset, csa2.SHARD_TOKENS,
                                           b.tscore, b.tid, b.ws_idx, self.max_visible, global_pool=b.pool)
        gs, gi = gather_rows(b.tscore, W, self.group), gather_rows(b.tid, W, self.group)
        csa2.csa2_shard_merge_topk(gs, gi, W, B, csa2.TOP_K, 1, B, csa2.TOP_K, b.idx, b.ws_merge_t)
        self.have_set = True

    def _attend(self, q: torch.Tensor, sm_scale: float) -> torch.Tensor:
        b, B, W = self.buf, self.B, self.world
        csa2.csa2_sparse_attn_shard(self.cache, q, self.q_seq, self.shard_offset, b.idx, self.window_start, b.part,
                                    b.lse2, b.ws_attn, sm_scale)
        gp, gl = gather_rows(b.part, W, self.group), gather_rows(b.lse2, W, self.group)
        csa2.csa2_shard_combine(gp, gl, W, B, self.heads, 1, B, b.out)
        return b.out

    def full(self, idx_q: torch.Tensor, q: torch.Tensor, sm_scale: float = 1.0) -> torch.Tensor:
        """A Full layer: the global pool (block candidates, merged), then its tokens."""
        b, B, W = self.buf, self.B, self.world
        csa2.csa2_shard_indexer_candidates(self.cache, idx_q, self.q_seq, self.shard_offset, csa2.SHARD_BLOCKS,
                                           b.bscore, b.bid, b.ws_idx, self.max_visible)
        gs, gi = gather_rows(b.bscore, W, self.group), gather_rows(b.bid, W, self.group)
        csa2.csa2_shard_merge_topk(gs, gi, W, B, csa2.POOL_BLOCKS, 1, B, csa2.POOL_BLOCKS, b.pool, b.ws_merge_b)
        self.have_pool = True
        self._tokens(idx_q)
        return self._attend(q, sm_scale)

    def reindex(self, idx_q: torch.Tensor, q: torch.Tensor, sm_scale: float = 1.0) -> torch.Tensor:
        """A Reindex layer: the Full layer's global pool ranked with this layer's query."""
        if not self.have_pool:
            raise RuntimeError("Reindex layer before any Full layer")
        self._tokens(idx_q)
        return self._attend(q, sm_scale)

    def reuse(self, q: torch.Tensor, sm_scale: float = 1.0) -> torch.Tensor:
        """A Reuse layer: attention over the latest Full / Reindex index set."""
        if not self.have_set:
            raise RuntimeError("Reuse layer before any Full or Reindex layer")
        return self._attend(q, sm_scale)

    @property
    def pool(self) -> torch.Tensor:
        return self.buf.pool

    @property
    def idx(self) -> torch.Tensor:
        return self.buf.idx


class ShardedFullLayer(ShardedDecoder):
    """One hierarchical Full layer on this rank's shards (ShardedDecoder.full)."""

    def run(self, idx_q: torch.Tensor, q: torch.Tensor, sm_scale: float = 1.0) -> torch.Tensor:
        return self.full(idx_q, q, sm_scale)


def emulate_full_layer(cache: csa2.Cache, nshard: int, shard_offset: torch.Tensor, window_start: torch.Tensor,
                       idx_q: torch.Tensor, q: torch.Tensor, max_visible: int, sm_scale: float = 1.0):
    """All shards on one GPU: sequence b * nshard + s of `cache` is shard s of
    global sequence b; shard_offset [B * nshard]; window_start, idx_q, q per
    global sequence [B].  Returns (pool [B, 2048], idx [B, 512], out [B, H, 512])."""
    B = idx_q.shape[0]
    heads = q.shape[1]
    nq_s = B * nshard
    dev = idx_q.device
    b = _Buffers(nq_s, B, nshard, heads, max_visible, dev)
    q_seq = torch.arange(nq_s, dtype=torch.int32, device=dev)
    rep = lambda t: t.repeat_interleave(nshard, dim=0).contiguous()   # each shard's copy of a query input
    iq, qq, ws = rep(idx_q), rep(q), rep(window_start)
    csa2.csa2_shard_indexer_candidates(cache, iq, q_seq, shard_offset, csa2.SHARD_BLOCKS, b.bscore, b.bid,
                                       b.ws_idx, max_visible)
    # shard s of query q is row q * nshard + s
    csa2.csa2_shard_merge_topk(b.bscore, b.bid, nshard, B, csa2.POOL_BLOCKS, nshard, 1, csa2.POOL_BLOCKS,
                               b.pool, b.ws_merge_b)
    csa2.csa2_shard_indexer_candidates(cache, iq, q_seq, shard_offset, csa2.SHARD_TOKENS, b.tscore, b.tid,
                                       b.ws_idx, max_visible, global_pool=rep(b.pool))
    csa2.csa2_shard_merge_topk(b.tscore, b.tid, nshard, B, csa2.TOP_K, nshard, 1, csa2.TOP_K, b.idx, b.ws_merge_t)
    csa2.csa2_sparse_attn_shard(cache, qq, q_seq, shard_offset, rep(b.idx), ws, b.part, b.lse2, b.ws_attn,
                                sm_scale)
    csa2.csa2_shard_combine(b.part, b.lse2, nshard, B, heads, nshard, 1, b.out)
    return b.pool, b.idx, b.out, b.lse2


class EmulatedDecoder:
    """ShardedDecoder's layers with every shard on this GPU: sequence b * S + s
    of `cache` is shard s of global sequence b, and the gathered rows are read
    through strides (query stride S, shard stride 1) instead of being copied.
    shard_offset: int32 [B * S]; window_start: int32 [B] of the global lengths;
    the layer inputs (idx_q [B, 4, 64], q [B, H, 512]) are per global sequence."""

    def __init__(self, cache: csa2.Cache, nshard: int, shard_offset: torch.Tensor, window_start: torch.Tensor,
                 heads: int, max_visible: int):
        self.cache, self.S = cache, nshard
        self.B = window_start.numel()
        dev = shard_offset.device
        self.q_seq = torch.arange(self.B * nshard, dtype=torch.int32, device=dev)
        self.shard_offset, self.max_visible, self.heads = shard_offset, max_visible, heads
        self.wstart = self._rep(window_start)
        self.buf = _Buffers(self.B * nshard, self.B, nshard, heads, max_visible, dev)
        self.pool_rep = torch.empty((self.B * nshard, csa2.POOL_BLOCKS), dtype=torch.int32, device=dev)
        self.idx_rep = torch.empty((self.B * nshard, csa2.TOP_K), dtype=torch.int32, device=dev)
        self.iq_rep = torch.empty((self.B * nshard, 4, 64), dtype=torch.bfloat16, device=dev)
        self.q_rep = torch.empty((self.B * nshard, heads, csa2.LATENT_DIM), dtype=torch.bfloat16, device=dev)

    def _rep(self, t: torch.Tensor) -> torch.Tensor:   # each shard's copy of a per-sequence input
        return t.repeat_interleave(self.S, dim=0).contiguous()

    def _tokens(self, idx_q: torch.Tensor):
        b = self.buf
        self.iq_rep.copy_(idx_q.repeat_interleave(self.S, dim=0))
        csa2.csa2_shard_indexer_candidates(self.cache, self.iq_rep, self.q_seq, self.shard_offset, csa2.SHARD_TOKENS,
                                           b.tscore, b.tid, b.ws_idx, self.max_visible, global_pool=self.pool_rep)
        csa2.csa2_shard_merge_topk(b.tscore, b.tid, self.S, self.B, csa2.TOP_K, self.S, 1, csa2.TOP_K, b.idx,
                                   b.ws_merge_t)
        self.idx_rep.copy_(b.idx.repeat_interleave(self.S, dim=0))

    def _attend(self, q: torch.Tensor, sm_scale: float) -> torch.Tensor:
        b = self.buf
        self.q_rep.copy_(q.repeat_interleave(self.S, dim=0))
        csa2.csa2_sparse_attn_shard(self.cache, self.q_rep, self.q_seq, self.shard_offset, self.idx_rep, self.wstart,
                                    b.part, b.lse2, b.ws_attn, sm_scale)
        csa2.csa2_shard_combine(b.part, b.lse2, self.S, self.B, self.heads, self.S, 1, b.out)
        return b.out

    def full(self, idx_q: torch.Tensor, q: torch.Tensor, sm_scale: float = 1.0) -> torch.Tensor:
        b = self.buf
        self.iq_rep.copy_(idx_q.repeat_interleave(self.S, dim=0))
        csa2.csa2_shard_indexer_candidates(self.cache, self.iq_rep, self.q_seq, self.shard_offset, csa2.SHARD_BLOCKS,
                                           b.bscore, b.bid, b.ws_idx, self.max_visible)
        csa2.csa2_shard_merge_topk(b.bscore, b.bid, self.S, self.B, csa2.POOL_BLOCKS, self.S, 1, csa2.POOL_BLOCKS,
                                   b.pool, b.ws_merge_b)
        self.pool_rep.copy_(b.pool.repeat_interleave(self.S, dim=0))
        self._tokens(idx_q)
        return self._attend(q, sm_scale)

    def reindex(self, idx_q: torch.Tensor, q: torch.Tensor, sm_scale: float = 1.0) -> torch.Tensor:
        self._tokens(idx_q)
        return self._attend(q, sm_scale)

    def reuse(self, q: torch.Tensor, sm_scale: float = 1.0) -> torch.Tensor:
        return self._attend(q, sm_scale)
