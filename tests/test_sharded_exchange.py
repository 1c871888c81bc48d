"""Host side of the position-sharded decode on CPU: two gloo ranks gather their
candidate rows with the helper the multi-GPU layer uses, and the rows read back
through that layer's strides (query 1, shard B) give the exact top-k of the union
of the shards' candidates, lowest position first on ties; shard bounds cover the
sequence with aligned starts."""
import os
import socket

import numpy as np
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _local_candidates(rank: int, B: int, K: int, span: int):
    """Rank `rank` holds positions [rank span, (rank + 1) span); its K best of
    seeded scores (ties frequent), ascending, as (score, global position)."""
    rng = np.random.default_rng(100 + rank)
    sc = rng.integers(0, 6, (B, span)).astype(np.float32)
    score = np.full((B, K), -np.inf, np.float32)
    ids = np.full((B, K), -1, np.int32)
    for q in range(B):
        order = np.lexsort((np.arange(span), -sc[q]))[:K]
        sel = np.sort(order)
        score[q, :sel.size] = sc[q, sel]
        ids[q, :sel.size] = sel + rank * span
    return sc, score, ids


def _worker(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from fp4_kv_cache_decode_b200.sharded import gather_rows
    B, K, span = 3, 16, 40
    _, score, ids = _local_candidates(rank, B, K, span)
    gs = gather_rows(torch.from_numpy(score), world)
    gi = gather_rows(torch.from_numpy(ids), world)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, gs.numpy(), gi.numpy()))


def test_gathered_rows_merge_to_the_exact_top_k():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    world = 2
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=180) for _ in procs), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    B, K, span = 3, 16, 40
    gs, gi = res[0][1], res[0][2]
    assert np.array_equal(gs, res[1][1]) and np.array_equal(gi, res[1][2])   # every rank sees the same rows
    full = np.concatenate([_local_candidates(r, B, K, span)[0] for r in range(world)], axis=1)
    for qq in range(B):
        rows = [qq * 1 + s * B for s in range(world)]               # (query stride 1, shard stride B)
        cs = np.concatenate([gs[r] for r in rows])
        ci = np.concatenate([gi[r] for r in rows])
        assert np.all(np.diff(ci[ci >= 0]) > 0)                     # shard order = ascending positions
        valid = ci >= 0
        order = np.lexsort((ci[valid], -cs[valid]))[:K]
        merged = np.sort(ci[valid][order])
        want = np.sort(np.lexsort((np.arange(world * span), -full[qq]))[:K])
        np.testing.assert_array_equal(merged, want)


def test_shard_bounds():
    import sys
    sys.path.insert(0, ROOT)
    from fp4_kv_cache_decode_b200.sharded import shard_bounds
    for L in (1, 63, 64, 1000, 40000, 1 << 20):
        for n in (1, 2, 3, 8):
            b = shard_bounds(L, n)
            assert b[0][0] == 0 and b[-1][1] == L and len(b) == n
            assert all(lo <= hi and (lo % 64 == 0 or lo == hi == L) for lo, hi in b)
            assert all(b[i][1] == b[i + 1][0] for i in range(n - 1))
