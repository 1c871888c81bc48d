"""The position-sharded decoder driven by two real ranks (two processes, gloo).

Each rank holds one shard of every sequence in its own cache and runs
ShardedDecoder through a Full, a Reuse, a Reindex and a Reuse layer; the
all-gathers pass through host memory (gloo).  Both processes use the one GPU of
this machine: no kernel waits on another rank, each exchange is a host-side
collective between launches.  Checked here, after the ranks exit: both ranks
produced the same results; the global pool and the index sets equal those of
the unsharded calls bit for bit (the same kernels on the same scores) and the
oracle's under the index-set rule; every layer's output is within the parity
bound of the oracle over the whole sequence and of the unsharded output.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import workload as wl
from oracle import indexer as oidx
from oracle.formats import bf16_to_f64
from tests import parity
from tests.gpu_util import bits, small_workload

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LENGTHS = [40000, 20011, 3000]
HEADS = 16
LAYERS = ["F", "R", "RI", "R"]
SEED = 71


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank: int, world: int, port: int, q) -> None:
    import sys
    sys.path.insert(0, ROOT)
    from datetime import timedelta

    import torch.distributed as dist

    import workload
    from fp4_kv_cache_decode_b200 import synthetic
    from fp4_kv_cache_decode_b200.sharded import ShardedDecoder, shard_bounds
    from workload import device as wdev
    try:
        workload.build_cuda()
        torch.cuda.set_device(0)
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=120))
        B = len(LENGTHS)
        mine = [shard_bounds(L, world)[rank] for L in LENGTHS]          # this rank's shard of each sequence
        lens = [hi - lo for lo, hi in mine]
        w = small_workload(LENGTHS, seed=SEED, heads=HEADS, spare_pages=64)
        ws = small_workload(lens, seed=SEED, heads=HEADS, spare_pages=64)
        cache = synthetic.new_cache(ws, lengths=lens)
        synthetic.fill_sharded_cache(w, cache, [[b] for b in mine])
        off = torch.tensor([lo for lo, _ in mine], dtype=torch.int32, device="cuda")
        wstart = torch.tensor([max(0, L - 128) for L in LENGTHS], dtype=torch.int32, device="cuda")
        dec = ShardedDecoder(cache, off, wstart, HEADS, max(lens), world)
        res = {"pool": None, "idx": {}, "out": {}}
        for l, m in enumerate(LAYERS):
            qq = wdev.q_batch(w.seed, l, 0, B, HEADS)
            if m == "F":
                o = dec.full(wdev.idxq_batch(w.seed, l, 0, B), qq)
                res["pool"] = dec.pool.cpu().numpy()
            elif m == "RI":
                o = dec.reindex(wdev.idxq_batch(w.seed, l, 0, B), qq)
            else:
                o = dec.reuse(qq)
            if m != "R":
                res["idx"][l] = dec.idx.cpu().numpy()
            res["out"][l] = bits(o)
        from fp4_kv_cache_decode_b200 import csa2
        res["err"] = csa2.csa2_check_device_error(cache)
        dist.barrier()
        dist.destroy_process_group()
        q.put((rank, res))
    except Exception as e:   # report instead of leaving the other rank waiting
        q.put((rank, repr(e)))
        raise


@pytest.fixture(scope="module")
def ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=600) for _ in procs)
    for p in procs:
        p.join(timeout=120)
    for r in range(2):
        assert isinstance(res[r], dict), res[r]
        assert procs[r].exitcode == 0
    return res


def test_two_ranks_agree_and_match_the_unsharded_calls_and_the_oracle(csa2_lib, ranks):
    import workload
    workload.build_cuda()
    from fp4_kv_cache_decode_b200 import synthetic
    csa2 = csa2_lib
    r0, r1 = ranks[0], ranks[1]
    assert r0["err"] == 0 and r1["err"] == 0
    np.testing.assert_array_equal(r0["pool"], r1["pool"])
    for l in r0["idx"]:
        np.testing.assert_array_equal(r0["idx"][l], r1["idx"][l])
    for l in r0["out"]:
        np.testing.assert_array_equal(r0["out"][l], r1["out"][l])
    # the unsharded calls on one cache holding the whole sequences
    w = small_workload(LENGTHS, seed=SEED, heads=HEADS, spare_pages=64)
    w.layers = list(LAYERS)
    cache = synthetic.new_cache(w)
    synthetic.fill_decode_cache(w, cache)
    full = synthetic.DecodeStep(w, cache, layers=["F"])
    full.run(append=False)
    step = synthetic.DecodeStep(w, cache)
    step.run(append=False)
    torch.cuda.synchronize()
    assert csa2.csa2_check_device_error(cache) == 0
    np.testing.assert_array_equal(r0["pool"], full.iset.pool_blocks.cpu().numpy())
    np.testing.assert_array_equal(r0["idx"][0], full.iset.idx.cpu().numpy())
    np.testing.assert_array_equal(r0["idx"][2], step.iset.idx.cpu().numpy())
    for b, L in enumerate(LENGTHS):
        o = parity.OracleSeq(w, b, L)
        iq0 = wl.idxq_rows(w.seed, 0, b)
        pool, idx0, _ = oidx.full_indexer(iq0, o.keys, L)
        parity.check_index_set(r0["pool"][b], pool, lambda x: oidx.index_scores(iq0, oidx.block_keys(o.keys, L)[
            np.asarray(x)]), f"pool L={L}")
        sets = {0: r0["idx"][0][b], 1: r0["idx"][0][b], 2: r0["idx"][2][b], 3: r0["idx"][2][b]}
        if np.array_equal(r0["pool"][b], pool):
            parity.check_index_set(sets[0], idx0, parity.token_scorer(o, iq0), f"Full tokens L={L}")
            iq2 = wl.idxq_rows(w.seed, 2, b)
            idx2, _ = oidx.reindex_indexer(iq2, o.keys, L, pool)
            parity.check_index_set(sets[2], idx2, parity.token_scorer(o, iq2), f"Reindex tokens L={L}")
        for l in range(len(LAYERS)):
            ref = parity.oracle_attention(o, sets[l], wl.q_rows(w.seed, l, b, HEADS), L)
            err, bound = parity.attention_error(r0["out"][l][b], ref)
            assert err <= bound, f"layer {l} L={L}: err {err} > {bound}"
            un = bits(step.out[l])[b]
            err_u = float(np.max(np.abs(bf16_to_f64(r0["out"][l][b]) - bf16_to_f64(un))))
            assert err_u <= bound, f"layer {l} L={L}: sharded vs unsharded {err_u}"
