"""Host logic of the multi-rank bench, on CPU: two gloo ranks join the process group,
draw different batches, report the slowest rank's time, and only rank 0 runs the
reference arm.  (Under torchrun on GPUs the same functions run with NCCL.)"""
import os
import socket

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, q) -> None:
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    w, r, local = bench.rank_env()
    bench.init_ranks(w, "gloo")
    slowest = bench.max_over_ranks(1.0 + 0.5 * r, w, device="cpu")
    seed = bench.rank_seed(1, r)
    bench.barrier(w)
    ran_reference = True
    if r != 0:   # the reference arm returns at once on every rank but 0

        class A:
            steps, warmup, gpus = 1, 3, w
        bench.run_reference(A())
        ran_reference = False
    bench.finish_ranks(w)
    q.put((r, w, local, slowest, seed, ran_reference))


def test_two_gloo_ranks_time_by_the_slowest_and_split_the_batches():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [x[1] for x in res] == [2, 2] and [x[2] for x in res] == [0, 1]
    assert [x[3] for x in res] == [1.5, 1.5]          # both ranks see the slowest rank's time
    assert res[0][4] != res[1][4]                       # each rank draws its own batch
    assert res[1][5] is False                           # rank 1 did no reference work


def test_single_process_needs_no_group():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.0, 1) == 3.0
    assert bench.rank_seed(7, 0) == 7
    bench.init_ranks(1)
    bench.barrier(1)
    bench.finish_ranks(1)
