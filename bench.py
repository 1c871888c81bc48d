"""Benchmark of the CSA2 decode step over the FP4 KV cache (B200, sm_100a).

Workload: the 64K-context decode batch -- 32 sequences of 65,536 tokens, 64
query heads x 512 latent, FP4 KV in 64-token pages scattered over a 4 GiB
pool, one decoder group Full + 3 Reuse then one group Reindex + 3 Reuse.  A
step appends each sequence's newest token (csa2_kv_quant_append) and runs the
8 layers (csa2_indexer_score_topk for Full / Reindex, csa2_sparse_attn for
every layer).  Metric: layer-steps/s (one layer over the whole batch).

Timing: W warm-up steps, then K timed steps; L2 is flushed (a 256 MiB write)
before every step, outside the timed events; each step is bracketed by CUDA
events on the launching stream and the step time is their sum; with N ranks
(torchrun) every rank runs its own batch (weak scaling, no collective on the
data path) and the reported time is the max over ranks.

``--impl reference`` times the CPU oracle instead (bounded sample, host cores).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "CSA2 decode layer-steps/s at 64K ctx; achieved HBM GB/s vs B200 peak"
UNIT = "layer-steps/s"
CONFIG_ID = 1
# dram__bytes_read.sum + dram__bytes_write.sum of one attn_pipe_kernel launch on this
# workload (ncu, three launches: 9.709, 9.703, 9.799 MB read, 0 written), captured with
# the pool sized to the batch -- the same rows, queries and outputs per launch as the
# 4 GiB pool, only the rows' page addresses differ
ATTN_DRAM_BYTES_PER_LAUNCH = 9.74e6
L2_FLUSH_BYTES = 256 << 20
NOMINAL_HBM_GBS = 8000.0   # the B200's nominal HBM3e bandwidth, for context beside the measured peak


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def _config_json(w, n_gpus):
    return {"workload": "decode B=32 x 65536-token context, 64 heads x 512 latent, 8 layers "
                        "F,R,R,R,RI,R,R,R, 64-token pages in a 4 GiB pool",
            "batch": w.batch, "context": w.lengths[0], "heads": w.heads, "layers": w.layers,
            "pool_pages": w.n_pages_pool,
            "l2": "flushed before every step (256 MiB write outside the timed events)",
            "launch": "the whole step captured once as a CUDA graph and replayed per timed step",
            "parallelism": f"dp{n_gpus} (independent batches per GPU)"}


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = max(mx, float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

def _attended_rows(idx: np.ndarray, L: int) -> int:
    w0 = max(0, L - 128)
    sel = idx[(idx >= 0) & (idx < w0)]
    return int(sel.size + (L - w0))


# ---------------------------------------------------------------------------
# ranks (one process per GPU under torchrun; the host logic is tested with gloo)
# ---------------------------------------------------------------------------

def rank_env() -> tuple[int, int, int]:
    """(world, rank, local_rank) from the torchrun environment (1, 0, 0 alone)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init_ranks(world: int, backend: str = "nccl", device=None) -> None:
    """Join the process group (nothing to do alone).  A short timeout makes ranks
    that wait on a missing peer fail instead of hanging."""
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        kw = {"device_id": device} if device is not None else {}
        dist.init_process_group(backend, timeout=timedelta(seconds=120), **kw)


def rank_seed(seed: int, rank: int) -> int:
    """Every rank draws its own batch (weak scaling: no data is shared)."""
    return seed + 1000 * rank


def max_over_ranks(x: float, world: int, device: str = "cuda") -> float:
    """The slowest rank's time: the job is done when its last rank is."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int) -> None:
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def finish_ranks(world: int) -> None:
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


def run_gpu(args):
    import torch
    import torch.distributed as dist

    import workload as wl
    from fp4_kv_cache_decode_b200 import _build, csa2, synthetic

    world, rank, local = rank_env()
    if not os.path.exists(_build.LIB):
        raise SystemExit("libcsa2.so is not built: run `python -c 'import __graft_entry__ as g; g.build()'`")
    torch.cuda.set_device(local)
    init_ranks(world, "nccl", torch.device("cuda", local))
    w = wl.workload(CONFIG_ID)
    w.seed = rank_seed(w.seed, rank)
    if args.pool_pages:
        # profiling case only: a pool of exactly the pages the batch uses (same work per
        # call, compact addresses, ~1 GB on the device instead of ~5 GB)
        w.n_pages_pool = sum((l + 63) // 64 for l in w.lengths)
    torch.manual_seed(0)
    cache = synthetic.new_cache(w)
    synthetic.fill_decode_cache(w, cache)
    step = synthetic.DecodeStep(w, cache)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    torch.cuda.synchronize()
    assert csa2.csa2_check_device_error(cache) == 0

    calls = ["append"] + [f"L{i}:{m}" for i, m in enumerate(w.layers)]

    def timed_step(ev):
        ev[0].record(stream)
        step.append()
        ev[1].record(stream)
        for i in range(len(w.layers)):
            step.layer(i)
            ev[2 + i].record(stream)

    n_ev = 2 + len(w.layers)
    for _ in range(args.warmup):
        flush.fill_(1)
        step.run()
    torch.cuda.synchronize()
    # The decode step (append + every layer) is captured once as a CUDA graph and the
    # timed region replays it, as a serving loop does; the library calls are
    # capture-safe (no host synchronisation, no allocation).
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        step.run()
    stream.wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step.run()
    torch.cuda.synchronize()
    for _ in range(args.warmup):
        flush.fill_(1)
        graph.replay()
    torch.cuda.synchronize()
    barrier(world)

    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    torch.cuda.synchronize()
    barrier(world)
    for k in range(args.steps):
        flush.fill_(k & 0xFF)          # outside the events: the step starts with a cold L2
        events[k][0].record(stream)
        graph.replay()
        events[k][1].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clocks = sampler.stop()
    step_ms = np.array([events[k][0].elapsed_time(events[k][1]) for k in range(args.steps)])
    total_ms = float(step_ms.sum())
    # diagnostic outside the timed region: the same replays without the L2 flush
    # (inputs and kernel code left in L2 by the previous step)
    warm = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    for k in range(args.steps):
        warm[k][0].record(stream)
        graph.replay()
        warm[k][1].record(stream)
    torch.cuda.synchronize()
    warm_ms = float(np.median([e[0].elapsed_time(e[1]) for e in warm]))

    # diagnostics outside the timed region: (1) a per-call breakdown from eager steps
    # with an event between calls (each event adds a little to its call); (2) the
    # attention kernel's launch duration from a graph of back-to-back Reuse calls
    n_diag = 3
    diag = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(n_diag)]
    for k in range(n_diag):
        flush.fill_(k & 0xFF)
        timed_step(diag[k])
    torch.cuda.synchronize()
    per_call = np.zeros((n_diag, n_ev - 1))
    for k in range(n_diag):
        for j in range(n_ev - 1):
            per_call[k, j] = diag[k][j].elapsed_time(diag[k][j + 1])   # ms
    reuse_layers = [i for i, m in enumerate(w.layers) if m == "R" and i > w.layers.index("RI")]

    def reuse_run():   # the step's last Reuse layers, twice, back to back as in the step
        for _ in range(2):
            for i in reuse_layers:
                step.layer(i)
    n_attn = 2 * len(reuse_layers)
    attn_launch_ms = _graph_ms(reuse_run, flush, stream, reps=7) / n_attn

    def graph_ms(fn, reps=5):
        return _graph_ms(fn, flush, stream, reps)

    # the indexer calls alone, each as its own graph (Full at layer 0, then the
    # Reindex layer on the Full's pool)
    f_layer, ri_layer = w.layers.index("F"), w.layers.index("RI")
    idx_full_ms = graph_ms(lambda: csa2.csa2_indexer_score_topk(
        cache, step.idxq[f_layer], step.q_seq, csa2.FULL, f_layer, step.iset, step.ws_idx, step.max_visible))
    idx_ri_ms = graph_ms(lambda: csa2.csa2_indexer_score_topk(
        cache, step.idxq[ri_layer], step.q_seq, csa2.REINDEX, ri_layer, step.iset, step.ws_idx, step.max_visible))
    total_ms = max_over_ranks(total_ms, world)
    assert csa2.csa2_check_device_error(cache) == 0

    # --- algorithmic work of one step (from the sets the step produced) ---
    L = w.lengths[0]
    B = w.batch
    nb = (L + 7) // 8
    full_sets = synthetic.DecodeStep(w, cache, layers=["F"])
    full_sets.run(append=False)
    torch.cuda.synchronize()
    rows_full = sum(_attended_rows(r, L) for r in full_sets.iset.idx.cpu().numpy())
    rows_ri = sum(_attended_rows(r, L) for r in step.iset.idx.cpu().numpy())
    rows_per_layer = [rows_full if i < 4 else rows_ri for i in range(len(w.layers))]
    bytes_attn = [r * 288 for r in rows_per_layer]
    flops_attn = [4.0 * w.heads * 512 * r for r in rows_per_layer]
    bytes_full_idx = B * (nb * 128 + 16384 * 128)
    bytes_ri_idx = B * 16384 * 128
    step_bytes = bytes_full_idx + bytes_ri_idx + sum(bytes_attn)
    # compulsory bytes: the algorithmic bytes plus every layer's attention query and
    # output (bf16), the indexer queries and the index sets written (pool, Full and
    # Reindex token sets, int32)
    n_idx = sum(1 for m in w.layers if m in ("F", "RI"))
    qo_bytes = 2 * len(w.layers) * B * w.heads * 512 * 2
    set_bytes = B * (n_idx * 4 * 64 * 2 + 2048 * 4 + n_idx * 512 * 4)
    compulsory_bytes = step_bytes + qo_bytes + set_bytes
    mean_call = per_call.mean(axis=0)        # ms per call type (append, L0..L7)

    peaks = _peaks()
    # per call type: attention calls (Reuse layers are attention only)
    reuse_ms = float(np.mean([mean_call[1 + i] for i, m in enumerate(w.layers) if m == "R"]))
    reuse_call_ms = reuse_ms                 # eager, with per-call events
    reuse_ms = attn_launch_ms                # back-to-back launches in a graph
    reuse_flops = float(np.mean([flops_attn[i] for i, m in enumerate(w.layers) if m == "R"]))
    reuse_bytes = float(np.mean([bytes_attn[i] for i, m in enumerate(w.layers) if m == "R"]))
    # the Full layer = indexer + attention; its indexer share is Full - Reuse-like attention
    attn_total_ms = reuse_ms * len(w.layers)
    idx_total_ms = idx_full_ms + idx_ri_ms
    if attn_total_ms >= idx_total_ms:
        # f16 x f16 -> fp32 runs at the dense bf16 rate, so the measured bf16 peak applies
        dom = {"kernel": "csa2_sparse_attn (attn_pipe_kernel), Reuse layer",
               "bound": "tensor", "achieved": reuse_flops / (reuse_ms * 1e-3) / 1e12,
               "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
               "hbm_achieved_gbs": reuse_bytes / (reuse_ms * 1e-3) / 1e9}
    else:
        b = bytes_full_idx
        t = idx_full_ms * 1e-3
        dom = {"kernel": "csa2_indexer_score_topk (Full: block + pool scoring, two top-k)",
               "bound": "hbm", "achieved": b / t / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s",
               "launch_ms": idx_full_ms,
               "launches_timed": "the Full indexer call after an L2 flush, 10 in one CUDA graph minus the flushes"}
    if attn_total_ms >= idx_total_ms:
        dom["launch_ms"] = reuse_ms
        dom["launches_timed"] = ("2 x 3 Reuse attention calls back to back after an L2 flush, 10 such "
                                 "groups in one CUDA graph minus a graph of the 10 flushes")
    dom["frac"] = dom["achieved"] / dom["peak"]
    dom["peak_source"] = peaks["source"]
    # DRAM bytes per launch of the dominant kernel from an ncu capture of this
    # kernel version (profiles/attn_pipe_decode_64k_b32.md); None when unmeasured
    dom["traffic"] = ATTN_DRAM_BYTES_PER_LAUNCH if dom["kernel"].startswith("csa2_sparse_attn") else None

    units = len(w.layers) * args.steps * world
    value = units / (total_ms * 1e-3)
    ms_per_step = total_ms / args.steps
    hbm_gbs = step_bytes / (ms_per_step * 1e-3) / 1e9

    # --- end to end through the C ABI with host buffers ---
    e2e = run_e2e(args, w, step, stream, flush)
    e2e["ms"] = max_over_ranks(e2e["ms"], world)
    e2e_value = len(w.layers) * args.steps * world / (e2e["ms"] * 1e-3)

    result = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f16", "data": "synthetic (seeded)",
        "config": _config_json(w, world),
        "tokens_per_s": B * world * args.steps / (total_ms * 1e-3),
        "hbm_gbs_achieved": hbm_gbs, "hbm_frac": hbm_gbs / peaks["hbm_gbs"],
        "hbm_frac_of_nominal": hbm_gbs / NOMINAL_HBM_GBS,
        "step_algorithmic_bytes": step_bytes,
        "step_compulsory_bytes": compulsory_bytes,
        "compulsory_frac": compulsory_bytes / (ms_per_step * 1e-3) / 1e9 / peaks["hbm_gbs"],
        "ms_per_call": {c: float(m) for c, m in zip(calls, mean_call)},
        "ms_per_call_note": "diagnostic: eager steps outside the timed region, one event between calls",
        "ms_graph": {"attention_launch": reuse_ms, "indexer_full": idx_full_ms, "indexer_reindex": idx_ri_ms},
        "ms_per_step_warm_l2": warm_ms,
        "ms_per_step_warm_l2_note": "median of graph replays back to back with no L2 flush (diagnostic)",
        "roofline": dom,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": e2e["h2d"],
                "d2h_bytes_per_step": e2e["d2h"],
                "note": "copies of step k+1 (up) and k-1 (down) on two copy streams overlap step k's compute; "
                        "L2 flushed before every step inside the timed region"},
        "gpu_launches": args.steps * launches_per_step(w),
        "clocks": clocks,
    }
    if not args.no_extra_legs:   # diagnostics outside the timed region
        result["window_store"] = measure_window_store(w, cache, step, stream, flush, peaks, reuse_ms)
        result["max_pooled_blocks"] = measure_max_pool(w, cache, step, stream, flush, peaks, idx_full_ms)
        result["fp8_indexer_keys"] = measure_fp8_keys(
            w, stream, flush, peaks, {"step": ms_per_step, "full": idx_full_ms, "reindex": idx_ri_ms})
        result["workloads"] = measure_workloads(stream, flush, peaks, rank)
        result["sharded_1m"] = measure_sharded_1m(stream, flush, result["workloads"]["config2"]["step_ms"], rank)
        result["access_ceilings"] = measure_access_ceilings(
            stream, flush, {"attention_launch": reuse_ms, "indexer_reindex": idx_ri_ms})
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(args)
        if "workloads" in result:
            for k, v in workload_baselines().items():
                result["workloads"][k]["cpu_baseline"] = v
    finish_ranks(world)
    if rank == 0:
        print(json.dumps(result), flush=True)


def _graph_ms(fn, flush, stream, reps=5, n=10):
    """Device time of one fn() call with the L2 flushed before it: a CUDA graph of
    n x (flush + call) minus a graph of the same n flushes, divided by n, so that the
    graph's launch latency and the events' 2.048-us steps drop out; median of reps."""
    import torch

    def capture(with_call):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(n):
                flush.fill_(i & 0xFF)
                if with_call:
                    fn()
        return g

    def timed(g):
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        g.replay()
        a1.record(stream)
        torch.cuda.synchronize()
        return a0.elapsed_time(a1)

    g_call, g_flush = capture(True), capture(False)
    for _ in range(2):
        timed(g_call)
        timed(g_flush)
    ts = [(timed(g_call) - timed(g_flush)) / n for _ in range(reps)]
    del g_call, g_flush
    return float(np.median(ts))


def measure_window_store(w, cache, step, stream, flush, peaks, attn_global_ms):
    """The separate sliding-window store on the bench batch, outside the timed
    region: bounded replay (every sequence flagged) into the store at ratio 1 and 2
    and into the global cache at ratio 1, and the Reuse attention launch reading
    its window from the store.  The store is filled with the same entries as the
    global cache, so the step's outputs must not change by a bit."""
    import torch

    import workload as wl
    from workload import device as wdev
    from fp4_kv_cache_decode_b200 import csa2
    B = w.batch
    col = torch.from_numpy(wl.kv_col_scale(w.seed)).cuda()
    kv1 = torch.zeros((B, 128, 512), dtype=torch.bfloat16, device="cuda")
    k1 = torch.zeros((B, 128, 64), dtype=torch.bfloat16, device="cuda")
    kv2 = torch.zeros((B, 256, 512), dtype=torch.bfloat16, device="cuda")
    n_blocks = 0
    for b, L in enumerate(w.lengths):
        n = min(128, L)
        wdev.kv_rows(w.seed, b, L - n, n, out=kv1[b, 128 - n:], col_scale=col)
        wdev.idxk_rows(w.seed, b, L - n, n, out=k1[b, 128 - n:])
        wdev.kv_rows(w.seed + 1, b, 0, 2 * n, out=kv2[b, 256 - 2 * n:], col_scale=col)
        n_blocks += (L - 1) // 8 - (L - n) // 8 + 1
    n_entries = sum(min(128, L) for L in w.lengths)
    miss = torch.ones(B, dtype=torch.uint8, device="cuda")
    ref_out = [o.clone() for o in step.out]
    hbm = peaks["hbm_gbs"]

    def leg(ms, nbytes, launches):
        gbs = nbytes / (ms * 1e-3) / 1e9
        return {"ms": ms, "algorithmic_bytes": nbytes, "gbs": gbs, "frac_of_hbm": gbs / hbm,
                "launches": launches}

    # global cache, ratio 1: rows, keys and touched block keys rewritten (same values)
    t_glob = _graph_ms(lambda: csa2.csa2_swa_replay(cache, kv1, k1, miss), flush, stream)
    glob_bytes = n_entries * (1024 + 128 + 288 + 128) + n_blocks * (8 * 128 + 128)
    cache.swa_rows = torch.zeros((B, 128, 288), dtype=torch.uint8, device="cuda")
    cache.refresh()
    try:
        t_st1 = _graph_ms(lambda: csa2.csa2_swa_replay(cache, kv1, None, miss), flush, stream)
        step.run(append=False)             # sets and row caches resolved with the store attached
        torch.cuda.synchronize()
        same = all(torch.equal(a.view(torch.int16), b.view(torch.int16)) for a, b in zip(step.out, ref_out))
        reuse = [i for i, m in enumerate(w.layers) if m == "R" and i > w.layers.index("RI")]

        def reuse_calls():
            for _ in range(2):
                for i in reuse:
                    step.layer(i)
        t_attn = _graph_ms(reuse_calls, flush, stream) / (2 * len(reuse))
        t_st2 = _graph_ms(lambda: csa2.csa2_swa_replay(cache, kv2, None, miss, compress=2), flush, stream)
        assert csa2.csa2_check_device_error(cache) == 0
    finally:
        cache.swa_rows = None
        cache.refresh()
    return {
        "replay_global_ratio1": leg(t_glob, glob_bytes, 2),
        "replay_store_ratio1": leg(t_st1, n_entries * (1024 + 288), 1),
        "replay_store_ratio2": leg(t_st2, n_entries * (2048 + 288), 1),
        "attention_reuse_launch_ms": {"window_from_store": t_attn, "window_from_global_cache": attn_global_ms},
        "step_outputs_bit_identical": bool(same),
        "note": "CUDA graphs of one call (replay) or 2 x 3 Reuse calls (attention), L2 flushed first; "
                "bytes: bf16 rows read + FP4 rows (and keys) written",
    }


def measure_max_pool(w, cache, step, stream, flush, peaks, mean_full_ms):
    """The Full indexer with max-pooled block scores on the bench batch, outside the
    timed region: it scores every key (the flat score kernel also writing each
    block's maximum), then selects the pool and the tokens.  Also the recall of the
    mean-pooled hierarchy: the share of the exact top-512 (= the max-pooled one)
    that the step's mean-pooled Full layer selects."""
    import torch

    from fp4_kv_cache_decode_b200 import csa2
    f_layer = w.layers.index("F")
    iset = csa2.IndexSet(step.nq, row_cache=False)
    ws = torch.empty(csa2.csa2_workspace_bytes(csa2.OP_INDEXER, step.nq, 0, step.max_visible, csa2.HIER_MAX),
                     dtype=torch.uint8, device="cuda")

    def full_max():
        csa2.csa2_indexer_score_topk(cache, step.idxq[f_layer], step.q_seq, csa2.FULL, f_layer, iset, ws,
                                     step.max_visible, hierarchical=csa2.HIER_MAX)
    ms = _graph_ms(full_max, flush, stream)
    mean_set = csa2.IndexSet(step.nq, row_cache=False)
    csa2.csa2_indexer_score_topk(cache, step.idxq[f_layer], step.q_seq, csa2.FULL, f_layer, mean_set,
                                 step.ws_idx, step.max_visible, hierarchical=csa2.HIER_MEAN)
    full_max()
    torch.cuda.synchronize()
    assert csa2.csa2_check_device_error(cache) == 0
    exact, approx = iset.idx.cpu().numpy(), mean_set.idx.cpu().numpy()
    recall = float(np.mean([np.isin(a[a >= 0], e[e >= 0]).sum() / max(1, (e >= 0).sum())
                            for e, a in zip(exact, approx)]))
    key_bytes = sum(w.lengths[s] for s in step.seqs) * 128
    gbs = key_bytes / (ms * 1e-3) / 1e9
    return {"indexer_full_ms": ms, "indexer_full_ms_mean_pooled": mean_full_ms,
            "key_bytes": key_bytes, "gbs": gbs, "frac_of_hbm": gbs / peaks["hbm_gbs"],
            "mean_pooled_recall_of_exact_top512": recall,
            "note": "median of CUDA-graph replays, L2 flushed first; bytes = every visible bf16 key once"}


def _set_rows(idx, lens):
    """Attended rows of index sets (selected positions outside the window, plus
    the window) given each query's visible length."""
    return sum(_attended_rows(r, int(L)) for r, L in zip(idx, lens))


def measure_workloads(stream, flush, peaks, seed_rank: int = 0):
    """The other seeded workloads on this GPU, outside the timed region, each
    step captured once as a CUDA graph and replayed (median of 5, L2 flushed
    before each replay); inputs generated before the graph.  A decode
    layer-step is one layer over the whole batch.  Algorithmic bytes: gathered
    FP4 rows (288 B each, counted from the step's own index sets), indexer keys
    read (block keys and pool keys, 128 B each) and, for the ragged batch, the
    replay's rows in and out; the prefill is tensor-bound and reports FLOPs."""
    import torch

    import workload as wl
    from workload import device as wdev
    from fp4_kv_cache_decode_b200 import csa2, synthetic
    hbm = peaks["hbm_gbs"]
    out = {}

    def hbm_leg(w, ms, nbytes, units, what):
        gbs = nbytes / (ms * 1e-3) / 1e9
        return {"workload": w.name, "step": what, "step_ms": ms, "layer_steps_per_s": units / (ms * 1e-3),
                "tokens_per_s": w.batch / (ms * 1e-3), "algorithmic_bytes": nbytes, "hbm_gbs": gbs,
                "hbm_frac": gbs / hbm}

    for cid in (0, 2):
        w = wl.workload(cid)
        w.seed = rank_seed(w.seed, seed_rank)
        cache = synthetic.new_cache(w)
        synthetic.fill_decode_cache(w, cache)
        step = synthetic.DecodeStep(w, cache)
        step.run()
        full = synthetic.DecodeStep(w, cache, layers=["F"])
        full.run(append=False)
        torch.cuda.synchronize()
        assert csa2.csa2_check_device_error(cache) == 0
        ms = _graph_ms(step.run, flush, stream)
        lens = [w.lengths[s] for s in step.seqs]
        rows_f = _set_rows(full.iset.idx.cpu().numpy(), lens)
        rows_ri = _set_rows(step.iset.idx.cpu().numpy(), lens)
        nbytes, group = 0, rows_f
        for m in w.layers:
            if m == "RI":
                group = rows_ri
            nbytes += group * 288
            nb = [(L + 7) // 8 for L in lens]
            if m == "F":   # flat: every key; hierarchical: block keys + the pool's keys
                nbytes += sum(n * 8 * 128 if n <= 2048 else n * 128 + 16384 * 128 for n in nb)
            elif m == "RI":
                nbytes += sum(min(n, 2048) * 8 * 128 for n in nb)
        out[f"config{cid}"] = hbm_leg(w, ms, nbytes, len(w.layers), "append + every layer")
        del step, full, cache
        torch.cuda.empty_cache()

    w = wl.workload(4)
    w.seed = rank_seed(w.seed, seed_rank)
    cache = synthetic.new_cache(w)
    synthetic.fill_decode_cache(w, cache)
    st = synthetic.RaggedStep(w, cache)
    st.setup()
    st.run()
    torch.cuda.synchronize()
    assert csa2.csa2_check_device_error(cache) == 0
    ms = _graph_ms(st.run, flush, stream)
    ri, ru = st.groups["ri"], st.groups["ru"]
    rows = (_set_rows(ri["iset"].idx.cpu().numpy(), [w.lengths[s] for s in st.ri]) +
            _set_rows(ru["iset"].idx.cpu().numpy(), [w.lengths[s] for s in st.ru]))
    pool_keys = sum(min((w.lengths[s] + 7) // 8, 2048) * 8 * 128 for s in st.ri)
    n_rep = sum(min(128, w.lengths[b]) if w.miss_mask[b] else 1 for b in range(w.batch))
    nbytes = rows * 288 + pool_keys + n_rep * (1024 + 128 + 288 + 128)
    out["config4"] = hbm_leg(w, ms, nbytes, 1, "replay + one layer (16 Reindex, 48 Reuse)")
    del st, cache
    torch.cuda.empty_cache()

    # encoder chunked prefill, the whole sequence: 16 chunks, each the append of
    # its 8,192 raw tokens, the flat indexer of its 8,192 queries and the Full +
    # 5 Reuse attention layers (one query tensor serves every layer and chunk:
    # the work does not depend on the values)
    w = wl.workload(3)
    w.seed = rank_seed(w.seed, seed_rank)
    cache = synthetic.new_cache(w)
    nchunk = w.raw_tokens // w.chunk
    n_e = w.chunk // w.compress
    last_vis = w.raw_tokens // w.compress
    ws = torch.empty(csa2.csa2_workspace_bytes(csa2.OP_INDEXER, w.chunk, 0, last_vis, False), dtype=torch.uint8,
                     device="cuda")
    obuf = torch.empty((w.chunk, w.heads, 512), dtype=torch.bfloat16, device="cuda")
    col = torch.from_numpy(wl.kv_col_scale(w.seed)).cuda()
    chunks, inputs = [], []
    for ci in range(nchunk):
        r0 = ci * w.chunk
        chunks.append(synthetic.PrefillChunk(w, cache, ci, ws_idx=ws, out=obuf))
        inputs.append((wdev.kv_rows(w.seed, 0, r0, w.chunk, col_scale=col), wdev.idxk_rows(w.seed, 0, r0, w.chunk),
                       torch.zeros(n_e, dtype=torch.int32, device="cuda"),
                       torch.arange(r0 // w.compress, r0 // w.compress + n_e, dtype=torch.int32, device="cuda")))
    q = chunks[-1].queries(0).clone()
    cache.seq_lens[0] = last_vis

    def prefill():
        for ch, (kv, k, eseq, epos) in zip(chunks, inputs):
            csa2.csa2_kv_quant_append(cache, kv, k, eseq, epos, w.compress)
            ch.indexer()
            for layer in range(len(w.layers)):
                ch.attention(layer, q=q)
    # one eager pass: attended rows of every query (for the FLOP count)
    rows = 0
    for ch, (kv, k, eseq, epos) in zip(chunks, inputs):
        csa2.csa2_kv_quant_append(cache, kv, k, eseq, epos, w.compress)
        ch.indexer()
        torch.cuda.synchronize()
        rows += _set_rows(ch.iset.idx.cpu().numpy(), ch.q_vis.cpu().numpy())
    assert csa2.csa2_check_device_error(cache) == 0
    ms = _graph_ms(prefill, flush, stream, reps=3, n=1)   # 16 chunks: launch latency is negligible
    vis = np.concatenate([ch.q_vis.cpu().numpy() for ch in chunks]).astype(np.float64)
    flops_attn = 4.0 * w.heads * 512 * rows * len(w.layers)
    flops_idx = 2.0 * 4 * 64 * float(vis.sum())
    tf = (flops_attn + flops_idx) / (ms * 1e-3) / 1e12
    out["config3"] = {"workload": w.name, "step": f"the whole prefill: {nchunk} chunks of {w.chunk} queries",
                      "step_ms": ms, "tokens_per_s": w.raw_tokens / (ms * 1e-3),
                      "layer_steps_per_s": len(w.layers) * nchunk / (ms * 1e-3),
                      "flops": flops_attn + flops_idx, "flops_attention": flops_attn, "flops_indexer": flops_idx,
                      "tflops": tf, "bound": "tensor", "tensor_frac": tf / peaks["bf16_tflops"],
                      "append_bytes": w.raw_tokens * (1024 + 128) + last_vis * (288 + 128)}
    del chunks, inputs, cache, ws, obuf
    torch.cuda.empty_cache()
    return out


def measure_sharded_1m(stream, flush, unsharded_ms: float | None, seed_rank: int = 0, nshard: int = 4):
    """The 4 x 1M decode step position-sharded over `nshard` shards, every shard
    emulated on this GPU (the shards are separate sequences of one cache; the
    all-gathers become strided reads): Full, Reindex and Reuse layers of the
    20-layer schedule through the sharded calls, as one CUDA graph.  The time is
    the sum of all shards' work on one GPU -- what one GPU of S would do is
    about a 1/S share of the sharded calls plus the exchanges."""
    import torch

    import workload as wl
    from workload import device as wdev
    from fp4_kv_cache_decode_b200 import synthetic
    from fp4_kv_cache_decode_b200.sharded import EmulatedDecoder, shard_bounds
    w = wl.workload(2)
    w.seed = rank_seed(w.seed, seed_rank)
    bounds = [shard_bounds(L, nshard) for L in w.lengths]
    lens = [hi - lo for sh in bounds for lo, hi in sh]
    cache = synthetic.new_cache(w, lengths=lens)
    synthetic.fill_sharded_cache(w, cache, bounds)
    B = w.batch
    off = torch.tensor([lo for sh in bounds for lo, _ in sh], dtype=torch.int32, device="cuda")
    wstart = torch.tensor([max(0, L - 128) for L in w.lengths], dtype=torch.int32, device="cuda")
    dec = EmulatedDecoder(cache, nshard, off, wstart, w.heads, max(lens))
    iq = {l: wdev.idxq_batch(w.seed, l, 0, B) for l, m in enumerate(w.layers) if m in ("F", "RI")}
    q = [wdev.q_batch(w.seed, l, 0, B, w.heads) for l in range(len(w.layers))]

    def step():
        for l, m in enumerate(w.layers):
            if m == "F":
                dec.full(iq[l], q[l])
            elif m == "RI":
                dec.reindex(iq[l], q[l])
            else:
                dec.reuse(q[l])
    step()
    torch.cuda.synchronize()
    ms = _graph_ms(step, flush, stream)
    del dec, cache
    torch.cuda.empty_cache()
    return {"workload": w.name, "shards": nshard, "step_ms": ms, "layer_steps_per_s": len(w.layers) / (ms * 1e-3),
            "unsharded_step_ms": unsharded_ms,
            "note": "all shards emulated on one GPU (sum of every shard's work), CUDA graph, L2 flushed first"}


def measure_fp8_keys(w, stream, flush, peaks, bf16_ms):
    """The same decode step on a cache whose indexer keys are FP8 (64 E4M3 codes
    + one fp32 scale, 68 B per token instead of 128 B), outside the timed region:
    the step as one CUDA graph, and the Full and Reindex indexer calls alone."""
    import torch

    from fp4_kv_cache_decode_b200 import csa2, synthetic
    cache = synthetic.new_cache(w, cache_id=3, idxk_format=csa2.IDXK_FP8)
    synthetic.fill_decode_cache(w, cache)
    step = synthetic.DecodeStep(w, cache)
    step.run()
    torch.cuda.synchronize()
    assert csa2.csa2_check_device_error(cache) == 0
    step_ms = _graph_ms(step.run, flush, stream, reps=7)
    f_layer, ri_layer = w.layers.index("F"), w.layers.index("RI")
    full_ms = _graph_ms(lambda: csa2.csa2_indexer_score_topk(
        cache, step.idxq[f_layer], step.q_seq, csa2.FULL, f_layer, step.iset, step.ws_idx, step.max_visible),
        flush, stream)
    ri_ms = _graph_ms(lambda: csa2.csa2_indexer_score_topk(
        cache, step.idxq[ri_layer], step.q_seq, csa2.REINDEX, ri_layer, step.iset, step.ws_idx,
        step.max_visible), flush, stream)
    assert csa2.csa2_check_device_error(cache) == 0
    B, L = w.batch, w.lengths[0]
    nb = (L + 7) // 8
    full_bytes = B * (nb * 128 + 16384 * 68)
    ri_bytes = B * 16384 * 68
    del step, cache
    torch.cuda.empty_cache()
    return {
        "layer_steps_per_s": len(w.layers) / (step_ms * 1e-3),
        "step_ms": step_ms,
        "step_ms_bf16_keys": bf16_ms["step"],
        "indexer_full_ms": full_ms, "indexer_full_ms_bf16_keys": bf16_ms["full"],
        "indexer_reindex_ms": ri_ms, "indexer_reindex_ms_bf16_keys": bf16_ms["reindex"],
        "indexer_full_gbs": full_bytes / (full_ms * 1e-3) / 1e9,
        "indexer_reindex_gbs": ri_bytes / (ri_ms * 1e-3) / 1e9,
        "hbm_peak_gbs": peaks["hbm_gbs"],
        "bytes_per_token": {"main_kv": 288, "indexer_key": 68, "block_key_share": 16},
        "note": "median of CUDA-graph replays, L2 flushed first; Full bytes = block keys (bf16) + "
                "16,384 pool keys x 68 B per query; the step's timed line above uses bf16 keys",
    }


def launches_per_step(w) -> int:
    n = 2                                   # append: rows + block keys
    for m in w.layers:
        n += 1                              # attention (ranges merged inside the kernel)
        if m == "F":
            n += 4                          # block scores, block top-k, pool scores, pool top-k
        elif m == "RI":
            n += 2                          # pool scores, top-k
    return n


def measure_access_ceilings(stream, flush, ms_graph: dict) -> dict:
    """The least time this GPU takes to move the bytes of each CSA2 kernel in its
    access pattern (kernels that load, sum and discard: the ceilings library),
    timed like the calls (flush-subtracted CUDA graphs, L2 flushed before each
    launch unless stated), each checked to have read every byte it was given
    (the sum of its loaded words against torch's sum of the same words)."""
    import ctypes

    import torch

    from fp4_kv_cache_decode_b200 import _build
    lib = ctypes.CDLL(_build.CEIL_LIB)
    P, I = ctypes.c_void_p, ctypes.c_int
    lib.csa2c_sink_slots.restype = ctypes.c_longlong
    lib.csa2c_sink_slots.argtypes = [I, I]
    lib.csa2c_stream.argtypes = [P, ctypes.c_longlong, P, I, P]
    lib.csa2c_gather_units.argtypes = [P, P, I, P, I, P]
    lib.csa2c_gather_rows.argtypes = [P, P, I, P, I, P]
    lib.csa2c_attn_inputs.argtypes = [P, P, P, P, P, I, P]
    lib.csa2c_cta_load.argtypes = [P, I, P, P]
    dev = torch.device("cuda")
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    cur = lambda: P(torch.cuda.current_stream().cuda_stream)   # the capturing stream inside a graph
    pool_bytes = 4 << 30
    pool = torch.empty(pool_bytes, dtype=torch.uint8, device=dev)
    pool.view(torch.int64).random_()
    rng = np.random.default_rng(11)
    n_units, n_rows = 65536, 128 * 160     # one Reindex call's pool units; one Reuse launch's rows
    ids_u = torch.from_numpy(rng.integers(0, pool_bytes // 1024, n_units).astype(np.int32)).to(dev)
    ids_r = torch.from_numpy(rng.integers(0, pool_bytes // 288, n_rows).astype(np.int32)).to(dev)
    q = torch.empty(32 * 65536, dtype=torch.uint8, device=dev)
    q.view(torch.int64).random_()
    part = torch.empty(128 * 65536, dtype=torch.uint8, device=dev)
    src = torch.empty(32 * 65536, dtype=torch.uint8, device=dev)
    src.view(torch.int64).random_()
    sink = torch.zeros(1 << 20, dtype=torch.int32, device=dev)
    small = torch.empty(4096, dtype=torch.uint8, device=dev)   # "flush" that leaves L2 as it is
    ptr = lambda t: P(t.data_ptr())

    def words(t):   # sum of a byte tensor's 32-bit words mod 2^32
        return int(t.contiguous().view(torch.int32).to(torch.int64).sum().item()) & 0xFFFFFFFF

    def call(rc):
        if rc != 0:
            raise RuntimeError(f"ceilings kernel failed: {rc}")

    out = {"note": "kernels that only load (and sum) the bytes of each pattern; flush-subtracted "
                   "CUDA graphs of 10 launches, L2 flushed before each unless stated"}
    cases = [
        ("contiguous_read_64MiB", 64 << 20, 0, 8 * sms,
         lambda g: lib.csa2c_stream(ptr(pool), (64 << 20) // 16, ptr(sink), g, cur()),
         lambda: words(pool[: 64 << 20]), flush, "the copy-peak pattern at the pool scorer's size"),
        ("units_1KiB_random_64MiB", n_units * 1024, 1, 4 * sms,
         lambda g: lib.csa2c_gather_units(ptr(pool), ptr(ids_u), n_units, ptr(sink), g, cur()),
         lambda: words(pool.view(-1, 1024)[ids_u.long()]), flush,
         "one Reindex call's pool scoring: 32 x 2,048 random 1-KiB key units"),
        ("units_1KiB_random_32MiB", n_units * 512, 1, 4 * sms,
         lambda g: lib.csa2c_gather_units(ptr(pool), ptr(ids_u), n_units // 2, ptr(sink), g, cur()),
         lambda: words(pool.view(-1, 1024)[ids_u[: n_units // 2].long()]), flush,
         "the Full call's block-key scoring size (32 x 1,024 units)"),
        ("rows_288B_random_5.9MB", n_rows * 288, 2, 4 * sms,
         lambda g: lib.csa2c_gather_rows(ptr(pool), ptr(ids_r), n_rows, ptr(sink), g, cur()),
         lambda: words(pool[: pool_bytes // 288 * 288].view(-1, 288)[ids_r.long()]), flush,
         "one Reuse attention launch's FP4 rows (32 x 640), gathered by warps spread over every SM"),
        ("attention_inputs", 128 * 65536 + n_rows * 288, 3, 128,
         lambda g: lib.csa2c_attn_inputs(ptr(q), ptr(pool), ptr(ids_r), None, ptr(sink), 0, cur()),
         lambda: (4 * words(q) + words(pool[: pool_bytes // 288 * 288].view(-1, 288)[ids_r.long()]))
         & 0xFFFFFFFF, flush,
         "the attention's split: 128 CTAs, each its query (64 KiB, shared by 4) and 160 rows"),
        ("attention_inputs_and_slices", 128 * 65536 * 2 + n_rows * 288, 3, 128,
         lambda g: lib.csa2c_attn_inputs(ptr(q), ptr(pool), ptr(ids_r), ptr(part), ptr(sink), 1, cur()),
         lambda: (4 * words(q) + words(pool[: pool_bytes // 288 * 288].view(-1, 288)[ids_r.long()]))
         & 0xFFFFFFFF, flush, "the same, then each CTA stores a 64-KiB f16 slice (the range merge's store)"),
        ("topk_score_load_l2", 32 * 65536, 4, 32,
         lambda g: lib.csa2c_cta_load(ptr(src), g, ptr(sink), cur()),
         lambda: words(src), small, "32 CTAs x 1,024 threads, 64 KiB of L2-resident scores each (no flush)"),
    ]
    for name, nbytes, kernel, grid, launch, expect, fl, what in cases:
        slots = int(lib.csa2c_sink_slots(kernel, grid))
        sink.zero_()
        call(launch(grid))
        torch.cuda.synchronize()
        got = int(sink[:slots].to(torch.int64).sum().item()) & 0xFFFFFFFF
        ms = _graph_ms(lambda: call(launch(grid)), fl, stream, reps=5, n=10)
        out[name] = {"us": ms * 1e3, "bytes": nbytes, "gbs": nbytes / (ms * 1e-3) / 1e9,
                     "verified": got == expect(), "pattern": what}
    a = out["attention_inputs_and_slices"]["us"]
    out["attention_launch_over_data_floor"] = ms_graph["attention_launch"] * 1e3 / a
    floor_ri = out["units_1KiB_random_64MiB"]["us"] + out["topk_score_load_l2"]["us"]
    out["indexer_reindex_over_data_floor"] = ms_graph["indexer_reindex"] * 1e3 / floor_ri
    del pool, q, part, src, sink, ids_u, ids_r
    torch.cuda.empty_cache()
    return out


def run_e2e(args, w, step, stream, flush):
    """Same step through the C ABI as a serving loop runs it: every step copies its
    inputs from pinned host memory and reads its outputs back, inside the timed
    region, with the copies pipelined against the compute -- step k+1's inputs go
    up (one copy stream) and step k-1's outputs come down (another) while step k
    computes, two sets of device buffers alternating.  The L2 flush before each
    step's compute stays in the timed region (the bench repeats identical steps)."""
    import torch

    from fp4_kv_cache_decode_b200 import synthetic
    sets = [step, synthetic.DecodeStep(w, step.cache)]

    # a step's inputs (new token, indexer and attention queries) are views of one
    # device buffer: one host->device copy per step
    pinned = torch.empty(step.inputs.shape, dtype=step.inputs.dtype, pin_memory=True)
    pinned.copy_(step.inputs)
    outs = [torch.empty(st.out_all.shape, dtype=st.out_all.dtype, pin_memory=True) for st in sets]
    h2d = pinned.numel() * pinned.element_size()
    d2h = outs[0].numel() * outs[0].element_size()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()

    def pipeline(n: int):
        ev = lambda: torch.cuda.Event()
        ready, done, back = [ev() for _ in range(n)], [ev() for _ in range(n)], [ev() for _ in range(n)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(up)
        stream.wait_event(t0)
        down.wait_event(t0)
        for k in range(n):
            st = sets[k % 2]
            with torch.cuda.stream(up):   # inputs of step k (its buffer set was last used by step k-2)
                if k >= 2:
                    up.wait_event(done[k - 2])
                st.inputs.copy_(pinned, non_blocking=True)
                ready[k].record(up)
            stream.wait_event(ready[k])
            if k >= 2:
                stream.wait_event(back[k - 2])   # step k-2's outputs (same set) are read back
            flush.fill_(k & 0xFF)
            st.run()
            done[k].record(stream)
            with torch.cuda.stream(down):
                down.wait_event(done[k])
                outs[k % 2].copy_(st.out_all, non_blocking=True)
                back[k].record(down)
        down.wait_event(done[n - 1])
        t1.record(down)
        return t0, t1

    pipeline(max(3, args.warmup))
    torch.cuda.synchronize()
    t0, t1 = pipeline(args.steps)
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1)
    return {"ms": ms, "h2d": h2d, "d2h": d2h}


# ---------------------------------------------------------------------------
# CPU oracle arm
# ---------------------------------------------------------------------------

def host_threads() -> int:
    """Host cores this process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def _cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def prefill_queries(w, n: int = 1024) -> np.ndarray:
    """Stratified sample of prefill query positions: every chunk's first and last
    position, the rest a seeded draw from all positions (ascending)."""
    import workload as wl
    fixed = set()
    for c in range(w.raw_tokens // w.chunk):
        fixed.update((c * w.chunk, (c + 1) * w.chunk - 1))
    perm = wl.permutation(w.seed, wl.stream_id(wl.TAG_LENS, 3), w.raw_tokens)
    extra = [int(p) for p in perm if int(p) not in fixed][:n - len(fixed)]
    return np.asarray(sorted(fixed | set(extra)), dtype=np.int64)


def c_decode_baseline(cid: int, seed: int, warmup: int, steps: int, threads: int | None = None):
    """Decode steps of the C oracle (oracle/c/csa2_oracle.c) over a workload's whole
    batch on host threads, one sequence per thread at a time: wall seconds of each
    timed step.  Inputs are drawn before the timing; a KV row is drawn from the
    seeded generator the first time a set needs it and kept (the warm-up step)."""
    import workload as wl
    from oracle import c_oracle as co
    w = wl.workload(cid)
    seqs = [{"L": w.lengths[s], "seq": s, "keys": wl.idxk_rows(seed, s, 0, w.lengths[s]),
             "iq": {l: wl.idxq_rows(seed, l, s) for l, m in enumerate(w.layers) if m in ("F", "RI")},
             "q": {l: wl.q_rows(seed, l, s, w.heads) for l in range(len(w.layers))},
             "new": wl.kv_rows(seed, s, w.lengths[s] - 1, 1)} for s in range(w.batch)]
    threads = max(1, min(threads or host_threads(), w.batch))
    ds = co.DecodeSteps(w.layers, w.heads, seed, seqs)
    for _ in range(warmup):
        ds.step(threads)
    ts = []
    for _ in range(steps):
        t0 = time.perf_counter()
        ds.step(threads)
        ts.append(time.perf_counter() - t0)
    return w, ts, threads


def c_ragged_baseline(seed: int, warmup: int, steps: int, threads: int | None = None):
    """Ragged decode steps with bounded replay (the 64-sequence workload) on the C
    oracle: per sequence the Full layer's pool and set are computed before the timing
    (as on the GPU, where an earlier Full layer made them), then each timed step
    replays, re-ranks (Reindex sequences) or keeps the set (Reuse) and attends."""
    from concurrent.futures import ThreadPoolExecutor

    import workload as wl
    from oracle import c_oracle as co
    w = wl.workload(4)
    threads = max(1, min(threads or host_threads(), w.batch))

    def one(s):
        L = w.lengths[s]
        keys = wl.idxk_rows(seed, s, 0, L)
        pool, idx = co.full_indexer(wl.idxq_rows(seed, 0, s), keys, L)
        n = min(128, L)
        kv_last = np.zeros((128, 512), np.uint16)
        kv_last[128 - n:] = wl.kv_rows(seed, s, L - n, n)
        return {"L": L, "seq": s, "ri": bool(w.reindex_mask[s]), "miss": bool(w.miss_mask[s]), "kv_last": kv_last,
                "keys": keys, "pool": pool, "set": idx, "iq": wl.idxq_rows(seed, 1, s),
                "q": wl.q_rows(seed, 1, s, w.heads)}
    with ThreadPoolExecutor(max_workers=threads) as ex:   # the C calls release the GIL
        seqs = list(ex.map(one, range(w.batch)))
    rs = co.RaggedSteps(w.heads, seed, seqs)
    for _ in range(warmup):
        rs.step(threads)
    ts = []
    for _ in range(steps):
        t0 = time.perf_counter()
        rs.step(threads)
        ts.append(time.perf_counter() - t0)
    return w, ts, threads


def c_prefill_baseline(seed: int, threads: int | None = None):
    """The encoder prefill on the C oracle: the whole append (2:1 compression, FP4
    encode, stored keys) timed in full, and the stratified query sample (flat causal
    indexer + every layer's attention) timed and scaled to all queries.  Inputs are
    drawn before the timing.  Returns (workload, append s, sample s, queries, threads)."""
    import workload as wl
    from oracle import c_oracle as co
    w = wl.workload(3)
    threads = threads or host_threads()
    raw_kv = wl.kv_rows(seed, 0, 0, w.raw_tokens)
    raw_k = wl.idxk_rows(seed, 0, 0, w.raw_tokens)
    keys = co.key_entries(raw_k, w.compress)
    qs = [{"P": int(P), "iq": wl.idxq_rows(seed, 0, int(P)),
           "q": np.stack([wl.q_rows(seed, l, int(P), w.heads) for l in range(len(w.layers))])}
          for P in prefill_queries(w)]
    pq = co.PrefillQueries(len(w.layers), w.heads, w.compress, keys, raw_kv, raw_k, qs)
    t0 = time.perf_counter()
    pq.append(threads)
    t_app = time.perf_counter() - t0
    t0 = time.perf_counter()
    pq.queries(threads)
    t_q = time.perf_counter() - t0
    return w, t_app, t_q, len(qs), threads


def cpu_baseline(args, steps: int = 3, seed: int | None = None):
    """The C oracle's whole decode step (all 32 sequences, 8 layers) on the host cores."""
    import workload as wl
    w0 = wl.workload(CONFIG_ID)
    w, ts, threads = c_decode_baseline(CONFIG_ID, w0.seed if seed is None else seed, 1, steps)
    sec = float(np.median(ts))
    return {"value": len(w.layers) / sec, "unit": UNIT, "cores": threads, "nproc": host_threads(),
            "cpu": _cpu_model(), "kind": "oracle", "impl": "C (oracle/c/csa2_oracle.c), pthreads",
            "ms_per_step": sec * 1e3,
            "sample": f"the whole step: {w.batch} of {w.batch} sequences, all {len(w.layers)} layers "
                      f"(append, indexer, fp64 attention); median of {steps} steps after 1 warm-up, "
                      f"{threads} host threads"}


def workload_baselines(seed_rank: int = 0):
    """The oracle on the other workloads (bounded samples, host cores)."""
    import workload as wl
    out = {}
    for cid, unit_per_step in ((0, 1), (2, 20)):   # decode workloads: the C oracle
        w0 = wl.workload(cid)
        w, ts, threads = c_decode_baseline(cid, rank_seed(w0.seed, seed_rank), 1, 2)
        sec = float(np.median(ts))
        out[f"config{cid}"] = {
            "value": unit_per_step / sec, "unit": UNIT, "cores": threads, "kind": "oracle",
            "impl": "C, pthreads", "tokens_per_s": w.batch / sec, "ms_per_step": sec * 1e3,
            "sample": f"the whole step ({w.batch} sequences); median of 2 steps after 1 warm-up"}
    # ragged decode with bounded replay
    w0 = wl.workload(4)
    w, ts, threads = c_ragged_baseline(rank_seed(w0.seed, seed_rank), 1, 2)
    sec = float(np.median(ts))
    out["config4"] = {
        "value": 1 / sec, "unit": UNIT, "cores": threads, "kind": "oracle", "impl": "C, pthreads",
        "tokens_per_s": w.batch / sec, "ms_per_step": sec * 1e3,
        "sample": f"the whole step ({w.batch} sequences: replay, then one Reindex or Reuse layer); "
                  f"median of 2 steps after 1 warm-up"}
    # prefill: the whole append plus a stratified sample of queries, extrapolated
    w, t_app, t_q, nq, threads = c_prefill_baseline(rank_seed(wl.workload(3).seed, seed_rank))
    n_e = w.raw_tokens // w.compress
    total = t_app + t_q * w.raw_tokens / nq
    out["config3"] = {
        "value": w.raw_tokens / total, "unit": "tokens/s", "cores": threads, "kind": "oracle",
        "impl": "C, pthreads", "extrapolated": True, "prefill_s": total, "append_s": t_app,
        "sample": f"the whole append ({w.raw_tokens} raw tokens -> {n_e} entries) timed in full; "
                  f"{nq} stratified queries (every chunk's first and last position + seeded draws; "
                  f"flat indexer + {len(w.layers)} attention layers) timed and scaled x{w.raw_tokens / nq:g} "
                  f"to all {w.raw_tokens} queries"}
    return out


def run_reference(args):
    """The C oracle as it stands on the host cores, on the same workload and metric:
    every timed step is the whole decode step of all 32 sequences."""
    world, rank, _ = rank_env()
    if rank != 0:
        return
    import workload as wl
    w0 = wl.workload(CONFIG_ID)
    w, ts, threads = c_decode_baseline(CONFIG_ID, w0.seed, args.warmup, args.steps)
    total = float(sum(ts))
    value = len(w.layers) * args.steps / total
    result = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded)", "config": _config_json(w, world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "nproc": host_threads(),
                         "cpu": _cpu_model(), "kind": "oracle", "impl": "C (oracle/c/csa2_oracle.c), pthreads",
                         "sample": f"the whole step every step: {w.batch} of {w.batch} sequences, all "
                                   f"{len(w.layers)} layers, {threads} host threads"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(result), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--pool-pages", action="store_true",
                    help="profiling case: size the paged pool to the batch (not a bench number)")
    ap.add_argument("--no-extra-legs", action="store_true",
                    help="skip the diagnostic legs after the timed step (window store, max-pooled blocks, "
                         "FP8 keys, other workloads): profiling runs keep a few GB on the device")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
