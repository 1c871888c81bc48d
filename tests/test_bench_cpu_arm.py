"""The benchmark's CPU oracle arm, on CPU: the C oracle's threaded decode steps
time a small workload's whole step; the prefill query sample holds every
chunk's first and last position and nothing twice."""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def test_prefill_query_sample_is_stratified():
    import bench
    import workload as wl
    w = wl.workload(3)
    qs = bench.prefill_queries(w)
    assert len(qs) == 1024 and np.all(np.diff(qs) > 0)
    assert qs[0] >= 0 and qs[-1] < w.raw_tokens
    for c in range(w.raw_tokens // w.chunk):
        assert c * w.chunk in qs and (c + 1) * w.chunk - 1 in qs
    np.testing.assert_array_equal(qs, bench.prefill_queries(w))     # seeded


def test_c_oracle_decode_steps_time_a_whole_step():
    import bench
    w, ts, threads = bench.c_decode_baseline(0, 0, warmup=1, steps=2, threads=4)
    assert threads == 1 and len(ts) == 2 and all(t > 0 for t in ts)   # one sequence: one thread
