"""CPU oracle for the CSA2 step over an FP4 KV cache -- TEST INFRASTRUCTURE ONLY.

A plain, slow, obviously correct restatement of what the CSA2 hot path
computes, written from the pages' description of the method:

* ``formats``   -- the E2M1, E4M3 and bfloat16 number formats (closed forms);
* ``codec``     -- FP4 main-KV encode/decode, 2:1 sequence compression;
* ``indexer``   -- block keys, indexer scores, lowest-position top-k, the
                   hierarchical 2,048 x 8 candidate pool, Full/Reindex selection;
* ``attention`` -- the attended set (selected tokens joined with the 128-token
                   sliding window) and exact softmax attention in fp64;
* ``modes``     -- the Full / Reindex / Reuse layer schedule and the replay rule;
* ``c_oracle``  -- a second restatement of the decode path in plain C
                   (``c/csa2_oracle.c``, brute-force roundings, fp64 attention,
                   whole decode steps on host threads), pinned on its own and
                   checked against the numpy functions; the benchmark's CPU
                   baseline for the decode workloads.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its CPU
baseline and reference arm) may import this package.  It shares no code with
the CUDA path (``fp4_kv_cache_decode_b200``) and never imports it; the only
thing both sides use is the seeded input generator in ``workload``.

Precision: the codec and the block-key/score arithmetic that decides integer
results (FP4 codes, scale bytes, bf16 block keys, top-k membership) are exact
or fp32 in a fixed order, as the kernels decide them; attention is fp64.

Parity status of each function is stated in its docstring ("pinned by ..." or
"parity unpinned").
"""
