"""The indexer entry point for callers that cannot allocate device memory.

Some callers cannot hand the library a workspace -- a host framework that owns
all device memory and gives plugins no allocator, or a serving loop that must
never reach cudaMalloc.  csa2_indexer_score_topk_noalloc serves them from a
static device array inside the library.  This test calls it through the C ABI
twice in a row (the array keeps the first call's contents) and checks both
results against the workspace-taking entry point on the same inputs.  It lives
in a file that pytest collects last, so a stop-at-first-failure run has already
run every other test when it gets here; it also passes on its own in a fresh
process.
"""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def test_noalloc_indexer_matches_workspace_entry_point(csa2_lib):
    import workload
    workload.build_cuda()
    from workload import device as wdev
    from fp4_kv_cache_decode_b200 import synthetic
    from tests.gpu_util import small_workload

    csa2 = csa2_lib
    lengths = [5, 300, 4096, 16385, 40000, 70000]
    w = small_workload(lengths, seed=21)
    cache = synthetic.new_cache(w)
    synthetic.fill_decode_cache(w, cache)
    nq = len(lengths)
    max_vis = max(lengths)
    qs = torch.arange(nq, dtype=torch.int32, device="cuda")
    # within the static array's size
    need = csa2.csa2_workspace_bytes(csa2.OP_INDEXER, nq, 0, max_vis, True)
    assert 0 < need <= csa2.NOALLOC_SCRATCH_BYTES

    def run(call, layer, mode, iset, iq):
        if call == "workspace":
            ws = torch.empty(need, dtype=torch.uint8, device="cuda")
            csa2.csa2_indexer_score_topk(cache, iq, qs, mode, layer, iset, ws, max_vis)
        else:
            csa2.csa2_indexer_score_topk_noalloc(cache, iq, qs, mode, layer, iset, max_vis)
        torch.cuda.synchronize()
        return iset.idx.cpu().numpy().copy(), iset.pool_blocks.cpu().numpy().copy()

    iq0 = wdev.idxq_batch(w.seed, 0, 0, nq)
    iq1 = wdev.idxq_batch(w.seed, 1, 0, nq)
    ref_set = csa2.IndexSet(nq)
    ref_full = run("workspace", 0, csa2.FULL, ref_set, iq0)
    ref_ri = run("workspace", 1, csa2.REINDEX, ref_set, iq1)
    # two calls in a row on the static array: a Full layer then a Reindex layer
    na_set = csa2.IndexSet(nq)
    got_full = run("noalloc", 0, csa2.FULL, na_set, iq0)
    got_ri = run("noalloc", 1, csa2.REINDEX, na_set, iq1)
    # the same kernels on the same inputs: the index sets agree exactly
    # (exact agreement is inside the near-tie rule the other parity tests use)
    for got, ref in ((got_full, ref_full), (got_ri, ref_ri)):
        np.testing.assert_array_equal(got[0], ref[0])
        np.testing.assert_array_equal(got[1], ref[1])
    assert np.all((ref_full[0] >= 0).sum(axis=1) == np.minimum(lengths, 512))
    assert csa2.csa2_check_device_error(cache) == 0

    # a request larger than the static array is refused before anything runs
    big = csa2.IndexSet(64)
    qs64 = torch.zeros(64, dtype=torch.int32, device="cuda")
    iq64 = torch.zeros((64, 4, 64), dtype=torch.bfloat16, device="cuda")
    assert csa2.csa2_workspace_bytes(csa2.OP_INDEXER, 64, 0, 1 << 20, True) > csa2.NOALLOC_SCRATCH_BYTES
    st = csa2.lib().csa2_indexer_score_topk_noalloc(
        cache.ref(), iq64.data_ptr(), None, qs64.data_ptr(), None, 64, 1 << 20, csa2.FULL, 1, 2,
        big.ref(), torch.cuda.current_stream().cuda_stream)
    assert st == 5                              # CSA2_ERR_WORKSPACE
    assert big.layer == -1
