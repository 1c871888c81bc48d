"""A bounded device wait that runs out, on the GPU, without a fault or a hang.

Every mbarrier wait in the attention and tensor-core scorer kernels is bounded;
when one runs out the kernel raises CSA2_DEVERR_TIMEOUT in the cache's error
word, lets the tensor-core work it issued drain, releases its tensor memory and
returns, so the context stays usable.  This test drives that path with the test
build of the library (lib/libcsa2_test.so: the same kernels with shorter wait
limits and a hook that, while bit 31 of the error word is set, makes the
attention's MMA thread -- after its first Q.K^T commit -- or the scorer's MMA
thread wait on an mbarrier that nothing completes).  For each kernel: the call
returns, csa2_check_device_error reports the timeout, and the next call on the
same context reproduces the production library's result bit for bit.
"""
import ctypes
import contextlib

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

STALL_BIT = 0x80000000
DEVERR_TIMEOUT = 8


@contextlib.contextmanager
def _test_library(csa2):
    """Route the binding's calls to the test build for the duration."""
    from fp4_kv_cache_decode_b200 import _build
    lib = ctypes.CDLL(_build.TEST_LIB)
    for name, (res, args) in csa2.SIGNATURES.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    saved = csa2.lib()
    csa2._lib = lib
    try:
        yield lib
    finally:
        csa2._lib = saved


def _arm(cache):
    cache.error_word.fill_(STALL_BIT - (1 << 32))   # int32 view of bit 31
    torch.cuda.synchronize()


@pytest.mark.parametrize("lengths", [[70000, 40000, 5000, 300], [70000] * 32])
def test_wait_runs_out_then_the_next_call_is_exact(csa2_lib, lengths):
    import workload
    workload.build_cuda()
    from fp4_kv_cache_decode_b200 import synthetic
    from tests.gpu_util import small_workload

    csa2 = csa2_lib
    w = small_workload(lengths, seed=31)
    cache = synthetic.new_cache(w)
    synthetic.fill_decode_cache(w, cache)
    step = synthetic.DecodeStep(w, cache, layers=["F", "R"])
    # production library: the reference index set and outputs
    step.run(append=False)
    torch.cuda.synchronize()
    assert csa2.csa2_check_device_error(cache) == 0
    ref_idx = step.iset.idx.clone()
    ref_out = [o.clone() for o in step.out]

    with _test_library(csa2):
        # attention: the MMA thread stalls after its first commit
        for o in step.out:
            o.zero_()
        _arm(cache)
        csa2.csa2_sparse_attn(cache, step.q[0], step.q_seq, csa2.FULL, 0, step.iset, step.out[0], step.ws_attn,
                              synthetic.SM_SCALE)
        bits = csa2.csa2_check_device_error(cache)   # synchronises: the call returned
        assert bits & DEVERR_TIMEOUT, hex(bits)
        # the context is usable: the same layers again give the production outputs
        step.layer(0)
        step.layer(1)
        torch.cuda.synchronize()
        assert csa2.csa2_check_device_error(cache) == 0
        for got, want in zip(step.out, ref_out):
            assert torch.equal(got.view(torch.int16), want.view(torch.int16))

        # tensor-core scorer: the MMA thread stalls before its first MMA
        _arm(cache)
        csa2.csa2_indexer_score_topk(cache, step.idxq[0], step.q_seq, csa2.FULL, 0, step.iset, step.ws_idx,
                                     step.max_visible)
        bits = csa2.csa2_check_device_error(cache)
        assert bits & DEVERR_TIMEOUT, hex(bits)
        csa2.csa2_indexer_score_topk(cache, step.idxq[0], step.q_seq, csa2.FULL, 0, step.iset, step.ws_idx,
                                     step.max_visible)
        torch.cuda.synchronize()
        assert csa2.csa2_check_device_error(cache) == 0
        np.testing.assert_array_equal(step.iset.idx.cpu().numpy(), ref_idx.cpu().numpy())
