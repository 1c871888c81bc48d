"""The access-pattern ceilings library that the benchmark times beside the CSA2
kernels: it builds, exports its calls and rejects bad arguments on the host (CPU),
and on the GPU each kernel reads exactly the bytes it is given (the sum of its
loaded 32-bit words against numpy's sum of the same words)."""
import ctypes

import numpy as np
import pytest

NAMES = ["csa2c_sink_slots", "csa2c_stream", "csa2c_gather_units", "csa2c_gather_rows", "csa2c_attn_inputs",
         "csa2c_cta_load"]


def _lib():
    from fp4_kv_cache_decode_b200 import _build
    _build.build()
    lib = ctypes.CDLL(_build.CEIL_LIB)
    P, I = ctypes.c_void_p, ctypes.c_int
    lib.csa2c_sink_slots.restype = ctypes.c_longlong
    lib.csa2c_sink_slots.argtypes = [I, I]
    lib.csa2c_stream.argtypes = [P, ctypes.c_longlong, P, I, P]
    lib.csa2c_gather_units.argtypes = [P, P, I, P, I, P]
    lib.csa2c_gather_rows.argtypes = [P, P, I, P, I, P]
    lib.csa2c_attn_inputs.argtypes = [P, P, P, P, P, I, P]
    lib.csa2c_cta_load.argtypes = [P, I, P, P]
    return lib


def _words(a: np.ndarray) -> int:
    return int(np.ascontiguousarray(a).view(np.uint32).astype(np.uint64).sum()) & 0xFFFFFFFF


def test_ceilings_library_exports_and_checks_arguments():
    lib = _lib()
    for n in NAMES:
        assert hasattr(lib, n), n
    assert lib.csa2c_sink_slots(0, 10) == 2560
    assert lib.csa2c_sink_slots(3, 1) == 128 * 416
    assert lib.csa2c_sink_slots(4, 32) == 32 * 1024
    # rejected before any launch
    assert lib.csa2c_stream(None, 16, None, 1, None) == -1
    assert lib.csa2c_gather_units(None, None, 1, None, 1, None) == -1
    assert lib.csa2c_gather_rows(None, None, 1, None, 1, None) == -1
    assert lib.csa2c_attn_inputs(None, None, None, None, None, 0, None) == -1
    assert lib.csa2c_cta_load(None, 1, None, None) == -1


@pytest.mark.gpu
def test_ceiling_kernels_read_exactly_their_bytes():
    import torch
    lib = _lib()
    dev = torch.device("cuda:0")
    rng = np.random.default_rng(3)
    pool_h = rng.integers(0, 256, 8 << 20, dtype=np.uint8)
    pool = torch.from_numpy(pool_h).to(dev)
    sink = torch.zeros(1 << 20, dtype=torch.int32, device=dev)
    P = ctypes.c_void_p
    ptr = lambda t: P(t.data_ptr())
    st = P(torch.cuda.current_stream().cuda_stream)

    def run(kernel, grid, rc):
        assert rc == 0
        torch.cuda.synchronize()
        n = lib.csa2c_sink_slots(kernel, grid)
        return int(sink[:n].cpu().numpy().view(np.uint32).astype(np.uint64).sum()) & 0xFFFFFFFF

    # contiguous read with a ragged tail (n16 not a multiple of the grid)
    n16 = (1 << 20) // 16 + 5
    sink.zero_()
    assert run(0, 37, lib.csa2c_stream(ptr(pool), n16, ptr(sink), 37, st)) == _words(pool_h[: 16 * n16])
    # random 1-KiB units, an odd count, repeats allowed
    ids = rng.integers(0, (8 << 20) // 1024, 1001).astype(np.int32)
    ids_d = torch.from_numpy(ids).to(dev)
    sink.zero_()
    got = run(1, 13, lib.csa2c_gather_units(ptr(pool), ptr(ids_d), len(ids), ptr(sink), 13, st))
    assert got == _words(pool_h.reshape(-1, 1024)[ids])
    # random 288-B rows, a count that leaves a partial round
    nrows = (8 << 20) // 288
    rids = rng.integers(0, nrows, 1000).astype(np.int32)
    rids_d = torch.from_numpy(rids).to(dev)
    sink.zero_()
    got = run(2, 7, lib.csa2c_gather_rows(ptr(pool), ptr(rids_d), len(rids), ptr(sink), 7, st))
    assert got == _words(pool_h[: nrows * 288].reshape(-1, 288)[rids])
    # the attention's inputs: 4 x every query + 128 x 160 rows; the slice store variant too
    q_h = rng.integers(0, 256, 32 * 65536, dtype=np.uint8)
    q = torch.from_numpy(q_h).to(dev)
    aids = rng.integers(0, nrows, 128 * 160).astype(np.int32)
    aids_d = torch.from_numpy(aids).to(dev)
    part = torch.zeros(128 * 65536, dtype=torch.uint8, device=dev)
    want = (4 * _words(q_h) + _words(pool_h[: nrows * 288].reshape(-1, 288)[aids])) & 0xFFFFFFFF
    for store in (0, 1):
        sink.zero_()
        got = run(3, 128, lib.csa2c_attn_inputs(ptr(q), ptr(pool), ptr(aids_d), ptr(part), ptr(sink), store, st))
        assert got == want
    # every CTA wrote its whole slice
    assert int((part.view(torch.int32).view(128, 4096, 4)[:, :, 1] ==
                torch.arange(4096, device=dev, dtype=torch.int32)).all().item())
    # 64 KiB per CTA
    sink.zero_()
    assert run(4, 32, lib.csa2c_cta_load(ptr(q), 32, ptr(sink), st)) == _words(q_h)
