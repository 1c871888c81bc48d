"""The shared seeded generator: published SplitMix64 outputs, counter independence,
distribution sanity and the five workload definitions."""
import ctypes

import numpy as np


def test_splitmix64_reference_outputs(host_gen):
    # first outputs of SplitMix64 started at state 0 (the reference sequence
    # published with Vigna's splitmix64.c)
    st = ctypes.c_uint64(0)
    lib = host_gen.host_lib()
    got = [lib.wl_splitmix64_next(ctypes.byref(st)) for _ in range(3)]
    assert got == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_counter_based_rows_are_position_independent(host_gen):
    a = host_gen.kv_rows(1, 3, 0, 20)
    b = host_gen.kv_rows(1, 3, 10, 5)
    np.testing.assert_array_equal(a[10:15], b)
    assert not np.array_equal(host_gen.kv_rows(1, 4, 0, 20), a)
    assert not np.array_equal(host_gen.kv_rows(2, 3, 0, 20), a)


def test_normal_distribution_sanity(host_gen):
    x = host_gen.normal_f32(0, 12345, 0, 400000).astype(np.float64)
    assert abs(x.mean()) < 0.01 and abs(x.var() - 1.0) < 0.01
    assert np.abs(x).max() < 6.0
    # one int->float rounding then an exact power-of-two scale
    assert np.all(x * 2.0 ** 24 == np.round(x * 2.0 ** 24))


def test_outliers_and_query_scale(host_gen):
    ch = host_gen.outlier_channels(0)
    assert ch.size == 5 and np.unique(ch).size == 5 and ch.max() < 512
    kv = host_gen.kv_rows(0, 0, 0, 4096)
    from oracle.formats import bf16_to_f64
    v = bf16_to_f64(kv)
    sd = v.std(axis=0)
    assert np.all(sd[ch] > 6.0) and np.median(sd) < 1.1
    q = bf16_to_f64(host_gen.q_rows(0, 0, 0, 16))
    assert abs(q.std() * np.sqrt(512) - 1.0) < 0.05


def test_page_table_and_workloads(host_gen):
    w1 = host_gen.workload(1)
    assert w1.n_pages_pool == 233016 and w1.batch == 32 and w1.max_pages == 1024
    pt = host_gen.page_table(w1.seed, w1.n_pages_pool, [w1.max_pages] * w1.batch, w1.max_pages)
    assert np.unique(pt).size == pt.size and pt.min() >= 0 and pt.max() < 233016
    w4 = host_gen.workload(4)
    lens = np.array(w4.lengths)
    assert lens.min() >= 4096 and lens.max() <= 1048576 and len(lens) == 64
    assert w4.reindex_mask.sum() == 16 and w4.miss_mask.sum() == 6
    w3 = host_gen.workload(3)
    assert w3.raw_tokens // w3.compress == 65536 and w3.raw_tokens // w3.chunk == 16
    perm = host_gen.permutation(9, 1, 1000)
    assert sorted(perm.tolist()) == list(range(1000))
