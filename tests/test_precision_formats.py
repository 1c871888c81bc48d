"""Which operand formats can the attention's tensor-core products use?

The oracle's attention rerun with the query or the softmax weights rounded to
the low-precision formats the tensor cores take (tests/precision_formats.py),
on the 64K decode workload: four sequences' Full-layer index sets with the Full
and a Reuse layer's queries.  The kernel's own choice (bf16 query and exact
f16 keys, f16 weights) must stay well inside the parity bound; a query in FP8
or in the cache's NVFP4 codec must not -- which is why the Q.K^T product is not
run block-scaled (kind::mxf4nvf4) or in FP8.
"""
import pytest

from tests import precision_formats as pf


@pytest.fixture(scope="module")
def worst():
    return pf.table(pf.decode_sample())


def test_kernel_formats_stay_inside_the_bound(worst):
    # the output's own bf16 rounding is about a third of the bound
    assert worst["exact"] < 0.5
    for k in ("p_f16", "p_bf16"):
        assert worst[k] < 0.5, (k, worst[k])


def test_low_precision_queries_break_the_bound(worst):
    for k in ("q_fp8", "q_nvfp4", "q_nvfp4_g", "q_fp8_p_fp8"):
        assert worst[k] > 1.0, (k, worst[k])


def test_fp8_weights_alone_fit_but_without_margin(worst):
    assert 0.5 < worst["p_fp8"] <= 1.0
