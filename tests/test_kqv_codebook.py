"""The library's KQV codebook (kvq_kqv_codebook, host code, no GPU needed)
against the oracle's: both compute the Lloyd-Max quantizer of N(0, 1) by
their own iteration (thresholds versus centroids first), and the fp32 tables
the codes are decided with must agree bit for bit."""

import numpy as np
import pytest

import oracle


@pytest.fixture(scope="module")
def kvq():
    from quantized_decode_attention_kvq_b200 import build
    build.build()
    from quantized_decode_attention_kvq_b200 import kvq as m
    return m


@pytest.mark.parametrize("bits", [1, 2, 3, 4, 5])
@pytest.mark.parametrize("d", [64, 128])
def test_codebook_equals_the_oracle(kvq, oracle_lib, bits, d):
    cent, thr = kvq.kqv_codebook(bits, d)
    ocent, othr = oracle.kqv_tables(bits, d)
    assert np.array_equal(cent.view(np.uint32), ocent.view(np.uint32))
    assert np.array_equal(thr.view(np.uint32), othr.view(np.uint32))
    assert np.all(np.diff(cent) > 0) and np.all((thr > cent[:-1]) & (thr < cent[1:]))
    assert thr[thr.size // 2] == 0.0 and np.array_equal(cent, -cent[::-1])
