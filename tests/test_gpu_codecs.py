"""Every codec the library builds a kernel for, against the oracle: head_dim 64
and 128, 8- and 4-bit keys in groups of 32, 64 and 128 (those dividing
head_dim), with and without the Hadamard rotation, and the three ways four
query rows can share a kv head (4 GQA heads x 1 query, 2 x 2, 1 x 4).  Pool
bytes and eta bit-exact, outputs and bounds within the parity tolerances."""

import itertools

import numpy as np
import pytest
import torch

import oracle
from gpu_cases import (TOL_BOUND_REL, TOL_MAXABS, TOL_RELL2, compare_outputs, oracle_pool,
                       run_gpu)
from oracle_cases import device_pool, max_err
from quantized_decode_attention_kvq_b200 import inputs as synth

pytestmark = pytest.mark.gpu

CODECS = [(d, kb, kg) for d, kb, kg in itertools.product((64, 128), (8, 4), (32, 64, 128))
          if d % kg == 0]
ROWS = [(4, 1), (2, 2), (1, 4)]   # (GQA group, queries per sequence)


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("the GPU tests need a CUDA device")


@pytest.mark.parametrize("d,kb,kg", CODECS)
@pytest.mark.parametrize("rotate", [False, True])
def test_codec_parity(d, kb, kg, rotate):
    g_, nq = ROWS[(d + kb + kg + int(rotate)) % len(ROWS)]
    inp = synth.make("llama8b", 5, num_seqs=2, num_kv_heads=2, num_q_heads=2 * g_,
                     num_queries=nq, head_dim=d, ctx=211, k_bits=kb, k_group=kg,
                     k_rotate=rotate)
    k, v = inp.kv()
    q = inp.q()
    g = run_gpu(inp, k, v, q)
    assert g["err"] == 0
    oc = oracle_pool(inp, k, v)
    assert np.array_equal(g["cache"].pool.cpu().numpy(), device_pool(oc))
    assert np.array_equal(g["cache"].eta.cpu().numpy().view(np.uint32), oc.eta.view(np.uint32))
    o_hat, bound, _, _ = oc.decode(q, inp.page_table, inp.seq_lens)
    emax, rel = compare_outputs(g["out"], o_hat)
    assert emax <= TOL_MAXABS and rel <= TOL_RELL2, (emax, rel)
    assert (np.abs(g["bound"] - bound) <= TOL_BOUND_REL * bound).all()
    o_dense = oracle.dense(q, k, v, inp.seq_lens)
    assert (g["bound"] >= max_err(o_dense, g["out"])).all()
