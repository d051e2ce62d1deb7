"""The CUDA path's certified bound on the hand-worked cases of
tests/golden/bound_hand_worked.txt ("Runtime-Certified Bounded-Error Quantized
Attention", Methodology 2): the bound within the parity tolerance of the
values derived by hand, and the output within tolerance of the oracle's."""

import numpy as np
import pytest
import torch

import oracle
from gpu_cases import TOL_BOUND_REL, TOL_MAXABS
from test_oracle_bound_golden import CASES, D

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("the GPU tests need a CUDA device")
    from quantized_decode_attention_kvq_b200 import build
    build.build()


@pytest.mark.parametrize("case", CASES, ids=[c["name"] for c in CASES])
def test_gpu_bound_matches_hand_worked(case):
    from quantized_decode_attention_kvq_b200 import kvq
    cfg = case["cfg"]
    pt = np.array([[int(p) for p in cfg["page_table"].split(",")]], np.int32)
    n = len(case["tokens"])
    k = np.stack([t[0] for t in case["tokens"]])[None, None]
    v = np.stack([t[1] for t in case["tokens"]])[None, None]
    q = case["q"].reshape(1, 1, 1, D)
    c = kvq.PagedCache(1, D, pt.shape[1], k_bits=int(cfg["kbits"]), k_group=int(cfg["kgroup"]),
                       k_rotate=cfg["rotate"] == "1", rot_signs=case["signs"])
    ptd = torch.from_numpy(pt).cuda()
    sl = torch.tensor([n], dtype=torch.int32, device="cuda")
    c.append(torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda(), ptd,
             torch.zeros(1, dtype=torch.int32, device="cuda"), sl)
    ws = c.workspace(1, 1, 1, pt.shape[1])
    out, bound, flags = c.decode(torch.from_numpy(q).cuda(), ptd, sl, ws)
    torch.cuda.synchronize()
    assert c.device_error() == 0
    want = case["expect"]["bound"]
    got = float(bound.cpu()[0, 0, 0])
    assert abs(got - want) <= TOL_BOUND_REL * want, (got, want)
    oc = oracle.Cache(D, 1, pt.shape[1], k_bits=int(cfg["kbits"]), k_group=int(cfg["kgroup"]),
                      k_rotate=cfg["rotate"] == "1", rot_signs=case["signs"])
    assert oc.append(k, v, pt, np.zeros(1, np.int32)) == 0
    o_hat, _, _, _ = oc.decode(q, pt, np.array([n], np.int32))
    assert np.abs(out.cpu().numpy().reshape(-1) - o_hat[0]).max() <= TOL_MAXABS
