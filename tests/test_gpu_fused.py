"""kvq_decode_attention_append (the step's append fused into the decode) against
the two separate calls on the same cache: identical pool bytes and eta (the
same codec arithmetic), identical flags, and outputs and bounds equal up to
the fp32 summation order (the fused launch gives its last split fewer pages,
so splits can sum pages in another grouping).  Ragged lengths include 0
(nothing appended) and 1 (the new token is the whole context)."""

import math

import numpy as np
import pytest
import torch

from gpu_cases import gpu_cache, to_torch
from oracle_cases import small
from quantized_decode_attention_kvq_b200 import inputs as synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("the GPU tests need a CUDA device")


def _cases():
    yield "llama8b", small("llama8b", 2), 5.0
    yield "rotated", small("rotated", 1), math.inf
    yield "tiny", small("tiny", 0), math.inf
    # pages are allocated for 200 tokens per sequence; the lengths are then cut
    inp = synth.make("serving", 3, num_seqs=6, num_q_heads=8, num_kv_heads=2, ctx=200,
                     ctx_min=200)
    inp.seq_lens[:] = [199, 0, 1, 16, 17, 200]   # 16: the new token fills a page's last
    yield "serving-ragged", inp, 1.0              # slot; 17: it opens a new page


@pytest.mark.parametrize("case", list(range(4)))
def test_fused_step_equals_append_then_decode(case):
    from quantized_decode_attention_kvq_b200 import kvq
    name, inp, tau = list(_cases())[case]
    wl = inp.wl
    k, v = inp.kv()
    q = inp.q()
    kd, vd, qd = to_torch(k), to_torch(v), to_torch(q)
    pt = torch.from_numpy(inp.page_table).cuda()
    lens = np.array(inp.seq_lens, np.int32)
    sl = torch.from_numpy(lens).cuda()
    before = torch.from_numpy(np.maximum(lens - 1, 0)).cuda()      # context before the step
    zeros = torch.zeros(wl.num_seqs, dtype=torch.int32, device="cuda")
    last = torch.from_numpy(np.maximum(lens - 1, 0).astype(np.int64)).cuda()
    idx = last.view(-1, 1, 1, 1).expand(-1, wl.num_kv_heads, 1, wl.head_dim)
    k_new = torch.gather(kd, 2, idx).contiguous()                  # [S][Hkv][1][d]
    v_new = torch.gather(vd, 2, idx).contiguous()
    dt = kvq.KVQ_BF16 if kd.dtype == torch.bfloat16 else kvq.KVQ_F32
    S, NQ, HQ, d = q.shape

    results = []
    for fused in (False, True):
        c = gpu_cache(inp)
        c.append(kd, vd, pt, zeros, before)
        ws = c.workspace(S, NQ, HQ, pt.shape[1])
        out = torch.full((S, NQ, HQ, d), float("nan"), dtype=torch.float32, device="cuda")
        bound = torch.full((S, NQ, HQ), float("nan"), dtype=torch.float32, device="cuda")
        flags = torch.full((S, NQ, HQ), 7, dtype=torch.uint8, device="cuda")
        if fused:
            rc = kvq.kvq_decode_attention_append(
                c.desc, k_new, v_new, dt, k_new.stride(0), k_new.stride(1), qd,
                kvq.KVQ_BF16 if qd.dtype == torch.bfloat16 else kvq.KVQ_F32, S, NQ, HQ, pt,
                pt.shape[1], sl, 0.0, tau, out, bound, flags, ws, ws.numel())
            assert rc == kvq.KVQ_OK, kvq.last_error()
        else:
            has_new = torch.from_numpy((lens > 0).astype(np.int32)).cuda()
            c.append(k_new, v_new, pt, before, has_new)
            c.decode(qd, pt, sl, ws, tau=tau, out=out, bound=bound, flags=flags)
        torch.cuda.synchronize()
        assert c.device_error() == 0
        results.append((c.pool.cpu().numpy(), c.eta.cpu().numpy(), out.cpu().numpy(),
                        bound.cpu().numpy(), flags.cpu().numpy()))
    (pa, ea, oa, ba, fa), (pb, eb, ob, bb, fb) = results
    assert np.array_equal(pa, pb), name
    assert np.array_equal(ea.view(np.uint32), eb.view(np.uint32)), name
    assert np.abs(oa - ob).max() <= 1e-5 * max(1.0, np.abs(oa).max()), name
    assert (np.abs(ba - bb) <= 1e-5 * ba).all(), name
    near = np.abs(ba - tau) <= 1e-4 * abs(tau) if math.isfinite(tau) else np.zeros_like(fa, bool)
    assert np.array_equal(fa[~near], fb[~near]), name


def test_fused_step_rejects_bad_arguments():
    from quantized_decode_attention_kvq_b200 import kvq
    inp = small("llama8b", 0)
    c = gpu_cache(inp)
    dummy = torch.zeros(16, dtype=torch.int32, device="cuda")
    rc = kvq.kvq_decode_attention_append(c.desc, None, dummy, kvq.KVQ_BF16, 0, 0, dummy,
                                         kvq.KVQ_BF16, 2, 1, 8, dummy, 4, dummy, 0.0, math.inf,
                                         dummy, dummy, dummy, dummy, 1 << 20)
    assert rc == kvq.KVQ_ERR_INVALID_ARG
    rc = kvq.kvq_decode_attention_append(c.desc, dummy, dummy, 9, 0, 0, dummy, kvq.KVQ_BF16, 2,
                                         1, 8, dummy, 4, dummy, 0.0, math.inf, dummy, dummy,
                                         dummy, dummy, 1 << 20)
    assert rc == kvq.KVQ_ERR_INVALID_ARG
