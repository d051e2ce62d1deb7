"""kvq_decode_attention_noalloc: the decode entry point for callers that cannot
allocate device memory where they call it -- an allocator-free runtime, a host
framework that hands the library fixed buffers, or code that runs where a
cudaMalloc is forbidden or would synchronize the device.  It uses the
library's static device scratch instead of a caller workspace.

Checked here through the C ABI against kvq_decode_attention with a workspace,
on two calls in a row (the scratch keeps the previous call's contents), within
the tolerances of the other parity tests.  This file is collected last."""

import math

import numpy as np
import pytest
import torch

from gpu_cases import TOL_BOUND_REL, TOL_MAXABS, TOL_RELL2, compare_outputs, run_gpu
from oracle_cases import small

pytestmark = pytest.mark.gpu


def _buffers(inp):
    wl = inp.wl
    S, NQ, HQ, d = wl.num_seqs, wl.num_queries, wl.num_q_heads, wl.head_dim
    return (torch.empty((S, NQ, HQ, d), dtype=torch.float32, device="cuda"),
            torch.empty((S, NQ, HQ), dtype=torch.float32, device="cuda"),
            torch.empty((S, NQ, HQ), dtype=torch.uint8, device="cuda"))


def _noalloc(g, inp, tau, bufs, stream=None):
    """One call into caller-owned buffers (poisoned first); no torch allocation
    happens between the poisoning and the read-back."""
    from quantized_decode_attention_kvq_b200 import kvq
    wl = inp.wl
    S, NQ, HQ, d = wl.num_seqs, wl.num_queries, wl.num_q_heads, wl.head_dim
    out, bound, flags = bufs
    s = stream if stream is not None else torch.cuda.current_stream()
    with torch.cuda.stream(s):
        out.fill_(float("nan"))
        bound.fill_(float("nan"))
        flags.fill_(7)
        q = g["q"]
        rc = kvq.kvq_decode_attention_noalloc(
            g["cache"].desc, q, kvq.KVQ_BF16 if q.dtype == torch.bfloat16 else kvq.KVQ_F32, S,
            NQ, HQ, g["pt"], g["pt"].shape[1], g["sl"], 0.0, tau, out, bound, flags, s)
    assert rc == kvq.KVQ_OK, kvq.last_error()
    torch.cuda.synchronize()
    return (out.cpu().numpy().reshape(-1, d).astype(np.float64),
            bound.cpu().numpy().reshape(-1).astype(np.float64), flags.cpu().numpy().reshape(-1))


def _check(res, g):
    out, bound, flags = res
    emax, rel = compare_outputs(out, g["out"])
    assert emax <= TOL_MAXABS and rel <= TOL_RELL2, (emax, rel)
    assert (np.abs(bound - g["bound"]) <= TOL_BOUND_REL * g["bound"]).all()
    assert np.array_equal(flags, g["flags"])


@pytest.mark.parametrize("name,tau", [("llama8b", 5.0), ("serving", math.inf)])
def test_noalloc_matches_workspace_entry_point(name, tau):
    if not torch.cuda.is_available():
        pytest.fail("the GPU tests need a CUDA device")
    inp = small(name, 3)
    g = run_gpu(inp, tau=tau)                       # kvq_decode_attention with a workspace
    bufs = _buffers(inp)
    for _ in range(2):                              # two calls in a row share the scratch
        _check(_noalloc(g, inp, tau, bufs), g)
    assert g["cache"].device_error() == 0


def test_noalloc_allocates_nothing_and_runs_on_any_stream():
    """After a first call (which may load the library's device code), further
    calls leave the device's free memory unchanged, on the default stream and on
    a stream of the caller's."""
    if not torch.cuda.is_available():
        pytest.fail("the GPU tests need a CUDA device")
    inp = small("llama8b", 5)
    g = run_gpu(inp, tau=5.0)
    bufs = _buffers(inp)
    side = torch.cuda.Stream()
    _check(_noalloc(g, inp, 5.0, bufs), g)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    _check(_noalloc(g, inp, 5.0, bufs), g)
    _check(_noalloc(g, inp, 5.0, bufs, stream=side), g)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0, (free0, free1)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    from quantized_decode_attention_kvq_b200 import kvq
    if not torch.cuda.is_available():
        pytest.fail("the GPU tests need a CUDA device")
    inp = small("llama8b", 0)
    c = kvq.PagedCache(inp.wl.num_kv_heads, inp.wl.head_dim, inp.num_pages)
    seqs, max_pages = 4096, 4096                    # far more split-K scratch than it holds
    need = kvq.kvq_workspace_size(c.desc, seqs, 1, inp.wl.num_q_heads, max_pages)
    assert need > kvq.NOALLOC_SCRATCH_BYTES
    dummy = torch.zeros(16, dtype=torch.int32, device="cuda")
    rc = kvq.kvq_decode_attention_noalloc(c.desc, dummy, kvq.KVQ_BF16, seqs, 1,
                                          inp.wl.num_q_heads, dummy, max_pages, dummy, 0.0,
                                          math.inf, dummy, dummy, dummy)
    assert rc == kvq.KVQ_ERR_UNSUPPORTED
    assert "static scratch" in kvq.last_error()


def test_noalloc_on_a_kqv_cache():
    """The same entry point over a cache of the KQV codec (its split kernel and
    merge use the static scratch too): bit for bit the workspace decode."""
    from quantized_decode_attention_kvq_b200 import kvq
    from gpu_cases import to_torch
    if not torch.cuda.is_available():
        pytest.fail("the GPU tests need a CUDA device")
    inp = small("serving", 7)
    wl = inp.wl
    k, v = inp.kv()
    q = inp.q()
    g = kvq.PagedCache(wl.num_kv_heads, wl.head_dim, inp.num_pages, codec="kqv",
                       rot_signs=inp.rotation_signs(), qjl_matrix=inp.qjl_matrix())
    pt = torch.from_numpy(inp.page_table).cuda()
    sl = torch.tensor(inp.seq_lens, dtype=torch.int32, device="cuda")
    g.append(to_torch(k), to_torch(v), pt, torch.zeros(wl.num_seqs, dtype=torch.int32,
                                                       device="cuda"), sl)
    qd = to_torch(q)
    S, NQ, HQ, d = q.shape
    ws = g.workspace(S, NQ, HQ, pt.shape[1])
    out_w, bound_w, flags_w = g.decode(qd, pt, sl, ws, tau=20.0)
    out, bound, flags = _buffers(inp)
    out.fill_(float("nan"))
    qdt = kvq.KVQ_BF16 if qd.dtype == torch.bfloat16 else kvq.KVQ_F32
    rc = kvq.kvq_decode_attention_noalloc(g.desc, qd, qdt, S, NQ, HQ, pt, pt.shape[1], sl, 0.0,
                                          20.0, out, bound, flags)
    assert rc == kvq.KVQ_OK, kvq.last_error()
    torch.cuda.synchronize()
    assert g.device_error() == 0
    assert torch.equal(out, out_w.view_as(out)) and torch.equal(bound, bound_w.view_as(bound))
    assert torch.equal(flags, flags_w.view_as(flags))


def test_noalloc_on_an_hqmq_cache():
    """The same entry point over a cache of the HQMQ codec: bit for bit the
    workspace decode."""
    from quantized_decode_attention_kvq_b200 import kvq
    from gpu_cases import to_torch
    if not torch.cuda.is_available():
        pytest.fail("the GPU tests need a CUDA device")
    inp = small("serving", 8)
    wl = inp.wl
    k, v = inp.kv()
    q = inp.q()
    g = kvq.PagedCache(wl.num_kv_heads, wl.head_dim, inp.num_pages, codec="hqmq",
                       hq_secondary=inp.hqmq_secondary(32))
    pt = torch.from_numpy(inp.page_table).cuda()
    sl = torch.tensor(inp.seq_lens, dtype=torch.int32, device="cuda")
    g.append(to_torch(k), to_torch(v), pt, torch.zeros(wl.num_seqs, dtype=torch.int32,
                                                       device="cuda"), sl)
    qd = to_torch(q)
    S, NQ, HQ, d = q.shape
    ws = g.workspace(S, NQ, HQ, pt.shape[1])
    out_w, bound_w, flags_w = g.decode(qd, pt, sl, ws, tau=20.0)
    out, bound, flags = _buffers(inp)
    out.fill_(float("nan"))
    qdt = kvq.KVQ_BF16 if qd.dtype == torch.bfloat16 else kvq.KVQ_F32
    rc = kvq.kvq_decode_attention_noalloc(g.desc, qd, qdt, S, NQ, HQ, pt, pt.shape[1], sl, 0.0,
                                          20.0, out, bound, flags)
    assert rc == kvq.KVQ_OK, kvq.last_error()
    torch.cuda.synchronize()
    assert g.device_error() == 0
    assert torch.equal(out, out_w.view_as(out)) and torch.equal(bound, bound_w.view_as(bound))
    assert torch.equal(flags, flags_w.view_as(flags))
