"""GPU parity: the CUDA path (through the C ABI) against the oracle on the same
seeded inputs.  Codes, scales, eta and flags bit-exact; outputs within max-abs
2e-3 and relative L2 1e-3; the bound within 1e-4 relative and never below the
observed error against exact attention."""

import math

import numpy as np
import pytest
import torch

import oracle
from gpu_cases import (TOL_BOUND_REL, TOL_MAXABS, TOL_RELL2, compare_flags, compare_outputs,
                       record_margin,
                       gpu_cache, oracle_pool, run_gpu, to_torch)
from oracle_cases import SMALL, device_pool, max_err, small
from quantized_decode_attention_kvq_b200 import inputs as synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("the GPU tests need a CUDA device")
    from quantized_decode_attention_kvq_b200 import build
    build.build()


def _check_decode(inp, g, o_hat, bound, flags, tau):
    wl = inp.wl
    record_margin(f"{wl.name} B={wl.num_seqs} ctx<={max(inp.seq_lens)} seed={inp.seed}",
                  g["out"], o_hat, spike_seqs=list(inp.spike_seqs),
                  rows_per_seq=wl.num_queries * wl.num_q_heads)
    emax, rel = compare_outputs(g["out"], o_hat)
    assert emax <= TOL_MAXABS and rel <= TOL_RELL2, (emax, rel)
    brel = np.abs(g["bound"] - bound) / np.maximum(bound, 1e-30)
    assert brel.max() <= TOL_BOUND_REL, brel.max()
    bad, tie = compare_flags(g["flags"], flags, bound, tau)
    assert bad == 0, (bad, tie)


@pytest.mark.parametrize("name", list(SMALL))
@pytest.mark.parametrize("seed", [0, 1])
def test_append_bit_exact(name, seed):
    inp = small(name, seed)
    k, v = inp.kv()
    g = run_gpu(inp, k, v)
    oc = oracle_pool(inp, k, v)
    assert g["err"] == 0
    pool = g["cache"].pool.cpu().numpy()
    opool = device_pool(oc)
    assert np.array_equal(pool, opool), np.flatnonzero(pool != opool)[:10]
    eta = g["cache"].eta.cpu().numpy()
    assert np.array_equal(eta.view(np.uint32), oc.eta.view(np.uint32))


@pytest.mark.parametrize("name", list(SMALL))
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_decode_matches_oracle(name, seed):
    inp = small(name, seed)
    k, v = inp.kv()
    q = inp.q()
    g = run_gpu(inp, k, v, q)
    oc = oracle_pool(inp, k, v)
    o_hat, bound, flags, _ = oc.decode(q, inp.page_table, inp.seq_lens, tau=inp.wl.tau)
    assert g["err"] == 0
    _check_decode(inp, g, o_hat, bound, flags, inp.wl.tau)
    # certified: the GPU's own output is within its bound of exact attention
    o_dense = oracle.dense(q, k, v, inp.seq_lens)
    assert (g["bound"] >= max_err(o_dense, g["out"])).all()


@pytest.mark.parametrize("name", ["llama8b", "serving"])
def test_flags_with_finite_tau(name):
    """Flags bit-exact at a tau inside the bound distribution (about half flagged)."""
    inp = small(name, 4)
    k, v = inp.kv()
    q = inp.q()
    oc = oracle_pool(inp, k, v)
    _, bound, _, _ = oc.decode(q, inp.page_table, inp.seq_lens)
    tau = float(np.float32(np.median(bound)))
    o_hat, bound, flags, _ = oc.decode(q, inp.page_table, inp.seq_lens, tau=tau)
    g = run_gpu(inp, k, v, q, tau=tau)
    assert 0 < flags.sum() < flags.size
    _check_decode(inp, g, o_hat, bound, flags, tau)


def test_bound_only_entry_point_matches():
    inp = small("llama8b", 0)
    k, v = inp.kv()
    a = run_gpu(inp, k, v, tau=5.0)
    b = run_gpu(inp, k, v, tau=5.0, bound_only=True)
    assert np.array_equal(a["bound"], b["bound"]) and np.array_equal(a["flags"], b["flags"])


def test_page_permutation_invariance():
    """Outputs depend on logical order only: another physical permutation of the
    same pages gives bit-identical results."""
    inp = small("llama8b", 1)
    k, v = inp.kv()
    q = inp.q()
    a = run_gpu(inp, k, v, q)
    rng = np.random.default_rng(123)
    perm = rng.permutation(inp.num_pages).astype(np.int32)
    pt2 = np.where(inp.page_table >= 0, perm[np.maximum(inp.page_table, 0)], -1).astype(np.int32)
    b = run_gpu(inp, k, v, q, page_table=pt2)
    assert np.array_equal(a["out"], b["out"]) and np.array_equal(a["bound"], b["bound"])


@pytest.mark.parametrize("pps", [1, 3, 7])
def test_split_count_invariance(monkeypatch, pps):
    """Split-K with other split sizes agrees with the single-pass oracle."""
    monkeypatch.setenv("KVQ_PAGES_PER_SPLIT", str(pps))
    inp = small("long128k", 0)
    k, v = inp.kv()
    q = inp.q()
    g = run_gpu(inp, k, v, q)
    oc = oracle_pool(inp, k, v)
    o_hat, bound, flags, _ = oc.decode(q, inp.page_table, inp.seq_lens)
    _check_decode(inp, g, o_hat, bound, flags, math.inf)


def test_ragged_and_empty_contexts():
    inp = synth.make("serving", 7, num_seqs=5, num_q_heads=8, num_kv_heads=2, ctx=70, ctx_min=1)
    inp.seq_lens[2] = 0          # an empty context
    inp.seq_lens[3] = 16         # exactly one page
    k, v = inp.kv()
    q = inp.q()
    g = run_gpu(inp, k, v, q, tau=math.inf)
    oc = oracle_pool(inp, k, v)
    o_hat, bound, flags, _ = oc.decode(q, inp.page_table, inp.seq_lens)
    _check_decode(inp, g, o_hat, bound, flags, math.inf)
    rows = slice(2 * 8, 3 * 8)
    assert (g["out"][rows] == 0).all() and (g["bound"][rows] == 0).all()


def test_device_errors_are_reported():
    inp = small("llama8b", 0)
    k, v = inp.kv()
    c = gpu_cache(inp)
    kd, vd = to_torch(k), to_torch(v)
    pt = inp.page_table.copy()
    pt[0, 1] = inp.num_pages + 5                       # outside the pool
    ptd = torch.from_numpy(pt).cuda()
    sp = torch.zeros(inp.wl.num_seqs, dtype=torch.int32, device="cuda")
    sl = torch.tensor(inp.seq_lens, dtype=torch.int32, device="cuda")
    c.append(kd, vd, ptd, sp, sl)
    from quantized_decode_attention_kvq_b200 import kvq
    assert c.device_error() == kvq.KVQ_ERR_INVALID_ARG
    assert c.device_error() == 0                        # cleared
    ws = c.workspace(inp.wl.num_seqs, 1, inp.wl.num_q_heads, pt.shape[1])
    c.decode(to_torch(inp.q()), ptd, sl, ws)
    assert c.device_error() == kvq.KVQ_ERR_INVALID_ARG
    # non-finite input
    kn = k.copy()
    kn[0, 0, 3, 5] = 0x7FC0                            # bf16 NaN
    c2 = gpu_cache(inp)
    c2.append(to_torch(kn), vd, torch.from_numpy(inp.page_table).cuda(), sp, sl)
    assert c2.device_error() == kvq.KVQ_ERR_RANGE


@pytest.mark.parametrize("name", ["llama8b", "long128k", "rotated"])
def test_full_size_parity(name):
    """The workloads at full size, every output element against the oracle."""
    inp = synth.make(name, 0)
    k, v = inp.kv()
    q = inp.q()
    g = run_gpu(inp, k, v, q)
    assert g["err"] == 0
    oc = oracle_pool(inp, k, v)
    assert np.array_equal(g["cache"].pool.cpu().numpy(), device_pool(oc))
    o_hat, bound, flags, _ = oc.decode(q, inp.page_table, inp.seq_lens, tau=inp.wl.tau)
    _check_decode(inp, g, o_hat, bound, flags, inp.wl.tau)


@pytest.mark.parametrize("name,seed", [("llama8b", 0), ("llama8b", 1), ("long128k", 0)])
def test_fused_step_full_size(name, seed):
    """The configuration the benchmark times, at full size: the context up to the
    last token appended, then one kvq_decode_attention_append launch that encodes
    the last token of every sequence and decodes.  The pool and eta must equal the
    oracle's full append bit for bit; every output, bound and flag is checked
    against the oracle's decode."""
    from quantized_decode_attention_kvq_b200 import kvq
    inp = synth.make(name, seed)
    wl = inp.wl
    k, v = inp.kv()
    q = inp.q()
    kd, vd, qd = to_torch(k), to_torch(v), to_torch(q)
    pt = torch.from_numpy(inp.page_table).cuda()
    lens = np.array(inp.seq_lens, np.int32)
    sl = torch.from_numpy(lens).cuda()
    before = torch.from_numpy(np.maximum(lens - 1, 0)).cuda()
    zeros = torch.zeros(wl.num_seqs, dtype=torch.int32, device="cuda")
    last = torch.from_numpy(np.maximum(lens - 1, 0).astype(np.int64)).cuda()
    idx = last.view(-1, 1, 1, 1).expand(-1, wl.num_kv_heads, 1, wl.head_dim)
    k_new = torch.gather(kd, 2, idx).contiguous()
    v_new = torch.gather(vd, 2, idx).contiguous()
    c = gpu_cache(inp)
    c.append(kd, vd, pt, zeros, before)
    S, NQ, HQ, d = q.shape
    ws = c.workspace(S, NQ, HQ, pt.shape[1])
    out = torch.full((S, NQ, HQ, d), float("nan"), dtype=torch.float32, device="cuda")
    bound = torch.full((S, NQ, HQ), float("nan"), dtype=torch.float32, device="cuda")
    flags = torch.full((S, NQ, HQ), 7, dtype=torch.uint8, device="cuda")
    dt = kvq.KVQ_BF16 if kd.dtype == torch.bfloat16 else kvq.KVQ_F32
    rc = kvq.kvq_decode_attention_append(
        c.desc, k_new, v_new, dt, k_new.stride(0), k_new.stride(1), qd,
        kvq.KVQ_BF16 if qd.dtype == torch.bfloat16 else kvq.KVQ_F32, S, NQ, HQ, pt,
        pt.shape[1], sl, 0.0, wl.tau, out, bound, flags, ws, ws.numel())
    assert rc == kvq.KVQ_OK, kvq.last_error()
    torch.cuda.synchronize()
    assert c.device_error() == 0
    oc = oracle_pool(inp, k, v)
    assert np.array_equal(c.pool.cpu().numpy(), device_pool(oc))
    assert np.array_equal(c.eta.cpu().numpy().view(np.uint32), oc.eta.view(np.uint32))
    o_hat, ob, of, _ = oc.decode(q, inp.page_table, inp.seq_lens, tau=wl.tau)
    g = dict(out=out.cpu().numpy().reshape(-1, d).astype(np.float64),
             bound=bound.cpu().numpy().reshape(-1).astype(np.float64),
             flags=flags.cpu().numpy().reshape(-1))
    _check_decode(inp, g, o_hat, ob, of, wl.tau)


@pytest.mark.parametrize("pages_per_split", [None, "64"])
def test_unread_page_leaves_no_certified_bound(monkeypatch, pages_per_split):
    """A page index outside the pool is never copied: the error word is set and
    every row of that (sequence, kv head) gets bound = +inf and flag = 1, even
    with tau = inf, so the exact fallback recomputes it.  A context longer than
    the page table does the same.  Other units are untouched."""
    from quantized_decode_attention_kvq_b200 import kvq
    if pages_per_split:
        monkeypatch.setenv("KVQ_PAGES_PER_SPLIT", pages_per_split)
    inp = small("llama8b", 0)
    wl = inp.wl
    g = run_gpu(inp)
    assert g["err"] == 0
    G = wl.num_q_heads // wl.num_kv_heads
    # sequence 1, logical page 5 -> an index one past the pool (kv head 0 and 1)
    pt = inp.page_table.copy()
    pt[1, 5] = inp.num_pages
    ptd = torch.from_numpy(pt).cuda()
    ws = g["cache"].workspace(wl.num_seqs, wl.num_queries, wl.num_q_heads, pt.shape[1])
    out, bound, flags = g["cache"].decode(g["q"], ptd, g["sl"], ws, tau=math.inf)
    torch.cuda.synchronize()
    assert g["cache"].device_error() == kvq.KVQ_ERR_INVALID_ARG
    b = bound.cpu().numpy().reshape(wl.num_seqs, -1)
    f = flags.cpu().numpy().reshape(wl.num_seqs, -1)
    assert np.isinf(b[1]).all() and (f[1] == 1).all()
    ref_b = g["bound"].reshape(wl.num_seqs, -1)
    assert np.array_equal(b[0], ref_b[0].astype(np.float32)) and (f[0] == 0).all()
    ref_o = g["out"].reshape(wl.num_seqs, -1)
    assert np.array_equal(out.cpu().numpy().reshape(wl.num_seqs, -1)[0], ref_o[0].astype(np.float32))
    # a context longer than the page table: sequence 0 is cut, marked uncertified
    sl = g["sl"].clone()
    sl[0] = pt.shape[1] * 16 + 1
    out, bound, flags = g["cache"].decode(g["q"], g["pt"], sl, ws, tau=math.inf)
    torch.cuda.synchronize()
    assert g["cache"].device_error() == kvq.KVQ_ERR_INVALID_ARG
    b = bound.cpu().numpy().reshape(wl.num_seqs, -1)
    f = flags.cpu().numpy().reshape(wl.num_seqs, -1)
    assert np.isinf(b[0]).all() and (f[0] == 1).all()
    assert np.isfinite(b[1]).all() and (f[1] == 0).all()
    assert G == 4
