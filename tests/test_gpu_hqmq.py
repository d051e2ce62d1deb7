"""GPU parity of the HQMQ codec ("Hurwitz Quaternion Multiplicative
Quantization for KV Cache Compression", Method 1-2) through the C ABI against
the oracle on the same seeded inputs: pool bytes (chunk codes, E4M3 radii,
|k|, eps, value range) and eta bit for bit after the append; outputs within
max-abs 2e-3 and relative L2 1e-3, the bound within 1e-4 relative and never
below the error against exact attention, flags equal outside the tie band."""

import math

import numpy as np
import pytest
import torch

import oracle
from gpu_cases import (TOL_BOUND_REL, TOL_MAXABS, TOL_RELL2, compare_flags, compare_outputs,
                       record_margin, to_torch)
from oracle_cases import SMALL, max_err, small
from quantized_decode_attention_kvq_b200 import inputs as synth

pytestmark = pytest.mark.gpu
SPIKES = dict(spike_seq_frac=0.5, spike_token_frac=0.05)
S_DEFAULT = 32


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("the GPU tests need a CUDA device")
    from quantized_decode_attention_kvq_b200 import build
    build.build()


def _caches(inp, S=S_DEFAULT, outliers=False):
    from quantized_decode_attention_kvq_b200 import kvq
    wl = inp.wl
    sec = inp.hqmq_secondary(S)
    g = kvq.PagedCache(wl.num_kv_heads, wl.head_dim, inp.num_pages, codec="hqmq",
                       hq_secondary=sec, outliers=outliers)
    o = oracle.HqCache(wl.head_dim, wl.num_kv_heads, inp.num_pages, sec, outliers=outliers)
    return g, o


def _run(inp, k, v, q, tau=None, seqs=None, bound_only=False, S=S_DEFAULT, outliers=False):
    wl = inp.wl
    g, o = _caches(inp, S, outliers)
    pt = torch.from_numpy(inp.page_table).cuda()
    sl = torch.tensor(inp.seq_lens, dtype=torch.int32, device="cuda")
    g.append(to_torch(k), to_torch(v), pt, torch.zeros(wl.num_seqs, dtype=torch.int32,
                                                       device="cuda"), sl)
    ws = g.workspace(wl.num_seqs, wl.num_queries, wl.num_q_heads, pt.shape[1])
    tau = wl.tau if tau is None else tau
    out, bound, flags = g.decode(to_torch(q), pt, sl, ws, tau=tau, bound_only=bound_only)
    torch.cuda.synchronize()
    res = dict(cache=g, err=g.device_error(),
               bound=bound.cpu().numpy().reshape(-1).astype(np.float64),
               flags=flags.cpu().numpy().reshape(-1))
    if out is not None:
        res["out"] = out.cpu().numpy().reshape(-1, wl.head_dim).astype(np.float64)
    sel = list(range(wl.num_seqs)) if seqs is None else seqs
    lens = np.array(inp.seq_lens, np.int32)
    assert o.append(k[sel], v[sel], inp.page_table[sel], np.zeros(len(sel), np.int32),
                    valid=lens[sel]) == 0
    res["oracle"] = o
    res["sel"] = sel
    return res


@pytest.mark.parametrize("name", list(SMALL))
@pytest.mark.parametrize("seed", [0, 1])
def test_append_bit_exact(name, seed):
    inp = small(name, seed, **SPIKES)
    k, v = inp.kv()
    r = _run(inp, k, v, inp.q())
    assert r["err"] == 0
    pool = r["cache"].pool.cpu().numpy()
    opool = r["oracle"].pool
    assert np.array_equal(pool, opool), np.flatnonzero(pool != opool)[:10]
    eta = r["cache"].eta.cpu().numpy()
    assert np.array_equal(eta.view(np.uint32), r["oracle"].eta.view(np.uint32))


@pytest.mark.parametrize("S", [1, 7, 64])
def test_append_bit_exact_secondary_sizes(S):
    inp = small("llama8b", 4, **SPIKES)
    k, v = inp.kv()
    r = _run(inp, k, v, inp.q(), S=S)
    assert r["err"] == 0
    assert np.array_equal(r["cache"].pool.cpu().numpy(), r["oracle"].pool)
    assert np.array_equal(r["cache"].eta.cpu().numpy().view(np.uint32),
                          r["oracle"].eta.view(np.uint32))


def _check(inp, r, q, tau, label, rows=None):
    wl = inp.wl
    lens = np.array(inp.seq_lens, np.int32)
    sel = r["sel"]
    o_hat, bound, flags, _ = r["oracle"].decode(q[sel], inp.page_table[sel], lens[sel], tau=tau)
    if rows is None:
        rows = np.concatenate([np.arange(s * wl.num_queries * wl.num_q_heads,
                                         (s + 1) * wl.num_queries * wl.num_q_heads) for s in sel])
    if "out" in r:
        record_margin(label, r["out"][rows], o_hat, rows_per_seq=wl.num_queries * wl.num_q_heads)
        emax, rel = compare_outputs(r["out"][rows], o_hat)
        assert emax <= TOL_MAXABS and rel <= TOL_RELL2, (emax, rel)
    brel = np.abs(r["bound"][rows] - bound) / np.maximum(bound, 1e-30)
    assert brel.max() <= TOL_BOUND_REL, brel.max()
    bad, tie = compare_flags(r["flags"][rows], flags, bound, tau)
    assert bad == 0, (bad, tie)
    return rows, o_hat


@pytest.mark.parametrize("name", list(SMALL))
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_decode_matches_oracle(name, seed):
    inp = small(name, seed, **SPIKES)
    k, v = inp.kv()
    q = inp.q()
    r = _run(inp, k, v, q)
    assert r["err"] == 0
    _check(inp, r, q, inp.wl.tau, f"hqmq {name} seed={seed}")
    o_dense = oracle.dense(q, k, v, inp.seq_lens)
    assert (max_err(o_dense, r["out"]) <= r["bound"]).all()


@pytest.mark.parametrize("S", [1, 64])
def test_decode_secondary_sizes(S):
    inp = small("serving", 2, **SPIKES)
    k, v = inp.kv()
    q = inp.q()
    r = _run(inp, k, v, q, S=S)
    _check(inp, r, q, inp.wl.tau, f"hqmq serving S={S}")


@pytest.mark.parametrize("pps", ["1", "3"])
def test_split_invariance(monkeypatch, pps):
    monkeypatch.setenv("KVQ_PAGES_PER_SPLIT", pps)
    inp = small("serving", 3, **SPIKES)
    k, v = inp.kv()
    q = inp.q()
    r = _run(inp, k, v, q)
    _check(inp, r, q, inp.wl.tau, f"hqmq serving pps={pps}")


def test_bound_only_and_finite_tau():
    inp = small("llama8b", 5)
    k, v = inp.kv()
    q = inp.q()
    tau = float(np.median(_run(inp, k, v, q)["bound"]))   # a threshold inside the bounds' spread
    full = _run(inp, k, v, q, tau=tau)
    bo = _run(inp, k, v, q, tau=tau, bound_only=True)
    assert "out" not in bo
    assert np.array_equal(bo["bound"], full["bound"]) and np.array_equal(bo["flags"], full["flags"])
    _check(inp, full, q, tau, "hqmq llama8b finite tau")
    assert 0 < full["flags"].sum() < full["flags"].size


def test_ragged_and_empty_contexts():
    inp = small("serving", 6, **SPIKES)
    lens = list(inp.seq_lens)
    lens[0] = 0
    lens[1] = 1
    lens[2] = 17
    inp.seq_lens = lens
    k, v = inp.kv()
    q = inp.q()
    r = _run(inp, k, v, q)
    rows_per = inp.wl.num_queries * inp.wl.num_q_heads
    assert np.all(r["out"][:rows_per] == 0) and np.all(r["bound"][:rows_per] == 0)
    _check(inp, r, q, inp.wl.tau, "hqmq ragged")


@pytest.mark.parametrize("name", ["tiny", "llama8b"])   # d = 64 and d = 128 (one warp per role)
def test_non_finite_input_is_reported(name):
    from quantized_decode_attention_kvq_b200 import kvq
    inp = small(name, 0)
    k, v = inp.kv()
    k = k.copy()
    v = v.copy()
    bf16 = k.dtype == np.uint16     # bf16 bit patterns: +inf 0x7f80, a quiet NaN 0x7fc0
    k[0, 0, 3, 5] = 0x7F80 if bf16 else np.inf
    v[0, 0, 7, 9] = 0x7FC0 if bf16 else np.nan
    wl = inp.wl
    g, o = _caches(inp)
    pt = torch.from_numpy(inp.page_table).cuda()
    sl = torch.tensor(inp.seq_lens, dtype=torch.int32, device="cuda")
    g.append(to_torch(k), to_torch(v), pt, torch.zeros(wl.num_seqs, dtype=torch.int32,
                                                       device="cuda"), sl)
    torch.cuda.synchronize()
    assert g.device_error() == kvq.KVQ_ERR_RANGE
    assert o.append(k, v, inp.page_table, np.zeros(wl.num_seqs, np.int32),
                    valid=np.array(inp.seq_lens, np.int32)) == oracle.ERR_RANGE
    # codes, radii and the finite annotations agree; the blocks of the two
    # tokens carry eta = +inf (and the key token eps = +inf) on both sides
    bb = o.block_bytes
    gp = g.pool.cpu().numpy().reshape(-1, bb)
    op = o.pool.reshape(-1, bb)
    nc = wl.head_dim // 4
    assert np.array_equal(gp[:, :96 * nc], op[:, :96 * nc])
    geta, oeta = g.eta.cpu().numpy(), o.eta
    assert np.array_equal(np.isinf(geta), np.isinf(oeta)) and np.isinf(oeta).any()
    fin = np.isfinite(oeta)
    assert np.array_equal(geta[fin], oeta[fin])


def test_unsupported_entry_points_and_arguments():
    from quantized_decode_attention_kvq_b200 import kvq
    inp = small("llama8b", 0)
    wl = inp.wl
    g, _ = _caches(inp)
    assert kvq.kvq_adaptive_work_size(g.desc, wl.num_seqs, 1, wl.num_q_heads, 4) == 0
    pt = torch.from_numpy(inp.page_table).cuda()
    sl = torch.tensor(inp.seq_lens, dtype=torch.int32, device="cuda")
    ws = g.workspace(wl.num_seqs, 1, wl.num_q_heads, pt.shape[1])
    q = to_torch(inp.q())
    kn = torch.zeros((wl.num_seqs, wl.num_kv_heads, 1, wl.head_dim), dtype=torch.bfloat16,
                     device="cuda")
    out = torch.zeros((wl.num_seqs, 1, wl.num_q_heads, wl.head_dim), device="cuda")
    bound = torch.zeros((wl.num_seqs, 1, wl.num_q_heads), device="cuda")
    flags = torch.zeros((wl.num_seqs, 1, wl.num_q_heads), dtype=torch.uint8, device="cuda")
    rc = kvq.kvq_decode_attention_append(g.desc, kn, kn, kvq.KVQ_BF16, kn.stride(0),
                                         kn.stride(1), q, kvq.KVQ_BF16, wl.num_seqs, 1,
                                         wl.num_q_heads, pt, pt.shape[1], sl, 0.0, math.inf,
                                         out, bound, flags, ws, ws.numel())
    assert rc == kvq.KVQ_ERR_UNSUPPORTED
    # a secondary set beyond the decode's shared-memory tables is refused
    g.desc.hq_s = kvq.KVQ_HQMQ_MAX_S + 1
    assert kvq.kvq_workspace_size(g.desc, wl.num_seqs, 1, wl.num_q_heads, 4) == 0


def test_full_size_sampled():
    """Full size (llama8b): the GPU appends and decodes every sequence; the
    oracle checks the pool and eta of two sequences bit for bit, and their rows."""
    inp = synth.make("llama8b", 0)
    wl = inp.wl
    k, v = inp.kv()
    q = inp.q()
    seqs = [0, wl.num_seqs - 1]
    r = _run(inp, k, v, q, seqs=seqs)
    assert r["err"] == 0
    bb = r["oracle"].block_bytes
    gpool = r["cache"].pool.cpu().numpy().reshape(inp.num_pages, wl.num_kv_heads, bb)
    opool = r["oracle"].pool.reshape(inp.num_pages, wl.num_kv_heads, bb)
    pages = np.concatenate([inp.page_table[s, :inp.pages_per_seq[s]] for s in seqs])
    assert np.array_equal(gpool[pages], opool[pages])
    assert np.array_equal(r["cache"].eta.cpu().numpy()[pages], r["oracle"].eta[pages])
    rows, o_hat = _check(inp, r, q, wl.tau, "hqmq llama8b full size")
    o_dense = oracle.dense(q[seqs], k[seqs], v[seqs], np.array(inp.seq_lens)[seqs])
    assert (max_err(o_dense, r["out"][rows]) <= r["bound"][rows]).all()


def test_exact_fallback_on_an_hqmq_cache():
    """The exact fallback recomputes the flagged rows of an HQMQ cache from the
    pinned originals (exact attention) and leaves the others as decoded."""
    from quantized_decode_attention_kvq_b200 import kvq
    inp = small("serving", 7, **SPIKES)
    wl = inp.wl
    k, v = inp.kv()
    q = inp.q()
    r = _run(inp, k, v, q)
    tau = float(np.median(r["bound"]))
    g = r["cache"]
    pt = torch.from_numpy(inp.page_table).cuda()
    sl = torch.tensor(inp.seq_lens, dtype=torch.int32, device="cuda")
    qd = to_torch(q)
    S, NQ, HQ, d = q.shape
    ws = g.workspace(S, NQ, HQ, pt.shape[1])
    out, bound, flags = g.decode(qd, pt, sl, ws, tau=tau)
    torch.cuda.synchronize()
    fl = flags.cpu().numpy().reshape(-1).astype(bool)
    assert 0 < fl.sum() < fl.size
    T = k.shape[2]
    kh = (torch.from_numpy(k.view(np.int16)).view(torch.bfloat16) if k.dtype == np.uint16
          else torch.from_numpy(k)).pin_memory()
    vh = (torch.from_numpy(v.view(np.int16)).view(torch.bfloat16) if v.dtype == np.uint16
          else torch.from_numpy(v)).pin_memory()
    dt = kvq.KVQ_BF16 if k.dtype == np.uint16 else kvq.KVQ_F32
    qdt = kvq.KVQ_BF16 if qd.dtype == torch.bfloat16 else kvq.KVQ_F32
    st_bytes = kvq.kvq_fallback_staging_size(g.desc, dt, max(inp.seq_lens)) * 4
    staging = torch.empty(st_bytes, dtype=torch.uint8, device="cuda")
    fh = torch.zeros(fl.size, dtype=torch.uint8).pin_memory()
    sl_h = np.array(inp.seq_lens, np.int32)
    decoded = out.cpu().numpy().reshape(-1, d).copy()
    rc, n = kvq.kvq_fallback_exact(g.desc, kh, vh, dt, wl.num_kv_heads * T * d, T * d, qd, qdt,
                                   S, NQ, HQ, sl_h.ctypes.data, 0.0, flags, fh, out, staging,
                                   st_bytes, None, torch.cuda.Stream(), 20000)
    torch.cuda.synchronize()
    assert rc == kvq.KVQ_OK, kvq.last_error()
    assert n == int(fl.sum())
    res = out.cpu().numpy().reshape(-1, d).astype(np.float64)
    od = oracle.dense(q, k, v, inp.seq_lens)
    assert max_err(od[fl], res[fl]).max() <= 1e-4
    assert np.array_equal(res[~fl], decoded[~fl].astype(np.float64))


@pytest.mark.parametrize("name", list(SMALL))
@pytest.mark.parametrize("seed", [0, 1])
def test_med3_over_hqmq_parity(name, seed):
    """Med3x over the HQMQ codec (the page's combination): pool bytes (the
    outlier section included) and eta bit for bit, the decode against the
    oracle, and the bound against dense attention."""
    inp = small(name, seed, **SPIKES)
    k, v = inp.kv()
    q = inp.q()
    r = _run(inp, k, v, q, outliers=True)
    assert r["err"] == 0
    pool = r["cache"].pool.cpu().numpy()
    assert np.array_equal(pool, r["oracle"].pool), np.flatnonzero(pool != r["oracle"].pool)[:10]
    assert np.array_equal(r["cache"].eta.cpu().numpy().view(np.uint32),
                          r["oracle"].eta.view(np.uint32))
    _check(inp, r, q, inp.wl.tau, f"hqmq+med3 {name} seed={seed}")
    o_dense = oracle.dense(q, k, v, inp.seq_lens)
    assert (max_err(o_dense, r["out"]) <= r["bound"]).all()


def test_med3_over_hqmq_full_size_sampled():
    inp = synth.make("llama8b", 0)
    wl = inp.wl
    k, v = inp.kv()
    q = inp.q()
    seqs = [0, wl.num_seqs - 1]
    r = _run(inp, k, v, q, seqs=seqs, outliers=True)
    assert r["err"] == 0
    bb = r["oracle"].block_bytes
    gpool = r["cache"].pool.cpu().numpy().reshape(inp.num_pages, wl.num_kv_heads, bb)
    opool = r["oracle"].pool.reshape(inp.num_pages, wl.num_kv_heads, bb)
    pages = np.concatenate([inp.page_table[s, :inp.pages_per_seq[s]] for s in seqs])
    assert np.array_equal(gpool[pages], opool[pages])
    rows, _ = _check(inp, r, q, wl.tau, "hqmq+med3 llama8b full size")
    o_dense = oracle.dense(q[seqs], k[seqs], v[seqs], np.array(inp.seq_lens)[seqs])
    assert (max_err(o_dense, r["out"][rows]) <= r["bound"][rows]).all()
