"""The mixed-length serving workload at full size: 64 sequences with lengths
uniform in [1024, 32768], spikes of magnitude 50 in one sequence, tau = 1e-2,
bf16 originals in pinned host memory.

The GPU appends and decodes every sequence; the oracle (far too slow for all
of them) checks sampled sequences -- the spike sequence, the shortest and the
longest -- on the pool bytes, eta, outputs, bounds and flags.  Then every
flagged row is recomputed by the exact fallback, and the sampled rows are
checked against fp64 dense attention over the originals."""

import numpy as np
import pytest
import torch

import oracle
from gpu_cases import (TOL_BOUND_REL, TOL_MAXABS, TOL_RELL2, compare_flags, compare_outputs,
                       run_gpu)
from oracle_cases import device_pool, max_err, oracle_cache
from quantized_decode_attention_kvq_b200 import inputs as synth

pytestmark = pytest.mark.gpu


def _host(x: np.ndarray) -> torch.Tensor:
    t = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16) if x.dtype == np.uint16 \
        else torch.from_numpy(x)
    return t.contiguous().pin_memory()


def test_serving_full_size_sampled_sequences():
    from quantized_decode_attention_kvq_b200 import kvq
    if not torch.cuda.is_available():
        pytest.fail("the GPU tests need a CUDA device")
    inp = synth.make("serving", 0)
    wl = inp.wl
    k, v = inp.kv()
    q = inp.q()
    g = run_gpu(inp, k, v, q)
    assert g["err"] == 0
    lens = np.array(inp.seq_lens)
    sel = sorted({*inp.spike_seqs, int(lens.argmin()), int(lens.argmax())})
    assert len(sel) >= 2

    # pool bytes and eta of every page of the sampled sequences, bit-exact
    oc = oracle_cache(inp)
    pt = inp.page_table[sel]
    assert oc.append(k[sel], v[sel], pt, np.zeros(len(sel), np.int32),
                     valid=lens[sel].astype(np.int32)) == 0
    pages = np.concatenate([pt[i, :inp.pages_per_seq[s]] for i, s in enumerate(sel)])
    bb = oc.block_bytes
    gpool = g["cache"].pool.cpu().numpy().reshape(inp.num_pages, wl.num_kv_heads, bb)
    opool = device_pool(oc).reshape(inp.num_pages, wl.num_kv_heads, bb)
    assert np.array_equal(gpool[pages], opool[pages])
    assert np.array_equal(g["cache"].eta.cpu().numpy()[pages], oc.eta[pages])

    # decode of the sampled rows against the oracle
    rows = np.concatenate([np.arange(s * wl.num_q_heads, (s + 1) * wl.num_q_heads) for s in sel])
    o_hat, bound, flags, _ = oc.decode(q[sel], pt, lens[sel], tau=wl.tau)
    emax, rel = compare_outputs(g["out"][rows], o_hat)
    assert emax <= TOL_MAXABS and rel <= TOL_RELL2, (emax, rel)
    brel = np.abs(g["bound"][rows] - bound) / np.maximum(bound, 1e-30)
    assert brel.max() <= TOL_BOUND_REL, brel.max()
    bad, _ = compare_flags(g["flags"][rows], flags, bound, wl.tau)
    assert bad == 0

    # the bound is never below the observed error against exact attention
    o_dense = oracle.dense(q[sel], k[sel], v[sel], lens[sel])
    assert (max_err(o_dense, g["out"][rows]) <= g["bound"][rows]).all()

    # exact fallback of every flagged row, from pinned host originals
    T = k.shape[2]
    kh, vh = _host(k), _host(v)
    out = torch.from_numpy(g["out"].astype(np.float32)).cuda()
    flags_d = torch.from_numpy(g["flags"]).cuda()
    flags_h = torch.zeros(g["flags"].size, dtype=torch.uint8).pin_memory()
    st_bytes = kvq.kvq_fallback_staging_size(g["cache"].desc, kvq.KVQ_BF16, int(lens.max())) * 8
    staging = torch.empty(st_bytes, dtype=torch.uint8, device="cuda")
    side = torch.cuda.Stream()
    sl_h = lens.astype(np.int32)
    rc, n = kvq.kvq_fallback_exact(g["cache"].desc, kh, vh, kvq.KVQ_BF16,
                                   wl.num_kv_heads * T * wl.head_dim, T * wl.head_dim, g["q"],
                                   kvq.KVQ_BF16, wl.num_seqs, wl.num_queries, wl.num_q_heads,
                                   sl_h.ctypes.data, 0.0, flags_d, flags_h, out, staging,
                                   st_bytes, None, side, 60000)
    torch.cuda.synchronize()
    assert rc == kvq.KVQ_OK, kvq.last_error()
    flagged = g["flags"].astype(bool)
    assert n == int(flagged.sum())
    out = out.cpu().numpy().astype(np.float64)
    fl = flagged[rows]
    if fl.any():
        assert max_err(o_dense[fl], out[rows][fl]).max() <= 1e-4
    assert np.array_equal(out[~flagged], g["out"][~flagged])
    print(f"serving seed 0: fallback rate {flagged.mean():.4f} ({int(flagged.sum())} of "
          f"{flagged.size} rows); sampled bound / observed error median "
          f"{np.median(bound / np.maximum(max_err(o_dense, o_hat), 1e-30)):.1f}")


def test_serving_full_size_adaptive_precision():
    """The adaptive-precision ladder at full size (tau = 1e-2, 99.5% of the
    estimated mass on exact keys, value promotion above 1e-4, ranking slack
    0.1) on every flagged row; the sampled sequences against the oracle."""
    from test_gpu_adaptive import BAND, ambiguous_rows, run_adaptive
    inp = synth.make("serving", 0)
    wl = inp.wl
    k, v = inp.kv()
    q = inp.q()
    tau_cov, v_tol, rank_tol = 0.995, 1e-4, 0.1
    res = run_adaptive(inp, k, v, q, wl.tau, tau_cov, v_tol, rank_tol, timeout_ms=120000)
    assert res["rc"] == 0, res.get("msg")
    assert res["err"] == 0
    flagged = res["g"]["flags"].astype(bool)
    lens = np.array(inp.seq_lens)
    sel = sorted({*inp.spike_seqs, int(lens.argmin()), int(lens.argmax())})
    oc = oracle_cache(inp)
    pt = inp.page_table[sel]
    assert oc.append(k[sel], v[sel], pt, np.zeros(len(sel), np.int32),
                     valid=lens[sel].astype(np.int32)) == 0
    rows = np.concatenate([np.arange(s * wl.num_q_heads, (s + 1) * wl.num_q_heads) for s in sel])
    fl = flagged[rows]
    ref = oc.decode_adaptive(q[sel], pt, lens[sel], k[sel], v[sel], tau_cov, v_tol, rank_tol,
                             tau=wl.tau, row_mask=fl.astype(np.uint8))
    amb = ambiguous_rows(oc, q[sel], k[sel], pt, lens[sel], wl.group, ref, tau_cov, v_tol,
                         rank_tol, wl.tau, inp.as_f32, row_mask=fl)
    # with ~2000 blocks per row, masses near the coverage boundary are dense and
    # near-ties common: maps and flags are compared where no decision is within
    # the band, outputs and bounds on every flagged row
    ok = fl & ~amb
    assert ok.sum() >= 0.75 * fl.sum() and ok.any()
    for gr, orow in zip(rows[ok], np.flatnonzero(ok)):
        npg = inp.pages_per_seq[sel[orow // wl.num_q_heads]]
        assert np.array_equal(res["kp"][gr, :npg], ref["kprom"][orow, :npg])
        assert np.array_equal(res["vp"][gr, :npg], ref["vprom"][orow, :npg])
    assert np.array_equal(res["flags"][rows[ok]], ref["flags"][ok])
    emax = np.abs(res["out"][rows[fl]] - ref["out"][fl]).max()
    assert emax <= TOL_MAXABS, emax
    brel = np.abs(res["bound"][rows[fl]] - ref["bound"][fl]) / ref["bound"][fl]
    assert brel.max() <= TOL_BOUND_REL, brel.max()
    mp = pt.shape[1]
    o_dense = oracle.dense(q[sel], k[sel], v[sel], lens[sel])
    assert (max_err(o_dense, res["out"][rows]) <= res["bound"][rows]).all()
    print(f"serving seed 0 ladder: {int(flagged.sum())} rows in, {res['nflag']} flagged after "
          f"({res['nflag'] / flagged.size:.4f}); {int(amb.sum())} sampled rows in the band")
    assert mp > 0 and BAND > 0
