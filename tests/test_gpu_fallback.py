"""Certified fallback: flagged queries are recomputed exactly from the pinned
host originals (side stream, cudaMemcpyAsync); the others keep the quantized
output.  The staging layouts (one region; two halves; two halves that each
carry several launches), row groups of more than 8 queries per (sequence,
kv head), token ranges split into merged chunks, and fp32 / d=64 originals
are covered.  Host-side failures (deadline, injected copy failure) leave out
as it was and return a clean status; no GPU fault is provoked."""

import numpy as np
import pytest
import torch

import oracle
from gpu_cases import TOL_MAXABS, compare_outputs, run_gpu
from oracle_cases import max_err, small

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("the GPU tests need a CUDA device")


def _host(x: np.ndarray) -> torch.Tensor:
    t = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16) if x.dtype == np.uint16 \
        else torch.from_numpy(x)
    return t.contiguous().pin_memory()


def _fallback(inp, g, k, v, timeout_ms=10000, mult=3):
    from quantized_decode_attention_kvq_b200 import kvq
    wl = inp.wl
    kh, vh = _host(k), _host(v)
    out = torch.from_numpy(g["out"].astype(np.float32)).cuda().reshape(
        wl.num_seqs, wl.num_queries, wl.num_q_heads, wl.head_dim)
    flags = torch.from_numpy(g["flags"]).cuda()
    flags_host = torch.zeros(g["flags"].size, dtype=torch.uint8).pin_memory()
    T = k.shape[2]
    dt = kvq.KVQ_BF16 if k.dtype == np.uint16 else kvq.KVQ_F32
    st_bytes = kvq.kvq_fallback_staging_size(g["cache"].desc, dt, max(inp.seq_lens)) * mult
    staging = torch.empty(st_bytes, dtype=torch.uint8, device="cuda")
    side = torch.cuda.Stream()
    sl_host = np.array(inp.seq_lens, np.int32)
    rc, n = kvq.kvq_fallback_exact(g["cache"].desc, kh, vh, dt, wl.num_kv_heads * T * wl.head_dim,
                                   T * wl.head_dim, g["q"], kvq.KVQ_BF16 if g["q"].dtype ==
                                   torch.bfloat16 else kvq.KVQ_F32, wl.num_seqs, wl.num_queries,
                                   wl.num_q_heads, sl_host.ctypes.data, 0.0, flags, flags_host,
                                   out, staging, st_bytes, None, side, timeout_ms)
    torch.cuda.synchronize()
    return rc, n, out.cpu().numpy().reshape(-1, wl.head_dim).astype(np.float64), \
        flags_host.numpy().copy()


def test_fallback_recovers_exact_attention():
    inp = small("serving", 0)
    k, v = inp.kv()
    q = inp.q()
    o_dense = oracle.dense(q, k, v, inp.seq_lens)
    g = run_gpu(inp, k, v, q, tau=float(np.float32(0.79)))  # about half the rows flagged
    flagged = g["flags"].astype(bool)
    assert 0 < flagged.sum() < flagged.size
    rc, n, out, fh = _fallback(inp, g, k, v)
    assert rc == 0 and n == int(flagged.sum())
    assert np.array_equal(fh, g["flags"])
    emax, _ = compare_outputs(out[flagged], o_dense[flagged])
    assert emax <= 1e-4                                     # exact attention, fp32
    assert np.array_equal(out[~flagged], g["out"][~flagged])
    # every row is now bounded or recovered exactly
    err = max_err(o_dense, out)
    assert (err <= np.where(flagged, 1e-4, g["bound"])).all()


def test_fallback_all_rows_at_tau_1e2():
    inp = small("serving", 1)
    k, v = inp.kv()
    q = inp.q()
    g = run_gpu(inp, k, v, q)                               # tau = 1e-2
    rc, n, out, _ = _fallback(inp, g, k, v)
    assert rc == 0 and n == int(g["flags"].sum())
    o_dense = oracle.dense(q, k, v, inp.seq_lens)
    flagged = g["flags"].astype(bool)
    assert compare_outputs(out[flagged], o_dense[flagged])[0] <= 1e-4


def test_fallback_deadline_zero_times_out_cleanly():
    from quantized_decode_attention_kvq_b200 import kvq
    inp = small("serving", 2)
    k, v = inp.kv()
    g = run_gpu(inp, k, v)
    rc, n, out, _ = _fallback(inp, g, k, v, timeout_ms=0)
    assert rc == kvq.KVQ_ERR_TIMEOUT and n == 0
    assert np.array_equal(out, g["out"])


def test_fallback_injected_copy_failure(monkeypatch):
    from quantized_decode_attention_kvq_b200 import kvq
    monkeypatch.setenv("KVQ_FAULT", "memcpy")
    inp = small("serving", 3)
    k, v = inp.kv()
    g = run_gpu(inp, k, v)
    assert g["flags"].any()
    rc, n, out, _ = _fallback(inp, g, k, v)
    assert rc == kvq.KVQ_ERR_CUDA and n == 0
    assert "injected" in kvq.last_error()
    assert np.array_equal(out, g["out"])


def _check_recovered(inp, g, out, q, k, v):
    o_dense = oracle.dense(q, k, v, inp.seq_lens)
    flagged = g["flags"].astype(bool)
    assert flagged.any()
    assert compare_outputs(out[flagged], o_dense[flagged])[0] <= 1e-4
    assert np.array_equal(out[~flagged], g["out"][~flagged])


@pytest.mark.parametrize("mult", [1, 3, 40])
def test_fallback_staging_layouts_and_row_groups(mult):
    # 30 sequences x 2 kv heads with 12 q heads each: up to 12 flagged rows per
    # (sequence, kv head), so two row groups; lengths above 128 split in two
    # chunks.  The flags are seeded (the fallback reads only q, flags and out;
    # the decode takes at most 4 rows per kv head).  mult 1: one staging
    # region (each batch's copies wait for the previous recompute); 3: two
    # halves; 40: two halves, each holding more items than one launch takes.
    from gpu_cases import gpu_cache, to_torch
    inp = small("serving", 4, num_seqs=30, num_q_heads=24, num_kv_heads=2)
    k, v = inp.kv()
    q = inp.q()
    rng = np.random.default_rng(40 + mult)
    flags = (rng.random(q.shape[:3]) < 0.7).astype(np.uint8).reshape(-1)
    flags[:12] = 1                                         # one full pair of 12 rows
    g = dict(cache=gpu_cache(inp), q=to_torch(q), flags=flags,
             out=rng.standard_normal((flags.size, inp.wl.head_dim)).astype(np.float32))
    rc, n, out, fh = _fallback(inp, g, k, v, mult=mult)
    assert rc == 0 and n == int(flags.sum())
    assert np.array_equal(fh, flags)
    _check_recovered(inp, g, out, q, k, v)


def test_fallback_fp32_head_dim_64():
    inp = small("tiny", 5)                                  # fp32 originals, d=64, 4 queries
    k, v = inp.kv()
    q = inp.q()
    g = run_gpu(inp, k, v, q, tau=0.0)                      # every row flagged
    assert g["flags"].all()
    rc, n, out, _ = _fallback(inp, g, k, v, mult=1)
    assert rc == 0 and n == g["flags"].size
    _check_recovered(inp, g, out, q, k, v)
