"""GPU parity of adaptive precision ("Runtime-Certified Bounded-Error Quantized
Attention", Methodology 3: top-K* key promotion from a light scoring pass,
the ranking-consistency check, value promotion) against the oracle's
oc_decode_adaptive, through the C ABI.

Key- and value-promotion maps and flags are compared bit for bit; outputs
within max-abs 2e-3 and relative L2 1e-3; bounds within 1e-4 relative.  The
selections are integer decisions taken on floating-point masses (fp32 on the
GPU, fp64 in the oracle): a row whose decision lies within a relative 1e-5 of
its threshold on the oracle's own values (the coverage sum at K*, a block's
mass x eta at v_tol, an exact log-mass gap at rank_tol, the bound at tau) is
only checked for validity, and such rows are counted (none are expected at
these seeds)."""

import math

import numpy as np
import pytest
import torch

import oracle
from gpu_cases import TOL_BOUND_REL, TOL_MAXABS, TOL_RELL2, run_gpu, to_torch
from oracle_cases import max_err, oracle_cache, small

pytestmark = pytest.mark.gpu
BAND = 1e-5


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("the GPU tests need a CUDA device")
    from quantized_decode_attention_kvq_b200 import build
    build.build()


def _pinned(x):
    t = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16) if x.dtype == np.uint16 \
        else torch.from_numpy(np.ascontiguousarray(x))
    return t.pin_memory()


def run_adaptive(inp, k, v, q, tau, tau_cov, v_tol, rank_tol, staging_bytes=None,
                 timeout_ms=20000, outliers=False):
    """Decode on the GPU, then kvq_adaptive_precision on its flagged rows."""
    from quantized_decode_attention_kvq_b200 import kvq
    wl = inp.wl
    g = run_gpu(inp, k, v, q, tau=tau, outliers=outliers)
    assert g["err"] == 0
    c, qd, pt, sl = g["cache"], g["q"], g["pt"], g["sl"]
    B, NQ, HQ, d = q.shape
    rows = B * NQ * HQ
    mp = pt.shape[1]
    # the decode's results, on the device again (run_gpu returned host copies)
    out = torch.from_numpy(g["out"].astype(np.float32).reshape(B, NQ, HQ, d)).cuda()
    bound = torch.from_numpy(g["bound"].astype(np.float32).reshape(B, NQ, HQ)).cuda()
    flags = torch.from_numpy(g["flags"].reshape(B, NQ, HQ).copy()).cuda()
    dt = kvq.KVQ_BF16 if k.dtype == np.uint16 else kvq.KVQ_F32
    kh, vh = _pinned(k), _pinned(v)
    T = k.shape[2]
    work = torch.zeros(kvq.kvq_adaptive_work_size(c.desc, B, NQ, HQ, mp), dtype=torch.uint8,
                       device="cuda")
    host = torch.zeros(kvq.kvq_adaptive_host_size(c.desc, B, mp), dtype=torch.uint8).pin_memory()
    if staging_bytes is None:
        staging_bytes = kvq.kvq_adaptive_staging_size(c.desc, dt, mp) * B * wl.num_kv_heads
    staging = torch.empty(staging_bytes, dtype=torch.uint8, device="cuda")
    kp = torch.zeros((rows, mp), dtype=torch.uint8, device="cuda")
    vp = torch.zeros((rows, mp), dtype=torch.uint8, device="cuda")
    fh = torch.zeros(rows, dtype=torch.uint8).pin_memory()
    sl_h = np.array(inp.seq_lens, np.int32)
    side = torch.cuda.Stream()
    rc, nrows, nflag = kvq.kvq_adaptive_precision(
        c.desc, kh, vh, dt, wl.num_kv_heads * T * d, T * d, qd,
        kvq.KVQ_BF16 if qd.dtype == torch.bfloat16 else kvq.KVQ_F32, B, NQ, HQ, pt, mp, sl,
        sl_h.ctypes.data, 0.0, tau, tau_cov, v_tol, rank_tol, flags, fh, out, bound, kp, vp,
        work, work.numel(), host, host.numel(), staging, staging.numel(), None, side, timeout_ms)
    torch.cuda.synchronize()
    res = dict(rc=rc, nrows=nrows, nflag=nflag, g=g, err=c.device_error(),
               out=out.cpu().numpy().reshape(rows, d).astype(np.float64),
               bound=bound.cpu().numpy().reshape(-1).astype(np.float64),
               flags=flags.cpu().numpy().reshape(-1), flags_host=fh.numpy().copy(),
               kp=kp.cpu().numpy(), vp=vp.cpu().numpy())
    if rc:
        res["msg"] = kvq.last_error()
    return res


def ambiguous_rows(c, q, k, page_table, seq_lens, group, ref, tau_cov, v_tol, rank_tol, tau,
                   as_f32, row_mask=None):
    """Rows whose integer decisions lie within BAND of a threshold, decided on the
    oracle's fp64 values (q, k of the sequences the oracle cache holds)."""
    B, NQ, HQ, d = q.shape
    amb = np.zeros(B * NQ * HQ, bool)
    s_att = float(oracle.default_scale(d))
    for b in range(B):
        n = int(seq_lens[b])
        if n == 0:
            continue
        npg = (n + 15) // 16
        for i in range(NQ):
            for h in range(HQ):
                row = (b * NQ + i) * HQ + h
                if row_mask is not None and not row_mask[row]:
                    continue
                z, _ = c.decode_terms(q, page_table, n, b, i, h)
                p = np.exp(z - z.max())
                p /= p.sum()
                m = np.add.reduceat(p, np.arange(0, n, 16))
                order = sorted(range(npg), key=lambda x: (-m[x], x))
                cum = np.cumsum(m[order])
                K = int(ref["nkey"][row])
                if tau_cov > 0:
                    if K >= 1 and abs(cum[K - 1] - tau_cov) <= BAND * tau_cov:
                        amb[row] = True
                    if K >= 2 and abs(cum[K - 2] - tau_cov) <= BAND * tau_cov:
                        amb[row] = True
                    if 1 <= K < npg and abs(m[order[K - 1]] - m[order[K]]) <= BAND * m[order[K - 1]]:
                        amb[row] = True
                kv = h // group
                eta = c.eta[page_table[b, :npg], kv].astype(np.float64)
                if np.isfinite(v_tol) and (np.abs(m * eta - v_tol) <= BAND * abs(v_tol)).any():
                    amb[row] = True
                blocks = order[:K]
                if len(blocks) > 1:
                    qf = as_f32(q[b, i, h]).astype(np.float64)
                    kf = as_f32(k[b, kv, :n]).astype(np.float64)
                    zz = s_att * (kf @ qf)
                    e = np.exp(zz - zz.max())
                    L = np.log(np.add.reduceat(e, np.arange(0, n, 16)))[blocks] + zz.max()
                    gap = L[1:] - np.minimum.accumulate(L)[:-1]
                    if (np.abs(gap - rank_tol) <= BAND).any():
                        amb[row] = True
                if math.isfinite(tau) and abs(ref["bound"][row] - tau) <= 1e-4 * abs(tau):
                    amb[row] = True
    return amb


def _oracle_row_decisions(inp, c, q, k, r, tau_cov, v_tol, rank_tol, tau):
    return ambiguous_rows(c, q, k, inp.page_table, inp.seq_lens, inp.wl.group, r, tau_cov,
                          v_tol, rank_tol, tau, inp.as_f32)


def _check(inp, res, ref, amb, flagged):
    assert res["rc"] == 0, res.get("msg")
    assert res["err"] == 0
    ok = flagged & ~amb
    assert ok.sum() > 0
    mp = res["kp"].shape[1]
    npg_row = np.repeat([(n + 15) // 16 for n in inp.seq_lens],
                        inp.wl.num_queries * inp.wl.num_q_heads)
    for row in np.flatnonzero(ok):
        assert np.array_equal(res["kp"][row, :npg_row[row]], ref["kprom"][row, :npg_row[row]]), row
        assert np.array_equal(res["vp"][row, :npg_row[row]], ref["vprom"][row, :npg_row[row]]), row
    emax = np.abs(res["out"][ok] - ref["out"][ok]).max()
    rel = np.linalg.norm(res["out"][ok] - ref["out"][ok]) / np.linalg.norm(ref["out"][ok])
    assert emax <= TOL_MAXABS and rel <= TOL_RELL2, (emax, rel)
    brel = np.abs(res["bound"][ok] - ref["bound"][ok]) / np.maximum(ref["bound"][ok], 1e-30)
    assert brel.max() <= TOL_BOUND_REL, brel.max()
    assert np.array_equal(res["flags"][ok], ref["flags"][ok])
    # rows the ladder did not run on are the decode's
    un = ~flagged
    assert np.array_equal(res["flags"][un], res["g"]["flags"][un])
    assert np.array_equal(res["bound"][un], res["g"]["bound"][un].astype(np.float32))
    assert res["nrows"] == int(flagged.sum())
    assert res["nflag"] == int(res["flags"].astype(bool).sum())
    assert np.array_equal(res["flags_host"], res["flags"])
    return int((flagged & amb).sum())


CASES = [
    # name, seed, tau, tau_cov, v_tol, rank_tol
    ("llama8b", 0, 0.0, 0.9, math.inf, 0.0),
    ("llama8b", 1, 5.0, 0.995, 1e-3, 0.05),
    ("serving", 0, 0.2, 0.995, 1e-3, 0.0),
    ("serving", 2, 0.0, 0.5, 1e-2, 1.0),
    ("rotated", 0, 0.0, 0.9, 1e-3, 0.0),
    ("long128k", 0, 0.0, 0.995, math.inf, 0.02),
    ("tiny", 0, 0.0, 0.8, 1e-3, 0.0),
]


@pytest.mark.parametrize("name,seed,tau,tau_cov,v_tol,rank_tol", CASES)
def test_adaptive_matches_oracle(name, seed, tau, tau_cov, v_tol, rank_tol):
    inp = small(name, seed)
    k, v = inp.kv()
    q = inp.q()
    res = run_adaptive(inp, k, v, q, tau, tau_cov, v_tol, rank_tol)
    oc = oracle_cache(inp)
    assert oc.append(k, v, inp.page_table, np.zeros(inp.wl.num_seqs, np.int32),
                     valid=np.array(inp.seq_lens, np.int32)) == 0
    flagged = res["g"]["flags"].astype(bool)
    ref = oc.decode_adaptive(q, inp.page_table, inp.seq_lens, k, v, tau_cov, v_tol, rank_tol,
                             tau=tau, row_mask=flagged.astype(np.uint8))
    amb = _oracle_row_decisions(inp, oc, q, k, ref, tau_cov, v_tol, rank_tol, tau)
    n_amb = _check(inp, res, ref, amb, flagged)
    assert n_amb == 0, f"{n_amb} rows within the decision band"
    # certified: the GPU's own output is within its bound of exact attention
    od = oracle.dense(q, k, v, inp.seq_lens)
    assert (res["bound"][flagged] >= max_err(od, res["out"])[flagged]).all()


EXTRACTION_CASES = [
    # name, seed, tau, tau_cov, v_tol, rank_tol (spikes in half the sequences)
    ("serving", 0, 0.0, 0.995, 1e-3, 0.0),
    ("llama8b", 2, 0.0, 0.9, 1e-3, 0.05),
    ("rotated", 1, 0.0, 0.9, math.inf, 0.0),
    ("tiny", 0, 0.0, 0.8, 1e-3, 0.0),
]


@pytest.mark.parametrize("name,seed,tau,tau_cov,v_tol,rank_tol", EXTRACTION_CASES)
def test_adaptive_with_extraction_matches_oracle(name, seed, tau, tau_cov, v_tol, rank_tol):
    """The ladder over a cache with Med3x outlier extraction: scores, values,
    Delta and range include the extracted chunks, as the oracle's do."""
    inp = small(name, seed, spike_seq_frac=0.5, spike_token_frac=0.05)
    k, v = inp.kv()
    q = inp.q()
    res = run_adaptive(inp, k, v, q, tau, tau_cov, v_tol, rank_tol, outliers=True)
    oc = oracle_cache(inp, outliers=True)
    assert oc.append(k, v, inp.page_table, np.zeros(inp.wl.num_seqs, np.int32),
                     valid=np.array(inp.seq_lens, np.int32)) == 0
    flagged = res["g"]["flags"].astype(bool)
    ref = oc.decode_adaptive(q, inp.page_table, inp.seq_lens, k, v, tau_cov, v_tol, rank_tol,
                             tau=tau, row_mask=flagged.astype(np.uint8))
    amb = _oracle_row_decisions(inp, oc, q, k, ref, tau_cov, v_tol, rank_tol, tau)
    _check(inp, res, ref, amb, flagged)
    od = oracle.dense(q, k, v, inp.seq_lens)
    assert (res["bound"][flagged] >= max_err(od, res["out"])[flagged]).all()


def test_nothing_promoted_reproduces_the_decode():
    inp = small("serving", 1)
    k, v = inp.kv()
    q = inp.q()
    res = run_adaptive(inp, k, v, q, 0.0, 0.0, math.inf, 0.0)
    assert res["rc"] == 0, res.get("msg")
    g = res["g"]
    emax = np.abs(res["out"] - g["out"]).max()
    assert emax <= TOL_MAXABS
    assert (np.abs(res["bound"] - g["bound"]) <= TOL_BOUND_REL * g["bound"]).all()
    assert not res["kp"].any() and not res["vp"].any()


def test_everything_promoted_is_exact_attention_with_small_staging():
    """tau_cov > 1 and v_tol < 0 promote every block: the output is exact dense
    attention; a staging buffer of one (sequence, kv head) forces one batch per
    unit."""
    from quantized_decode_attention_kvq_b200 import kvq
    inp = small("llama8b", 2)
    k, v = inp.kv()
    q = inp.q()
    c = kvq.PagedCache(inp.wl.num_kv_heads, inp.wl.head_dim, inp.num_pages)
    one = kvq.kvq_adaptive_staging_size(c.desc, kvq.KVQ_BF16, inp.page_table.shape[1])
    res = run_adaptive(inp, k, v, q, 0.0, 2.0, -1.0, 1e9, staging_bytes=one)
    assert res["rc"] == 0, res.get("msg")
    od = oracle.dense(q, k, v, inp.seq_lens)
    assert np.abs(res["out"] - od).max() <= 1e-4
    assert (res["bound"] >= max_err(od, res["out"])).all()
    assert (res["bound"] < 0.05).all()
    assert res["kp"][:, :(max(inp.seq_lens) + 15) // 16].all()


def test_timeout_and_injected_copy_failure(monkeypatch):
    inp = small("serving", 3)
    k, v = inp.kv()
    q = inp.q()
    from quantized_decode_attention_kvq_b200 import kvq
    res = run_adaptive(inp, k, v, q, 0.0, 0.9, math.inf, 0.0, timeout_ms=0)
    assert res["rc"] == kvq.KVQ_ERR_TIMEOUT
    monkeypatch.setenv("KVQ_FAULT", "memcpy")
    res = run_adaptive(inp, k, v, q, 0.0, 0.9, math.inf, 0.0)
    assert res["rc"] == kvq.KVQ_ERR_CUDA and "injected" in res["msg"]


@pytest.mark.parametrize("name,seed,v_tol", [("llama8b", 0, 1e-3), ("serving", 1, 1e-3),
                                             ("rotated", 2, 3e-3)])
def test_value_promotion_matches_its_oracle(name, seed, v_tol):
    """Rung 2 alone (tau_cov = 0): outputs, bounds, promoted counts and flags
    against oc_decode_promote_values."""
    inp = small(name, seed)
    k, v = inp.kv()
    q = inp.q()
    tau = 0.0
    res = run_adaptive(inp, k, v, q, tau, 0.0, v_tol, 0.0)
    assert res["rc"] == 0, res.get("msg")
    oc = oracle_cache(inp)
    assert oc.append(k, v, inp.page_table, np.zeros(inp.wl.num_seqs, np.int32),
                     valid=np.array(inp.seq_lens, np.int32)) == 0
    o, b, f, npro, _ = oc.decode_promote_values(q, inp.page_table, inp.seq_lens, v, v_tol,
                                                tau=tau)
    ref = dict(nkey=np.zeros_like(npro), bound=b)
    amb = ambiguous_rows(oc, q, k, inp.page_table, inp.seq_lens, inp.wl.group, ref, 0.0, v_tol,
                         0.0, tau, inp.as_f32)
    ok = ~amb
    assert ok.sum() == ok.size
    assert np.array_equal(res["vp"].sum(axis=1)[ok], npro[ok])
    assert not res["kp"].any()
    emax = np.abs(res["out"][ok] - o[ok]).max()
    assert emax <= TOL_MAXABS, emax
    assert (np.abs(res["bound"][ok] - b[ok]) <= TOL_BOUND_REL * b[ok]).all()
    assert np.array_equal(res["flags"][ok], f[ok])
