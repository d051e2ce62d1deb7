"""GPU parity of outlier extraction (the median-multiplier rule, Med3x, of
"Hurwitz Quaternion Multiplicative Quantization for KV Cache Compression",
Method 3) through the C ABI, against the oracle on the same seeded inputs:
the pool bytes (codes, scales, chunk indices, fp16 chunk values) and eta bit
for bit after the append, outputs within max-abs 2e-3 and relative L2 1e-3,
the bound within 1e-4 relative and never below the observed error against
exact attention, flags equal outside the tie band."""

import math

import numpy as np
import pytest
import torch

import oracle
from gpu_cases import (TOL_BOUND_REL, TOL_MAXABS, TOL_RELL2, compare_flags, compare_outputs,
                       gpu_cache, oracle_pool, record_margin, run_gpu, to_torch)
from oracle_cases import SMALL, device_pool, max_err, small
from quantized_decode_attention_kvq_b200 import inputs as synth

pytestmark = pytest.mark.gpu

NO = 0xFF
# spikes in half the sequences, so that values are extracted as well as keys
SPIKES = dict(spike_seq_frac=0.5, spike_token_frac=0.05)


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("the GPU tests need a CUDA device")
    from quantized_decode_attention_kvq_b200 import build
    build.build()


def _extracted(cache_pool, block_bytes, out_off):
    """Chunk indices of every (page, kv head, slot): K [..., 16], V [..., 16]."""
    blk = cache_pool.reshape(-1, block_bytes)
    return blk[:, out_off:out_off + 16], blk[:, out_off + 16:out_off + 32]


def _check(inp, g, o_hat, bound, flags, tau, label):
    record_margin(label, g["out"], o_hat, rows_per_seq=inp.wl.num_queries * inp.wl.num_q_heads)
    emax, rel = compare_outputs(g["out"], o_hat)
    assert emax <= TOL_MAXABS and rel <= TOL_RELL2, (emax, rel)
    brel = np.abs(g["bound"] - bound) / np.maximum(bound, 1e-30)
    assert brel.max() <= TOL_BOUND_REL, brel.max()
    bad, tie = compare_flags(g["flags"], flags, bound, tau)
    assert bad == 0, (bad, tie)


@pytest.mark.parametrize("name", list(SMALL))
@pytest.mark.parametrize("seed", [0, 1])
def test_append_bit_exact_with_extraction(name, seed):
    inp = small(name, seed, **SPIKES)
    k, v = inp.kv()
    g = run_gpu(inp, k, v, outliers=True)
    oc = oracle_pool(inp, k, v, outliers=True)
    assert g["err"] == 0
    pool = g["cache"].pool.cpu().numpy()
    opool = device_pool(oc)
    assert pool.size == opool.size
    assert np.array_equal(pool, opool), np.flatnonzero(pool != opool)[:10]
    eta = g["cache"].eta.cpu().numpy()
    assert np.array_equal(eta.view(np.uint32), oc.eta.view(np.uint32))
    # the case exercises the extraction: some keys and some values have a chunk out
    wl = inp.wl
    out_off = oc.block_bytes - 288
    ki, vi = _extracted(pool, oc.block_bytes, out_off)
    assert (ki != NO).any() and (vi != NO).any()
    assert ((ki == NO) | (ki < wl.head_dim // 4)).all()


@pytest.mark.parametrize("name", list(SMALL))
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_decode_with_extraction_matches_oracle(name, seed):
    inp = small(name, seed, **SPIKES)
    wl = inp.wl
    k, v = inp.kv()
    q = inp.q()
    g = run_gpu(inp, k, v, q, outliers=True)
    assert g["err"] == 0
    oc = oracle_pool(inp, k, v, outliers=True)
    o_hat, bound, flags, _ = oc.decode(q, inp.page_table, inp.seq_lens, tau=wl.tau)
    _check(inp, g, o_hat, bound, flags, wl.tau, f"med3 {name} seed={seed}")
    o_dense = oracle.dense(q, k, v, inp.seq_lens)
    assert (max_err(o_dense, g["out"]) <= g["bound"]).all()


@pytest.mark.parametrize("pps", ["1", "5"])
def test_split_merge_with_extraction(monkeypatch, pps):
    """Value corrections ride in the tensor-core accumulators: any split of the
    context merges to the same result."""
    monkeypatch.setenv("KVQ_PAGES_PER_SPLIT", pps)
    inp = small("serving", 3, **SPIKES)
    k, v = inp.kv()
    q = inp.q()
    g = run_gpu(inp, k, v, q, outliers=True)
    oc = oracle_pool(inp, k, v, outliers=True)
    o_hat, bound, flags, _ = oc.decode(q, inp.page_table, inp.seq_lens, tau=inp.wl.tau)
    _check(inp, g, o_hat, bound, flags, inp.wl.tau, f"med3 serving pps={pps}")


def test_hand_worked_spike_token_on_gpu():
    """The hand-worked token of the oracle's pins (d = 64): V = 0.25 except
    channel 9 = 50 and channel 33 = -0.5, K = 1 except channel 60 = 40; V chunk 2
    and K chunk 15 are extracted, stored as (0.25, 50, 0.25, 0.25) and
    (40, 1, 1, 1); the K scale is 1033 * 2^-17."""
    from quantized_decode_attention_kvq_b200 import kvq
    d = 64
    v = np.full(d, 0.25, np.float32)
    v[9] = 50.0
    v[33] = -0.5
    k = np.ones(d, np.float32)
    k[60] = 40.0
    c = kvq.PagedCache(1, d, 1, k_bits=8, k_group=d, outliers=True)
    pt = torch.zeros((1, 1), dtype=torch.int32, device="cuda")
    z = torch.zeros(1, dtype=torch.int32, device="cuda")
    c.append(torch.from_numpy(k.reshape(1, 1, 1, d)).cuda(),
             torch.from_numpy(v.reshape(1, 1, 1, d)).cuda(), pt, z)
    torch.cuda.synchronize()
    assert c.device_error() == 0
    blk = c.pool.cpu().numpy()
    oc = oracle.Cache(d, 1, 1, k_bits=8, k_group=d, outliers=True)
    assert oc.append(k.reshape(1, 1, 1, d), v.reshape(1, 1, 1, d), np.zeros((1, 1), np.int32),
                     np.zeros(1, np.int32)) == 0
    assert np.array_equal(blk, device_pool(oc))
    out = 16 * d + 16 * d // 2 + 16 * 2 + 16 * (d // 32) * 4
    assert blk[out] == 15 and blk[out + 16] == 2
    assert list(blk[out + 32:out + 40].view(np.float16).astype(np.float64)) == [40, 1, 1, 1]
    assert list(blk[out + 160:out + 168].view(np.float16).astype(np.float64)) == \
        [0.25, 50, 0.25, 0.25]
    ks = blk[16 * d + 16 * d // 2:][:2].view(np.float16)[0]
    assert float(ks) == 1033 * 2.0 ** -17


def test_extracted_value_out_of_fp16_range_is_reported():
    """An extracted chunk value that is not finite or above 65504 in magnitude is
    stored as 0 and raises KVQ_ERR_RANGE, as the oracle does."""
    from quantized_decode_attention_kvq_b200 import kvq
    inp = small("tiny", 0)
    wl = inp.wl
    k, v = inp.kv()
    k = k.copy()
    v = v.copy()
    k[0, 0, 5, 17] = np.inf
    v[0, 0, 9, 40] = 1.0e6
    c = gpu_cache(inp, outliers=True)
    pt = torch.from_numpy(inp.page_table).cuda()
    sl = torch.tensor(inp.seq_lens, dtype=torch.int32, device="cuda")
    c.append(to_torch(k), to_torch(v), pt, torch.zeros(wl.num_seqs, dtype=torch.int32,
                                                       device="cuda"), sl)
    torch.cuda.synchronize()
    assert c.device_error() == kvq.KVQ_ERR_RANGE
    oc = oracle.Cache(wl.head_dim, wl.num_kv_heads, inp.num_pages, k_bits=wl.k_bits,
                      k_group=wl.k_group, outliers=True)
    rc = oc.append(k, v, inp.page_table, np.zeros(wl.num_seqs, np.int32),
                   valid=np.array(inp.seq_lens, np.int32))
    assert rc == oracle.ERR_RANGE
    assert np.array_equal(c.pool.cpu().numpy(), device_pool(oc))


def _fused_step(inp, k, v, q, outliers):
    """Context up to the last token appended, then kvq_decode_attention_append."""
    from quantized_decode_attention_kvq_b200 import kvq
    wl = inp.wl
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
    c = gpu_cache(inp, outliers=outliers)
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
    g = dict(out=out.cpu().numpy().reshape(-1, d).astype(np.float64),
             bound=bound.cpu().numpy().reshape(-1).astype(np.float64),
             flags=flags.cpu().numpy().reshape(-1))
    return c, g


@pytest.mark.parametrize("name", ["llama8b", "rotated", "serving", "tiny"])
def test_fused_step_with_extraction(name):
    inp = small(name, 4, **SPIKES)
    k, v = inp.kv()
    q = inp.q()
    c, g = _fused_step(inp, k, v, q, True)
    oc = oracle_pool(inp, k, v, outliers=True)
    assert np.array_equal(c.pool.cpu().numpy(), device_pool(oc))
    assert np.array_equal(c.eta.cpu().numpy().view(np.uint32), oc.eta.view(np.uint32))
    o_hat, ob, of, _ = oc.decode(q, inp.page_table, inp.seq_lens, tau=inp.wl.tau)
    _check(inp, g, o_hat, ob, of, inp.wl.tau, f"med3 fused {name}")


def test_fused_step_full_size_with_extraction():
    """The benchmark's llama8b step (8 x 8192 tokens, 32/8 heads, INT8 keys) with
    extraction, at full size: pool and eta bit-exact, every row against the
    oracle's decode."""
    inp = synth.make("llama8b", 0)
    k, v = inp.kv()
    q = inp.q()
    c, g = _fused_step(inp, k, v, q, True)
    oc = oracle_pool(inp, k, v, outliers=True)
    assert np.array_equal(c.pool.cpu().numpy(), device_pool(oc))
    assert np.array_equal(c.eta.cpu().numpy().view(np.uint32), oc.eta.view(np.uint32))
    o_hat, ob, of, _ = oc.decode(q, inp.page_table, inp.seq_lens, tau=inp.wl.tau)
    _check(inp, g, o_hat, ob, of, inp.wl.tau, "med3 llama8b full size")


def test_extraction_tightens_the_bound_on_spikes():
    """Spiked values widen a group's range and its eta; with the spike's chunk
    out of the codec eta drops, and so does the bound's E_val share."""
    inp = small("serving", 5, spike_seq_frac=1.0, spike_token_frac=0.05)
    k, v = inp.kv()
    q = inp.q()
    g0 = run_gpu(inp, k, v, q, outliers=False)
    g1 = run_gpu(inp, k, v, q, outliers=True)
    e0 = g0["cache"].eta.cpu().numpy()
    e1 = g1["cache"].eta.cpu().numpy()
    assert (e1 <= e0 * (1 + 1e-6)).all() and e1.max() < 0.5 * e0.max()
    assert np.median(g1["bound"] / g0["bound"]) < 1.0
    o_dense = oracle.dense(q, k, v, inp.seq_lens)
    assert (max_err(o_dense, g1["out"]) <= g1["bound"]).all()
    assert math.isfinite(g1["bound"].max())
