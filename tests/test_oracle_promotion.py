"""Pins of the oracle's value promotion (rung 2 of the fallback ladder of
"Runtime-Certified Bounded-Error Quantized Attention", Methodology 3): blocks
whose estimated share of E_val (attention mass x eta) exceeds v_tol take the
original values.  Pinned against the decode it extends (nothing promoted), a
closed form (everything promoted: softmax of the quantized scores over the
original values, E_val = 0), a hand-worked case with uniform scores,
monotonicity in v_tol, and the certified inequality against exact attention."""

import math

import numpy as np
import pytest

import oracle
from oracle_cases import max_err, oracle_cache, small

KAPPA = 1.0 + 2.0 ** -10


def _setup(name, seed, **kw):
    inp = small(name, seed, **kw)
    wl = inp.wl
    k, v = inp.kv()
    q = inp.q()
    c = oracle_cache(inp)
    assert c.append(k, v, inp.page_table, np.zeros(wl.num_seqs, np.int32),
                    valid=np.array(inp.seq_lens, np.int32)) == 0
    return inp, c, q, k, v


def _v64(v):
    """Original values as fp64 (bf16 bits widened exactly)."""
    if v.dtype == np.uint16:
        return (v.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return v.astype(np.float64)


@pytest.mark.parametrize("name", ["tiny", "llama8b", "rotated", "serving"])
def test_nothing_promoted_is_the_decode(name):
    inp, c, q, k, v = _setup(name, 0)
    o, b, f, diag = c.decode(q, inp.page_table, inp.seq_lens, tau=inp.wl.tau)
    o2, b2, f2, n2, d2 = c.decode_promote_values(q, inp.page_table, inp.seq_lens, v, math.inf,
                                                 tau=inp.wl.tau)
    assert (n2 == 0).all()
    assert np.array_equal(o, o2) and np.array_equal(b, b2) and np.array_equal(f, f2)
    assert np.array_equal(diag, d2)


@pytest.mark.parametrize("name", ["tiny", "llama8b", "rotated"])
def test_everything_promoted_is_softmax_of_quantized_scores_over_originals(name):
    inp, c, q, k, v = _setup(name, 1)
    wl = inp.wl
    o, b, f, n, diag = c.decode_promote_values(q, inp.page_table, inp.seq_lens, v, -1.0)
    v64 = _v64(v)
    G = wl.num_q_heads // wl.num_kv_heads
    B, NQ, HQ, d = q.shape
    for s in range(B):
        ln = inp.seq_lens[s]
        npg = -(-ln // 16)
        for i in range(NQ):
            for h in range(HQ):
                row = (s * NQ + i) * HQ + h
                assert n[row] == npg
                z, _ = c.decode_terms(q, inp.page_table, ln, s, i, h)
                p = np.exp(z - z.max())
                p /= p.sum()
                ref = p @ v64[s, h // G, :ln]
                assert np.abs(o[row] - ref).max() <= 1e-12 * max(1.0, np.abs(ref).max())
    assert (diag[:, 2] == 0).all()                       # no value error left
    assert np.allclose(b, KAPPA * diag[:, 1], rtol=1e-15, atol=0)


def test_uniform_scores_hand_case():
    # q = 0: every score is 0, so p^ is uniform (1/n) and a block's mass is its
    # share of the tokens.  With 40 tokens the blocks hold 16, 16 and 8 of them,
    # so c_b = (n_b / n) eta_b, and v_tol between the two smallest shares
    # promotes the other two blocks.  Then o' = o + (1/n) sum over the promoted
    # blocks' tokens of (v - v^), with o the decode's mean of v^ and each
    # block's sum of v^ from the decode of that block alone.
    inp, c, q, k, v = _setup("tiny", 2, ctx=40)
    q = np.zeros_like(q)
    n = 40
    sizes = np.array([16, 16, 8])
    eta = c.eta[inp.page_table[0, :3], 0].astype(np.float64)
    share = sizes / n * eta
    order = np.argsort(share)
    v_tol = 0.5 * (share[order[0]] + share[order[1]])
    o, b, f, prom, diag = c.decode_promote_values(q, inp.page_table[:1], [n], v, v_tol)
    assert (prom == 2).all()
    promoted = np.zeros(3, bool)
    promoted[order[1:]] = True
    o0, _, _, _ = c.decode(q, inp.page_table[:1], [n])
    v64 = _v64(v)[0, 0, :n]
    diff = np.zeros(v64.shape[1])
    for blk in np.flatnonzero(promoted):
        t0, t1 = blk * 16, blk * 16 + sizes[blk]
        ob, _, _, _ = c.decode(q, inp.page_table[:1, blk:blk + 1], [t1 - t0])
        diff += v64[t0:t1].sum(axis=0) - ob[0] * (t1 - t0)
    expect = o0[0] + diff / n
    assert np.abs(o[0] - expect).max() <= 1e-12 * max(1.0, np.abs(expect).max())
    assert math.isclose(diag[0, 2], float((share * ~promoted).sum()), rel_tol=1e-12)


@pytest.mark.parametrize("name,seed", [("serving", 0), ("llama8b", 1), ("rotated", 2)])
def test_monotone_in_v_tol(name, seed):
    inp, c, q, k, v = _setup(name, seed)
    last_ev, last_n = None, None
    for v_tol in [math.inf, 1e-2, 1e-3, 1e-4, 1e-5, 0.0, -1.0]:
        _, _, _, n, diag = c.decode_promote_values(q, inp.page_table, inp.seq_lens, v, v_tol)
        if last_ev is not None:
            assert (diag[:, 2] <= last_ev + 1e-15).all()
            assert (n >= last_n).all()
        last_ev, last_n = diag[:, 2], n


@pytest.mark.parametrize("name,seed", [("tiny", 3), ("llama8b", 2), ("rotated", 0),
                                       ("serving", 1)])
def test_bound_covers_the_error_against_exact_attention(name, seed):
    inp, c, q, k, v = _setup(name, seed)
    dense = oracle.dense(q, k, v, inp.seq_lens)
    _, _, _, _, diag0 = c.decode_promote_values(q, inp.page_table, inp.seq_lens, v, math.inf)
    med = float(np.median(diag0[:, 2])) / 8          # a tolerance that promotes some blocks
    for v_tol in [math.inf, med, 0.0, -1.0]:
        o, b, f, n, diag = c.decode_promote_values(q, inp.page_table, inp.seq_lens, v, v_tol)
        err = max_err(dense, o)
        assert (err <= b).all(), (v_tol, float((err - b).max()))
