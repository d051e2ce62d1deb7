"""Pins of the oracle's adaptive precision ("Runtime-Certified Bounded-Error
Quantized Attention", Methodology 3: adaptive top-K* block selection from a
light scoring pass with the quantized keys, promotion to full-precision keys,
the ranking-consistency check, and value promotion).

Against things other than its own code:
* special cases that reduce to other pinned routines: nothing promoted is the
  plain decode; value promotion alone is the value-promotion oracle;
  everything promoted is exact dense attention (itself pinned to torch SDPA);
* the selection's defining properties, checked on block masses computed here
  from the per-token scores: the promoted blocks are a top set, cover tau_cov
  and are the fewest that do; sets are nested in tau_cov;
* a brute-force, pairwise version of the ranking check on the originals;
* a hand-worked two-block case where the quantized keys invert the order;
* the bound never below the error against exact attention;
* five planted mistakes compiled into copies of the oracle are each caught.
"""

import math

import numpy as np
import pytest

import oracle
from oracle_cases import SMALL, max_err, oracle_cache, small


def _setup(name, seed):
    inp = small(name, seed)
    wl = inp.wl
    k, v = inp.kv()
    q = inp.q()
    c = oracle_cache(inp)
    assert c.append(k, v, inp.page_table, np.zeros(wl.num_seqs, np.int32),
                    valid=np.array(inp.seq_lens, np.int32)) == 0
    return inp, c, q, k, v


def _rows(inp):
    wl = inp.wl
    for b in range(wl.num_seqs):
        for i in range(wl.num_queries):
            for h in range(wl.num_q_heads):
                yield (b * wl.num_queries + i) * wl.num_q_heads + h, b, i, h


def _est_masses(inp, c, q, b, i, h):
    """Block masses under the quantized softmax, from the per-token scores."""
    n = inp.seq_lens[b]
    z, _ = c.decode_terms(q, inp.page_table, n, b, i, h)
    p = np.exp(z - z.max())
    p /= p.sum()
    npg = (n + 15) // 16
    return np.array([p[16 * k:16 * k + 16].sum() for k in range(npg)])


@pytest.mark.parametrize("name", list(SMALL))
def test_nothing_promoted_is_the_plain_decode(oracle_lib, name):
    inp, c, q, k, v = _setup(name, 0)
    o, b, f, dg = c.decode(q, inp.page_table, inp.seq_lens, tau=0.5)
    r = c.decode_adaptive(q, inp.page_table, inp.seq_lens, k, v, tau_cov=0.0, tau=0.5)
    assert np.array_equal(r["out"], o) and np.array_equal(r["bound"], b)
    assert np.array_equal(r["flags"], f) and np.array_equal(r["diag"], dg)
    assert (r["nkey"] == 0).all() and (r["nval"] == 0).all() and (r["rank_fail"] == 0).all()


@pytest.mark.parametrize("name", ["llama8b", "serving", "rotated"])
def test_values_only_is_value_promotion(oracle_lib, name):
    inp, c, q, k, v = _setup(name, 1)
    for vt in (1e-3, 1e-2):
        o, b, f, npro, dg = c.decode_promote_values(q, inp.page_table, inp.seq_lens, v, vt,
                                                    tau=0.2)
        r = c.decode_adaptive(q, inp.page_table, inp.seq_lens, k, v, tau_cov=0.0, v_tol=vt,
                              tau=0.2)
        assert np.array_equal(r["out"], o) and np.array_equal(r["bound"], b)
        assert np.array_equal(r["flags"], f) and np.array_equal(r["nval"], npro)


@pytest.mark.parametrize("name", list(SMALL))
def test_everything_promoted_is_dense_attention(oracle_lib, name):
    inp, c, q, k, v = _setup(name, 2)
    r = c.decode_adaptive(q, inp.page_table, inp.seq_lens, k, v, tau_cov=2.0, v_tol=-1.0)
    od = oracle.dense(q, k, v, inp.seq_lens)
    assert np.array_equal(r["out"], od)
    # no value error left, and the key term only carries the fp32 allowance of
    # the exact scores, far below 2^-15 s_att |q|_2 |k|_2
    assert (r["diag"][:, 2] == 0).all()
    qn = np.linalg.norm(inp.as_f32(q).astype(np.float64), axis=-1).max()
    kn = np.linalg.norm(inp.as_f32(k).astype(np.float64), axis=-1).max()
    s_att = float(oracle.default_scale(inp.wl.head_dim))
    assert (r["diag"][:, 3] <= 2.0 ** -15 * s_att * qn * kn).all()
    npg = np.array([(n + 15) // 16 for n in inp.seq_lens])
    wl = inp.wl
    per_row = np.repeat(npg, wl.num_queries * wl.num_q_heads)
    assert np.array_equal(r["nkey"], per_row) and np.array_equal(r["nval"], per_row)


@pytest.mark.parametrize("name", ["llama8b", "long128k", "serving", "rotated"])
def test_selection_is_the_smallest_top_set_covering_tau_cov(oracle_lib, name):
    inp, c, q, k, v = _setup(name, 0)
    prev = None
    for tc in (0.3, 0.7, 0.95, 0.995):
        r = c.decode_adaptive(q, inp.page_table, inp.seq_lens, k, v, tau_cov=tc)
        for row, b, i, h in _rows(inp):
            m = _est_masses(inp, c, q, b, i, h)
            sel = r["kprom"][row, :m.size].astype(bool)
            assert r["nkey"][row] == sel.sum()
            assert not r["kprom"][row, m.size:].any()
            tol = 1e-12
            # covers tau_cov ...
            assert m[sel].sum() >= tc - tol or sel.all()
            # ... with the fewest blocks: without its lightest block it would not
            if sel.any():
                assert m[sel].sum() - m[sel].min() < tc + tol
            # top set: no unselected block is heavier than a selected one
            if sel.any() and (~sel).any():
                assert m[~sel].max() <= m[sel].min() + tol
            if prev is not None:   # nested in tau_cov
                assert (prev[row] <= r["kprom"][row]).all()
        prev = r["kprom"].copy()


def _exact_block_logmass(inp, q, k, b, i, h, blocks):
    """log sum_j e^{z_j} per block from the originals (fp64, unrotated)."""
    wl = inp.wl
    kv = h // wl.group
    qf = inp.as_f32(q[b, i, h]).astype(np.float64)
    kf = inp.as_f32(k[b, kv, :inp.seq_lens[b]]).astype(np.float64)
    z = float(oracle.default_scale(wl.head_dim)) * (kf @ qf)
    return {blk: np.log(np.exp(z[16 * blk:16 * blk + 16] - z.max()).sum()) + z.max()
            for blk in blocks}


@pytest.mark.parametrize("name,rank_tol", [("llama8b", 0.0), ("serving", 0.0),
                                           ("serving", 0.05), ("rotated", 0.0)])
def test_ranking_check_matches_pairwise_brute_force(oracle_lib, name, rank_tol):
    inp, c, q, k, v = _setup(name, 3)
    r = c.decode_adaptive(q, inp.page_table, inp.seq_lens, k, v, tau_cov=0.9,
                          rank_tol=rank_tol)
    seen = {0: 0, 1: 0}
    for row, b, i, h in _rows(inp):
        m = _est_masses(inp, c, q, b, i, h)
        blocks = [int(x) for x in np.flatnonzero(r["kprom"][row, :m.size])]
        order = sorted(blocks, key=lambda x: (-m[x], x))     # the estimated ranking
        L = _exact_block_logmass(inp, q, k, b, i, h, blocks)
        fail = any(L[order[y]] - L[order[x]] > rank_tol
                   for x in range(len(order)) for y in range(x + 1, len(order)))
        assert bool(r["rank_fail"][row]) == fail, (row, order)
        seen[int(fail)] += 1
        if fail:
            assert r["flags"][row] == 1
    assert seen[0] and (seen[1] or rank_tol > 0)


def _two_block_case():
    """Hand-worked: d = 64, INT4 keys in groups of 32, one query q = e0, two
    pages of 16 identical tokens.
      page 0 keys a = 0.5 e0 + 7 e1: absmax 7, s = 7/7 = 1, code(0.5) = rint(0.5)
             = 0 (ties to even): k^_a = 7 e1, so z^_a = 0.125 * 0 = 0;
             exact z_a = 0.125 * 0.5 = 0.0625.
      page 1 keys b = 0.4375 e0: s = 0.4375/7 = 0.0625 exactly, code 7:
             k^_b = k_b, z^_b = z_b = 0.125 * 0.4375 = 0.0546875.
    Estimated masses M^_1 = 1 / (1 + e^-0.0546875) = 0.51366..., M^_0 = 0.48633...
    so the estimated order is (page 1, page 0) and tau_cov = 0.5 promotes page 1
    alone, 0.6 both.  Exact log-masses: L_0 - L_1 = 0.0625 - 0.0546875
    = 0.0078125 > 0 with page 0 ranked after page 1: the ranking is
    inconsistent for rank_tol < 0.0078125 and consistent above."""
    d = 64
    k = np.zeros((1, 1, 32, d), np.float32)
    k[0, 0, :16, 0] = 0.5
    k[0, 0, :16, 1] = 7.0
    k[0, 0, 16:, 0] = 0.4375
    v = np.zeros_like(k)
    v[0, 0, :, 0] = np.linspace(-1, 1, 32, dtype=np.float32)
    q = np.zeros((1, 1, 1, d), np.float32)
    q[0, 0, 0, 0] = 1.0
    pt = np.array([[0, 1]], np.int32)
    c = oracle.Cache(d, 1, 2, k_bits=4, k_group=32)
    assert c.append(k, v, pt, np.zeros(1, np.int32)) == 0
    return c, q, k, v, pt


def test_hand_worked_inversion(oracle_lib):
    c, q, k, v, pt = _two_block_case()
    r = c.decode_adaptive(q, pt, [32], k, v, tau_cov=0.5)
    assert list(r["kprom"][0]) == [0, 1] and r["nkey"][0] == 1 and r["rank_fail"][0] == 0
    for tol, fail in [(0.0, 1), (0.0078, 1), (0.0079, 0), (1.0, 0)]:
        r = c.decode_adaptive(q, pt, [32], k, v, tau_cov=0.6, rank_tol=tol)
        assert list(r["kprom"][0]) == [1, 1] and r["nkey"][0] == 2
        assert r["rank_fail"][0] == fail and r["flags"][0] == fail
    # with both blocks on exact keys the scores are exact: p = softmax(z) with
    # z = 0.0625 on page 0 and 0.0546875 on page 1
    r = c.decode_adaptive(q, pt, [32], k, v, tau_cov=0.6, rank_tol=1.0, v_tol=-1.0)
    w0 = 1.0 / (1.0 + math.exp(0.0546875 - 0.0625))
    vv = v[0, 0, :, 0].astype(np.float64)
    want = w0 * vv[:16].mean() + (1 - w0) * vv[16:].mean()
    assert abs(r["out"][0, 0] - want) < 1e-15


@pytest.mark.parametrize("name", list(SMALL))
@pytest.mark.parametrize("tau_cov,v_tol", [(0.5, math.inf), (0.9, math.inf), (0.995, 1e-3),
                                            (0.9, 1e-2)])
def test_adaptive_bound_dominates_observed_error(oracle_lib, name, tau_cov, v_tol):
    inp, c, q, k, v = _setup(name, 1)
    r = c.decode_adaptive(q, inp.page_table, inp.seq_lens, k, v, tau_cov=tau_cov, v_tol=v_tol)
    od = oracle.dense(q, k, v, inp.seq_lens)
    assert (r["bound"] >= max_err(od, r["out"])).all()


# ------------------------------------------------- planted mistakes ---------
# (name, text in kvq_oracle.c, replacement): plausible slips in the oracle's
# adaptive precision, each of which one of the pins above must catch.
MUTANTS = [
    ("coverage_one_block_short", "while (kstar < npg && cum < tau_cov) cum += ord[kstar++].m;",
     "while (kstar + 1 < npg && cum < tau_cov) cum += ord[kstar++].m;"),
    ("ascending_order", "  if (a->m > b->m) return -1;\n  if (a->m < b->m) return 1;",
     "  if (a->m < b->m) return -1;\n  if (a->m > b->m) return 1;"),
    ("ranking_check_reversed", "if (L - lmin > rank_tol) fail = 1;",
     "if (lmin - L > rank_tol) fail = 1;"),
    ("value_promotion_on_eta_only", "vp[lp] = ord[lp].m * et[lp * OC_PAGE] > v_tol ? 1 : 0;",
     "vp[lp] = et[lp * OC_PAGE] > v_tol ? 1 : 0;"),
    ("promoted_values_keep_eval", "for (int ch = 0; ch < d; ++ch) o[ch] += p[j] * (double)vf[ch];\n"
     "          } else {",
     "for (int ch = 0; ch < d; ++ch) o[ch] += p[j] * (double)vf[ch];\n"
     "            Ev += p[j] * et[j];\n          } else {"),
]

# the pins a mutant is run against, cheapest first
PROBES = [
    (test_hand_worked_inversion, {}),
    (test_selection_is_the_smallest_top_set_covering_tau_cov, {"name": "llama8b"}),
    (test_everything_promoted_is_dense_attention, {"name": "tiny"}),
    (test_values_only_is_value_promotion, {"name": "llama8b"}),
    (test_ranking_check_matches_pairwise_brute_force, {"name": "llama8b", "rank_tol": 0.0}),
]


@pytest.fixture(scope="module")
def mutant_dir(tmp_path_factory):
    return str(tmp_path_factory.mktemp("adaptive_mutants"))


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(oracle_lib, mutant_dir, name, old, new):
    src = oracle.source_text()
    assert src.count(old) == 1, f"mutation target of {name} not found once in the oracle"
    so = oracle.compile_variant(src.replace(old, new), mutant_dir, name)
    caught = None
    with oracle.library_override(so):
        for fn, kw in PROBES:
            try:
                fn(oracle_lib, **kw)
            except AssertionError:
                caught = fn.__name__
                break
    assert caught, f"no pin catches the planted mistake {name}"
