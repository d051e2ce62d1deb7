"""Pins of the oracle's Med3x outlier extraction ("Hurwitz Quaternion
Multiplicative Quantization for KV Cache Compression", Method 3: 4-element
chunks whose norm exceeds 3x the median chunk norm are kept in fp16 with a
flag; the bulk codec quantizes the rest).

Against things other than its own code:
* binary16 round-to-nearest against numpy's float16 conversion;
* the chunk choice against the definition in fp64 (numpy's median), on
  random and spiked vectors whose decision is not within 1e-6 of the
  threshold;
* a hand-worked token with one spike;
* extraction lowers eta (the largest |v - v^| of a block) in spike
  sequences and raises it nowhere; the bound dominates the error against
  exact attention;
* with no chunk above the threshold, the decode equals the one without
  extraction;
* eta covers the fp16 rounding of an extracted value (a hand case);
* four planted mistakes compiled into copies of the oracle are each caught.
"""

import math

import numpy as np
import pytest

import oracle
from oracle_cases import max_err, small


def test_f16_round_to_nearest_matches_numpy(oracle_lib):
    rng = np.random.default_rng(7)
    x = (10.0 ** rng.uniform(-8, 4.7, 3000) * rng.choice([-1, 1], 3000)).astype(np.float32)
    ties = np.array([1 + 2 ** -11, 1 + 3 * 2 ** -11, 2 ** -24 * 1.5, 2 ** -24 * 2.5, 65504.0,
                     -0.0, 0.0, 3 * 2 ** -25], np.float32)
    x = np.concatenate([x, ties])
    got = oracle.f16_rn(x)
    want = x.astype(np.float16).view(np.uint16)
    assert np.array_equal(got, want), x[got != want][:5]


def _fp64_choice(x):
    r = np.sqrt((x.astype(np.float64).reshape(-1, 4) ** 2).sum(axis=1))
    thr = 3.0 * np.median(r)
    over = np.flatnonzero(r > thr)
    margin = np.abs(r / thr - 1.0).min()
    return (int(over[np.argmax(r[over])]) if over.size else -1), margin, r


@pytest.mark.parametrize("d", [64, 128])
def test_chunk_choice_matches_definition(oracle_lib, d):
    rng = np.random.default_rng(d)
    checked = picked = 0
    for t in range(2000):
        x = rng.standard_normal(d).astype(np.float32)
        if t % 3 == 0:                                   # one or two spikes
            x[rng.integers(d)] = np.float32(rng.choice([-1, 1]) * rng.uniform(2, 60))
        if t % 7 == 0:
            x[rng.integers(d)] = np.float32(rng.uniform(-40, 40))
        want, margin, r = _fp64_choice(x)
        if margin < 1e-6:
            continue
        # the largest of two chunks above the threshold must be clear as well
        over = np.sort(r[r > 3.0 * np.median(r)])
        if over.size > 1 and over[-1] - over[-2] < 1e-6 * over[-1]:
            continue
        assert oracle.med3_chunk(x) == want, (t, want)
        checked += 1
        picked += want >= 0
    assert checked > 1800 and picked > 300


def _one_token_cache(k, v, d=64, **kw):
    c = oracle.Cache(d, 1, 1, k_bits=8, k_group=d, outliers=True, **kw)
    assert c.append(k.reshape(1, 1, 1, d), v.reshape(1, 1, 1, d), np.zeros((1, 1), np.int32),
                    np.zeros(1, np.int32)) == 0
    return c


def test_hand_worked_spike_token(oracle_lib):
    """d = 64: V = 0.25 everywhere except channel 9 = 50 and channel 33 = -0.5;
    K = 1.0 everywhere except channel 60 = 40.
      V chunk norms: chunk 2 (channels 8-11) sqrt(3 * 0.0625 + 2500) = 50.00187...,
      the others 0.5 (chunk 8: sqrt(3 * 0.0625 + 0.25) = 0.6614...); median of the
      16 norms = 0.5 -> threshold 1.5 -> chunk 2 is extracted.
      Group 0 without channels 8-11: all 0.25 -> z = 0.25, s = 0, codes 0, error 0.
      Group 1: min -0.5 = z, max 0.25: s = fp16 up of 0.75/15 = 0.05 -> 1639*2^-15;
      0.25 -> rint(0.75 / s) = rint(14.9954...) = 15 -> v^ = -0.5 + 15 s = 0.25022888...,
      error 2.2888e-4.  The stored chunk: fp16(50) = 50, fp16(0.25) = 0.25: exact.
      eta = nextafter(2.2888184e-4).
      K: chunk 15 (channels 60-63) norm sqrt(1600 + 3) = 40.04, the others 2;
      median 2 -> threshold 6 -> chunk 15 extracted, stored (40, 1, 1, 1); the
      bulk absmax is 1.0 ->
      s = fp16 up of 1/127 (= 1032.06 * 2^-17) = 1033*2^-17 = 0.0078812..., codes
      rint(1/s) = 127, and channels 60-63 get code 0."""
    d = 64
    v = np.full(d, 0.25, np.float32)
    v[9] = 50.0
    v[33] = -0.5
    k = np.ones(d, np.float32)
    k[60] = 40.0
    assert oracle.med3_chunk(v) == 2 and oracle.med3_chunk(k) == 15
    c = _one_token_cache(k, v)
    blk = c.pool
    L = dict(kcode=16 * d, vcode=16 * d // 2, ks=16 * 2, vm=16 * (d // 32) * 4)
    out = L["kcode"] + L["vcode"] + L["ks"] + L["vm"]
    assert blk[out] == 15 and blk[out + 16] == 2            # K chunk, V chunk of slot 0
    k16 = blk[out + 32:out + 32 + 8].view(np.float16)
    v16 = blk[out + 32 + 128:out + 32 + 128 + 8].view(np.float16)
    # channel 60 opens chunk 15; channel 9 is the second of chunk 2 (channels 8-11)
    assert list(k16.astype(np.float64)) == [40.0, 1.0, 1.0, 1.0]
    assert list(v16.astype(np.float64)) == [0.25, 50.0, 0.25, 0.25]
    ks = blk[L["kcode"] + L["vcode"]:L["kcode"] + L["vcode"] + 2].view(np.float16)[0]
    assert float(ks) == 1033 * 2.0 ** -17
    vm = blk[L["kcode"] + L["vcode"] + L["ks"]:][:8].view(np.float16)
    assert float(vm[0]) == 0.0 and float(vm[1]) == 0.25      # group 0: s = 0, z = 0.25
    assert float(vm[2]) == 1639 * 2.0 ** -15 and float(vm[3]) == -0.5
    want_eta = np.nextafter(np.float32(abs(np.float32(0.25) - np.float32(
        np.float32(-0.5) + np.float32(15) * np.float32(1639 * 2.0 ** -15)))), np.float32(1))
    assert c.eta[0, 0] == want_eta


@pytest.mark.parametrize("name", ["serving", "llama8b", "rotated", "tiny"])
def test_roundtrip_and_bound_with_extraction(oracle_lib, name):
    inp = small(name, 1, **({"spike_seq_frac": 0.5} if name == "serving" else {}))
    wl = inp.wl
    k, v = inp.kv()
    q = inp.q()
    c = oracle.Cache(wl.head_dim, wl.num_kv_heads, inp.num_pages, k_bits=wl.k_bits,
                     k_group=wl.k_group, k_rotate=wl.k_rotate, rot_signs=inp.rot_signs,
                     outliers=True)
    assert c.append(k, v, inp.page_table, np.zeros(wl.num_seqs, np.int32),
                    valid=np.array(inp.seq_lens, np.int32)) == 0
    o, bound, _, _ = c.decode(q, inp.page_table, inp.seq_lens)
    od = oracle.dense(q, k, v, inp.seq_lens)
    assert (bound >= max_err(od, o)).all()
    # extraction lowers eta where the spikes are and raises it nowhere
    c0 = oracle.Cache(wl.head_dim, wl.num_kv_heads, inp.num_pages, k_bits=wl.k_bits,
                      k_group=wl.k_group, k_rotate=wl.k_rotate, rot_signs=inp.rot_signs)
    assert c0.append(k, v, inp.page_table, np.zeros(wl.num_seqs, np.int32),
                     valid=np.array(inp.seq_lens, np.int32)) == 0
    if inp.spike_seqs:
        s = inp.spike_seqs[0]
        pages = inp.page_table[s, :inp.pages_per_seq[s]]
        assert c.eta[pages].max() < 0.5 * c0.eta[pages].max()
    assert (c.eta <= c0.eta + 1e-6).all()


def test_no_outlier_means_same_decode(oracle_lib):
    """Gaussian data with no chunk above 3x the median: the codes and the decode
    equal those without extraction."""
    inp = small("llama8b", 3, outlier_frac=0.0)
    wl = inp.wl
    k, v = inp.kv()
    q = inp.q()
    kf, vf = inp.as_f32(k), inp.as_f32(v)
    flat = np.concatenate([kf.reshape(-1, wl.head_dim), vf.reshape(-1, wl.head_dim)])
    assert all(oracle.med3_chunk(x) < 0 for x in flat[::7])
    res = []
    for out in (False, True):
        c = oracle.Cache(wl.head_dim, wl.num_kv_heads, inp.num_pages, k_bits=wl.k_bits,
                         k_group=wl.k_group, outliers=out)
        assert c.append(k, v, inp.page_table, np.zeros(wl.num_seqs, np.int32),
                        valid=np.array(inp.seq_lens, np.int32)) == 0
        res.append(c.decode(q, inp.page_table, inp.seq_lens))
    if all(oracle.med3_chunk(x) < 0 for x in flat):
        assert np.array_equal(res[0][0], res[1][0]) and np.array_equal(res[0][1], res[1][1])


def test_eta_covers_the_fp16_rounding_of_an_extracted_value(oracle_lib):
    """d = 64: V = 0.25 everywhere except channel 9 = 50.0123, which fp16
    rounds to 50.0 (spacing 2^-5 there); the other values are exact for the
    INT4 group codec (a constant group), so eta is the fp16 error, 0.0123,
    raised by one ulp."""
    d = 64
    k = np.ones(d, np.float32)
    v = np.full(d, 0.25, np.float32)
    v[9] = np.float32(50.0123)
    c = _one_token_cache(k, v, d)
    err16 = abs(float(v[9]) - float(np.float16(v[9])))
    assert 0.012 < err16 < 0.013
    assert err16 <= c.eta[0, 0] <= err16 * (1 + 1e-6) + 1e-30


# ------------------------------------------------- planted mistakes ---------
# (name, text in kvq_oracle.c, replacement): plausible slips in the oracle's
# Med3x, each of which one of the pins above must catch.
MUTANTS = [
    ("threshold_2x", "float thr = 3.0f * med;", "float thr = 2.0f * med;"),
    ("median_upper_only", "float med = 0.5f * (srt[nc / 2 - 1] + srt[nc / 2]);",
     "float med = srt[nc / 2];"),
    ("first_not_largest", "if (r[i] > thr && (best < 0 || r[i] > r[best])) best = i;",
     "if (r[i] > thr && best < 0) best = i;"),
    ("eta_without_fp16_error", "float err = fabsf(x - (float)oc_f16_value(hv));",
     "float err = 0.0f;"),
]

# the pins a mutant is run against, cheapest first
PROBES = [
    (test_hand_worked_spike_token, {}),
    (test_eta_covers_the_fp16_rounding_of_an_extracted_value, {}),
    (test_chunk_choice_matches_definition, {"d": 64}),
]


@pytest.fixture(scope="module")
def mutant_dir(tmp_path_factory):
    return str(tmp_path_factory.mktemp("med3_mutants"))


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
