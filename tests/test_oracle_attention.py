"""Pins of the oracle's rotation, attention and certified bound.

Against: scipy's Sylvester Hadamard matrix, an fp64 matrix product, torch's
fp64 scaled-dot-product attention, the two-token logistic closed form, an
independent numpy dequantization of the group quantizers' output, brute force
over score perturbations (the total-variation lemma behind E_key), and fp64
dense attention on the originals (bound dominance on every query); four
planted mistakes compiled into copies of the oracle are each caught.
"""

import math

import numpy as np
import pytest
import scipy.linalg
import torch

import oracle
from quantized_decode_attention_kvq_b200 import inputs as synth
from oracle_cases import SMALL, max_err, oracle_cache, run_oracle, small


# --------------------------------------------------------------- rotation --
@pytest.mark.parametrize("d", [64, 128])
def test_rotation_columns_are_scaled_hadamard(oracle_lib, d):
    c = np.float32(1.0 / math.sqrt(d))
    eye = np.eye(d, dtype=np.float32)
    cols = oracle.rotate(eye, np.ones(d, np.int8))          # row i = R e_i
    H = scipy.linalg.hadamard(d).astype(np.float64)
    assert np.array_equal(cols.T.astype(np.float64), c * H)


@pytest.mark.parametrize("d", [64, 128])
def test_rotation_matches_fp64_and_preserves_products(oracle_lib, d):
    rng = np.random.default_rng(d)
    sig = np.where(rng.integers(0, 2, d) == 1, 1, -1).astype(np.int8)
    x = rng.standard_normal((50, d)).astype(np.float32)
    x[:, :3] *= 20
    y = oracle.rotate(x, sig).astype(np.float64)
    H = scipy.linalg.hadamard(d).astype(np.float64)
    ref = (x.astype(np.float64) * sig) @ H.T * np.float64(np.float32(1 / math.sqrt(d)))
    nrm = np.linalg.norm(x.astype(np.float64), axis=1, keepdims=True)
    assert (np.abs(y - ref) <= 2 ** -20 * nrm).all()
    # inner products survive to fp32 accuracy (orthogonal up to c^2 d = 1 +- 2^-23)
    G = y @ y.T
    G0 = x.astype(np.float64) @ x.astype(np.float64).T
    assert np.abs(G - G0).max() <= 2 ** -18 * (nrm @ nrm.T).max()


# ------------------------------------------------------------------ dense --
def test_dense_two_token_closed_form(oracle_lib):
    d = 4
    q = np.array([[[[0.5, -1.0, 2.0, 0.25]]]], np.float32)
    k = np.array([[[[1, 0, 0, 0], [0, 0, 1, 0]]]], np.float32)
    v = np.array([[[[1, 2, 3, 4], [-1, 0, 5, 2]]]], np.float32)
    s = np.float64(np.float32(0.5))
    o = oracle.dense(q, k, v, [2], scale=0.5)[0]
    z1, z2 = s * 0.5, s * 2.0
    p1 = 1.0 / (1.0 + math.exp(z2 - z1))                     # logistic form
    v64 = v.astype(np.float64)
    assert np.allclose(o, p1 * v64[0, 0, 0] + (1 - p1) * v64[0, 0, 1], rtol=0, atol=1e-14)


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_dense_matches_torch_sdpa_fp64(oracle_lib, dtype):
    inp = synth.make("llama8b", 3, num_seqs=2, num_q_heads=8, num_kv_heads=2, ctx=77,
                     num_queries=2, dtype=dtype)
    q, (k, v) = inp.q(), inp.kv()
    got = oracle.dense(q, k, v, inp.seq_lens)
    qt = torch.from_numpy(inp.as_f32(q)).double()                 # [B, nq, Hq, d]
    kt = torch.from_numpy(inp.as_f32(k)).double()                 # [B, Hkv, T, d]
    vt = torch.from_numpy(inp.as_f32(v)).double()
    G = inp.wl.group
    kt = kt.repeat_interleave(G, dim=1)
    vt = vt.repeat_interleave(G, dim=1)
    ref = torch.nn.functional.scaled_dot_product_attention(
        qt.permute(0, 2, 1, 3), kt, vt, scale=float(oracle.default_scale(inp.wl.head_dim)))
    ref = ref.permute(0, 2, 1, 3).reshape(-1, inp.wl.head_dim).numpy()
    assert np.abs(got - ref).max() < 1e-12


# ------------------------------------------------------ quantized decode --
@pytest.mark.parametrize("name", ["tiny", "llama8b", "rotated"])
def test_decode_equals_attention_on_dequantized_cache(oracle_lib, name):
    """o_hat from the page pool == fp64 attention over k_hat, v_hat built from the
    group quantizers' codes and scales (independent of the page layout)."""
    inp = small(name)
    wl = inp.wl
    r = run_oracle(inp)
    k, v = r["k"], r["v"]
    kf, vf = inp.as_f32(k), inp.as_f32(v)
    q = r["q"]
    if wl.k_rotate:
        kf = oracle.rotate(kf, inp.rot_signs)
        qf = oracle.rotate(inp.as_f32(q), inp.rot_signs)
    else:
        qf = inp.as_f32(q)
    khat = np.zeros(kf.shape, np.float64)
    vhat = np.zeros(vf.shape, np.float64)
    B, H, T, d = kf.shape
    for b in range(B):
        for h in range(H):
            for t in range(inp.seq_lens[b]):
                for g in range(d // wl.k_group):
                    sl = slice(g * wl.k_group, (g + 1) * wl.k_group)
                    rc, sb, codes = oracle.quantize_sym(kf[b, h, t, sl], wl.k_bits)
                    khat[b, h, t, sl] = oracle.f16_value([sb])[0] * codes
                for g in range(d // 32):
                    sl = slice(g * 32, (g + 1) * 32)
                    rc, sb, zb, codes, e = oracle.quantize_asym(vf[b, h, t, sl])
                    s, z = oracle.f16_value([sb, zb])
                    vhat[b, h, t, sl] = s * codes + z
    # dense() reads fp32 inputs: k_hat and v_hat are exact in fp32
    ref = oracle.dense(qf, khat.astype(np.float32), vhat.astype(np.float32), inp.seq_lens)
    assert np.abs(r["o_hat"] - ref).max() < 1e-12


def test_exact_recovery_makes_decode_exact(oracle_lib):
    """Inputs representable by the codec: o_hat equals dense attention and the
    value term vanishes."""
    rng = np.random.default_rng(5)
    B, H, T, d, HQ = 1, 1, 40, 64, 2
    k = np.zeros((B, H, T, d), np.float32)
    v = np.zeros((B, H, T, d), np.float32)
    for t in range(T):
        for g in range(d // 32):
            sl = slice(g * 32, (g + 1) * 32)
            ck = rng.integers(-127, 128, 32)
            ck[0] = 127
            k[0, 0, t, sl] = 2.0 ** -5 * ck
            cv = rng.integers(0, 16, 32)
            cv[0], cv[1] = 0, 15
            v[0, 0, t, sl] = np.float16(rng.standard_normal()) + 2.0 ** -3 * cv
    q = rng.standard_normal((B, 1, HQ, d)).astype(np.float32)
    c = oracle.Cache(d, H, 3, k_bits=8, k_group=32)
    pt = np.array([[1, 2, 0]], np.int32)
    assert c.append(k, v, pt, [0]) == 0
    o_hat, bound, flags, diag = c.decode(q, pt, [T])
    o_dense = oracle.dense(q, k, v, [T])
    assert np.abs(o_hat - o_dense).max() < 1e-13
    assert (diag[:, 2] < 1e-40).all()                  # E_val ~ one subnormal ulp
    assert (bound >= 0).all()


@pytest.mark.parametrize("name", ["tiny", "llama8b", "rotated", "serving"])
def test_score_perturbation_bounded_by_delta(oracle_lib, name):
    """|z_j - z^_j| <= Delta_j for every token (z from the originals in fp64)."""
    inp = small(name)
    r = run_oracle(inp)
    wl = inp.wl
    qf = inp.as_f32(r["q"]).astype(np.float64)
    kf = inp.as_f32(r["k"]).astype(np.float64)
    sc = np.float64(oracle.default_scale(wl.head_dim))
    for b in range(wl.num_seqs):
        n = inp.seq_lens[b]
        for h in range(0, wl.num_q_heads, max(1, wl.group // 2)):
            zq, dl = r["cache"].decode_terms(r["q"], inp.page_table, n, b, 0, h)
            z = sc * kf[b, h // wl.group, :n] @ qf[b, 0, h]
            assert (np.abs(z - zq) <= dl).all()
            assert (dl > 0).all()


def _tv_bounds(p, dl):
    A = np.sum(p * np.expm1(dl))
    B = np.sum(p * np.exp(-dl))
    return min(math.tanh(dl.max() / 2), A / B)


def test_tv_lemma_brute_force():
    """For p ~ p^ exp(a), |a_j| <= Delta_j: TV(p, p^) <= min(tanh(max Delta/2), A/B)."""
    rng = np.random.default_rng(9)
    worst = 0.0
    for trial in range(3000):
        n = rng.integers(2, 7)
        p = rng.dirichlet(np.full(n, rng.uniform(0.1, 3)))
        dl = rng.uniform(0, rng.choice([0.01, 0.3, 2.0]), n)
        bound = _tv_bounds(p, dl)
        # corners of the perturbation box, plus random interior points
        corners = np.array(np.meshgrid(*[[-1, 1]] * n)).reshape(n, -1).T
        pts = np.concatenate([corners, rng.uniform(-1, 1, (20, n))])
        for s in pts:
            pp = p * np.exp(s * dl)
            pp /= pp.sum()
            tv = 0.5 * np.abs(pp - p).sum()
            assert tv <= bound * (1 + 1e-12) + 1e-15
            worst = max(worst, tv / bound if bound > 0 else 0)
    assert worst > 0.5          # the bound is not vacuous: corners come close


@pytest.mark.parametrize("name", list(SMALL))
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_bound_dominates_observed_error(oracle_lib, name, seed):
    """Every query: bound >= |o_dense - o_hat|_inf (fp64 brute force)."""
    inp = small(name, seed)
    r = run_oracle(inp)
    err = max_err(r["o_dense"], r["o_hat"])
    assert (r["bound"] >= err).all(), (r["bound"][r["bound"] < err], err[r["bound"] < err])
    assert (r["bound"] > 0).all()
    # the key term is the TV bound times the value range
    d = r["diag"]
    assert (d[:, 0] <= 1.0).all() and (d[:, 1] >= 0).all() and (d[:, 2] > 0).all()


@pytest.mark.parametrize("name", ["tiny", "llama8b", "serving"])
def test_true_tv_below_certified_tv(oracle_lib, name):
    inp = small(name)
    r = run_oracle(inp)
    wl = inp.wl
    qf = inp.as_f32(r["q"]).astype(np.float64)
    kf = inp.as_f32(r["k"]).astype(np.float64)
    sc = np.float64(oracle.default_scale(wl.head_dim))
    for b in range(wl.num_seqs):
        n = inp.seq_lens[b]
        for h in range(wl.num_q_heads):
            row = (b * wl.num_queries) * wl.num_q_heads + h
            zq, _ = r["cache"].decode_terms(r["q"], inp.page_table, n, b, 0, h)
            z = sc * kf[b, h // wl.group, :n] @ qf[b, 0, h]
            p = np.exp(z - z.max()); p /= p.sum()
            ph = np.exp(zq - zq.max()); ph /= ph.sum()
            assert 0.5 * np.abs(p - ph).sum() <= r["diag"][row, 0] * (1 + 1e-12)


def test_flags_and_certified_output(oracle_lib):
    inp = small("serving")
    r = run_oracle(inp)
    assert inp.spike_seqs
    flags = r["flags"].astype(bool)
    assert np.array_equal(flags, r["bound"] > inp.wl.tau)
    out = oracle.certified(r["o_hat"], r["o_dense"], r["flags"])
    assert np.array_equal(out[flags], r["o_dense"][flags])
    err = max_err(r["o_dense"], out)
    assert (err <= np.where(flags, 0.0, r["bound"])).all()      # bounded or exact


def test_empty_context_row(oracle_lib):
    inp = synth.make("llama8b", 0, num_seqs=2, num_q_heads=4, num_kv_heads=1, ctx=40)
    k, v = inp.kv()
    c = oracle_cache(inp)
    assert c.append(k, v, inp.page_table, [0, 0], valid=[40, 0]) == 0
    o_hat, bound, flags, diag = c.decode(inp.q(), inp.page_table, [40, 0], tau=0.0)
    assert (o_hat[4:] == 0).all() and (bound[4:] == 0).all() and (flags[4:] == 0).all()
    assert (flags[:4] == 1).all()


# ------------------------------------------------- planted mistakes ---------
# (name, text in kvq_oracle.c, replacement): plausible slips in the oracle's
# rotation and dense attention, each of which one of the pins above must catch.
_DENSE_K = ("oc_load_vec(k, kv_is_f32, b * seq_stride + kv * head_stride + j * tok_stride, d, kf);\n"
            "          double dot = 0.0;\n"
            "          for (int ch = 0; ch < d; ++ch) dot += (double)qf[ch] * (double)kf[ch];\n"
            "          z[j] = sc * dot;\n          if (z[j] > m) m = z[j];")
_DENSE_P = ("double p = exp(z[j] - m) / l;\n"
            "          oc_load_vec(v, kv_is_f32, b * seq_stride + kv * head_stride + j * tok_stride, d, vf);")
MUTANTS = [
    ("butterfly_sign", "y[j + h] = a - b;", "y[j + h] = b - a;"),
    ("rotation_scale", "float c = (float)(1.0 / sqrt((double)d));", "float c = (float)(1.0 / d);"),
    ("dense_unnormalized", _DENSE_P, _DENSE_P.replace("exp(z[j] - m) / l", "exp(z[j] - m)")),
    ("dense_scale_twice", _DENSE_K, _DENSE_K.replace("z[j] = sc * dot;", "z[j] = sc * sc * dot;")),
]

# the pins a mutant is run against, cheapest first
PROBES = [
    (test_rotation_columns_are_scaled_hadamard, {"d": 64}),
    (test_dense_two_token_closed_form, {}),
    (test_dense_matches_torch_sdpa_fp64, {"dtype": "fp32"}),
]


@pytest.fixture(scope="module")
def mutant_dir(tmp_path_factory):
    return str(tmp_path_factory.mktemp("attention_mutants"))


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
