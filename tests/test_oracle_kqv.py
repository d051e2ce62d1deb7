"""Pins of the oracle's KQV codec ("Statistical Inference and Quality Measures
of KV Cache Quantisations Inspired by TurboQuant", Quantisation schemes: KQV:
Walsh-Hadamard rotation of K and V, K by the 4-bit scalar MSE (Lloyd-Max)
quantizer, V by the 3-bit one plus the 1-bit QJL sketch of its residual).

Against things other than its own code:
* the Lloyd-Max quantizer of N(0, 1) against Max's published table (1960) and
  the closed form sqrt(2/pi) of the 1-bit case; its fixed-point conditions by
  scipy quadrature; its mean squared errors against the table;
* the page's Beta((d-1)/2, (d-1)/2) marginal: under that density (scipy) the
  scaled Gaussian codebook's mean squared error is within 1% of what Lloyd's
  iteration on the Beta density reaches, at d = 64 and 128;
* codes are the nearest centroid and sketch bits the signs of S r (fp64);
* the QJL estimate is unbiased and its variance is the page's
  (pi/2)|r|^2 |y|^2 / m (less <y, r>^2 / m) over many draws of S;
* an independent numpy reader of the documented block layout reproduces the
  decode, and the stored eps, eta and value range cover the errors;
* the bound never falls below the error against exact attention, and Delta
  is tight for a rotated query that makes Hoelder's inequality an equality;
* five planted mistakes compiled into copies of the oracle are each caught.
"""

import math

import numpy as np
import pytest
import scipy.integrate
import scipy.linalg
import scipy.stats

import oracle
from oracle_cases import max_err, small

# Max (1960), optimum quantizer for a unit normal: positive output levels, MSE
MAX_TABLE = {
    1: ([0.7980], 0.3634),
    2: ([0.4528, 1.510], 0.1175),
    3: ([0.2451, 0.7560, 1.344, 2.152], 0.03454),
    4: ([0.1284, 0.3881, 0.6568, 0.9424, 1.256, 1.618, 2.069, 2.733], 0.009497),
}


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_lloyd_max_matches_max_table(oracle_lib, bits):
    c = oracle.lloyd_max(bits)
    n = c.size // 2
    assert np.array_equal(c[:n], -c[n:][::-1])            # symmetric
    levels, mse_tab = MAX_TABLE[bits]
    assert np.allclose(c[n:], levels, atol=6e-4, rtol=0)
    if bits == 1:
        assert abs(c[1] - math.sqrt(2 / math.pi)) < 1e-12
    # fixed point: each centroid is its cell's conditional mean (quadrature),
    # the thresholds are midpoints; the mean squared error is the table's
    t = np.concatenate([[-np.inf], 0.5 * (c[:-1] + c[1:]), [np.inf]])
    mse = 0.0
    for i in range(c.size):
        mass = scipy.stats.norm.cdf(t[i + 1]) - scipy.stats.norm.cdf(t[i])
        mean = scipy.integrate.quad(lambda x: x * scipy.stats.norm.pdf(x), t[i], t[i + 1])[0]
        assert abs(mean / mass - c[i]) < 1e-9
        mse += scipy.integrate.quad(lambda x: (x - c[i]) ** 2 * scipy.stats.norm.pdf(x),
                                    t[i], t[i + 1])[0]
    assert abs(mse - mse_tab) < 5e-4 * max(1.0, mse_tab * 100)


def _beta_lloyd_max(bits, d, iters=400):
    """Lloyd-Max for a coordinate of a uniform point on the sphere S^(d-1):
    (x + 1)/2 ~ Beta((d-1)/2, (d-1)/2)."""
    a = (d - 1) / 2.0
    dist = scipy.stats.beta(a, a, loc=-1.0, scale=2.0)
    L = 1 << bits
    c = np.linspace(-2.5, 2.5, L) / math.sqrt(d)
    for _ in range(iters):
        t = np.concatenate([[-1.0], 0.5 * (c[:-1] + c[1:]), [1.0]])
        new = np.empty_like(c)
        for i in range(L):
            mass = dist.cdf(t[i + 1]) - dist.cdf(t[i])
            new[i] = dist.expect(lambda x: x, lb=t[i], ub=t[i + 1]) / mass
        c = new
    return c


@pytest.mark.parametrize("d", [64, 128])
def test_gaussian_codebook_close_to_the_beta_marginal(oracle_lib, d):
    """The reading takes the Gaussian limit of the page's Beta marginal: at
    d = 64 and 128 its codebook's mean squared error under the Beta density is
    within 1% of what Lloyd's iteration on the Beta density itself reaches."""
    cent, thr = oracle.kqv_tables(oracle.KQV_KBITS, d)
    beta = _beta_lloyd_max(oracle.KQV_KBITS, d, iters=100)
    assert np.allclose(cent, beta, rtol=0.04, atol=0)
    a = (d - 1) / 2.0
    dist = scipy.stats.beta(a, a, loc=-1.0, scale=2.0)

    def mse(cb):
        t = np.concatenate([[-1.0], 0.5 * (cb[:-1] + cb[1:]), [1.0]])
        return sum(dist.expect(lambda x: (x - cb[i]) ** 2, lb=t[i], ub=t[i + 1])
                   for i in range(cb.size))
    assert mse(cent.astype(np.float64)) <= 1.01 * mse(beta)
    c = oracle.lloyd_max(oracle.KQV_KBITS)
    assert np.array_equal(cent, (c / math.sqrt(d)).astype(np.float32))
    assert np.array_equal(thr, ((c[:-1] + c[1:]) / (2 * math.sqrt(d))).astype(np.float32))
    assert thr[thr.size // 2] == 0.0


def _setup(name, seed, **kw):
    inp = small(name, seed, **kw)
    wl = inp.wl
    k, v = inp.kv()
    q = inp.q()
    c = oracle.KqvCache(wl.head_dim, wl.num_kv_heads, inp.num_pages, inp.rotation_signs(),
                        inp.qjl_matrix())
    assert c.append(k, v, inp.page_table, np.zeros(wl.num_seqs, np.int32),
                    valid=np.array(inp.seq_lens, np.int32)) == 0
    return inp, c, k, v, q


class _Reader:
    """numpy reader of the documented KQV block layout."""

    def __init__(self, c):
        self.c, self.d, self.bb = c, c.cfg.d, c.block_bytes

    def block(self, page, kv):
        off = (page * self.c.cfg.hkv + kv) * self.bb
        return self.c.pool[off:off + self.bb]

    def token(self, page, kv, slot):
        d, blk = self.d, self.block(page, kv)
        nib = lambda row: np.stack([row & 15, row >> 4], axis=1).reshape(-1)  # noqa: E731
        kc = nib(blk[slot * d // 2:(slot + 1) * d // 2])
        vc = nib(blk[16 * d // 2 + slot * d // 2:16 * d // 2 + (slot + 1) * d // 2])
        sb = blk[16 * d + slot * d // 8:16 * d + (slot + 1) * d // 8]
        bits = np.unpackbits(sb, bitorder="little").astype(np.float64) * 2 - 1
        f = blk[16 * d + 16 * d // 8:].view(np.float32)
        return dict(kc=kc, vc=vc, bits=bits, nk=f[slot], eps=f[16 + slot], nv=f[32 + slot],
                    rn=f[48 + slot], rg=f[64:64 + 2 * (d // 32)].reshape(-1, 2))


def _rot64(x, signs):
    """Exact-arithmetic Walsh-Hadamard rotation, fp64 (scipy's Hadamard matrix)."""
    d = x.shape[-1]
    H = scipy.linalg.hadamard(d).astype(np.float64) / math.sqrt(d)
    return (np.asarray(x, np.float64) * signs) @ H.T


@pytest.mark.parametrize("name", ["llama8b", "tiny", "serving"])
def test_codes_bits_and_error_annotations(oracle_lib, name):
    inp, c, k, v, q = _setup(name, 0, **({"spike_seq_frac": 0.5} if name == "serving" else {}))
    wl = inp.wl
    d = wl.head_dim
    R = _Reader(c)
    kcent, kthr = oracle.kqv_tables(4, d)
    vcent, vthr = oracle.kqv_tables(3, d)
    S = inp.qjl_matrix().astype(np.float64)
    H = scipy.linalg.hadamard(d).astype(np.float64) / math.sqrt(d)
    sig = inp.rotation_signs().astype(np.float64)
    kf, vf = inp.as_f32(k), inp.as_f32(v)
    checked = 0
    for b in range(wl.num_seqs):
        for t in range(0, inp.seq_lens[b], 7):
            page = inp.page_table[b, t // 16]
            for h in range(wl.num_kv_heads):
                tok = R.token(page, h, t % 16)
                kr, vr = _rot64(kf[b, h, t], sig), _rot64(vf[b, h, t], sig)
                # codes: the nearest centroid of the unit coordinates (away from midpoints)
                uk = kr / np.linalg.norm(kr)
                near = np.abs(uk[:, None] - kcent[None, :].astype(np.float64))
                best = near.argmin(axis=1)
                gap = np.sort(near, axis=1)[:, 1] - np.sort(near, axis=1)[:, 0]
                ok = gap > 1e-5
                assert np.array_equal(tok["kc"][ok], best[ok])
                assert abs(tok["nk"] - np.linalg.norm(kr)) <= 1e-5 * np.linalg.norm(kr)
                # eps covers |k' - k^'|
                kh = tok["nk"] * kcent[tok["kc"]].astype(np.float64)
                assert np.abs(kr - kh).max() <= tok["eps"] * (1 + 1e-5) + 1e-6
                uv = vr / np.linalg.norm(vr)
                nearv = np.abs(uv[:, None] - vcent[None, :].astype(np.float64))
                gapv = np.diff(np.sort(nearv, axis=1)[:, :2], axis=1)[:, 0]
                okv = gapv > 1e-5
                assert np.array_equal(tok["vc"][okv], nearv.argmin(axis=1)[okv])
                # sketch bits: signs of S r (fp64), away from zero
                r = uv - vcent[tok["vc"]].astype(np.float64)
                proj = S @ r
                okb = np.abs(proj) > 1e-4 * np.linalg.norm(r) * math.sqrt(d)
                assert np.array_equal(tok["bits"][okb], np.where(proj >= 0, 1.0, -1.0)[okb])
                # eta and the range cover the reconstruction
                vh_rot = float(tok["nv"]) * (vcent[tok["vc"]] + math.sqrt(math.pi / 2) / d *
                                             float(tok["rn"]) * (S.T @ tok["bits"]))
                vh = (H @ vh_rot) * sig
                assert np.abs(vf[b, h, t] - vh).max() <= c.eta[page, h]
                rg = tok["rg"]
                for g in range(d // 32):
                    seg = vh[32 * g:32 * g + 32]
                    assert rg[g, 0] >= max(seg.max(), 0) - 1e-5 and rg[g, 1] <= min(seg.min(), 0) + 1e-5
                checked += 1
    assert checked > 30


def test_qjl_is_unbiased_with_the_page_variance(oracle_lib):
    """<y, r~> over many draws of S: mean <y, r>, variance
    (pi/2) |r|^2 |y|^2 / m - <y, r>^2 / m with m = d projections."""
    d, N = 32, 20000
    rng = np.random.default_rng(5)
    r = rng.standard_normal(d).astype(np.float32)
    y = rng.standard_normal(d)
    est = np.empty(N)
    for i in range(N):
        S = rng.standard_normal((d, d)).astype(np.float32)
        _, rsum = oracle.qjl(r, S)
        rt = math.sqrt(math.pi / 2) / d * np.linalg.norm(r.astype(np.float64)) * rsum
        est[i] = y @ rt
    r64 = r.astype(np.float64)
    yr, rr, yy = y @ r64, r64 @ r64, y @ y
    var = (math.pi / 2) * rr * yy / d - yr ** 2 / d
    assert abs(est.mean() - yr) < 5 * math.sqrt(var / N)
    assert abs(est.var() / var - 1) < 0.05


@pytest.mark.parametrize("name", ["llama8b", "tiny"])
def test_decode_matches_an_independent_reader(oracle_lib, name):
    inp, c, k, v, q = _setup(name, 1)
    wl = inp.wl
    d = wl.head_dim
    R = _Reader(c)
    kcent, _ = oracle.kqv_tables(4, d)
    vcent, _ = oracle.kqv_tables(3, d)
    S = inp.qjl_matrix().astype(np.float64)
    sig = inp.rotation_signs()
    H = scipy.linalg.hadamard(d).astype(np.float64) / math.sqrt(d)
    o, bound, _, _ = c.decode(q, inp.page_table, inp.seq_lens)
    qf = inp.as_f32(q)
    scale = float(oracle.default_scale(d))
    row = 0
    for b in range(wl.num_seqs):
        n = inp.seq_lens[b]
        toks = [R.token(inp.page_table[b, t // 16], 0, t % 16) for t in range(n)]  # kv head 0
        for i in range(wl.num_queries):
            for h in range(wl.num_q_heads):
                if h // wl.group == 0:
                    qr = oracle.rotate(qf[b, i, h], sig).astype(np.float64)
                    kh = np.stack([np.float32(tk["nk"]) * kcent[tk["kc"]] for tk in toks]).astype(np.float64)
                    z = scale * (kh @ qr)
                    p = np.exp(z - z.max())
                    p /= p.sum()
                    vr = np.stack([float(tk["nv"]) * (vcent[tk["vc"]] + math.sqrt(math.pi / 2) /
                                                      d * float(tk["rn"]) * (S.T @ tk["bits"]))
                                   for tk in toks])
                    want = (H @ (p @ vr)) * sig
                    assert np.allclose(o[row], want, rtol=1e-9, atol=1e-9)
                row += 1


@pytest.mark.parametrize("name", ["llama8b", "tiny", "serving", "long128k"])
@pytest.mark.parametrize("seed", [0, 1])
def test_bound_dominates_observed_error(oracle_lib, name, seed):
    inp, c, k, v, q = _setup(name, seed, **({"spike_seq_frac": 0.5} if name == "serving" else {}))
    o, bound, _, diag = c.decode(q, inp.page_table, inp.seq_lens)
    od = oracle.dense(q, k, v, inp.seq_lens)
    err = max_err(od, o)
    assert (bound >= err).all()
    assert (diag[:, 0] <= 1.0).all() and (diag[:, 1] >= 0).all() and (diag[:, 2] > 0).all()


def test_delta_is_tight_for_a_one_hot_rotated_query(oracle_lib):
    """One token: with q' (the rotated query) one-hot on the channel where
    |k' - k^'| is largest, |z - z^| = s |q'| eps exactly (Hoelder's inequality
    is tight), and the oracle's Delta exceeds it by no more than kappa and the
    rotation allowance (a Delta with |q'|_2 in place of |q'|_1, a factor 2 or a
    dropped term fails one side)."""
    d = 128
    inp = small("llama8b", 0)
    rng = np.random.default_rng(8)
    k = rng.standard_normal(d).astype(np.float32)
    v = rng.standard_normal(d).astype(np.float32)
    sig = inp.rotation_signs()
    c = oracle.KqvCache(d, 1, 1, sig, inp.qjl_matrix())
    assert c.append(k.reshape(1, 1, 1, d), v.reshape(1, 1, 1, d), np.zeros((1, 1), np.int32),
                    np.zeros(1, np.int32)) == 0
    R = _Reader(c)
    tok = R.token(0, 0, 0)
    kcent, _ = oracle.kqv_tables(4, d)
    kr = _rot64(k, sig.astype(np.float64))
    kh = float(tok["nk"]) * kcent[tok["kc"]].astype(np.float64)
    cstar = int(np.abs(kr - kh).argmax())
    # q with q' = 3 e_cstar: the inverse rotation is sigma o (H x') / sqrt(d)
    onehot = np.zeros(d)
    onehot[cstar] = 3.0
    H = scipy.linalg.hadamard(d).astype(np.float64) / math.sqrt(d)
    q = (sig * (H @ onehot)).astype(np.float32)
    qr = _rot64(q, sig.astype(np.float64))
    _, _, _, diag = c.decode(q.reshape(1, 1, 1, d), np.zeros((1, 1), np.int32),
                             np.array([1], np.int32))
    s = float(oracle.default_scale(d))
    exact = s * abs(qr @ (kr - kh))
    e_inf = np.abs(kr - kh).max()
    assert exact == pytest.approx(s * 3.0 * e_inf, rel=1e-5)
    allowance = s * np.linalg.norm(qr) * 2 ** -16 * float(tok["nk"])
    slack = 1 + 2 ** -10
    assert exact * (1 - 1e-5) <= diag[0, 3] <= slack * (exact * (1 + 1e-4) + allowance) + 1e-12
    # q' = 3 sign(k' - k^') on every channel: |q' . e| = 3 |e|_1, which only
    # the 1-norm of q' covers (|q'|_2 eps falls short for a spread error)
    q2 = (sig * (H @ (3.0 * np.sign(kr - kh)))).astype(np.float32)
    qr2 = _rot64(q2, sig.astype(np.float64))
    _, _, _, diag2 = c.decode(q2.reshape(1, 1, 1, d), np.zeros((1, 1), np.int32),
                              np.array([1], np.int32))
    exact2 = s * abs(qr2 @ (kr - kh))
    assert exact2 == pytest.approx(s * 3.0 * np.abs(kr - kh).sum(), rel=1e-4)
    assert diag2[0, 3] >= exact2


# ------------------------------------------------- planted mistakes ---------
# (name, text in kvq_oracle.c, replacement): plausible slips in the KQV
# oracle, each of which one of the pins above must catch.
MUTANTS = [
    ("sketch_bit_sign", "if (oq_dot(S + (int64_t)i * d, r, d) >= 0.0f) bits[i / 8]",
     "if (oq_dot(S + (int64_t)i * d, r, d) < 0.0f) bits[i / 8]"),
    ("codebook_scale", "for (int i = 0; i < L; ++i) cent[i] = (float)(c[i] / sd);",
     "for (int i = 0; i < L; ++i) cent[i] = (float)(c[i] / d);"),
    ("eps_not_inf_norm", "if (nk > 0.0f && e > eps) eps = e;", "if (nk > 0.0f) eps = e;"),
    ("delta_l2_for_l1", "dl[j] = OC_KAPPA * sc * (qn1 * (double)oq_rdf(",
     "dl[j] = OC_KAPPA * sc * (qn2 * (double)oq_rdf("),
    ("decode_sketch_constant", "double rho = sqrt(OQ_PI / 2.0) / d * (double)oq_rdf(",
     "double rho = sqrt(OQ_PI) / d * (double)oq_rdf("),
]

# the pins a mutant is run against, cheapest first
PROBES = [
    (test_codes_bits_and_error_annotations, {"name": "tiny"}),
    (test_decode_matches_an_independent_reader, {"name": "tiny"}),
    (test_delta_is_tight_for_a_one_hot_rotated_query, {}),
    (test_gaussian_codebook_close_to_the_beta_marginal, {"d": 64}),
]


@pytest.fixture(scope="module")
def mutant_dir(tmp_path_factory):
    return str(tmp_path_factory.mktemp("kqv_mutants"))


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
