"""Pins of the oracle's HQMQ codec ("Hurwitz Quaternion Multiplicative
Quantization for KV Cache Compression", Method 1-2: every 4-channel chunk of K
and V split into its radius and its direction on S^3, the direction coded by
the product codebook {q_p q_s : q_p in 2T, q_s in a random secondary set}).

Against things other than its own code:
* the 24 primary units are the binary tetrahedral group 2T: unit, distinct,
  closed under a quaternion product written here (4x4 matrices, fp64), with
  2T's element orders (1, 1, 8, 6, 8 elements of order 1, 2, 3, 4, 6) and 60
  degrees between nearest neighbours;
* each codeword is q_p q_s to fp32 rounding (and to fp16 rounding in the
  reconstruction), and each secondary unit maps 2T isometrically (the page's
  argument for calibration-free codebooks);
* the direction code is the codeword of largest inner product, by brute force
  in fp64 over all 24 S codewords;
* covering: every direction lies within 45 degrees (the 24-cell's covering
  radius, attained at (1 + i)/sqrt 2) of a codeword for any S, and the mean
  angular error falls with S like (24 S)^(-1/3) (the page's Proposition 3.1);
* the radius in fp8 E4M3 against torch's float8_e4m3fn cast and hand values;
* exact recovery of chunks that are representable (r^ c16 with r^ in E4M3);
* an independent numpy reader of the documented block layout reproduces the
  decode; eps, eta and the value range cover the errors; the bound never falls
  below the error against exact attention, and Delta is tight when q is
  parallel to a token's error vector.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from oracle_cases import max_err, small


def _lmat(a):
    """Left multiplication by quaternion a as a 4x4 matrix (a b = L(a) b)."""
    a0, a1, a2, a3 = (float(x) for x in a)
    return np.array([[a0, -a1, -a2, -a3],
                     [a1, a0, -a3, a2],
                     [a2, a3, a0, -a1],
                     [a3, -a2, a1, a0]])


def _qmul(a, b):
    return _lmat(a) @ np.asarray(b, np.float64)


def _primaries():
    return np.stack([oracle.hq_primary(p).astype(np.float64) for p in range(24)])


def _key(q):
    return tuple(np.round(q * 2).astype(int))


def test_primary_units_are_2T(oracle_lib):
    P = _primaries()
    assert np.allclose(np.linalg.norm(P, axis=1), 1.0)
    keys = {_key(p) for p in P}
    assert len(keys) == 24
    for a in P:                                  # closed under the product
        for b in P:
            assert _key(_qmul(a, b)) in keys
    one = np.array([1.0, 0, 0, 0])
    orders = []
    for a in P:
        x, k = a.copy(), 1
        while not np.allclose(x, one):
            x, k = _qmul(x, a), k + 1
        orders.append(k)
    assert sorted(orders) == [1] + [2] + [3] * 8 + [4] * 6 + [6] * 8
    G = P @ P.T
    off = G[~np.eye(24, dtype=bool)]
    assert off.max() == 0.5                      # nearest neighbours 60 degrees apart
    assert set(np.round(off * 2).astype(int)) <= {-2, -1, 0, 1}


def _secondary(S, seed):
    x = np.random.default_rng(seed).standard_normal((S, 4))
    return (x / np.linalg.norm(x, axis=1, keepdims=True)).astype(np.float32)


def _book64(sec):
    """All 24 S codewords in fp64, computed here (index 24 s + p)."""
    P = _primaries()
    return np.stack([_qmul(P[i % 24], sec[i // 24].astype(np.float64))
                     for i in range(24 * sec.shape[0])])


def test_codewords_are_products_and_isometric_copies(oracle_lib):
    sec = _secondary(5, 3)
    book = _book64(sec)
    got = np.stack([oracle.hq_codeword(sec, i) for i in range(book.shape[0])]).astype(np.float64)
    assert np.abs(got - book).max() < 2 ** -23
    assert np.allclose(np.linalg.norm(got, axis=1), 1.0, atol=1e-6)
    got16 = np.stack([oracle.hq_codeword16(sec, i) for i in range(book.shape[0])])
    assert np.array_equal(got16, got.astype(np.float32).astype(np.float16).astype(np.float32))
    P = _primaries()
    for s in range(sec.shape[0]):                # right multiplication by q_s is an isometry
        blk = got[24 * s:24 * s + 24]
        assert np.allclose(blk @ blk.T, P @ P.T, atol=1e-6)


@pytest.mark.parametrize("S", [1, 7, 64])
def test_direction_is_the_best_codeword(oracle_lib, S):
    sec = _secondary(S, S)
    book = _book64(sec)
    rng = np.random.default_rng(11)
    X = (rng.standard_normal((400, 4)) * rng.uniform(0.01, 30, (400, 1))).astype(np.float32)
    same = 0
    for x in X:
        i = oracle.hq_direction(x, sec)
        ip = book @ x.astype(np.float64)
        assert ip[i] >= ip.max() - 1e-6 * np.linalg.norm(x)
        same += i == int(ip.argmax())
    assert same >= 396
    # a zero chunk takes code 0
    assert oracle.hq_direction(np.zeros(4, np.float32), sec) == 0


def test_covering_radius_and_rate(oracle_lib):
    rng = np.random.default_rng(2)
    U = rng.standard_normal((3000, 4))
    U /= np.linalg.norm(U, axis=1, keepdims=True)
    U32 = U.astype(np.float32)
    # the 24-cell's covering radius is 45 degrees, at the centre of a cell
    one = np.array([[1.0, 0, 0, 0]], np.float32)
    deep = np.array([1, 1, 0, 0], np.float32) / np.float32(math.sqrt(2))
    c = oracle.hq_codeword(one, oracle.hq_direction(deep, one)).astype(np.float64)
    assert abs(c @ deep.astype(np.float64) - math.sqrt(0.5)) < 1e-6
    mean_angle = {}
    for S in (1, 4, 32, 256):
        sec = _secondary(S, 100 + S)
        ang = []
        for u in U32[:1000 if S == 256 else 3000]:
            cw = oracle.hq_codeword(sec, oracle.hq_direction(u, sec)).astype(np.float64)
            cosv = cw @ u.astype(np.float64) / np.linalg.norm(cw)
            assert cosv >= math.sqrt(0.5) - 1e-6
            ang.append(math.acos(min(1.0, cosv)))
        mean_angle[S] = float(np.mean(ang))
    # Proposition 3.1: covering rate O((24 S)^(-1/3)); the mean error follows
    for s1, s2 in ((4, 32), (32, 256)):
        ratio = mean_angle[s2] / mean_angle[s1]
        assert 0.35 < ratio < 0.7, (s1, s2, ratio)   # (1/8)^(1/3) = 0.5


def test_e4m3_radius(oracle_lib):
    assert oracle.e4m3_rn(1.0) == 0x38 and oracle.e4m3_value(0x38) == 1.0
    assert oracle.e4m3_rn(448.0) == 0x7E and oracle.e4m3_value(0x7E) == 448.0
    assert oracle.e4m3_rn(1e6) == 0x7E                      # saturates
    assert oracle.e4m3_rn(2.0 ** -9) == 0x01                # smallest subnormal
    assert oracle.e4m3_rn(2.0 ** -11) == 0x00               # below half of it
    assert oracle.e4m3_rn(1.0625) == 0x38                   # tie between 1 and 1.125: even
    assert oracle.e4m3_rn(1.1875) == 0x3A                   # tie between 1.125 and 1.25: even
    assert oracle.e4m3_rn(0.0) == 0
    rng = np.random.default_rng(4)
    x = np.concatenate([rng.uniform(0, 448, 4000), 2.0 ** rng.uniform(-12, 8.8, 4000)])
    x = x[x <= 448].astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_rn(v) for v in x], np.uint8)
    assert np.array_equal(got, ref)
    codes = np.arange(0x7F, dtype=np.uint8)
    vals = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.array([oracle.e4m3_value(int(c)) for c in codes]), vals)


def _setup(name, seed, S=16, **kw):
    inp = small(name, seed, **kw)
    wl = inp.wl
    k, v = inp.kv()
    q = inp.q()
    c = oracle.HqCache(wl.head_dim, wl.num_kv_heads, inp.num_pages, inp.hqmq_secondary(S))
    assert c.append(k, v, inp.page_table, np.zeros(wl.num_seqs, np.int32),
                    valid=np.array(inp.seq_lens, np.int32)) == 0
    return inp, c, k, v, q


class _Reader:
    """numpy reader of the documented HQMQ block layout."""

    def __init__(self, c):
        self.c, self.d, self.bb = c, c.cfg.d, c.block_bytes
        self.nc = self.d // 4
        self.E4 = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(
            torch.float64).numpy()
        self.books = [[_book64(c.sec[h, r]) for r in range(2)] for h in range(c.cfg.hkv)]
        # the reconstruction's codewords: fp16 of the fp32 products
        self.books16 = [[b.astype(np.float32).astype(np.float16).astype(np.float64) for b in bh]
                        for bh in self.books]

    def token(self, page, kv, slot):
        nc, blk = self.nc, self.c.pool[(page * self.c.cfg.hkv + kv) * self.bb:][:self.bb]
        ki = blk[:32 * nc].view(np.uint16).reshape(nc, 16)[:, slot]
        vi = blk[32 * nc:64 * nc].view(np.uint16).reshape(nc, 16)[:, slot]
        kr = self.E4[blk[64 * nc:80 * nc].reshape(nc, 16)[:, slot]]
        vr = self.E4[blk[80 * nc:96 * nc].reshape(nc, 16)[:, slot]]
        f = blk[96 * nc:].view(np.float32)
        kh = (kr[:, None] * self.books16[kv][0][ki]).reshape(-1)
        vh = (vr[:, None] * self.books16[kv][1][vi]).reshape(-1)
        return dict(ki=ki, vi=vi, kr=kr, vr=vr, kh=kh, vh=vh, nk=f[slot], eps=f[16 + slot],
                    rg=f[32:32 + 2 * (self.d // 32)].reshape(-1, 2))


@pytest.mark.parametrize("name", ["llama8b", "tiny", "serving"])
def test_codes_radii_and_error_annotations(oracle_lib, name):
    inp, c, k, v, q = _setup(name, 0, **({"spike_seq_frac": 0.5} if name == "serving" else {}))
    wl = inp.wl
    R = _Reader(c)
    kf, vf = inp.as_f32(k).astype(np.float64), inp.as_f32(v).astype(np.float64)
    checked = 0
    for b in range(wl.num_seqs):
        for t in range(0, inp.seq_lens[b], 5):
            page = inp.page_table[b, t // 16]
            for h in range(wl.num_kv_heads):
                tok = R.token(page, h, t % 16)
                for role, x in ((0, kf[b, h, t]), (1, vf[b, h, t])):
                    book = R.books[h][role]
                    idx, rad = (tok["ki"], tok["kr"]) if role == 0 else (tok["vi"], tok["vr"])
                    xc = x.reshape(-1, 4)
                    ip = xc @ book.T
                    best = ip.max(axis=1)
                    assert (ip[np.arange(len(idx)), idx] >= best - 1e-6 * np.linalg.norm(xc, axis=1)).all()
                    r = np.linalg.norm(xc, axis=1)
                    # the stored radius is the nearest E4M3 value of r
                    cand = R.E4[:0x7F]
                    near = np.abs(cand[None, :] - r[:, None]).min(axis=1)
                    assert np.allclose(np.abs(rad - r), near, rtol=0, atol=1e-6 * (1 + r))
                assert abs(tok["nk"] - np.linalg.norm(kf[b, h, t])) <= 1e-5 * np.linalg.norm(kf[b, h, t])
                ek = np.linalg.norm(kf[b, h, t] - tok["kh"])
                assert ek <= tok["eps"] <= ek * (1 + 1e-4) + 1e-30
                assert np.abs(vf[b, h, t] - tok["vh"]).max() <= c.eta[page, h]
                rg = tok["rg"]
                for g in range(wl.head_dim // 32):
                    seg = tok["vh"][32 * g:32 * g + 32]
                    assert rg[g, 0] >= max(seg.max(), 0) - 1e-5 and rg[g, 1] <= min(seg.min(), 0) + 1e-5
                checked += 1
    assert checked > 20


def test_exact_recovery_of_representable_chunks(oracle_lib):
    d, S = 128, 16
    rng = np.random.default_rng(9)
    sec = _secondary(S, 21)
    secs = np.stack([sec, _secondary(S, 22)])[None]          # [1][2][S][4]
    x = np.zeros((2, d), np.float32)
    codes = rng.integers(0, 24 * S, size=(2, d // 4))
    rads = rng.integers(0x20, 0x60, size=(2, d // 4)).astype(np.uint8)
    for role in range(2):
        for ch in range(d // 4):
            cw = oracle.hq_codeword16(secs[0, role], int(codes[role, ch]))
            x[role, 4 * ch:4 * ch + 4] = np.float32(oracle.e4m3_value(int(rads[role, ch]))) * cw
    c = oracle.HqCache(d, 1, 1, secs)
    k = x[0].reshape(1, 1, 1, d)
    v = x[1].reshape(1, 1, 1, d)
    assert c.append(k, v, np.zeros((1, 1), np.int32), np.zeros(1, np.int32)) == 0
    kh, vh = c.read_token(0, 0, 0)
    assert np.array_equal(kh, x[0]) and np.array_equal(vh, x[1])
    R = _Reader(c)
    tok = R.token(0, 0, 0)
    assert np.array_equal(tok["ki"], codes[0]) and np.array_equal(tok["vi"], codes[1])
    assert tok["eps"] < 1e-40
    assert c.eta[0, 0] <= np.linalg.norm(x[1]) * 2.0 ** -16 * (1 + 1e-6)


@pytest.mark.parametrize("name", ["llama8b", "tiny"])
def test_decode_matches_an_independent_reader(oracle_lib, name):
    inp, c, k, v, q = _setup(name, 1)
    wl = inp.wl
    R = _Reader(c)
    o, bound, _, _ = c.decode(q, inp.page_table, inp.seq_lens)
    qf = inp.as_f32(q).astype(np.float64)
    scale = float(oracle.default_scale(wl.head_dim))
    row = 0
    for b in range(wl.num_seqs):
        n = inp.seq_lens[b]
        for i in range(wl.num_queries):
            for h in range(wl.num_q_heads):
                kv = h // wl.group
                toks = [R.token(inp.page_table[b, t // 16], kv, t % 16) for t in range(n)]
                kh = np.stack([tk["kh"] for tk in toks])
                vh = np.stack([tk["vh"] for tk in toks])
                z = scale * (kh @ qf[b, i, h])
                p = np.exp(z - z.max())
                p /= p.sum()
                assert np.allclose(o[row], p @ vh, rtol=1e-5, atol=1e-6)
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


def test_delta_is_tight_for_a_query_along_the_error(oracle_lib):
    """One token: with q parallel to k - k^, |z - z^| = s |q| |k - k^| exactly,
    and the oracle's Delta (diag[3]) exceeds it by no more than kappa and the
    2^-16 |k| allowance (a Delta with |q|_1, a factor 2 or a dropped term fails)."""
    d, S = 128, 8
    rng = np.random.default_rng(6)
    secs = np.stack([_secondary(S, 31), _secondary(S, 32)])[None]
    k = rng.standard_normal(d).astype(np.float32)
    v = rng.standard_normal(d).astype(np.float32)
    c = oracle.HqCache(d, 1, 1, secs)
    assert c.append(k.reshape(1, 1, 1, d), v.reshape(1, 1, 1, d), np.zeros((1, 1), np.int32),
                    np.zeros(1, np.int32)) == 0
    kh, _ = c.read_token(0, 0, 0)
    e = k.astype(np.float64) - kh.astype(np.float64)
    q = (3.0 * e / np.linalg.norm(e)).astype(np.float32)
    _, _, _, diag = c.decode(q.reshape(1, 1, 1, d), np.zeros((1, 1), np.int32),
                             np.array([1], np.int32))
    s = float(oracle.default_scale(d))
    qn = np.linalg.norm(q.astype(np.float64))
    exact = s * abs(q.astype(np.float64) @ e)
    assert exact == pytest.approx(s * qn * np.linalg.norm(e), rel=1e-6)
    slack = 1 + 2 ** -10
    allowance = s * qn * 2 ** -16 * np.linalg.norm(k.astype(np.float64))
    assert exact <= diag[0, 3] <= slack * (exact * (1 + 1e-4) + allowance) + 1e-12


def _setup_ext(name, seed, S=16, **kw):
    inp = small(name, seed, **kw)
    wl = inp.wl
    k, v = inp.kv()
    q = inp.q()
    caches = []
    for ext in (False, True):
        c = oracle.HqCache(wl.head_dim, wl.num_kv_heads, inp.num_pages, inp.hqmq_secondary(S),
                           outliers=ext)
        assert c.append(k, v, inp.page_table, np.zeros(wl.num_seqs, np.int32),
                        valid=np.array(inp.seq_lens, np.int32)) == 0
        caches.append(c)
    return inp, caches, k, v, q


def test_med3_extraction_in_the_hqmq_codec(oracle_lib):
    """Method 3 over the HQMQ codec: the chunk oc_med3_chunk picks (pinned in
    test_oracle_med3) is stored in fp16 (numpy's float16 of the inputs), takes
    code 0 and radius 0 and reconstructs to its fp16 values; every other chunk
    is coded exactly as without extraction; the tokens' key error falls where
    a chunk is extracted and stays where none is."""
    inp, (plain, ext), k, v, q = _setup_ext("serving", 0, spike_seq_frac=0.5)
    wl = inp.wl
    d, nc = wl.head_dim, wl.head_dim // 4
    kf, vf = inp.as_f32(k), inp.as_f32(v)
    bp, be = plain.block_bytes, ext.block_bytes
    assert be == bp + 288
    extracted = fell = 0
    for b in range(wl.num_seqs):
        for t in range(inp.seq_lens[b]):
            page = inp.page_table[b, t // 16]
            slot = t % 16
            for h in range(wl.num_kv_heads):
                P = plain.pool[(page * wl.num_kv_heads + h) * bp:][:bp]
                X = ext.pool[(page * wl.num_kv_heads + h) * be:][:be]
                os_ = X[bp:]
                kh, vh = ext.read_token(page, h, slot)
                for role, x, xh in ((0, kf[b, h, t], kh), (1, vf[b, h, t], vh)):
                    cx = int(os_[role * 16 + slot])
                    want = oracle.med3_chunk(x)
                    assert cx == (0xFF if want < 0 else want)
                    idx_p = P[role * 32 * nc:(role + 1) * 32 * nc].view(np.uint16).reshape(nc, 16)[:, slot]
                    idx_e = X[role * 32 * nc:(role + 1) * 32 * nc].view(np.uint16).reshape(nc, 16)[:, slot]
                    rad_p = P[64 * nc + role * 16 * nc:][:16 * nc].reshape(nc, 16)[:, slot]
                    rad_e = X[64 * nc + role * 16 * nc:][:16 * nc].reshape(nc, 16)[:, slot]
                    keep = np.arange(nc) != cx
                    assert np.array_equal(idx_p[keep], idx_e[keep])
                    assert np.array_equal(rad_p[keep], rad_e[keep])
                    if cx != 0xFF:
                        extracted += 1
                        assert idx_e[cx] == 0 and rad_e[cx] == 0
                        h16 = os_[32 + role * 128 + slot * 8:][:8].view(np.float16)
                        assert np.array_equal(h16, x[4 * cx:4 * cx + 4].astype(np.float16))
                        assert np.array_equal(xh[4 * cx:4 * cx + 4], h16.astype(np.float32))
                eps_p = P[96 * nc + 64:][:64].view(np.float32)[slot]
                eps_e = X[96 * nc + 64:][:64].view(np.float32)[slot]
                if os_[slot] == 0xFF:
                    assert eps_e == eps_p
                else:
                    fell += eps_e < eps_p
    assert extracted > 10
    assert fell > 0


@pytest.mark.parametrize("name", ["llama8b", "serving", "tiny"])
@pytest.mark.parametrize("seed", [0, 1])
def test_med3_hqmq_bound_dominates_observed_error(oracle_lib, name, seed):
    inp, (plain, ext), k, v, q = _setup_ext(name, seed, spike_seq_frac=0.5)
    o, bound, _, _ = ext.decode(q, inp.page_table, inp.seq_lens)
    od = oracle.dense(q, k, v, inp.seq_lens)
    err = max_err(od, o)
    assert (bound >= err).all()
    # the decode over the extraction cache is attention over its reconstructions
    o2, _, _, _ = plain.decode(q, inp.page_table, inp.seq_lens)
    assert np.isfinite(o2).all()


# ------------------------------------------------- planted mistakes ---------
# (name, text in kvq_oracle.c, replacement): plausible slips in the HQMQ
# oracle, each of which one of the pins above must catch.
MUTANTS = [
    ("y_component_sign", "y[1] = fmaf(x[3], b[2], fmaf(-x[2], b[3], fmaf(x[1], b[0], -x[0] * b[1])));",
     "y[1] = fmaf(x[3], b[2], fmaf(x[2], b[3], fmaf(x[1], b[0], -x[0] * b[1])));"),
    ("half_unit_scale", "float h = 0.5f * (((a[0] + a[1]) + a[2]) + a[3]);",
     "float h = 0.45f * (((a[0] + a[1]) + a[2]) + a[3]);"),
    ("product_sign", "{a[0] * b[1], a[1] * b[0], a[2] * b[3], -(a[3] * b[2])},",
     "{a[0] * b[1], a[1] * b[0], -(a[2] * b[3]), (a[3] * b[2])},"),
    ("primary_sign_bits", "q[n] = ((p - 8) >> n) & 1 ? -0.5f : 0.5f;",
     "q[n] = ((p - 8) >> (3 - n)) & 1 ? -0.5f : 0.5f;"),
    ("e4m3_ties_up", "return (uint8_t)((lo & 1) ? lo + 1 : lo);", "return (uint8_t)(lo + 1);"),
    ("eps_doubled", "nextafterf(fmaf(en, 1.0f / 65536.0f, en), INFINITY)",
     "nextafterf(2.0f * en, INFINITY)"),
    ("delta_scaled_norm", "dl[j] = OC_KAPPA * sc * qn2 *", "dl[j] = OC_KAPPA * sc * 1.5 * qn2 *"),
    ("med3_chunk_dropped", "xh[4 * cx + i] = (float)oc_f16_value(h);", "xh[4 * cx + i] = 0.0f;"),
]

# the pins a mutant is run against, cheapest first
PROBES = [
    (test_primary_units_are_2T, {}),
    (test_e4m3_radius, {}),
    (test_codewords_are_products_and_isometric_copies, {}),
    (test_direction_is_the_best_codeword, {"S": 7}),
    (test_exact_recovery_of_representable_chunks, {}),
    (test_delta_is_tight_for_a_query_along_the_error, {}),
    (test_codes_radii_and_error_annotations, {"name": "tiny"}),
    (test_med3_extraction_in_the_hqmq_codec, {}),
]


@pytest.fixture(scope="module")
def mutant_dir(tmp_path_factory):
    return str(tmp_path_factory.mktemp("hqmq_mutants"))


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
