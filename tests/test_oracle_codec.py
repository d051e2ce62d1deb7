"""Pins of the oracle's codec against things other than itself.

* binary16 directed rounding vs numpy's float16 (round-to-nearest) stepped
  with numpy.nextafter -- an independent implementation of the same
  definition;
* hand-worked group quantizations (tests/golden/codec_hand_worked.txt);
* the round-trip invariant |x - deq(q(x))| <= s/2 (plus fp32 slack);
* exact recovery of representable inputs;
* the packed page layout is a bijection and matches the documented formula;
* five planted mistakes compiled into copies of the oracle are each caught.
"""

import os

import numpy as np
import pytest

import oracle
from quantized_decode_attention_kvq_b200 import inputs as synth

GOLD = os.path.join(os.path.dirname(__file__), "golden", "codec_hand_worked.txt")


def _np_round(x, up):
    """binary16 directed rounding from numpy's RN conversion + nextafter."""
    x = np.asarray(x, np.float32)
    with np.errstate(over="ignore"):
        rn = x.astype(np.float16)
        out = rn.copy()
        for i, (xi, ri) in enumerate(zip(x, rn)):
            if up and np.float64(ri) < np.float64(xi):
                out[i] = np.nextafter(ri, np.float16(np.inf))
            elif not up and np.float64(ri) > np.float64(xi):
                out[i] = np.nextafter(ri, np.float16(-np.inf))
            # overflow: RN gives inf; rounding toward the other side stays finite
            if np.isinf(ri) and np.sign(ri) != (1 if up else -1):
                out[i] = np.float16(np.sign(ri) * 65504.0)
    return out


def test_f16_directed_rounding_matches_numpy_definition(oracle_lib):
    rng = np.random.default_rng(1)
    mags = 10.0 ** rng.uniform(-9, 5.2, 4000)
    x = (mags * rng.choice([-1, 1], mags.size)).astype(np.float32)
    specials = np.array([0.0, -0.0, 65504.0, -65504.0, 65505.0, -65505.0, 7e4, -7e4,
                         2.0 ** -24, 2.0 ** -25, 3 * 2.0 ** -26, 1.0, 1.0 + 2 ** -11,
                         np.nextafter(np.float32(1.0), 2), 0.1, -0.1, 6.1e-5],
                        dtype=np.float32)
    x = np.concatenate([x, specials])
    for up in (True, False):
        got = oracle.f16_round(x, up).view(np.float16)
        ref = _np_round(x, up)
        both = np.isclose(got.astype(np.float64), ref.astype(np.float64), rtol=0, atol=0)
        both |= (np.isinf(got) & np.isinf(ref) & (np.sign(got) == np.sign(ref)))
        assert both.all(), (x[~both][:5], got[~both][:5], ref[~both][:5])
        # directed: never on the wrong side of x
        g = got.astype(np.float64)
        if up:
            assert (g >= x.astype(np.float64)).all()
        else:
            assert (g <= x.astype(np.float64)).all()


def test_f16_zero_sign_rule(oracle_lib):
    h = oracle.f16_round([-1e-9, 1e-9, -0.0, 0.0], up=True)
    assert list(h) == [0x8000, 0x0001, 0x8000, 0x0000]
    h = oracle.f16_round([-1e-9, 1e-9, -0.0, 0.0], up=False)
    assert list(h) == [0x8001, 0x0000, 0x8000, 0x0000]


def _dyadic(s):
    m, e = s.split("*2^")
    return float(m) * 2.0 ** int(e)


def _gold_cases():
    for line in open(GOLD):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        kind, xs, sc, zr, codes, err = [f.strip() for f in line.split("|")]
        yield kind, [float(t) for t in xs.split()], _dyadic(sc), zr, [int(t) for t in codes.split()], err


@pytest.mark.parametrize("case", list(_gold_cases()), ids=lambda c: c[0] + ":" + str(c[1]))
def test_hand_worked_groups(oracle_lib, case):
    kind, xs, scale, zero, codes, err = case
    if kind.startswith("sym"):
        rc, sb, got = oracle.quantize_sym(xs, 8 if kind == "sym8" else 4)
        assert rc == 0
        assert oracle.f16_value([sb])[0] == scale
        assert list(got) == codes
    else:
        rc, sb, zb, got, e = oracle.quantize_asym(xs)
        assert rc == 0
        assert oracle.f16_value([sb])[0] == scale
        assert oracle.f16_value([zb])[0] == _dyadic(zero) if "*" in zero else float(zero)
        assert list(got) == codes
        assert np.float32(e) == np.float32(float(err))


def _groups(rng, n, size):
    """Groups in the shapes the workloads produce: N(0,1), x20 outliers, +-50 spikes,
    bf16-rounded, plus tiny and huge magnitudes."""
    out = []
    for i in range(n):
        x = rng.standard_normal(size).astype(np.float32)
        kind = i % 5
        if kind == 1:
            x[rng.integers(0, size, 3)] *= 20
        elif kind == 2:
            x[rng.integers(0, size)] = rng.choice([-50.0, 50.0])
        elif kind == 3:
            x *= np.float32(10.0 ** rng.uniform(-6, 3))
        x = synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(x)) if kind != 4 else x
        out.append(x)
    return out


@pytest.mark.parametrize("bits", [8, 4])
def test_roundtrip_invariant_symmetric(oracle_lib, bits):
    Q = 127 if bits == 8 else 7
    rng = np.random.default_rng(bits)
    for x in _groups(rng, 400, 128 if bits == 8 else 32):
        rc, sb, codes = oracle.quantize_sym(x, bits)
        assert rc == 0
        s = oracle.f16_value([sb])[0]
        assert s >= np.abs(x).max() / Q * (1 - 2 ** -23)          # codes never clip
        err = np.abs(x.astype(np.float64) - s * codes)
        assert (err <= s / 2 * (1 + 2 ** -14)).all()
        assert np.abs(codes).max() <= Q


def test_roundtrip_invariant_asymmetric(oracle_lib):
    rng = np.random.default_rng(7)
    for x in _groups(rng, 400, 32):
        rc, sb, zb, codes, e = oracle.quantize_asym(x)
        assert rc == 0
        s, z = oracle.f16_value([sb, zb])
        assert z <= x.min()
        assert z + 15 * s >= x.max() - 2 ** -22 * (abs(x.max()) + abs(z))
        vhat = np.float32(s) * codes.astype(np.float32) + np.float32(z)   # numpy fp32
        ex = np.abs(x.astype(np.float64) - (s * codes + z))
        slack = 2 ** -22 * (np.abs(x) + abs(z) + 15 * s)
        assert (ex <= s / 2 + slack).all()
        assert e >= np.abs(x - vhat).max() * (1 - 2 ** -20) - 1e-30


@pytest.mark.parametrize("bits", [8, 4])
def test_exact_recovery_symmetric(oracle_lib, bits):
    Q = 127 if bits == 8 else 7
    rng = np.random.default_rng(11)
    for e in range(-20, 8, 3):
        s = 2.0 ** e
        codes = rng.integers(-Q, Q + 1, 32)
        codes[rng.integers(0, 32)] = Q * rng.choice([-1, 1])
        x = (s * codes).astype(np.float32)
        rc, sb, got = oracle.quantize_sym(x, bits)
        assert rc == 0 and oracle.f16_value([sb])[0] == s
        assert (got == codes).all()


def test_exact_recovery_asymmetric(oracle_lib):
    rng = np.random.default_rng(12)
    for e in range(-14, 5, 3):
        s = 2.0 ** e
        z = float(np.float16(rng.standard_normal()))
        codes = rng.integers(0, 16, 32)
        codes[0], codes[1] = 0, 15
        x = (z + s * codes).astype(np.float32)
        assert np.array_equal(x.astype(np.float64), z + s * codes)   # representable
        rc, sb, zb, got, err = oracle.quantize_asym(x)
        assert rc == 0
        assert oracle.f16_value([sb])[0] == s and oracle.f16_value([zb])[0] == z
        assert (got == codes).all() and err == 0.0


def test_range_errors(oracle_lib):
    assert oracle.quantize_sym([1.0, np.nan], 8)[0] == oracle.ERR_RANGE
    assert oracle.quantize_sym([1.0, np.inf], 8)[0] == oracle.ERR_RANGE
    assert oracle.quantize_sym([1e7, 0.0], 4)[0] == oracle.ERR_RANGE     # scale > 65504
    assert oracle.quantize_sym([8e6, 0.0], 8)[0] == 0                    # 63000 fits
    assert oracle.quantize_asym([-7e4, 0.0])[0] == oracle.ERR_RANGE      # zero < -65504
    assert oracle.quantize_asym([-6e4, 1e6])[0] == oracle.ERR_RANGE      # scale > 65504


def _u16(buf, off):
    return int(buf[off]) | (int(buf[off + 1]) << 8)


def _k8_byte(d, ch):   # documented stripe order (8-bit keys), the oracle's pool
    nb, b, w = d // 32, ch // 32, ch % 32
    return (w // 8) * (8 * nb) + 8 * b + w % 8


def _k8_device_byte(d, ch, slot):   # the library's device layout of the same byte
    p = _k8_byte(d, ch)
    if d == 128:   # 128-byte rows: the 16-byte chunk index is XORed with slot % 8
        p = (((p >> 4) ^ (slot % 8)) << 4) | (p & 15)
    return p


def _k4_byte(d, ch):   # documented layout (4-bit keys)
    nb, b, w = d // 32, ch // 32, ch % 32
    return (w // 8) * (4 * nb) + 4 * b + (w % 8) // 2


def _v4_byte(d, ch):   # documented layout (4-bit values)
    nb, g, w = d // 32, ch // 32, ch % 32
    return (w // 4) * (2 * nb) + 2 * g + (w % 4) // 2


@pytest.mark.parametrize("d", [64, 128])
def test_nibble_layouts_are_bijections(d):
    for f in (_k4_byte, _v4_byte):
        slots = {(f(d, c), c % 2) for c in range(d)}
        assert len(slots) == d and max(b for b, _ in slots) == d // 2 - 1
    assert sorted(_k8_byte(d, c) for c in range(d)) == list(range(d))
    for slot in range(16):
        assert sorted(_k8_device_byte(d, c, slot) for c in range(d)) == list(range(d))
    # a thread of the decode kernel reads one contiguous stripe per token
    assert [_v4_byte(128, c) for c in (0, 1, 2, 3, 32, 34, 4)] == [0, 0, 1, 1, 2, 3, 8]
    assert [_k4_byte(128, c) for c in (0, 2, 6, 8, 32, 40)] == [0, 1, 3, 16, 4, 20]
    assert [_k8_byte(128, c) for c in (0, 7, 8, 32, 39, 40, 127)] == [0, 7, 32, 8, 15, 40, 127]
    # slot 3 of a 128-byte row: chunk q of the stripe order lands in chunk q ^ 3
    assert [_k8_device_byte(128, c, 3) for c in (0, 7, 8, 32, 39, 40, 127)] == \
        [48, 55, 16, 56, 63, 24, 79]
    assert [_k8_device_byte(64, c, 3) for c in (0, 8, 32)] == [0, 16, 8]   # 64-byte rows


def test_device_permutation_helper(oracle_lib):
    """device_pool (the test-side conversion of the oracle's logical pool into
    the library's documented device layout) moves each key code to the byte
    the documented formula gives, and nothing else."""
    from oracle_cases import device_pool
    rng = np.random.default_rng(11)
    d, H = 128, 2
    k = rng.standard_normal((1, H, 20, d)).astype(np.float32)
    v = rng.standard_normal((1, H, 20, d)).astype(np.float32)
    c = oracle.Cache(d, H, 2, k_bits=8, k_group=128)
    assert c.append(k, v, np.array([[1, 0]], np.int32), [0]) == 0
    dev = device_pool(c)
    bb = c.block_bytes
    for blk in range(2 * H):
        lo, do = c.pool[blk * bb:(blk + 1) * bb], dev[blk * bb:(blk + 1) * bb]
        assert np.array_equal(lo[16 * d:], do[16 * d:])
        for slot in range(16):
            for ch in range(d):
                assert do[slot * d + _k8_device_byte(d, ch, slot)] == lo[slot * d + _k8_byte(d, ch)]


@pytest.mark.parametrize("kbits,kgroup,d", [(8, 128, 128), (4, 32, 128), (8, 32, 64)])
def test_pack_roundtrip_through_pool(oracle_lib, kbits, kgroup, d):
    """Codes written to the page pool decode back to the group quantizer's output."""
    rng = np.random.default_rng(3)
    H, T = 2, 37
    k = rng.standard_normal((1, H, T, d)).astype(np.float32)
    v = rng.standard_normal((1, H, T, d)).astype(np.float32)
    npages = 3
    pt = np.array([[2, 0, 1]], np.int32)
    c = oracle.Cache(d, H, npages, k_bits=kbits, k_group=kgroup)
    assert c.append(k, v, pt, [0]) == 0
    bb = c.block_bytes
    kcode_bytes = 16 * d * kbits // 8
    for h in range(H):
        for t in range(T):
            blk = c.pool[(pt[0, t // 16] * H + h) * bb:][:bb]
            slot = t % 16
            for g in range(d // kgroup):
                rc, sb, codes = oracle.quantize_sym(k[0, h, t, g * kgroup:(g + 1) * kgroup], kbits)
                off = kcode_bytes + 16 * d // 2 + (slot * (d // kgroup) + g) * 2
                assert _u16(blk, off) == sb
                for i, cd in enumerate(codes):
                    ch = g * kgroup + i
                    if kbits == 8:
                        assert np.int8(blk[slot * d + _k8_byte(d, ch)]) == cd
                    else:
                        byte = int(blk[slot * d // 2 + _k4_byte(d, ch)])
                        nib = (byte >> 4) if ch % 2 else (byte & 15)
                        assert (nib - 16 if nib >= 8 else nib) == cd
            for g in range(d // 32):
                rc, sb, zb, codes, e = oracle.quantize_asym(v[0, h, t, g * 32:(g + 1) * 32])
                off = kcode_bytes + 16 * d // 2 + 16 * (d // kgroup) * 2 + (slot * (d // 32) + g) * 4
                assert _u16(blk, off) == sb
                assert _u16(blk, off + 2) == zb
                for i, cd in enumerate(codes):
                    ch = g * 32 + i
                    byte = blk[kcode_bytes + slot * d // 2 + _v4_byte(d, ch)]
                    assert ((byte >> 4) if ch % 2 else (byte & 15)) == cd
    # eta: max over the page's tokens of the group errors, one ulp up
    for lp, page in enumerate(pt[0]):
        for h in range(H):
            errs = [oracle.quantize_asym(v[0, h, t, g * 32:(g + 1) * 32])[4]
                    for t in range(lp * 16, min(T, lp * 16 + 16)) for g in range(d // 32)]
            assert c.eta[page, h] == np.nextafter(np.float32(max(errs)), np.float32(np.inf))


# ------------------------------------------------- planted mistakes ---------
# (name, text in kvq_oracle.c, replacement): plausible slips in the oracle's
# Tier-1 codec, each of which one of the pins above must catch.
MUTANTS = [
    ("key_scale_rounded_down", "float t = a / (float)Q;\n  uint16_t sb = oc_f16_round(t, 1);",
     "float t = a / (float)Q;\n  uint16_t sb = oc_f16_round(t, 0);"),
    ("key_scale_over_q_plus_one", "float t = a / (float)Q;", "float t = a / (float)(Q + 1);"),
    ("key_code_truncated", "float r = rintf(x[c] / s);", "float r = truncf(x[c] / s);"),
    ("value_zero_rounded_up", "uint16_t zb = oc_f16_round(lo, 0);", "uint16_t zb = oc_f16_round(lo, 1);"),
    ("value_sixteen_steps", "float t = (hi - z) / 15.0f;", "float t = (hi - z) / 16.0f;"),
]

# the pins a mutant is run against, cheapest first
PROBES = [
    (lambda lib: [test_hand_worked_groups(lib, c) for c in _gold_cases()], {}),
    (test_roundtrip_invariant_symmetric, {"bits": 8}),
    (test_roundtrip_invariant_asymmetric, {}),
    (test_exact_recovery_symmetric, {"bits": 4}),
    (test_exact_recovery_asymmetric, {}),
]


@pytest.fixture(scope="module")
def mutant_dir(tmp_path_factory):
    return str(tmp_path_factory.mktemp("codec_mutants"))


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
                caught = True
                break
    assert caught, f"no pin catches the planted mistake {name}"
