"""Pins of the certified bound's magnitude.

The oracle's bound ("Runtime-Certified Bounded-Error Quantized Attention",
Methodology 2) is checked term by term against hand-worked cases
(tests/golden/bound_hand_worked.txt): Delta, A, B, the tanh and A/B branches
of the total-variation bound, the value range per group, eta, E_key, E_val and
the bound.  Every code and scale in those cases is exact, so the expected
numbers are closed forms derived by hand in the file.

The second half plants, one at a time, the mistakes a reader could make in
the bound's formula into a copy of the oracle (the half in Delta, kappa, the
2 eta_max term, the range definition, min against max in TV, the rotation
allowance, the mass weighting of E_val, ...) and checks that the hand-worked
cases catch every one of them.
"""

import os

import numpy as np
import pytest

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden", "bound_hand_worked.txt")
D = 64


def _spec(text, n=D, dtype=np.float32):
    """'i=x' / 'i-j=x' items applied left to right onto zeros."""
    x = np.zeros(n, dtype=np.float64)
    for item in text.split():
        idx, val = item.split("=")
        if "-" in idx:
            a, b = idx.split("-")
            x[int(a):int(b) + 1] = float(val)
        else:
            x[int(idx)] = float(val)
    return x.astype(dtype)


def _cases():
    cases, cur = [], None
    for raw in open(GOLD):
        line = raw.strip()
        if not line or line.startswith("#"):
            continue
        head, _, rest = line.partition(" ")
        if head == "case":
            cur = dict(name=rest, tokens=[])
            cases.append(cur)
        elif head == "config":
            cfg = {}
            parts = rest.split(" signs=")
            for kv in parts[0].split():
                k, v = kv.split("=")
                cfg[k] = v
            cur["cfg"] = cfg
            cur["signs"] = _spec(parts[1], dtype=np.int8) if len(parts) > 1 else None
        elif head == "q":
            cur["q"] = _spec(rest)
        elif head == "token":
            reps = 1
            if rest.startswith("x"):
                r, _, rest = rest.partition(" ")
                reps = int(r[1:])
            ks, vs = rest.split("|")
            assert ks.strip().startswith("k ") and vs.strip().startswith("v ")
            k, v = _spec(ks.strip()[2:]), _spec(vs.strip()[2:])
            cur["tokens"] += [(k, v)] * reps
        elif head == "expect":
            cur["expect"] = {kv.split("=")[0]: float(kv.split("=")[1]) for kv in rest.split()}
        else:
            raise ValueError(f"bad golden line: {line}")
    return cases


CASES = _cases()
DIAG = ["tv", "ekey", "eval", "dmax", "A", "B", "range", "eta_max"]


def _run(case):
    """The oracle's diagnostics and bound for one hand-worked case."""
    cfg = case["cfg"]
    pt = np.array([[int(p) for p in cfg["page_table"].split(",")]], np.int32)
    n = len(case["tokens"])
    c = oracle.Cache(D, 1, pt.shape[1], k_bits=int(cfg["kbits"]), k_group=int(cfg["kgroup"]),
                     k_rotate=cfg["rotate"] == "1", rot_signs=case["signs"])
    k = np.stack([t[0] for t in case["tokens"]])[None, None]
    v = np.stack([t[1] for t in case["tokens"]])[None, None]
    assert c.append(k, v, pt, np.zeros(1, np.int32)) == 0
    q = case["q"].reshape(1, 1, 1, D)
    _, bound, _, diag = c.decode(q, pt, np.array([n], np.int32))
    got = dict(zip(DIAG, diag[0]))
    got["bound"] = bound[0]
    return got


def _mismatches(case, rtol=1e-12):
    got = _run(case)
    bad = []
    for key, want in case["expect"].items():
        if not np.isclose(got[key], want, rtol=rtol, atol=0.0):
            bad.append((key, got[key], want))
    return bad


def test_golden_file_has_every_branch():
    """The file covers both TV branches, a rotated case and two pages."""
    names = {c["name"] for c in CASES}
    assert {"T", "AB", "G2", "R", "P2"} <= names
    for c in CASES:
        e = c["expect"]
        assert set(e) == set(DIAG) | {"bound"}
    tanh_min = [c for c in CASES if c["expect"]["tv"] < c["expect"]["A"] / c["expect"]["B"]]
    ab_min = [c for c in CASES if np.isclose(c["expect"]["tv"], c["expect"]["A"] / c["expect"]["B"],
                                              rtol=1e-12)]
    assert tanh_min and ab_min


@pytest.mark.parametrize("case", CASES, ids=[c["name"] for c in CASES])
def test_bound_terms_match_hand_worked(oracle_lib, case):
    bad = _mismatches(case)
    assert not bad, bad


# ------------------------------------------------- planted mistakes ---------
# (name, text in kvq_oracle.c, replacement).  Each is a plausible misreading of
# the bound's derivation; every replacement must change the source.
MUTANTS = [
    ("delta_without_half", "qs += qn1[g] * ks[g] / 2.0;", "qs += qn1[g] * ks[g];"),
    ("delta_without_kappa", "dl[j] = OC_KAPPA * sc * (qs + rot * smax + qo +",
     "dl[j] = sc * (qs + rot * smax + qo +"),
    ("bound_without_kappa", "double bd = OC_KAPPA * (ekey + Ev);", "double bd = ekey + Ev;"),
    ("ekey_single_eta", "double ekey = tv * (range + 2.0 * eta_max);",
     "double ekey = tv * (range + eta_max);"),
    ("ekey_without_eta", "double ekey = tv * (range + 2.0 * eta_max);",
     "double ekey = tv * range;"),
    ("range_first_group_only", "range = vtop_max[g] - vz_min[g];",
     "range = vtop_max[0] - vz_min[0];"),
    ("range_top_16_steps", "vtop[g] = (double)fmaf(15.0f, (float)vs[g], (float)vz[g]);",
     "vtop[g] = (double)fmaf(16.0f, (float)vs[g], (float)vz[g]);"),
    ("tv_max_not_min", "if (A / B < tv) tv = A / B;", "if (A / B > tv) tv = A / B;"),
    ("tv_tanh_full_delta", "double tv = tanh(dmax / 2.0);", "double tv = tanh(dmax);"),
    ("b_wrong_sign", "B += p * exp(-dl[j]);", "B += p * exp(dl[j]);"),
    ("a_without_minus_one", "A += p * expm1(dl[j]);", "A += p * exp(dl[j]);"),
    ("no_rotation_allowance", "#define OC_ROT_SLACK (1.0 / 65536.0)", "#define OC_ROT_SLACK (0.0)"),
    ("eval_unweighted", "Ev += p * et[j];", "Ev += p * eta_max;"),
    ("delta_l2_not_l1", "qn1[ch / c->kgroup] += fabs((double)qp[ch]);",
     "qn1[ch / c->kgroup] += (double)qp[ch] * (double)qp[ch];"),
]


@pytest.fixture(scope="module")
def mutant_dir(tmp_path_factory):
    return str(tmp_path_factory.mktemp("oracle_mutants"))


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(oracle_lib, mutant_dir, name, old, new):
    src = oracle.source_text()
    assert old in src, f"mutation target of {name} not found in the oracle"
    so = oracle.compile_variant(src.replace(old, new), mutant_dir, name)
    with oracle.library_override(so):
        caught = [c["name"] for c in CASES if _mismatches(c)]
    assert caught, f"no hand-worked case catches the planted mistake {name}"
