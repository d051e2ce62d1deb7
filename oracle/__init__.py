"""CPU oracle for quantized-KV decode attention (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s
``cpu_baseline`` / ``--impl reference`` legs may import this package.  The
product path (the CUDA library and its binding) never imports or links it,
and the two share no code: the oracle is plain C (``kvq_oracle.c``) built
with gcc, fp32 codec arithmetic in a fixed order and fp64 attention.

Every function cites the page passage it follows; see ``kvq_oracle.c``.
Pinned by ``tests/test_oracle_*.py`` against hand-worked cases, closed forms,
library routines (scipy's Hadamard matrix, numpy's float16, torch's fp64
scaled-dot-product attention and float8_e4m3fn cast) and brute force; the bound's magnitude by
hand-worked cases (``tests/golden/bound_hand_worked.txt``).
"""

from __future__ import annotations

import contextlib
import ctypes
import math
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kvq_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "libkvq_oracle.so")

CFLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared", "-std=c11"]


def build(force: bool = False) -> str:
    """Compile the oracle with gcc into oracle/_build/libkvq_oracle.so."""
    os.makedirs(_BUILD, exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_lib: Optional[ctypes.CDLL] = None


def _configure(L: ctypes.CDLL) -> ctypes.CDLL:
    L.oc_f16_value.restype = ctypes.c_double
    L.oc_f16_value.argtypes = [ctypes.c_uint16]
    L.oc_f16_round.restype = ctypes.c_uint16
    L.oc_f16_round.argtypes = [ctypes.c_float, ctypes.c_int]
    L.oc_f16_rn.restype = ctypes.c_uint16
    L.oc_f16_rn.argtypes = [ctypes.c_float]
    L.oc_med3_chunk.restype = ctypes.c_int
    L.oc_block_bytes.restype = ctypes.c_int64
    if hasattr(L, "oq_block_bytes"):
        L.oq_block_bytes.restype = ctypes.c_int64
        for name in ("oq_lloyd_max", "oq_tables", "oq_append", "oq_decode"):
            getattr(L, name).restype = ctypes.c_int
    if hasattr(L, "oh_block_bytes"):
        L.oh_block_bytes.restype = ctypes.c_int64
        L.oh_e4m3_value.restype = ctypes.c_double
        L.oh_e4m3_value.argtypes = [ctypes.c_uint8]
        L.oh_e4m3_rn.restype = ctypes.c_uint8
        L.oh_e4m3_rn.argtypes = [ctypes.c_float]
        for name in ("oh_direction", "oh_append", "oh_decode"):
            getattr(L, name).restype = ctypes.c_int
    for name in ("oc_quantize_sym", "oc_quantize_asym", "oc_append", "oc_decode",
                 "oc_decode_promote_values", "oc_dense", "oc_f16_round_n"):
        getattr(L, name).restype = ctypes.c_int
    return L


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = _configure(ctypes.CDLL(build()))
    return _lib


@contextlib.contextmanager
def library_override(path: str):
    """Route every oracle call through another build of kvq_oracle.c while the
    block runs.  Test hook only: the tests that plant a mistake in a copy of
    the oracle use it to check that the pins catch that mistake."""
    global _lib
    saved = lib()
    _lib = _configure(ctypes.CDLL(os.path.abspath(path)))
    try:
        yield _lib
    finally:
        _lib = saved


def compile_variant(src_text: str, out_dir: str, name: str) -> str:
    """Compile C source text with the oracle's flags into out_dir/name.so."""
    src = os.path.join(out_dir, name + ".c")
    with open(src, "w") as f:
        f.write(src_text)
    so = os.path.join(out_dir, name + ".so")
    subprocess.check_call(["gcc", *CFLAGS, "-o", so, src, "-lm"])
    return so


def source_text() -> str:
    """The oracle's C source (for the planted-mistake tests)."""
    with open(_SRC) as f:
        return f.read()


class OcCfg(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("d", "hkv", "kbits", "kgroup", "krotate", "vbits", "vgroup", "num_pages",
                 "outliers")]


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


PAGE_SIZE = 16
OK, ERR_ARG, ERR_RANGE = 0, -1, -3


# ---------------------------------------------------------------- fp16 ----
def f16_round(x, up: bool) -> np.ndarray:
    """Directed rounding fp32 -> binary16 bits (up: toward +inf, else -inf)."""
    x = _c(x, np.float32).ravel()
    out = np.empty(x.shape, dtype=np.uint16)
    lib().oc_f16_round_n(_p(x), ctypes.c_int64(x.size), int(bool(up)), _p(out))
    return out


def f16_rn(x) -> np.ndarray:
    """Round fp32 to the nearest binary16 (ties to even): bits."""
    x = _c(x, np.float32).ravel()
    return np.array([lib().oc_f16_rn(ctypes.c_float(v)) for v in x], dtype=np.uint16)


def med3_chunk(x) -> int:
    """Med3x outlier chunk of one vector (index of 4-element chunk, or -1)."""
    x = _c(x, np.float32).ravel()
    return int(lib().oc_med3_chunk(_p(x), x.size))


def f16_value(h) -> np.ndarray:
    h = _c(h, np.uint16).ravel()
    out = np.empty(h.shape, dtype=np.float64)
    lib().oc_f16_value_n(_p(h), ctypes.c_int64(h.size), _p(out))
    return out


# ------------------------------------------------------------ rotation ----
def rotate(x, signs) -> np.ndarray:
    """Randomized Walsh-Hadamard rotation of the last axis, fp32, fixed order."""
    x = _c(x, np.float32)
    d = x.shape[-1]
    out = np.empty_like(x)
    lib().oc_rotate_n(_p(x), ctypes.c_int64(x.size // d), d, _p(_c(signs, np.int8)), _p(out))
    return out


# -------------------------------------------------------------- codecs ----
def quantize_sym(x, bits: int):
    """Symmetric group quantizer: returns (rc, scale_bits, codes int8)."""
    x = _c(x, np.float32).ravel()
    codes = np.zeros(x.size, dtype=np.int8)
    sb = np.zeros(1, dtype=np.uint16)
    rc = lib().oc_quantize_sym(_p(x), x.size, 127 if bits == 8 else 7, _p(sb), _p(codes))
    return rc, int(sb[0]), codes


def quantize_asym(x):
    """Asymmetric 4-bit group quantizer: (rc, scale_bits, zero_bits, codes, max_err)."""
    x = _c(x, np.float32).ravel()
    codes = np.zeros(x.size, dtype=np.uint8)
    sb = np.zeros(1, dtype=np.uint16)
    zb = np.zeros(1, dtype=np.uint16)
    e = np.zeros(1, dtype=np.float32)
    rc = lib().oc_quantize_asym(_p(x), x.size, _p(sb), _p(zb), _p(codes), _p(e))
    return rc, int(sb[0]), int(zb[0]), codes, float(e[0])


class Cache:
    """The oracle's own paged Tier-1 cache (same byte format as the library's)."""

    def __init__(self, head_dim, num_kv_heads, num_pages, k_bits=8, k_group=128,
                 k_rotate=False, v_bits=4, v_group=32, rot_signs=None, outliers=False):
        self.cfg = OcCfg(head_dim, num_kv_heads, k_bits, k_group, int(bool(k_rotate)),
                         v_bits, v_group, num_pages, int(bool(outliers)))
        bb = lib().oc_block_bytes(ctypes.byref(self.cfg))
        if bb < 0:
            raise ValueError("unsupported cache configuration")
        self.block_bytes = int(bb)
        self.pool = np.zeros(num_pages * num_kv_heads * self.block_bytes, dtype=np.uint8)
        self.eta = np.zeros((num_pages, num_kv_heads), dtype=np.float32)
        self.signs = None if rot_signs is None else _c(rot_signs, np.int8)

    @property
    def head_dim(self):
        return self.cfg.d

    def append(self, k, v, page_table, start_pos, valid=None):
        """Quantize k, v [num_seqs][Hkv][T][d] (fp32 or bf16 bits) into the pool."""
        k = np.ascontiguousarray(k)
        v = np.ascontiguousarray(v)
        assert k.shape == v.shape and k.dtype == v.dtype and k.ndim == 4
        B, H, T, d = k.shape
        is_f32 = int(k.dtype == np.float32)
        pt = _c(page_table, np.int32)
        sp = _c(start_pos, np.int32)
        vl = None if valid is None else _c(valid, np.int32)
        rc = lib().oc_append(ctypes.byref(self.cfg), _p(self.pool), _p(self.eta), _p(k), _p(v),
                             is_f32, ctypes.c_int64(H * T * d), ctypes.c_int64(T * d),
                             ctypes.c_int64(d), B, T, _p(vl), _p(pt), pt.shape[1], _p(sp),
                             _p(self.signs))
        return rc

    def decode(self, q, page_table, seq_lens, scale=None, tau=math.inf, row_mask=None):
        """Returns (o_hat f64 [rows][d], bound f64 [rows], flags u8 [rows], diag [rows][8])."""
        q = np.ascontiguousarray(q)
        B, NQ, HQ, d = q.shape
        rows = B * NQ * HQ
        scale = default_scale(d) if scale is None else np.float32(scale)
        out = np.zeros((rows, d), dtype=np.float64)
        bound = np.zeros(rows, dtype=np.float64)
        flags = np.zeros(rows, dtype=np.uint8)
        diag = np.zeros((rows, 8), dtype=np.float64)
        pt = _c(page_table, np.int32)
        sl = _c(seq_lens, np.int32)
        rm = None if row_mask is None else _c(row_mask, np.uint8)
        rc = lib().oc_decode(ctypes.byref(self.cfg), _p(self.pool), _p(self.eta), _p(q),
                             int(q.dtype == np.float32), B, NQ, HQ, _p(pt), pt.shape[1], _p(sl),
                             ctypes.c_float(scale), ctypes.c_float(tau), _p(self.signs),
                             _p(out), _p(bound), _p(flags), _p(diag), _p(rm))
        if rc != OK:
            raise ValueError(f"oracle decode failed: {rc}")
        return out, bound, flags, diag


    def decode_promote_values(self, q, page_table, seq_lens, v_orig, v_tol, scale=None,
                              tau=math.inf, row_mask=None):
        """Decode with rung 2 of the fallback ladder: blocks whose estimated share of
        E_val (mass x eta) exceeds v_tol take the original values v_orig
        [num_seqs][Hkv][T][d] (fp32, or bf16 bits as uint16).  Returns
        (o f64 [rows][d], bound f64 [rows], flags u8 [rows], promoted blocks i32
        [rows], diag [rows][8] with E_val of the blocks not promoted)."""
        q = np.ascontiguousarray(q)
        v_orig = np.ascontiguousarray(v_orig)
        B, NQ, HQ, d = q.shape
        _, H, T, dv = v_orig.shape
        assert dv == d and H == self.cfg.hkv
        rows = B * NQ * HQ
        scale = default_scale(d) if scale is None else np.float32(scale)
        out = np.zeros((rows, d), dtype=np.float64)
        bound = np.zeros(rows, dtype=np.float64)
        flags = np.zeros(rows, dtype=np.uint8)
        promoted = np.zeros(rows, dtype=np.int32)
        diag = np.zeros((rows, 8), dtype=np.float64)
        pt = _c(page_table, np.int32)
        sl = _c(seq_lens, np.int32)
        rm = None if row_mask is None else _c(row_mask, np.uint8)
        rc = lib().oc_decode_promote_values(
            ctypes.byref(self.cfg), _p(self.pool), _p(self.eta), _p(q),
            int(q.dtype == np.float32), B, NQ, HQ, _p(pt), pt.shape[1], _p(sl),
            ctypes.c_float(scale), ctypes.c_float(tau), _p(self.signs), _p(v_orig),
            int(v_orig.dtype == np.float32), ctypes.c_int64(H * T * d), ctypes.c_int64(T * d),
            ctypes.c_int64(d), ctypes.c_double(v_tol), _p(out), _p(bound), _p(flags),
            _p(promoted), _p(diag), _p(rm))
        if rc != OK:
            raise ValueError(f"oracle promoted decode failed: {rc}")
        return out, bound, flags, promoted, diag

    def decode_adaptive(self, q, page_table, seq_lens, k_orig, v_orig, tau_cov, v_tol=math.inf,
                        rank_tol=0.0, scale=None, tau=math.inf, row_mask=None):
        """Adaptive precision ("Runtime-Certified...", Methodology 3): per row the
        top-K* blocks covering tau_cov of the estimated mass take the original
        keys, blocks whose estimated mass x eta exceeds v_tol take the original values,
        and the ranking-consistency check over the key-promoted blocks (log-mass
        slack rank_tol) flags the row when it fails.  k_orig, v_orig
        [num_seqs][Hkv][T][d] (fp32, or bf16 bits as uint16).  Returns a dict:
        out f64 [rows][d], bound, flags, kprom/vprom u8 [rows][max_pages], nkey,
        nval, rank_fail per row, diag [rows][8]."""
        q = np.ascontiguousarray(q)
        k_orig = np.ascontiguousarray(k_orig)
        v_orig = np.ascontiguousarray(v_orig)
        assert k_orig.shape == v_orig.shape and k_orig.dtype == v_orig.dtype
        B, NQ, HQ, d = q.shape
        _, H, T, dv = v_orig.shape
        assert dv == d and H == self.cfg.hkv
        rows = B * NQ * HQ
        pt = _c(page_table, np.int32)
        mp = pt.shape[1]
        scale = default_scale(d) if scale is None else np.float32(scale)
        r = dict(out=np.zeros((rows, d)), bound=np.zeros(rows), flags=np.zeros(rows, np.uint8),
                 kprom=np.zeros((rows, mp), np.uint8), vprom=np.zeros((rows, mp), np.uint8),
                 nkey=np.zeros(rows, np.int32), nval=np.zeros(rows, np.int32),
                 rank_fail=np.zeros(rows, np.uint8), diag=np.zeros((rows, 8)))
        sl = _c(seq_lens, np.int32)
        rm = None if row_mask is None else _c(row_mask, np.uint8)
        rc = lib().oc_decode_adaptive(
            ctypes.byref(self.cfg), _p(self.pool), _p(self.eta), _p(q),
            int(q.dtype == np.float32), B, NQ, HQ, _p(pt), mp, _p(sl), ctypes.c_float(scale),
            ctypes.c_float(tau), _p(self.signs), _p(k_orig), _p(v_orig),
            int(v_orig.dtype == np.float32), ctypes.c_int64(H * T * d), ctypes.c_int64(T * d),
            ctypes.c_int64(d), ctypes.c_double(tau_cov), ctypes.c_double(v_tol),
            ctypes.c_double(rank_tol), _p(r["out"]), _p(r["bound"]), _p(r["flags"]),
            _p(r["kprom"]), _p(r["vprom"]), _p(r["nkey"]), _p(r["nval"]), _p(r["rank_fail"]),
            _p(r["diag"]), _p(rm))
        if rc != OK:
            raise ValueError(f"oracle adaptive decode failed: {rc}")
        return r

    def decode_terms(self, q, page_table, n, b, i, h, scale=None):
        """Per-token (z_hat, Delta) of one query row over the first n tokens."""
        q = np.ascontiguousarray(q)
        B, NQ, HQ, d = q.shape
        scale = default_scale(d) if scale is None else np.float32(scale)
        z = np.zeros(n, dtype=np.float64)
        dl = np.zeros(n, dtype=np.float64)
        pt = _c(page_table, np.int32)
        rc = lib().oc_decode_terms(ctypes.byref(self.cfg), _p(self.pool), _p(self.eta), _p(q),
                                   int(q.dtype == np.float32), NQ, HQ, b, i, h, _p(pt),
                                   pt.shape[1], n, ctypes.c_float(scale), _p(self.signs),
                                   _p(z), _p(dl))
        if rc != OK:
            raise ValueError(f"oracle decode_terms failed: {rc}")
        return z, dl


def default_scale(d: int) -> np.float32:
    """Scaled-dot-product default 1/sqrt(d), as the fp32 value the path receives."""
    return np.float32(1.0 / math.sqrt(d))


def dense(q, k, v, seq_lens, scale=None, row_mask=None) -> np.ndarray:
    """Exact fp64 attention over originals k, v [num_seqs][Hkv][T][d]."""
    q = np.ascontiguousarray(q)
    k = np.ascontiguousarray(k)
    v = np.ascontiguousarray(v)
    B, NQ, HQ, d = q.shape
    _, H, T, _ = k.shape
    scale = default_scale(d) if scale is None else np.float32(scale)
    out = np.zeros((B * NQ * HQ, d), dtype=np.float64)
    sl = _c(seq_lens, np.int32)
    rm = None if row_mask is None else _c(row_mask, np.uint8)
    rc = lib().oc_dense(_p(q), int(q.dtype == np.float32), _p(k), _p(v),
                        int(k.dtype == np.float32), ctypes.c_int64(H * T * d),
                        ctypes.c_int64(T * d), ctypes.c_int64(d), B, NQ, HQ, H, d, _p(sl),
                        ctypes.c_float(scale), _p(out), _p(rm))
    if rc != OK:
        raise ValueError(f"oracle dense failed: {rc}")
    return out


def certified(o_hat, o_dense, flags) -> np.ndarray:
    """Final output: exact dense attention for flagged rows, else o_hat."""
    return np.where(np.asarray(flags, bool)[:, None], o_dense, o_hat)


# ------------------------------------------------------------------ KQV ----
class OqCfg(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("d", "hkv", "num_pages")]


KQV_KBITS, KQV_VBITS = 4, 3


def lloyd_max(bits):
    """Lloyd-Max centroids of N(0, 1) with 2^bits levels (fp64, ascending)."""
    c = np.zeros(1 << bits, dtype=np.float64)
    it = lib().oq_lloyd_max(bits, _p(c))
    if it < 0:
        raise ValueError("bad bit count")
    return c


def kqv_tables(bits, d):
    """(centroids, thresholds) fp32 for unit vectors in dimension d."""
    cent = np.zeros(1 << bits, dtype=np.float32)
    thr = np.zeros((1 << bits) - 1, dtype=np.float32)
    if lib().oq_tables(bits, d, _p(cent), _p(thr)) != OK:
        raise ValueError("bad bit count")
    return cent, thr


def qjl(r, S):
    """The QJL sketch bits (packed, d/8 bytes) of r and sum_i S_ic b_i."""
    r = _c(r, np.float32)
    S = _c(S, np.float32)
    d = r.size
    bits = np.zeros(d // 8, dtype=np.uint8)
    rsum = np.zeros(d, dtype=np.float32)
    lib().oq_qjl(_p(r), _p(S), d, _p(bits), _p(rsum))
    return bits, rsum


class KqvCache:
    """The oracle's paged cache of the KQV codec ("Statistical Inference and
    Quality Measures of KV Cache Quantisations Inspired by TurboQuant",
    Quantisation schemes: KQV): rotated K in 4-bit Lloyd-Max codes, rotated V
    in 3-bit codes plus the 1-bit QJL sketch of the residual."""

    def __init__(self, head_dim, num_kv_heads, num_pages, rot_signs, qjl_matrix):
        self.cfg = OqCfg(head_dim, num_kv_heads, num_pages)
        bb = lib().oq_block_bytes(ctypes.byref(self.cfg))
        if bb < 0:
            raise ValueError("unsupported cache configuration")
        self.block_bytes = int(bb)
        self.pool = np.zeros(num_pages * num_kv_heads * self.block_bytes, dtype=np.uint8)
        self.eta = np.zeros((num_pages, num_kv_heads), dtype=np.float32)
        self.signs = _c(rot_signs, np.int8)
        self.S = _c(qjl_matrix, np.float32)
        assert self.S.shape == (head_dim, head_dim)

    def append(self, k, v, page_table, start_pos, valid=None):
        k = np.ascontiguousarray(k)
        v = np.ascontiguousarray(v)
        assert k.shape == v.shape and k.dtype == v.dtype and k.ndim == 4
        B, H, T, d = k.shape
        pt = _c(page_table, np.int32)
        sp = _c(start_pos, np.int32)
        vl = None if valid is None else _c(valid, np.int32)
        return lib().oq_append(ctypes.byref(self.cfg), _p(self.pool), _p(self.eta), _p(k),
                               _p(v), int(k.dtype == np.float32), ctypes.c_int64(H * T * d),
                               ctypes.c_int64(T * d), ctypes.c_int64(d), B, T, _p(vl), _p(pt),
                               pt.shape[1], _p(sp), _p(self.signs), _p(self.S))

    def decode(self, q, page_table, seq_lens, scale=None, tau=math.inf, row_mask=None):
        """Returns (o_hat f64 [rows][d], bound f64 [rows], flags u8 [rows], diag [rows][8])."""
        q = np.ascontiguousarray(q)
        B, NQ, HQ, d = q.shape
        rows = B * NQ * HQ
        scale = default_scale(d) if scale is None else np.float32(scale)
        out = np.zeros((rows, d), dtype=np.float64)
        bound = np.zeros(rows, dtype=np.float64)
        flags = np.zeros(rows, dtype=np.uint8)
        diag = np.zeros((rows, 8), dtype=np.float64)
        pt = _c(page_table, np.int32)
        sl = _c(seq_lens, np.int32)
        rm = None if row_mask is None else _c(row_mask, np.uint8)
        rc = lib().oq_decode(ctypes.byref(self.cfg), _p(self.pool), _p(self.eta), _p(q),
                             int(q.dtype == np.float32), B, NQ, HQ, _p(pt), pt.shape[1], _p(sl),
                             ctypes.c_float(scale), ctypes.c_float(tau), _p(self.signs),
                             _p(self.S), _p(out), _p(bound), _p(flags), _p(diag), _p(rm))
        if rc != OK:
            raise ValueError(f"oracle decode failed: {rc}")
        return out, bound, flags, diag


class OhCfg(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("d", "hkv", "num_pages", "S", "outliers")]


def hq_primary(p: int) -> np.ndarray:
    """Unit p of the binary tetrahedral group 2T, in the oracle's order."""
    out = np.zeros(4, dtype=np.float32)
    lib().oh_primary(int(p), _p(out))
    return out


def hq_codeword(sec, i: int) -> np.ndarray:
    """Codeword i = 24 s + p (the fp32 product q_p q_s) of a secondary set [S][4]."""
    sec = _c(sec, np.float32)
    out = np.zeros(4, dtype=np.float32)
    lib().oh_codeword(_p(sec), int(i), _p(out))
    return out


def hq_codeword16(sec, i: int) -> np.ndarray:
    """Codeword i rounded to fp16 per component (the one the reconstruction uses)."""
    sec = _c(sec, np.float32)
    out = np.zeros(4, dtype=np.float32)
    lib().oh_codeword16(_p(sec), int(i), _p(out))
    return out


def hq_direction(x, sec) -> int:
    """The direction code of one 4-channel chunk x against a secondary set [S][4]."""
    x = _c(x, np.float32)
    sec = _c(sec, np.float32)
    return int(lib().oh_direction(_p(x), _p(sec), int(sec.shape[0])))


def e4m3_value(code: int) -> float:
    return float(lib().oh_e4m3_value(int(code)))


def e4m3_rn(x) -> int:
    return int(lib().oh_e4m3_rn(ctypes.c_float(float(x))))


class HqCache:
    """The oracle's paged cache of the HQMQ codec ("Hurwitz Quaternion
    Multiplicative Quantization for KV Cache Compression", Method 1-2): every
    4-channel chunk of K and V coded by its radius (fp8 E4M3) and the index of
    the nearest product codeword q_p q_s (q_p in 2T, q_s from the secondary
    set of its kv head and role); with outliers, the Med3x chunk of K and of V
    kept in fp16 (Method 3)."""

    def __init__(self, head_dim, num_kv_heads, num_pages, secondary, outliers=False):
        sec = _c(secondary, np.float32)
        assert sec.ndim == 4 and sec.shape[0] == num_kv_heads and sec.shape[1] == 2 \
            and sec.shape[3] == 4
        self.cfg = OhCfg(head_dim, num_kv_heads, num_pages, sec.shape[2], int(bool(outliers)))
        bb = lib().oh_block_bytes(ctypes.byref(self.cfg))
        if bb < 0:
            raise ValueError("unsupported cache configuration")
        self.block_bytes = int(bb)
        self.pool = np.zeros(num_pages * num_kv_heads * self.block_bytes, dtype=np.uint8)
        self.eta = np.zeros((num_pages, num_kv_heads), dtype=np.float32)
        self.sec = sec

    def append(self, k, v, page_table, start_pos, valid=None):
        k = np.ascontiguousarray(k)
        v = np.ascontiguousarray(v)
        assert k.shape == v.shape and k.dtype == v.dtype and k.ndim == 4
        B, H, T, d = k.shape
        pt = _c(page_table, np.int32)
        sp = _c(start_pos, np.int32)
        vl = None if valid is None else _c(valid, np.int32)
        return lib().oh_append(ctypes.byref(self.cfg), _p(self.pool), _p(self.eta), _p(k),
                               _p(v), int(k.dtype == np.float32), ctypes.c_int64(H * T * d),
                               ctypes.c_int64(T * d), ctypes.c_int64(d), B, T, _p(vl), _p(pt),
                               pt.shape[1], _p(sp), _p(self.sec))

    def read_token(self, page: int, kv_head: int, slot: int):
        """(k^, v^) fp32 [d] of one slot, as the append reconstructed them."""
        d = self.cfg.d
        blk = self.pool[(page * self.cfg.hkv + kv_head) * self.block_bytes:][:self.block_bytes]
        kh = np.zeros(d, dtype=np.float32)
        vh = np.zeros(d, dtype=np.float32)
        lib().oh_read_token(ctypes.byref(self.cfg), _p(np.ascontiguousarray(blk)), int(slot),
                            _p(np.ascontiguousarray(self.sec[kv_head])), _p(kh), _p(vh))
        return kh, vh

    def decode(self, q, page_table, seq_lens, scale=None, tau=math.inf, row_mask=None):
        """Returns (o_hat f64 [rows][d], bound f64 [rows], flags u8 [rows], diag [rows][8])."""
        q = np.ascontiguousarray(q)
        B, NQ, HQ, d = q.shape
        rows = B * NQ * HQ
        scale = default_scale(d) if scale is None else np.float32(scale)
        out = np.zeros((rows, d), dtype=np.float64)
        bound = np.zeros(rows, dtype=np.float64)
        flags = np.zeros(rows, dtype=np.uint8)
        diag = np.zeros((rows, 8), dtype=np.float64)
        pt = _c(page_table, np.int32)
        sl = _c(seq_lens, np.int32)
        rm = None if row_mask is None else _c(row_mask, np.uint8)
        rc = lib().oh_decode(ctypes.byref(self.cfg), _p(self.pool), _p(self.eta), _p(q),
                             int(q.dtype == np.float32), B, NQ, HQ, _p(pt), pt.shape[1], _p(sl),
                             ctypes.c_float(scale), ctypes.c_float(tau), _p(self.sec), _p(out),
                             _p(bound), _p(flags), _p(diag), _p(rm))
        if rc != OK:
            raise ValueError(f"oracle decode failed: {rc}")
        return out, bound, flags, diag
