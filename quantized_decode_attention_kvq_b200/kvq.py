"""Thin ctypes binding of libkvq.so (include/kvq.h).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  PyTorch supplies device memory and streams.  Importing this module
loads the library and raises if it is missing -- there is no fallback.

Functions keep the C names (``kvq_decode_attention`` ...) and accept torch
tensors (their data pointers are passed), ints (raw pointers) or None.
``PagedCache`` owns the device buffers of one quantized cache.
"""

from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkvq.so")

KVQ_OK = 0
KVQ_ERR_INVALID_ARG = -1
KVQ_ERR_UNSUPPORTED = -2
KVQ_ERR_RANGE = -3
KVQ_ERR_CUDA = -4
KVQ_ERR_TIMEOUT = -5
KVQ_ERR_DEVICE = -6
KVQ_F32 = 0
KVQ_BF16 = 1
KVQ_CODEC_INT = 0
KVQ_CODEC_KQV = 1
KVQ_CODEC_HQMQ = 2
KVQ_HQMQ_MAX_S = 64
PAGE_SIZE = 16

EXPORTED = ("kvq_block_bytes", "kvq_pool_bytes", "kvq_quantize_append", "kvq_workspace_size",
            "kvq_decode_attention", "kvq_error_bound", "kvq_fallback_staging_size",
            "kvq_fallback_exact", "kvq_device_error", "kvq_status_string", "kvq_last_error",
            "kvq_decode_attention_noalloc", "kvq_decode_attention_append",
            "kvq_adaptive_work_size", "kvq_adaptive_host_size", "kvq_adaptive_staging_size",
            "kvq_adaptive_precision", "kvq_kqv_codebook")


class KvqError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}: {last_error()}")


class kvq_cache(ctypes.Structure):
    _fields_ = [("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("page_size", ctypes.c_int32), ("num_pages", ctypes.c_int32),
                ("k_bits", ctypes.c_int32), ("k_group", ctypes.c_int32),
                ("k_rotate", ctypes.c_int32), ("v_bits", ctypes.c_int32),
                ("v_group", ctypes.c_int32), ("pool", ctypes.c_void_p),
                ("v_eta", ctypes.c_void_p), ("rot_signs", ctypes.c_void_p),
                ("error_word", ctypes.c_void_p), ("outliers", ctypes.c_int32),
                ("codec", ctypes.c_int32), ("qjl", ctypes.c_void_p),
                ("hq_sec", ctypes.c_void_p), ("hq_s", ctypes.c_int32)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libkvq.so not built ({LIB_PATH}); run "
                          "python -m quantized_decode_attention_kvq_b200.build")
    L = ctypes.CDLL(LIB_PATH)
    P, I32, I64, SZ, F = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t,
                          ctypes.c_float)
    C = ctypes.POINTER(kvq_cache)
    sig = {
        "kvq_block_bytes": (SZ, [C]),
        "kvq_pool_bytes": (SZ, [C]),
        "kvq_quantize_append": (ctypes.c_int, [C, P, P, ctypes.c_int, I64, I64, I64, I32, I32,
                                               P, P, P, I32, P]),
        "kvq_workspace_size": (SZ, [C, I32, I32, I32, I32]),
        "kvq_decode_attention": (ctypes.c_int, [C, P, ctypes.c_int, I32, I32, I32, P, I32, P, F,
                                                F, P, P, P, P, SZ, P]),
        "kvq_error_bound": (ctypes.c_int, [C, P, ctypes.c_int, I32, I32, I32, P, I32, P, F, F,
                                           P, P, P, SZ, P]),
        "kvq_fallback_staging_size": (SZ, [C, ctypes.c_int, I32]),
        "kvq_fallback_exact": (ctypes.c_int, [C, P, P, ctypes.c_int, I64, I64, P, ctypes.c_int,
                                              I32, I32, I32, P, F, P, P, P, P, SZ, P, P, I32,
                                              ctypes.POINTER(I32)]),
        "kvq_device_error": (ctypes.c_int, [C, P, ctypes.POINTER(I32)]),
        "kvq_decode_attention_noalloc": (ctypes.c_int, [C, P, ctypes.c_int, I32, I32, I32, P,
                                                        I32, P, F, F, P, P, P, P]),
        "kvq_decode_attention_append": (ctypes.c_int, [C, P, P, ctypes.c_int, I64, I64, P,
                                                       ctypes.c_int, I32, I32, I32, P, I32, P, F,
                                                       F, P, P, P, P, SZ, P]),
        "kvq_adaptive_work_size": (SZ, [C, I32, I32, I32, I32]),
        "kvq_adaptive_host_size": (SZ, [C, I32, I32]),
        "kvq_adaptive_staging_size": (SZ, [C, ctypes.c_int, I32]),
        "kvq_adaptive_precision": (ctypes.c_int, [C, P, P, ctypes.c_int, I64, I64, P,
                                                  ctypes.c_int, I32, I32, I32, P, I32, P, P, F,
                                                  F, F, F, F, P, P, P, P, P, P, P, SZ, P, SZ, P,
                                                  SZ, P, P, I32, ctypes.POINTER(I32),
                                                  ctypes.POINTER(I32)]),
        "kvq_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "kvq_kqv_codebook": (ctypes.c_int, [I32, I32, P, P]),
        "kvq_last_error": (ctypes.c_char_p, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    return L


_lib = _load()


def lib() -> ctypes.CDLL:
    return _lib


def status_string(s: int) -> str:
    return _lib.kvq_status_string(s).decode()


def last_error() -> str:
    return _lib.kvq_last_error().decode()


def _ptr(x) -> Optional[int]:
    if x is None:
        return None
    if isinstance(x, torch.Tensor):
        return x.data_ptr() if x.numel() else None
    return int(x)


def _stream(s) -> Optional[int]:
    if s is None:
        # the caller's current torch stream; the legacy default stream without CUDA
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else 0
    if isinstance(s, torch.cuda.Stream):
        return s.cuda_stream
    return int(s)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return KVQ_F32
    if t.dtype == torch.bfloat16:
        return KVQ_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _check(rc: int, where: str) -> int:
    if rc != KVQ_OK:
        raise KvqError(rc, where)
    return rc


# ---- the C entry points (same names, same argument order) ---------------------------
def kvq_block_bytes(cache: kvq_cache) -> int:
    return _lib.kvq_block_bytes(ctypes.byref(cache))


def kvq_pool_bytes(cache: kvq_cache) -> int:
    return _lib.kvq_pool_bytes(ctypes.byref(cache))


def kvq_quantize_append(cache, k, v, in_dtype, seq_stride, head_stride, token_stride, num_seqs,
                        num_tokens, valid_tokens, start_pos, page_table, max_pages_per_seq,
                        stream=None) -> int:
    return _lib.kvq_quantize_append(ctypes.byref(cache), _ptr(k), _ptr(v), in_dtype, seq_stride,
                                    head_stride, token_stride, num_seqs, num_tokens,
                                    _ptr(valid_tokens), _ptr(start_pos), _ptr(page_table),
                                    max_pages_per_seq, _stream(stream))


def kvq_workspace_size(cache, num_seqs, num_queries, num_q_heads, max_pages_per_seq) -> int:
    return _lib.kvq_workspace_size(ctypes.byref(cache), num_seqs, num_queries, num_q_heads,
                                   max_pages_per_seq)


def kvq_decode_attention(cache, q, q_dtype, num_seqs, num_queries, num_q_heads, page_table,
                         max_pages_per_seq, seq_lens, softmax_scale, tau, out, bound, flags,
                         workspace, workspace_bytes, stream=None) -> int:
    return _lib.kvq_decode_attention(ctypes.byref(cache), _ptr(q), q_dtype, num_seqs,
                                     num_queries, num_q_heads, _ptr(page_table),
                                     max_pages_per_seq, _ptr(seq_lens), softmax_scale, tau,
                                     _ptr(out), _ptr(bound), _ptr(flags), _ptr(workspace),
                                     workspace_bytes, _stream(stream))


def kvq_error_bound(cache, q, q_dtype, num_seqs, num_queries, num_q_heads, page_table,
                    max_pages_per_seq, seq_lens, softmax_scale, tau, bound, flags, workspace,
                    workspace_bytes, stream=None) -> int:
    return _lib.kvq_error_bound(ctypes.byref(cache), _ptr(q), q_dtype, num_seqs, num_queries,
                                num_q_heads, _ptr(page_table), max_pages_per_seq,
                                _ptr(seq_lens), softmax_scale, tau, _ptr(bound), _ptr(flags),
                                _ptr(workspace), workspace_bytes, _stream(stream))


def kvq_decode_attention_noalloc(cache, q, q_dtype, num_seqs, num_queries, num_q_heads,
                                 page_table, max_pages_per_seq, seq_lens, softmax_scale, tau, out,
                                 bound, flags, stream=None) -> int:
    """kvq_decode_attention with the library's static device scratch instead of a
    caller workspace (for callers that cannot allocate device memory)."""
    return _lib.kvq_decode_attention_noalloc(ctypes.byref(cache), _ptr(q), q_dtype, num_seqs,
                                             num_queries, num_q_heads, _ptr(page_table),
                                             max_pages_per_seq, _ptr(seq_lens), softmax_scale,
                                             tau, _ptr(out), _ptr(bound), _ptr(flags),
                                             _stream(stream))


NOALLOC_SCRATCH_BYTES = 16 * 1024 * 1024


def kvq_decode_attention_append(cache, k_new, v_new, in_dtype, new_seq_stride, new_head_stride,
                                q, q_dtype, num_seqs, num_queries, num_q_heads, page_table,
                                max_pages_per_seq, seq_lens, softmax_scale, tau, out, bound,
                                flags, workspace, workspace_bytes, stream=None) -> int:
    """One decode step in one launch: the new token of every sequence is appended
    at position seq_lens - 1, then the decode runs over seq_lens tokens."""
    return _lib.kvq_decode_attention_append(ctypes.byref(cache), _ptr(k_new), _ptr(v_new),
                                            in_dtype, new_seq_stride, new_head_stride, _ptr(q),
                                            q_dtype, num_seqs, num_queries, num_q_heads,
                                            _ptr(page_table), max_pages_per_seq, _ptr(seq_lens),
                                            softmax_scale, tau, _ptr(out), _ptr(bound),
                                            _ptr(flags), _ptr(workspace), workspace_bytes,
                                            _stream(stream))


def kvq_fallback_staging_size(cache, orig_dtype, max_ctx) -> int:
    return _lib.kvq_fallback_staging_size(ctypes.byref(cache), orig_dtype, max_ctx)


def kvq_fallback_exact(cache, k_orig_host, v_orig_host, orig_dtype, orig_seq_stride,
                       orig_head_stride, q, q_dtype, num_seqs, num_queries, num_q_heads,
                       seq_lens_host, softmax_scale, flags, flags_host, out, staging,
                       staging_bytes, main_stream=None, side_stream=None, timeout_ms=10000):
    """Returns (status, number of recomputed queries)."""
    nfb = ctypes.c_int32(0)
    rc = _lib.kvq_fallback_exact(ctypes.byref(cache), _ptr(k_orig_host), _ptr(v_orig_host),
                                 orig_dtype, orig_seq_stride, orig_head_stride, _ptr(q), q_dtype,
                                 num_seqs, num_queries, num_q_heads, _ptr(seq_lens_host),
                                 softmax_scale, _ptr(flags), _ptr(flags_host), _ptr(out),
                                 _ptr(staging), staging_bytes, _stream(main_stream),
                                 _stream(side_stream), timeout_ms, ctypes.byref(nfb))
    return rc, nfb.value


def kvq_adaptive_work_size(cache, num_seqs, num_queries, num_q_heads, max_pages_per_seq) -> int:
    return _lib.kvq_adaptive_work_size(ctypes.byref(cache), num_seqs, num_queries, num_q_heads,
                                       max_pages_per_seq)


def kvq_adaptive_host_size(cache, num_seqs, max_pages_per_seq) -> int:
    return _lib.kvq_adaptive_host_size(ctypes.byref(cache), num_seqs, max_pages_per_seq)


def kvq_adaptive_staging_size(cache, orig_dtype, max_pages_per_seq) -> int:
    return _lib.kvq_adaptive_staging_size(ctypes.byref(cache), orig_dtype, max_pages_per_seq)


def kvq_adaptive_precision(cache, k_orig_host, v_orig_host, orig_dtype, orig_seq_stride,
                           orig_head_stride, q, q_dtype, num_seqs, num_queries, num_q_heads,
                           page_table, max_pages_per_seq, seq_lens, seq_lens_host, softmax_scale,
                           tau, tau_cov, v_tol, rank_tol, flags, flags_host, out, bound,
                           promoted_keys, promoted_values, work, work_bytes, host_work,
                           host_work_bytes, staging, staging_bytes, main_stream=None,
                           side_stream=None, timeout_ms=10000):
    """Returns (status, rows that ran through the ladder, rows flagged afterwards)."""
    nr, nf = ctypes.c_int32(0), ctypes.c_int32(0)
    rc = _lib.kvq_adaptive_precision(
        ctypes.byref(cache), _ptr(k_orig_host), _ptr(v_orig_host), orig_dtype, orig_seq_stride,
        orig_head_stride, _ptr(q), q_dtype, num_seqs, num_queries, num_q_heads, _ptr(page_table),
        max_pages_per_seq, _ptr(seq_lens), _ptr(seq_lens_host), softmax_scale, tau, tau_cov,
        v_tol, rank_tol, _ptr(flags), _ptr(flags_host), _ptr(out), _ptr(bound),
        _ptr(promoted_keys), _ptr(promoted_values), _ptr(work), work_bytes, _ptr(host_work),
        host_work_bytes, _ptr(staging), staging_bytes, _stream(main_stream), _stream(side_stream),
        timeout_ms, ctypes.byref(nr), ctypes.byref(nf))
    return rc, nr.value, nf.value


def kvq_device_error(cache, stream=None):
    code = ctypes.c_int32(0)
    rc = _lib.kvq_device_error(ctypes.byref(cache), _stream(stream), ctypes.byref(code))
    return rc, code.value


# ---- buffer ownership helper ---------------------------------------------------------
class PagedCache:
    """Device buffers of one quantized paged cache plus its kvq_cache descriptor."""

    def __init__(self, num_kv_heads: int, head_dim: int, num_pages: int, k_bits: int = 8,
                 k_group: int = 128, k_rotate: bool = False, rot_signs=None, v_bits: int = 4,
                 v_group: int = 32, outliers: bool = False, codec: str = "int", qjl_matrix=None,
                 hq_secondary=None, device="cuda"):
        """codec "int": the Tier-1 INT8/INT4 codec (k_bits, k_group, k_rotate,
        outliers apply); codec "kqv": the KQV codec (rotation with rot_signs, 4-bit
        Lloyd-Max keys, 3-bit values plus the QJL sketch with qjl_matrix [d][d]);
        codec "hqmq": the HQMQ codec (4-channel chunks as quaternions, the product
        codebook of 2T and the secondary units hq_secondary [Hkv][2][S][4])."""
        codes = {"int": KVQ_CODEC_INT, "kqv": KVQ_CODEC_KQV, "hqmq": KVQ_CODEC_HQMQ}
        if codec not in codes:
            raise ValueError(f"unknown codec {codec!r}")
        if codec == "kqv":
            k_bits, v_bits, k_group, v_group, k_rotate = 4, 3, head_dim, head_dim, True
        hq_s = 0
        if codec == "hqmq":   # outliers: Med3x over the HQMQ codec
            k_bits, v_bits, k_group, v_group, k_rotate = 6, 6, 4, 4, False
            hq_s = int(np.asarray(hq_secondary).shape[2])   # S secondary units per (head, role)
        self.desc = kvq_cache(num_kv_heads, head_dim, PAGE_SIZE, num_pages, k_bits, k_group,
                              int(bool(k_rotate)), v_bits, v_group, None, None, None, None,
                              int(bool(outliers)), codes[codec], None, None, hq_s)
        bb = kvq_block_bytes(self.desc)
        if bb == 0:
            raise KvqError(KVQ_ERR_UNSUPPORTED, "kvq_block_bytes")
        self.block_bytes = bb
        self.pool = torch.zeros(max(1, num_pages * num_kv_heads * bb), dtype=torch.uint8,
                                device=device)
        self.eta = torch.zeros((max(1, num_pages), num_kv_heads), dtype=torch.float32,
                               device=device)
        self.error_word = torch.zeros(1, dtype=torch.int32, device=device)
        self.signs = None
        if k_rotate:
            self.signs = torch.as_tensor(rot_signs, dtype=torch.int8).to(device)
        self.desc.pool = self.pool.data_ptr()
        self.desc.v_eta = self.eta.data_ptr()
        self.desc.rot_signs = None if self.signs is None else self.signs.data_ptr()
        self.desc.error_word = self.error_word.data_ptr()
        self.qjl = None
        if codec == "kqv":
            self.qjl = torch.as_tensor(qjl_matrix, dtype=torch.float32).to(device).contiguous()
            self.desc.qjl = self.qjl.data_ptr()
        self.hq_sec = None
        if codec == "hqmq":
            self.hq_sec = torch.as_tensor(np.asarray(hq_secondary, np.float32)).to(device).contiguous()
            assert tuple(self.hq_sec.shape) == (num_kv_heads, 2, hq_s, 4)
            self.desc.hq_sec = self.hq_sec.data_ptr()

    @property
    def head_dim(self) -> int:
        return self.desc.head_dim

    @property
    def num_kv_heads(self) -> int:
        return self.desc.num_kv_heads

    def append(self, k: torch.Tensor, v: torch.Tensor, page_table: torch.Tensor,
               start_pos: torch.Tensor, valid_tokens: Optional[torch.Tensor] = None,
               stream=None):
        """k, v: [num_seqs][Hkv][T][d] (fp32 or bf16) device tensors (any strides with
        contiguous channels)."""
        assert k.shape == v.shape and k.dtype == v.dtype and k.stride() == v.stride()
        assert k.stride(3) == 1
        S, H, T, d = k.shape
        _check(kvq_quantize_append(self.desc, k, v, _dtype_code(k), k.stride(0), k.stride(1),
                                   k.stride(2), S, T, valid_tokens, start_pos, page_table,
                                   page_table.shape[1], stream), "kvq_quantize_append")

    def workspace(self, num_seqs, num_queries, num_q_heads, max_pages_per_seq, device="cuda"):
        n = kvq_workspace_size(self.desc, num_seqs, num_queries, num_q_heads, max_pages_per_seq)
        if n == 0:
            raise KvqError(KVQ_ERR_INVALID_ARG, "kvq_workspace_size")
        return torch.zeros(n, dtype=torch.uint8, device=device)

    def decode(self, q: torch.Tensor, page_table: torch.Tensor, seq_lens: torch.Tensor,
               workspace: torch.Tensor, tau: float = math.inf, softmax_scale: float = 0.0,
               out=None, bound=None, flags=None, stream=None, bound_only=False):
        """q: [num_seqs][num_queries][Hq][d] device tensor.  Returns (out, bound, flags)."""
        S, NQ, HQ, d = q.shape
        dev = q.device
        if out is None and not bound_only:
            out = torch.empty((S, NQ, HQ, d), dtype=torch.float32, device=dev)
        if bound is None:
            bound = torch.empty((S, NQ, HQ), dtype=torch.float32, device=dev)
        if flags is None:
            flags = torch.empty((S, NQ, HQ), dtype=torch.uint8, device=dev)
        if bound_only:
            rc = kvq_error_bound(self.desc, q, _dtype_code(q), S, NQ, HQ, page_table,
                                 page_table.shape[1], seq_lens, softmax_scale, tau, bound, flags,
                                 workspace, workspace.numel(), stream)
            _check(rc, "kvq_error_bound")
        else:
            rc = kvq_decode_attention(self.desc, q, _dtype_code(q), S, NQ, HQ, page_table,
                                      page_table.shape[1], seq_lens, softmax_scale, tau, out,
                                      bound, flags, workspace, workspace.numel(), stream)
            _check(rc, "kvq_decode_attention")
        return out, bound, flags

    def device_error(self, stream=None) -> int:
        rc, code = kvq_device_error(self.desc, stream)
        _check(rc, "kvq_device_error")
        return code


def kqv_codebook(bits: int, head_dim: int):
    """The KQV codec's fp32 centroids and thresholds (kvq_kqv_codebook)."""
    import numpy as np
    cent = np.zeros(1 << bits, dtype=np.float32)
    thr = np.zeros((1 << bits) - 1, dtype=np.float32)
    _check(lib().kvq_kqv_codebook(bits, head_dim, cent.ctypes.data, thr.ctypes.data),
           "kvq_kqv_codebook")
    return cent, thr
