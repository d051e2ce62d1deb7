"""Seeded synthetic workloads for quantized-KV decode attention.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic (no quantization, no attention, no bound).  Both the CUDA
path and the CPU oracle are fed from it, so they see identical bytes.

Workloads follow the shapes the pages evaluate on ("Runtime-Certified
Bounded-Error Quantized Attention", Experimental Results: LLaMA 3.1-8B at
8K-128K context; "Hurwitz Quaternion Multiplicative Quantization", Memory and
latency: 128k context), represented by synthetic tensors of those shapes:

* ``tiny``     1 sequence, 1 q head / 1 kv head, d 64, 256 tokens, 4 decode
               queries, fp32 N(0,1); K INT8 g32, V INT4 g32; tau = inf.
* ``llama8b``  8 sequences, 32 q heads / 8 kv heads, d 128, 8192 tokens,
               bf16 N(0,1), a seeded 2% of K channels per kv head scaled x20;
               K INT8 g128, V INT4 g32; tau = inf.
* ``long128k`` as ``llama8b`` with 1 sequence of 131072 tokens.
* ``rotated``  as ``llama8b`` (same data) with a seeded randomized Hadamard
               rotation on K and symmetric INT4 K with g32.
* ``serving``  64 sequences, lengths uniform in [1024, 32768], bf16 N(0,1),
               no outlier channels; in a seeded 1% of sequences (at least one),
               1% of the tokens of every kv head carry one channel set to +-50
               in K and (independently drawn channel and sign) in V;
               K INT8 g128, V INT4 g32; tau = 1e-2.

Random streams.  Every tensor is drawn from its own numpy
``Generator(PCG64(SeedSequence(seed, spawn_key=(config, stream, index))))``,
so one sequence of a large workload can be regenerated without the others.
bf16 values are fp32 N(0,1) draws rounded to nearest-even.  Tensor layouts:

* q      [num_seqs][num_queries][num_q_heads][d]
* k, v   [num_seqs][num_kv_heads][ctx_stride][d]   (token-major per head)
* page_table [num_seqs][max_pages_per_seq] int32, -1 where unused; physical
  pages are a seeded random permutation of all pages the workload needs.
"""

from __future__ import annotations

import dataclasses
import math
import os
from concurrent.futures import ThreadPoolExecutor
from typing import Dict, List, Optional

import numpy as np

PAGE_SIZE = 16

# stream ids (fixed order: Q, K, V, outlier channels, spikes, Hadamard signs,
# page permutation, context lengths, the KQV codec's QJL projections)
_S_Q, _S_K, _S_V, _S_OUTLIER, _S_SPIKE, _S_SIGNS, _S_PERM, _S_LEN, _S_QJL, _S_HQ = range(10)

_CONFIG_IDS = {"tiny": 1, "llama8b": 2, "long128k": 3, "rotated": 4, "serving": 5}


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    ctx: int                      # fixed context, or the max of the range
    num_queries: int = 1
    dtype: str = "bf16"           # "bf16" | "fp32" for q, k, v
    k_bits: int = 8
    k_group: int = 128
    k_rotate: bool = False
    v_bits: int = 4
    v_group: int = 32
    outlier_frac: float = 0.0     # fraction of K channels per kv head
    outlier_scale: float = 20.0
    ctx_min: Optional[int] = None  # ragged lengths uniform in [ctx_min, ctx]
    spike_seq_frac: float = 0.0
    spike_token_frac: float = 0.01
    spike_value: float = 50.0
    tau: float = math.inf

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def max_pages_per_seq(self) -> int:
        return (self.ctx + PAGE_SIZE - 1) // PAGE_SIZE

    def scaled(self, **kw) -> "Workload":
        """Same recipe at other sizes (used for oracle-sized parity cases)."""
        return dataclasses.replace(self, **kw)


WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", 1, 1, 1, 64, 256, num_queries=4, dtype="fp32",
                     k_bits=8, k_group=32),
    "llama8b": Workload("llama8b", 8, 32, 8, 128, 8192, outlier_frac=0.02),
    "long128k": Workload("long128k", 1, 32, 8, 128, 131072, outlier_frac=0.02),
    "rotated": Workload("rotated", 8, 32, 8, 128, 8192, outlier_frac=0.02,
                        k_bits=4, k_group=32, k_rotate=True),
    "serving": Workload("serving", 64, 32, 8, 128, 32768, ctx_min=1024,
                        spike_seq_frac=0.01, tau=1e-2),
}


def _rng(seed: int, cfg: str, stream: int, index: int = 0) -> np.random.Generator:
    cid = _CONFIG_IDS.get(cfg.split("@")[0], 0)
    ss = np.random.SeedSequence(entropy=seed, spawn_key=(cid, stream, index))
    return np.random.Generator(np.random.PCG64(ss))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round finite fp32 to the nearest bf16 (ties to even); returns uint16 bits.
    (For a finite value the 32-bit sum below cannot wrap: the largest finite
    pattern 0xFF7FFFFF plus 0x8000 stays under 2^32.)"""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


class Inputs:
    """Lazily generated inputs of one workload at one seed."""

    def __init__(self, wl: Workload, seed: int = 0):
        self.wl = wl
        self.seed = seed
        self.name = wl.name
        self.seq_lens = self._seq_lens()
        self.pages_per_seq = [(n + PAGE_SIZE - 1) // PAGE_SIZE for n in self.seq_lens]
        self.num_pages = int(sum(self.pages_per_seq))
        self.page_table = self._page_table()
        self.outlier_channels = self._outliers()
        self.spike_seqs = self._spike_seqs()
        self.rot_signs = self._signs()

    # -- small metadata ---------------------------------------------------
    def _seq_lens(self) -> List[int]:
        wl = self.wl
        if wl.ctx_min is None:
            return [wl.ctx] * wl.num_seqs
        g = _rng(self.seed, wl.name, _S_LEN)
        return [int(x) for x in g.integers(wl.ctx_min, wl.ctx, size=wl.num_seqs,
                                           endpoint=True)]

    def _page_table(self) -> np.ndarray:
        wl = self.wl
        g = _rng(self.seed, wl.name, _S_PERM)
        perm = g.permutation(self.num_pages).astype(np.int32)
        pt = np.full((wl.num_seqs, wl.max_pages_per_seq), -1, dtype=np.int32)
        off = 0
        for b, npg in enumerate(self.pages_per_seq):
            pt[b, :npg] = perm[off:off + npg]
            off += npg
        return pt

    def _outliers(self) -> np.ndarray:
        wl = self.wl
        n = int(round(wl.outlier_frac * wl.head_dim))
        out = np.zeros((wl.num_kv_heads, n), dtype=np.int64)
        if n == 0:
            return out
        g = _rng(self.seed, wl.name, _S_OUTLIER)
        for h in range(wl.num_kv_heads):
            out[h] = np.sort(g.choice(wl.head_dim, size=n, replace=False))
        return out

    def _spike_seqs(self) -> List[int]:
        wl = self.wl
        if wl.spike_seq_frac <= 0:
            return []
        n = max(1, int(round(wl.spike_seq_frac * wl.num_seqs)))
        g = _rng(self.seed, wl.name, _S_SPIKE)
        return sorted(int(x) for x in g.choice(wl.num_seqs, size=n, replace=False))

    def _signs(self) -> Optional[np.ndarray]:
        return self.rotation_signs() if self.wl.k_rotate else None

    def rotation_signs(self) -> np.ndarray:
        """The Hadamard sign vector of the seed (drawn whether or not the
        workload's own codec rotates; the KQV codec always does)."""
        g = _rng(self.seed, self.wl.name, _S_SIGNS)
        return np.where(g.integers(0, 2, size=self.wl.head_dim) == 1, 1, -1).astype(np.int8)

    def qjl_matrix(self) -> np.ndarray:
        """The KQV codec's QJL projections: fp32 [d][d], i.i.d. N(0, 1)."""
        g = _rng(self.seed, self.wl.name, _S_QJL)
        d = self.wl.head_dim
        return g.standard_normal((d, d), dtype=np.float32)

    def hqmq_secondary(self, S: int = 64) -> np.ndarray:
        """The HQMQ codec's secondary sets: fp32 [Hkv][2 (K, V)][S][4] random
        unit quaternions (N(0, 1) 4-vectors normalized in fp64, then rounded
        to fp32)."""
        g = _rng(self.seed, self.wl.name, _S_HQ)
        x = g.standard_normal((self.wl.num_kv_heads, 2, S, 4))
        return (x / np.linalg.norm(x, axis=-1, keepdims=True)).astype(np.float32)

    # -- tensors ------------------------------------------------------------
    def _cast(self, x32: np.ndarray) -> np.ndarray:
        if self.wl.dtype == "fp32":
            return x32.astype(np.float32)
        return f32_to_bf16_bits(x32)

    def q(self) -> np.ndarray:
        """q [num_seqs][num_queries][Hq][d]: bf16 bits (uint16) or fp32."""
        wl = self.wl
        g = _rng(self.seed, wl.name, _S_Q)
        x = g.standard_normal((wl.num_seqs, wl.num_queries, wl.num_q_heads, wl.head_dim),
                              dtype=np.float32)
        return self._cast(x)

    def kv_seq(self, b: int, ctx_stride: Optional[int] = None, out=None):
        """(k, v) of sequence b as [Hkv][ctx_stride][d] (bf16 bits or fp32).

        Tokens at positions >= seq_lens[b] are zero.  With `out` = (k, v)
        arrays of that shape, they are filled in place and returned."""
        wl = self.wl
        n = self.seq_lens[b]
        T = ctx_stride if ctx_stride is not None else n
        shape = (wl.num_kv_heads, n, wl.head_dim)
        gk = _rng(self.seed, wl.name, _S_K, b)
        gv = _rng(self.seed, wl.name, _S_V, b)
        k = gk.standard_normal(shape, dtype=np.float32)
        v = gv.standard_normal(shape, dtype=np.float32)
        if self.outlier_channels.shape[1]:
            for h in range(wl.num_kv_heads):
                k[h][:, self.outlier_channels[h]] *= np.float32(wl.outlier_scale)
        if b in self.spike_seqs and n > 0:
            gs = _rng(self.seed, wl.name, _S_SPIKE, 1 + b)
            nt = max(1, int(round(wl.spike_token_frac * n)))
            for h in range(wl.num_kv_heads):
                toks = gs.choice(n, size=nt, replace=False)
                for arr in (k, v):
                    ch = gs.integers(0, wl.head_dim, size=nt)
                    sg = np.where(gs.integers(0, 2, size=nt) == 1, 1.0, -1.0)
                    arr[h, toks, ch] = (sg * wl.spike_value).astype(np.float32)
        kc, vc = self._cast(k), self._cast(v)
        if out is None:
            if T == n:
                return kc, vc
            out = (np.zeros((wl.num_kv_heads, T, wl.head_dim), dtype=kc.dtype),
                   np.zeros((wl.num_kv_heads, T, wl.head_dim), dtype=kc.dtype))
        ko, vo = out
        ko[:, :n] = kc
        vo[:, :n] = vc
        ko[:, n:] = 0
        vo[:, n:] = 0
        return ko, vo

    def kv(self, ctx_stride: Optional[int] = None, threads: Optional[int] = None):
        """(k, v) of all sequences as [num_seqs][Hkv][ctx_stride][d].

        Sequences are drawn from their own streams, so they are filled in
        parallel threads (numpy releases the interpreter lock while it fills
        large arrays) with values independent of the thread count."""
        wl = self.wl
        T = ctx_stride if ctx_stride is not None else max(self.seq_lens)
        dt = np.float32 if wl.dtype == "fp32" else np.uint16
        shape = (wl.num_seqs, wl.num_kv_heads, T, wl.head_dim)
        k, v = np.empty(shape, dtype=dt), np.empty(shape, dtype=dt)
        n = threads or min(wl.num_seqs, os.cpu_count() or 1, 16)
        if n <= 1:
            for b in range(wl.num_seqs):
                self.kv_seq(b, T, out=(k[b], v[b]))
        else:
            with ThreadPoolExecutor(max_workers=n) as ex:
                list(ex.map(lambda b: self.kv_seq(b, T, out=(k[b], v[b])), range(wl.num_seqs)))
        return k, v

    def as_f32(self, x: np.ndarray) -> np.ndarray:
        return x if x.dtype == np.float32 else bf16_bits_to_f32(x)


def make(name: str, seed: int = 0, **overrides) -> Inputs:
    wl = WORKLOADS[name]
    if overrides:
        wl = wl.scaled(**overrides)
    return Inputs(wl, seed)
