"""Benchmark of one decode step of quantized-KV attention with the certified bound.

A step is one pass of the whole hot path over one batch: quantize-on-append of
the step's new K/V token of every sequence into the paged cache, then the fused
split-K decode attention with its per-query bound and flags over the full
context (and, when tau is finite and a query is flagged, the exact fallback).
By default the append runs inside the decode launch (kvq_decode_attention_append,
one launch per step); --two-calls times kvq_quantize_append followed by
kvq_decode_attention instead.
The metric is KV token-heads processed per second (sum of context lengths x kv
heads per step) and the achieved HBM bandwidth of the decode kernel against the
measured peak.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload llama8b]
    python bench.py --impl reference ...   # the CPU oracle as the reference arm

Multi-GPU (torchrun): every rank runs its own replica of the workload (the path
has no exchange step); the time is the max over ranks and the value is the
work of all ranks over that time.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from quantized_decode_attention_kvq_b200 import inputs as synth  # noqa: E402

METRIC = ("quantized-KV decode attention: KV tokens·heads/s and achieved HBM GB/s "
          "vs peak")
UNIT = "KV token-heads/s"
L2_BYTES = 126 * 2 ** 20
SPEC_HBM_GBS = 8000.0     # nominal B200 HBM3e bandwidth (context for frac_vs_spec)
# adaptive-precision ladder of the serving line: the pages' example coverage
# (99.5% of the estimated mass on full-precision keys), value promotion of
# blocks whose estimated share of the value error exceeds 1e-4, and a ranking
# check that tolerates exact log-mass inversions up to 0.1
LADDER = {"tau_cov": 0.995, "v_tol": 1e-4, "rank_tol": 0.1}
# the sources of the decode kernel (and of the token codec its fused append runs)
DECODE_SRCS = [os.path.join(ROOT, "quantized_decode_attention_kvq_b200", "csrc", f)
               for f in ("decode_kernel.cuh", "quantize_token.cuh", "kvq_device.cuh")]


# secondary units per (kv head, role) of the HQMQ workloads' caches
HQ_S = 32


def _variant(name: str):
    """'llama8b' -> ('llama8b', ''); 'llama8b+med3' -> ('llama8b', 'med3'): the
    workload with Med3x outlier extraction in the cache; 'llama8b+kqv' and
    'llama8b+hqmq': the workload's data and shapes in a cache of the KQV or the
    HQMQ codec; 'llama8b+hqmq+med3': the HQMQ codec with Med3x."""
    base, _, ext = name.partition("+")
    if base not in synth.WORKLOADS or ext not in ("", "med3", "kqv", "hqmq", "hqmq+med3"):
        raise SystemExit(f"unknown workload {name}")
    return base, ext


def _describe(name: str) -> str:
    base, ext = _variant(name)
    wl = synth.WORKLOADS[base]
    if ext == "kqv":
        ctx = f"ctx {wl.ctx}" if wl.ctx_min is None else f"ctx U[{wl.ctx_min},{wl.ctx}]"
        return (f"{wl.name} data and shapes: B={wl.num_seqs}, Hq={wl.num_q_heads}, "
                f"Hkv={wl.num_kv_heads}, d={wl.head_dim}, {ctx}, KQV codec (Hadamard-rotated "
                f"K and V; K 4-bit Lloyd-Max, V 3-bit Lloyd-Max + 1-bit QJL sketch; fp32 "
                f"norms), 16-token pages (seeded permutation), tau={wl.tau}")
    if ext.startswith("hqmq"):
        ctx = f"ctx {wl.ctx}" if wl.ctx_min is None else f"ctx U[{wl.ctx_min},{wl.ctx}]"
        return (f"{wl.name} data and shapes: B={wl.num_seqs}, Hq={wl.num_q_heads}, "
                f"Hkv={wl.num_kv_heads}, d={wl.head_dim}, {ctx}, HQMQ codec (4-channel "
                f"chunks of K and V: 16-bit index into 2T x {HQ_S} secondary unit "
                f"quaternions, fp8 E4M3 radius)"
                + (", Med3x outlier extraction" if ext.endswith("med3") else "")
                + f", 16-token pages (seeded permutation), tau={wl.tau}")
    return _workload_desc(wl) + (
        ", Med3x outlier extraction (one 4-channel chunk of K and of V per token in fp16)"
        if ext == "med3" else "")


def _workload_desc(wl) -> str:
    ctx = f"ctx {wl.ctx}" if wl.ctx_min is None else f"ctx U[{wl.ctx_min},{wl.ctx}]"
    rot = "Hadamard-rotated " if wl.k_rotate else ""
    return (f"{wl.name}: B={wl.num_seqs}, Hq={wl.num_q_heads}, Hkv={wl.num_kv_heads}, "
            f"d={wl.head_dim}, {ctx}, {rot}INT{wl.k_bits}-K g{wl.k_group}, "
            f"INT{wl.v_bits}-V g{wl.v_group}, 16-token pages (seeded permutation), "
            f"tau={wl.tau}")


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


TRAFFIC_JSON = os.path.join(ROOT, "profiles", "decode_attention_traffic.json")


def decode_source_hash() -> str:
    """First 16 hex digits of the sha256 of the decode kernel's sources."""
    h = hashlib.sha256()
    for p in DECODE_SRCS:
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def _traffic_record(workload: str, two_calls: bool):
    """DRAM bytes per decode launch from the committed ncu record
    (profiles/decode_attention_traffic.json) for this workload and the fused
    step's launch, if it was taken on the current decode kernel source."""
    if two_calls or not os.path.exists(TRAFFIC_JSON):
        return None
    src_hash = decode_source_hash()
    with open(TRAFFIC_JSON) as f:
        recs = json.load(f).get("records", [])
    for r in recs:
        if r.get("workload") == workload and r.get("decode_source_sha256_16") == src_hash:
            try:
                return float(r["dram_bytes_per_launch"])
            except (KeyError, TypeError, ValueError):
                return None
    return None


def _smi_time(stamp: str):
    """nvidia-smi timestamp ('YYYY/MM/DD HH:MM:SS.mmm', local time) -> epoch seconds."""
    try:
        base, _, frac = stamp.strip().partition(".")
        t = time.mktime(time.strptime(base, "%Y/%m/%d %H:%M:%S"))
        return t + (float("0." + frac) if frac.isdigit() else 0.0)
    except ValueError:
        return None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    Q = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self, window=None):
        """Median clocks of the samples taken inside `window` (host epoch seconds)."""
        if self.proc is None:
            return None
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            if window is not None:
                t = _smi_time(f[0])
                if t is None or not (window[0] - 0.02 <= t <= window[1] + 0.02):
                    continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for nm, val in zip(names, f[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": float(max(mx)),
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------------- GPU --
def _dist_setup(n_gpus):
    import torch
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return rank, world, local


def _max_over_ranks(x: float, world: int) -> float:
    """The maximum of a per-rank number over all ranks (every rank gets it)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _rank_times(ms_total: float, dec_ms: float, e2e_ms: float, steps: int, world: int):
    """Per-step, per-decode and end-to-end times of the job: the slowest rank's."""
    ms_total = _max_over_ranks(ms_total, world)
    dec_ms = _max_over_ranks(dec_ms, world)
    e2e_ms = _max_over_ranks(e2e_ms, world)
    return ms_total / max(1, steps), dec_ms, e2e_ms


def _job_value(token_heads_per_rank: int, world: int, ms_per_step: float) -> float:
    """Whole-job throughput: the work of all ranks (independent replicas, one per
    rank) over the slowest rank's time per step."""
    return token_heads_per_rank * world / (ms_per_step * 1e-3)


def _barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def _cudart():
    """The CUDA runtime torch loaded, for the end-to-end loop's copies and events
    (thin calls: the loop issues about ten per step)."""
    import ctypes
    import glob

    import torch
    here = os.path.join(os.path.dirname(torch.__file__), "..", "nvidia", "cuda_runtime", "lib")
    for c in sorted(glob.glob(os.path.join(here, "libcudart.so*"))) + ["libcudart.so.12"]:
        try:
            rt = ctypes.CDLL(c)
            break
        except OSError:
            continue
    else:
        raise RuntimeError("libcudart not found")
    vp = ctypes.c_void_p
    rt.cudaMemcpyAsync.argtypes = [vp, vp, ctypes.c_size_t, ctypes.c_int, vp]
    rt.cudaEventRecord.argtypes = [vp, vp]
    rt.cudaStreamWaitEvent.argtypes = [vp, vp, ctypes.c_uint]
    rt.cudaEventCreateWithFlags.argtypes = [ctypes.POINTER(vp), ctypes.c_uint]
    rt.cudaEventDestroy.argtypes = [vp]
    return rt


def _packed(tensors):
    """One device byte buffer holding copies of `tensors` (256-byte aligned parts)
    and the views of it that replace them."""
    import torch
    sizes = [t.numel() * t.element_size() for t in tensors]
    offs, total = [], 0
    for n in sizes:
        offs.append(total)
        total += (n + 255) // 256 * 256
    buf = torch.empty(total, dtype=torch.uint8, device=tensors[0].device)
    views = []
    for t, o, n in zip(tensors, offs, sizes):
        v = buf[o:o + n].view(t.dtype).view(t.shape)
        v.copy_(t)
        views.append(v)
    return buf, views


class GpuStep:
    """Device-resident workload and the raw C-ABI calls of one step."""

    def __init__(self, wl_name: str, seed: int, replicas: int, two_calls: bool = False,
                 outliers: bool = False, codec: str = "int"):
        import ctypes

        import torch

        from quantized_decode_attention_kvq_b200 import kvq
        self.kvq = kvq
        self.torch = torch
        inp = synth.make(wl_name, seed)
        wl = inp.wl
        self.inp, self.wl = inp, wl
        k, v = inp.kv()
        q = inp.q()

        def dev(x):
            t = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16) if x.dtype == np.uint16 \
                else torch.from_numpy(x)
            return t.cuda()

        T = k.shape[2]
        self.kd, self.vd, self.qd = dev(k), dev(v), dev(q)
        self.pt = torch.from_numpy(inp.page_table).cuda()
        self.sl = torch.tensor(inp.seq_lens, dtype=torch.int32, device="cuda")
        ckw = dict(k_bits=wl.k_bits, k_group=wl.k_group, k_rotate=wl.k_rotate,
                   rot_signs=inp.rot_signs, outliers=outliers)
        if codec == "kqv":
            ckw = dict(codec="kqv", rot_signs=inp.rotation_signs(), qjl_matrix=inp.qjl_matrix())
        elif codec == "hqmq":
            ckw = dict(codec="hqmq", hq_secondary=inp.hqmq_secondary(HQ_S), outliers=outliers)
        base = kvq.PagedCache(wl.num_kv_heads, wl.head_dim, inp.num_pages, **ckw)
        zeros = torch.zeros(wl.num_seqs, dtype=torch.int32, device="cuda")
        base.append(self.kd, self.vd, self.pt, zeros, self.sl)
        torch.cuda.synchronize()
        # the step's new token: position seq_len - 1 of every sequence
        self.new_pos = (self.sl - 1).to(torch.int32)
        last = torch.tensor(inp.seq_lens, device="cuda").long() - 1
        idx = last.view(-1, 1, 1, 1).expand(-1, wl.num_kv_heads, 1, wl.head_dim)
        self.k_new = torch.gather(self.kd, 2, idx).contiguous()       # [B][Hkv][1][d]
        self.v_new = torch.gather(self.vd, 2, idx).contiguous()
        self.caches = [base]
        for _ in range(replicas - 1):
            c = kvq.PagedCache(wl.num_kv_heads, wl.head_dim, inp.num_pages, **ckw)
            c.pool.copy_(base.pool)
            c.eta.copy_(base.eta)
            self.caches.append(c)
        self.ws = [c.workspace(wl.num_seqs, wl.num_queries, wl.num_q_heads, self.pt.shape[1])
                   for c in self.caches]
        B, NQ, HQ, d = q.shape
        # one dedicated stream: the eager steps and the captured graph use it
        self.stream = torch.cuda.Stream()
        s = self.stream.cuda_stream
        L = kvq.lib()
        self.L = L
        dt = kvq.KVQ_BF16 if self.kd.dtype == torch.bfloat16 else kvq.KVQ_F32
        qdt = kvq.KVQ_BF16 if self.qd.dtype == torch.bfloat16 else kvq.KVQ_F32
        q0, kn0, vn0 = self.qd, self.k_new, self.v_new

        def io_set():
            """The step's inputs (q, new k, new v) and results (out, bound, flags),
            each group in one device buffer (one copy each way per step), and the
            pre-marshalled C-ABI arguments of the step's calls on them."""
            io_in, (qd, kn, vn) = _packed([q0, kn0, vn0])
            io_out, (out, bound, flags) = _packed(
                [torch.empty((B, NQ, HQ, d), dtype=torch.float32, device="cuda"),
                 torch.empty((B, NQ, HQ), dtype=torch.float32, device="cuda"),
                 torch.empty((B, NQ, HQ), dtype=torch.uint8, device="cuda")])
            append_args = [
                (ctypes.byref(c.desc), kn.data_ptr(), vn.data_ptr(), dt, kn.stride(0),
                 kn.stride(1), kn.stride(2), wl.num_seqs, 1, None, self.new_pos.data_ptr(),
                 self.pt.data_ptr(), self.pt.shape[1], s) for c in self.caches]
            decode_args = [
                (ctypes.byref(c.desc), qd.data_ptr(), qdt, B, NQ, HQ, self.pt.data_ptr(),
                 self.pt.shape[1], self.sl.data_ptr(), 0.0, wl.tau, out.data_ptr(),
                 bound.data_ptr(), flags.data_ptr(), w.data_ptr(), w.numel(), s)
                for c, w in zip(self.caches, self.ws)]
            # the fused step: the new token appended inside the decode launch
            fused_args = [
                (ctypes.byref(c.desc), kn.data_ptr(), vn.data_ptr(), dt, kn.stride(0),
                 kn.stride(1), qd.data_ptr(), qdt, B, NQ, HQ, self.pt.data_ptr(),
                 self.pt.shape[1], self.sl.data_ptr(), 0.0, wl.tau, out.data_ptr(),
                 bound.data_ptr(), flags.data_ptr(), w.data_ptr(), w.numel(), s)
                for c, w in zip(self.caches, self.ws)]
            return dict(io_in=io_in, qd=qd, k_new=kn, v_new=vn, io_out=io_out, out=out,
                        bound=bound, flags=flags, append_args=append_args,
                        decode_args=decode_args, fused_args=fused_args)

        # two sets: the end-to-end loop copies one step's inputs and the previous
        # step's results while the other set's step runs; the timed graph uses set 0
        self.io = [io_set(), io_set()]
        io0 = self.io[0]
        self.io_in, self.qd, self.k_new, self.v_new = io0["io_in"], io0["qd"], io0["k_new"], \
            io0["v_new"]
        self.io_out, self.out, self.bound, self.flags = io0["io_out"], io0["out"], \
            io0["bound"], io0["flags"]
        self.two_calls = two_calls
        self.token_heads = int(sum(inp.seq_lens)) * wl.num_kv_heads
        bb = base.block_bytes
        self.decode_bytes = (sum(inp.seq_lens) * wl.num_kv_heads * bb // 16
                             + sum(inp.pages_per_seq) * wl.num_kv_heads * 4)
        if not two_calls:   # plus the new token in (k and v) and its codes out
            es = 2 if dt == kvq.KVQ_BF16 else 4
            self.decode_bytes += wl.num_seqs * wl.num_kv_heads * (2 * wl.head_dim * es + bb // 16)
        self.cache_bytes = inp.num_pages * wl.num_kv_heads * bb
        self.replicas = replicas
        self.launches_per_step = (3 if codec in ("kqv", "hqmq") else 2) if two_calls else 1
        # finite tau: flagged rows are recomputed exactly from pinned host originals
        self.fallback = None
        self.ladder = None
        if math.isfinite(wl.tau):
            kh = (torch.from_numpy(k.view(np.int16)).view(torch.bfloat16) if k.dtype == np.uint16
                  else torch.from_numpy(k)).pin_memory()
            vh = (torch.from_numpy(v.view(np.int16)).view(torch.bfloat16) if v.dtype == np.uint16
                  else torch.from_numpy(v)).pin_memory()
            fb_bytes = kvq.kvq_fallback_staging_size(base.desc, dt, max(inp.seq_lens)) * 8
            self.fallback = dict(
                kh=kh, vh=vh, dt=dt, qdt=qdt, T=T, side=torch.cuda.Stream(),
                flags_h=torch.zeros(self.flags.numel(), dtype=torch.uint8).pin_memory(),
                sl_h=np.array(inp.seq_lens, np.int32),
                staging=torch.empty(fb_bytes, dtype=torch.uint8, device="cuda"), rows=0, calls=0,
                h2d=0)
        if self.fallback is not None and codec == "int":
            # the adaptive-precision ladder run before the exact fallback (it reads
            # the Tier-1 codec's caches, with or without outlier extraction)
            mp = self.pt.shape[1]
            rows = self.flags.numel()
            ad_host = kvq.kvq_adaptive_host_size(base.desc, B, mp)
            self.ladder = dict(
                work=torch.zeros(kvq.kvq_adaptive_work_size(base.desc, B, NQ, HQ, mp),
                                 dtype=torch.uint8, device="cuda"),
                host=torch.zeros(ad_host, dtype=torch.uint8).pin_memory(),
                kp=torch.zeros((rows, mp), dtype=torch.uint8, device="cuda"),
                vp=torch.zeros((rows, mp), dtype=torch.uint8, device="cuda"),
                rows_in=0, rows_after=0, calls=0, h2d=0)

    def fallback_exact(self, r=0):
        """The exact fallback of the rows the last decode flagged (host-synchronous)."""
        fb, wl, kvq = self.fallback, self.wl, self.kvq
        B, NQ, HQ, d = self.out.shape
        rc, n = kvq.kvq_fallback_exact(
            self.caches[r].desc, fb["kh"], fb["vh"], fb["dt"], wl.num_kv_heads * fb["T"] * d,
            fb["T"] * d, self.qd, fb["qdt"], B, NQ, HQ, fb["sl_h"].ctypes.data, 0.0, self.flags,
            fb["flags_h"], self.out, fb["staging"], fb["staging"].numel(), self.stream,
            fb["side"], 60000)
        if rc:
            raise RuntimeError(kvq.last_error())
        fl = fb["flags_h"].numpy().reshape(B, NQ, HQ).any(axis=1)     # (seq, q head)
        pairs = fl.reshape(B, wl.num_kv_heads, -1).any(axis=2)
        es = 2 if fb["dt"] == kvq.KVQ_BF16 else 4
        fb["h2d"] += int(2 * es * d * (pairs * fb["sl_h"][:, None]).sum())
        fb["rows"] += n
        fb["calls"] += 1
        return n

    def adaptive(self, r=0):
        """The adaptive-precision ladder on the rows the last decode flagged
        (host-synchronous): top-K* key promotion (tau_cov), value promotion
        (v_tol) and the ranking check (rank_tol); flags are rewritten for the
        exact fallback that follows."""
        fb, ad, wl, kvq = self.fallback, self.ladder, self.wl, self.kvq
        B, NQ, HQ, d = self.out.shape
        mp = self.pt.shape[1]
        rc, n_in, n_after = kvq.kvq_adaptive_precision(
            self.caches[r].desc, fb["kh"], fb["vh"], fb["dt"], wl.num_kv_heads * fb["T"] * d,
            fb["T"] * d, self.qd, fb["qdt"], B, NQ, HQ, self.pt, mp, self.sl,
            fb["sl_h"].ctypes.data, 0.0, wl.tau, LADDER["tau_cov"], LADDER["v_tol"],
            LADDER["rank_tol"], self.flags, fb["flags_h"], self.out, self.bound, ad["kp"],
            ad["vp"], ad["work"], ad["work"].numel(), ad["host"], ad["host"].numel(),
            fb["staging"], fb["staging"].numel(), self.stream, fb["side"], 60000)
        if rc:
            raise RuntimeError(kvq.last_error())
        # bytes paged in: the union of promoted pages per (sequence, kv head), K and V
        if n_in:
            fl = fb["flags_h"]
            um = (ad["kp"] | ad["vp"]).view(B, NQ, wl.num_kv_heads, -1, mp).amax(dim=(1, 3))
            es = 2 if fb["dt"] == kvq.KVQ_BF16 else 4
            th = self.torch
            sl = th.tensor(fb["sl_h"], dtype=th.int64, device=um.device)
            tok = th.clamp(sl[:, None, None] - 16 * th.arange(mp, device=um.device), 0, 16)
            ad["h2d"] += int((um.to(th.int64) * tok).sum().item()) * 2 * d * es
            ad["kp"].zero_()
            ad["vp"].zero_()
        ad["rows_in"] += n_in
        ad["rows_after"] += n_after
        ad["calls"] += 1
        return n_in, n_after

    def step(self, i, ev=None, io=0):
        r = i % self.replicas
        st = self.io[io]
        if not self.two_calls:
            if ev is not None:
                ev[0].record(self.stream)
            rc = self.L.kvq_decode_attention_append(*st["fused_args"][r])
            if rc:
                raise RuntimeError(self.kvq.last_error())
            if ev is not None:
                ev[1].record(self.stream)
            return
        rc = self.L.kvq_quantize_append(*st["append_args"][r])
        if rc:
            raise RuntimeError(self.kvq.last_error())
        if ev is not None:
            ev[0].record(self.stream)
        rc = self.L.kvq_decode_attention(*st["decode_args"][r])
        if rc:
            raise RuntimeError(self.kvq.last_error())
        if ev is not None:
            ev[1].record(self.stream)


def _timed_replay(st, args, world, rank, local):
    """W eager warm-up steps, the K timed steps captured into one CUDA graph,
    untimed replays of that graph (the first pays the graph's upload; the
    rest, about 0.2 s of them, put the GPU under the load the clocks are
    sampled in), then the timed replay between two events.  Returns (device
    ms of the K steps, mean decode-launch ms, clocks)."""
    import torch
    with torch.cuda.stream(st.stream):
        for r in range(st.replicas):      # setup: library descriptors and occupancy
            st.step(r)
        for i in range(args.warmup):
            st.step(i)
    torch.cuda.synchronize()
    err = st.caches[0].device_error()
    if err:
        raise RuntimeError(f"device error {err} during warm-up")
    # The default step is one launch, so the graph holds those launches alone and
    # a launch's duration is the region's time / K (an event pair around every
    # launch would add its own nodes to each step).  With --two-calls, events
    # around every decode launch separate it from the append.
    evs = [(torch.cuda.Event(enable_timing=True, external=True),
            torch.cuda.Event(enable_timing=True, external=True)) for _ in range(args.steps)] \
        if st.two_calls else [None] * args.steps
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=st.stream):
        for i in range(args.steps):
            st.step(args.warmup + i, evs[i])
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(st.stream):
        t0.record(st.stream)
        graph.replay()                    # untimed: uploads the graph
        t1.record(st.stream)
    torch.cuda.synchronize()
    one = max(1e-3, t0.elapsed_time(t1))
    pre = max(1, min(2000, int(200.0 / one)))
    pre = int(_max_over_ranks(float(pre), world))     # the same count on every rank
    sampler = ClockSampler(local) if rank == 0 else None
    _barrier(world)
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
        time.sleep(0.3)
    w0 = time.time()
    with torch.cuda.stream(st.stream):
        for _ in range(pre):
            graph.replay()
        t0.record(st.stream)
        graph.replay()
        t1.record(st.stream)
    torch.cuda.synchronize()
    w1 = time.time()
    clocks = sampler.stop((w0, w1)) if sampler else None
    if clocks is not None:
        clocks["window"] = (f"{pre} untimed replays of the same graph directly before the "
                            f"timed one, and the timed one")
    elif sampler:
        clocks = {"sm_mhz": None, "note": "no nvidia-smi sample inside the window"}
    _barrier(world)
    ms_total = t0.elapsed_time(t1)
    dec_ms = (float(np.mean([a.elapsed_time(b) for a, b in evs])) if st.two_calls
              else ms_total / max(1, args.steps))
    del graph
    return ms_total, dec_ms, clocks


def _e2e(st, args, world, ladder=False):
    """The same steps end to end through the C ABI with host buffers: per step the
    H2D of its packed inputs (q and the new K/V token) from pinned memory, the
    step's call(s), the D2H of its packed results (out, bound, flags); with a
    finite tau, also the host-synchronous exact fallback of the flagged rows.
    Returns (ms per step, h2d bytes per step, d2h bytes per step)."""
    import torch
    in_h = [st.io[k]["io_in"].cpu().pin_memory() for k in (0, 1)]
    out_h = [torch.empty(st.io_out.shape, dtype=torch.uint8).pin_memory() for _ in (0, 1)]
    h2d = st.qd.numel() * st.qd.element_size() + 2 * st.k_new.numel() * st.k_new.element_size()
    d2h = st.out.numel() * 4 + st.bound.numel() * 4 + st.flags.numel()
    # with a finite tau the step ends with the host-synchronous exact fallback of the
    # flagged rows, which pages in their originals: a few steps suffice
    e_steps = max(1, args.steps) if st.fallback is None else max(1, min(args.steps, 5))
    _barrier(world)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    if st.fallback is None:
        # Pipelined over the two buffer sets: step i's inputs go in on one copy
        # stream while step i-1 runs, and step i-1's results come back on another
        # while step i runs.  A set's inputs are overwritten only after the step
        # that read them ran, and its results only after they were copied out.
        import ctypes
        rt = _cudart()
        H2D, D2H, NO_TIMING = 1, 2, 2
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        sm, si, so = st.stream.cuda_stream, s_in.cuda_stream, s_out.cuda_stream
        evs = [[ctypes.c_void_p() for _ in (0, 1)] for _ in range(3)]
        for e in sum(evs, []):
            if rt.cudaEventCreateWithFlags(ctypes.byref(e), NO_TIMING):
                raise RuntimeError("cudaEventCreateWithFlags failed")
        ev_in, ev_ran, ev_out = evs
        d_in = [st.io[k]["io_in"].data_ptr() for k in (0, 1)]
        d_out = [st.io[k]["io_out"].data_ptr() for k in (0, 1)]
        h_in = [t.data_ptr() for t in in_h]
        h_out = [t.data_ptr() for t in out_h]
        n_in, n_out = st.io_in.numel(), st.io_out.numel()
        err = 0
        e0.record(st.stream)
        s_in.wait_event(e0)
        s_out.wait_event(e0)
        for i in range(e_steps):
            k = i & 1
            if i >= 2:
                err |= rt.cudaStreamWaitEvent(si, ev_ran[k], 0)
            err |= rt.cudaMemcpyAsync(d_in[k], h_in[k], n_in, H2D, si)
            err |= rt.cudaEventRecord(ev_in[k], si)
            err |= rt.cudaStreamWaitEvent(sm, ev_in[k], 0)
            if i >= 2:
                err |= rt.cudaStreamWaitEvent(sm, ev_out[k], 0)
            st.step(i, io=k)
            err |= rt.cudaEventRecord(ev_ran[k], sm)
            err |= rt.cudaStreamWaitEvent(so, ev_ran[k], 0)
            err |= rt.cudaMemcpyAsync(h_out[k], d_out[k], n_out, D2H, so)
            err |= rt.cudaEventRecord(ev_out[k], so)
        st.stream.wait_stream(s_out)
        e1.record(st.stream)
        torch.cuda.synchronize()
        for e in sum(evs, []):
            rt.cudaEventDestroy(e)
        if err:
            raise RuntimeError("a CUDA runtime call of the end-to-end loop failed")
        # every step computes the same batch: the results read back through either
        # set are the device results of the timed steps
        ref = st.io_out.cpu()
        if not all(torch.equal(t, ref) for t in out_h[:min(2, e_steps)]):
            raise RuntimeError("end-to-end results differ from the device results")
    else:
        with torch.cuda.stream(st.stream):
            e0.record(st.stream)
            for i in range(e_steps):
                st.io_in.copy_(in_h[0], non_blocking=True)
                st.step(i)
                if ladder:
                    st.adaptive(i % st.replicas)
                st.fallback_exact(i % st.replicas)
                out_h[0].copy_(st.io_out, non_blocking=True)
            e1.record(st.stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / e_steps, h2d, d2h


def measure_workload(name, args, world, rank, local):
    """One workload's measurement on this rank: the device-timed value and the
    decode kernel's roofline, the clocks, and the end-to-end number.  A name
    ending in "+med3" is the workload with outlier extraction in the cache."""
    import torch
    base, ext = _variant(name)
    wl = synth.WORKLOADS[base]
    reps = max(2, math.ceil(3 * L2_BYTES / max(1, _cache_bytes_estimate(wl, ext))))
    reps = min(reps, 8)
    # the KQV and HQMQ codecs have no fused step: theirs is the append and the decode
    codec = "kqv" if ext == "kqv" else "hqmq" if ext.startswith("hqmq") else "int"
    two_calls = args.two_calls or codec != "int"
    st = GpuStep(base, args.seed, reps, two_calls=two_calls, outliers=ext.endswith("med3"),
                 codec=codec)
    ms_total, dec_ms, clocks = _timed_replay(st, args, world, rank, local)
    e2e_ms, h2d, d2h = _e2e(st, args, world)
    lad_ms = None
    if st.ladder is not None:
        fb_rows, fb_calls, fb_h2d = st.fallback["rows"], st.fallback["calls"], st.fallback["h2d"]
        lad_ms, _, _ = _e2e(st, args, world, ladder=True)
        lad_ms = _max_over_ranks(lad_ms, world)
        lad_fb = (st.fallback["rows"] - fb_rows, st.fallback["calls"] - fb_calls,
                  st.fallback["h2d"] - fb_h2d)
        st.fallback["rows"], st.fallback["calls"], st.fallback["h2d"] = fb_rows, fb_calls, fb_h2d
    ms_step, dec_ms, e2e_ms = _rank_times(ms_total, dec_ms, e2e_ms, args.steps, world)
    peak, peak_kind = _peaks()
    achieved = st.decode_bytes / (dec_ms * 1e-3) / 1e9
    rec = {
        "value": _job_value(st.token_heads, world, ms_step),
        "unit": UNIT,
        # the same rate counted per query head (x Hq/Hkv: each kv head serves its GQA group)
        "value_q_heads": _job_value(st.token_heads, world, ms_step) * (wl.num_q_heads / wl.num_kv_heads),
        "ms_per_step": ms_step,
        "steps": args.steps,
        "config": {"workload": _describe(name),
                   "l2": f"inputs larger than L2: {reps} cache replicas of "
                         f"{st.cache_bytes / 1e6:.1f} MB rotated per step",
                   "step": ("kvq_quantize_append + kvq_decode_attention" if st.two_calls else
                            "kvq_decode_attention_append (append fused into the decode)"),
                   "token_heads_per_step": st.token_heads,
                   "decode_bytes_per_launch": st.decode_bytes},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": _traffic_record(name, st.two_calls),
                     "peak_kind": f"{peak_kind} copy bandwidth",
                     "frac_vs_spec": achieved / SPEC_HBM_GBS,
                     "spec_peak": SPEC_HBM_GBS,
                     "kernel": ("kqv_partial_kernel + kqv_merge_kernel" if ext == "kqv" else
                                "hqmq_partial_kernel + hqmq_merge_kernel" if codec == "hqmq" else
                                "decode_mma_kernel" + ("" if st.two_calls else " (append fused)")),
                     "kernel_ms": dec_ms,
                     "timing": ("events around every decode launch" if st.two_calls else
                                "events around the replay of K back-to-back launches, / K")},
        "e2e": {"value": _job_value(st.token_heads, world, e2e_ms), "unit": UNIT,
                "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                "note": ("each step: H2D of its packed inputs from pinned memory, the step's "
                         "call, D2H of its packed results; without a fallback the copies of "
                         "one step overlap the neighbouring steps' kernels (two buffer sets, "
                         "two copy streams)")},
        "gpu_launches": st.launches_per_step * args.steps,
        "clocks": clocks,
    }
    if st.fallback is not None:
        fb = st.fallback
        rows_per_step = fb["rows"] / max(1, fb["calls"])
        rows = st.out.shape[0] * st.out.shape[1] * st.out.shape[2]
        rec["fallback"] = {
            "tau": wl.tau, "rate": rows_per_step / rows, "rows_per_step": rows_per_step,
            "rows": rows, "h2d_bytes_per_step": fb["h2d"] / max(1, fb["calls"]),
            "note": "value times append + decode (graph); e2e adds the exact fallback of the "
                    "flagged rows (H2D of their originals + fp32 attention)"}
        rec["e2e"]["h2d_bytes_per_step"] = int(h2d + fb["h2d"] / max(1, fb["calls"]))
    if st.ladder is not None:
        ad = st.ladder
        calls = max(1, ad["calls"])
        rec["ladder"] = {
            "what": "kvq_adaptive_precision on the decode's flagged rows (top-K* key promotion, "
                    "value promotion, ranking check), then kvq_fallback_exact on the rows "
                    "still flagged",
            **LADDER,
            "rows_in_per_step": ad["rows_in"] / calls,
            "rows_flagged_after_ladder_per_step": ad["rows_after"] / calls,
            "fallback_rate": ad["rows_after"] / calls / rows,
            "promoted_h2d_bytes_per_step": ad["h2d"] / calls,
            "fallback_h2d_bytes_per_step": lad_fb[2] / max(1, lad_fb[1]),
            "e2e": {"value": _job_value(st.token_heads, world, lad_ms), "unit": UNIT,
                    "ms_per_step": lad_ms,
                    "h2d_bytes_per_step": int(h2d + ad["h2d"] / calls +
                                              lad_fb[2] / max(1, lad_fb[1])),
                    "d2h_bytes_per_step": int(d2h)}}
    del st
    torch.cuda.empty_cache()
    return rec


def run_gpu(args):
    rank, world, local = _dist_setup(args.gpus)
    main = measure_workload(args.workload, args, world, rank, local)
    also = [w for w in args.also.split(",") if w and w != "none" and w != args.workload]
    subs = {w: measure_workload(w, args, world, rank, local) for w in also}
    res = {
        "metric": METRIC,
        "value": main["value"],
        "unit": UNIT,
        "value_q_heads": main["value_q_heads"],
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": main["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "s8xs8->s32 (QK), f16xf16->f32 (PV), f32 softmax/bound",
        "data": "synthetic (seeded N(0,1) bf16 + outlier channels, as the workload states)",
        "config": dict(main["config"],
                       parallelism=f"replicas x{world}" if world > 1 else "1 GPU"),
        "roofline": main["roofline"],
        "e2e": main["e2e"],
        "gpu_launches": main["gpu_launches"],
        "clocks": main["clocks"],
    }
    if "fallback" in main:
        res["fallback"] = main["fallback"]
    if subs:
        res["workloads"] = subs
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(args.workload, args.seed, args.cpu_seconds)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)


def _cache_bytes_estimate(wl, ext="") -> int:
    per_tok = wl.head_dim * wl.k_bits // 8 + wl.head_dim // 2 + 2 * wl.head_dim // wl.k_group \
        + 4 * wl.head_dim // 32 + (18 if ext == "med3" else 0)
    if ext == "kqv":
        per_tok = wl.head_dim + wl.head_dim // 8 + 16 + wl.head_dim // 64
    if ext.startswith("hqmq"):
        per_tok = 3 * wl.head_dim // 2 + 8 + wl.head_dim // 64 + (18 if ext.endswith("med3") else 0)
    ctx = wl.ctx if wl.ctx_min is None else (wl.ctx + wl.ctx_min) // 2
    return wl.num_seqs * ctx * wl.num_kv_heads * per_tok


# ------------------------------------------------------------------------- CPU --
def _oracle_cache(workload: str, seed: int):
    """The workload's inputs and an empty oracle cache of its codec."""
    import oracle
    base, ext = _variant(workload)
    inp = synth.make(base, seed)
    wl = inp.wl
    if ext == "kqv":
        c = oracle.KqvCache(wl.head_dim, wl.num_kv_heads, inp.num_pages, inp.rotation_signs(),
                            inp.qjl_matrix())
    elif ext.startswith("hqmq"):
        c = oracle.HqCache(wl.head_dim, wl.num_kv_heads, inp.num_pages, inp.hqmq_secondary(HQ_S),
                           outliers=ext.endswith("med3"))
    else:
        c = oracle.Cache(wl.head_dim, wl.num_kv_heads, inp.num_pages, k_bits=wl.k_bits,
                         k_group=wl.k_group, k_rotate=wl.k_rotate, rot_signs=inp.rot_signs,
                         outliers=ext == "med3")
    return inp, c


def _oracle_setup(workload: str, seed: int, kv_heads=None):
    """The oracle's cache of sequence 0 of the workload; rows of the given kv heads."""
    inp, c = _oracle_cache(workload, seed)
    wl = inp.wl
    k, v = inp.kv_seq(0)
    pt = inp.page_table[:1]
    sl = np.array(inp.seq_lens[:1], np.int32)
    rc = c.append(k[None], v[None], pt, np.zeros(1, np.int32), valid=sl)
    assert rc == 0
    q = inp.q()[:1]
    heads = range(wl.num_kv_heads) if kv_heads is None else kv_heads
    mask = np.zeros((1, wl.num_queries, wl.num_q_heads), np.uint8)
    for h in heads:
        mask[:, :, h * wl.group:(h + 1) * wl.group] = 1
    return inp, c, q, pt, sl, mask.reshape(-1), len(list(heads))


def _oracle_decode_loop(workload: str, seed: int, heads, seconds: float):
    """Repeat the oracle's decode of sequence 0 (rows of the given kv heads, or all)
    for about `seconds`; returns (KV token-heads decoded, seconds, repeats)."""
    inp, c, q, pt, sl, mask, nh = _oracle_setup(workload, seed, heads)
    th = int(sl.sum()) * nh
    reps, t0 = 0, time.perf_counter()
    while True:
        c.decode(q, pt, sl, tau=inp.wl.tau, row_mask=mask)
        reps += 1
        el = time.perf_counter() - t0
        if el >= seconds or reps >= 1000:
            break
    return th * reps, el, reps


def _oracle_worker(job):
    return _oracle_decode_loop(*job)


def _oracle_codec_and_dense(workload: str, seed: int):
    """Single-thread rates of the oracle's other two stages on sequence 0 of the
    workload, all kv heads: the codec (append of every token) and the exact
    dense attention the fallback computes (every query row), in KV
    token-heads/s."""
    import oracle
    inp, c = _oracle_cache(workload, seed)
    wl = inp.wl
    k, v = inp.kv_seq(0)
    sl = np.array(inp.seq_lens[:1], np.int32)
    th = int(sl[0]) * wl.num_kv_heads
    t0 = time.perf_counter()
    rc = c.append(k[None], v[None], inp.page_table[:1], np.zeros(1, np.int32), valid=sl)
    t1 = time.perf_counter()
    assert rc == 0
    oracle.dense(inp.q()[:1], k[None], v[None], sl)
    t2 = time.perf_counter()
    return th / (t1 - t0), th / (t2 - t1)


def cpu_baseline(workload: str, seed: int, seconds: float):
    """The oracle's decode (fp64 attention + bound over the quantized cache) on whole
    sequences of the workload: one process per kv head of sequence 0 on the host's
    cores (spawned, so no CUDA state is inherited), each for about `seconds`, and
    the same single-threaded on all kv heads."""
    import multiprocessing
    wl = synth.WORKLOADS[_variant(workload)[0]]
    n = max(1, min(os.cpu_count() or 1, wl.num_kv_heads))
    with multiprocessing.get_context("spawn").Pool(n) as pool:
        res = pool.map(_oracle_worker, [(workload, seed, [h], seconds) for h in range(n)])
    value = sum(r[0] for r in res) / max(r[1] for r in res)
    th1, el1, reps1 = _oracle_decode_loop(workload, seed, None, seconds)
    codec, dense = _oracle_codec_and_dense(workload, seed)
    inp = synth.make(_variant(workload)[0], seed)
    return {"value": value, "unit": UNIT, "cores": n, "kind": "oracle",
            "single_core_value": th1 / el1,
            "single_core_codec_value": codec, "single_core_dense_value": dense,
            "sample": f"sequence 0 of {wl.name} ({int(inp.seq_lens[0])} tokens x "
                      f"{wl.num_q_heads // wl.num_kv_heads} q heads per kv head), decode + "
                      f"bound: {n} processes, one kv head each, about {seconds:.0f} s each; "
                      f"single-core figure over all {wl.num_kv_heads} kv heads, {reps1} "
                      f"repeat(s), {el1:.1f} s"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    wl = synth.WORKLOADS[_variant(args.workload)[0]]
    inp, c, q, pt, sl, mask, nh = _oracle_setup(args.workload, args.seed, [0])
    th = int(sl.sum()) * nh
    for _ in range(args.warmup):
        c.decode(q, pt, sl, tau=wl.tau, row_mask=mask)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        c.decode(q, pt, sl, tau=wl.tau, row_mask=mask)
    el = time.perf_counter() - t0
    ms = el * 1e3 / max(1, args.steps)
    value = th / (ms * 1e-3)
    res = {
        "impl": "reference",
        "metric": METRIC,
        "value": value,
        "unit": UNIT,
        "n_gpus": args.gpus,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64 (attention, bound), f32 (codec)",
        "data": "synthetic",
        "config": {"workload": _describe(args.workload),
                   "sample": f"each step: kv head 0 of sequence 0 ({int(sl[0])} tokens, "
                             f"{wl.group * wl.num_queries} query rows) of the workload"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": "kv head 0 of sequence 0 of the workload per step"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(res), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--workload", default="llama8b",
                    choices=sorted(synth.WORKLOADS) + [w + x for x in ("+med3", "+kqv", "+hqmq",
                                                                        "+hqmq+med3")
                                                        for w in sorted(synth.WORKLOADS)])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--impl", default="kvq", choices=["kvq", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--also", default=None,
                    help="comma-separated workloads measured in the same run and reported "
                         "under 'workloads'; a '+med3' suffix adds outlier extraction to the "
                         "cache, '+kqv' and '+hqmq' use the KQV and the HQMQ codec (default: "
                         "long128k,rotated,serving,llama8b+med3,serving+med3,llama8b+kqv,"
                         "llama8b+hqmq with llama8b; 'none')")
    ap.add_argument("--two-calls", action="store_true",
                    help="step = kvq_quantize_append + kvq_decode_attention (default: the fused "
                         "kvq_decode_attention_append)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.also is None:
        args.also = ("long128k,rotated,serving,llama8b+med3,serving+med3,llama8b+kqv,"
                     "llama8b+hqmq" if args.workload == "llama8b" else "none")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
