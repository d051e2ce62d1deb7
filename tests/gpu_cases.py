"""Helpers of the GPU parity tests: run the library through the C ABI on a seeded
workload, and the oracle on the same bytes.  Test helper only."""

import json
import math
import os

import numpy as np
import torch

import oracle
from quantized_decode_attention_kvq_b200 import inputs as synth
from oracle_cases import oracle_cache

TOL_MAXABS = 2e-3
TOL_RELL2 = 1e-3
TOL_BOUND_REL = 1e-4
TIE_BAND = 1e-4


def to_torch(x: np.ndarray, device="cuda") -> torch.Tensor:
    """Seeded numpy inputs (fp32, or bf16 bit patterns) -> torch tensor on device."""
    if x.dtype == np.uint16:
        t = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(np.ascontiguousarray(x))
    return t.to(device)


def gpu_cache(inp, num_pages=None, outliers=False):
    from quantized_decode_attention_kvq_b200 import kvq
    wl = inp.wl
    return kvq.PagedCache(wl.num_kv_heads, wl.head_dim, num_pages or inp.num_pages,
                          k_bits=wl.k_bits, k_group=wl.k_group, k_rotate=wl.k_rotate,
                          rot_signs=inp.rot_signs, outliers=outliers)


def run_gpu(inp, k=None, v=None, q=None, tau=None, page_table=None, bound_only=False,
            outliers=False):
    """Append the whole context and decode every row on the GPU."""
    wl = inp.wl
    if k is None:
        k, v = inp.kv()
    if q is None:
        q = inp.q()
    pt = inp.page_table if page_table is None else page_table
    c = gpu_cache(inp, outliers=outliers)
    kd, vd = to_torch(k), to_torch(v)
    ptd = torch.from_numpy(pt).cuda()
    sl = torch.tensor(inp.seq_lens, dtype=torch.int32, device="cuda")
    c.append(kd, vd, ptd, torch.zeros(wl.num_seqs, dtype=torch.int32, device="cuda"), sl)
    qd = to_torch(q)
    ws = c.workspace(wl.num_seqs, wl.num_queries, wl.num_q_heads, pt.shape[1])
    tau = wl.tau if tau is None else tau
    out, bound, flags = c.decode(qd, ptd, sl, ws, tau=tau, bound_only=bound_only)
    torch.cuda.synchronize()
    err = c.device_error()
    res = dict(cache=c, bound=bound.cpu().numpy().reshape(-1).astype(np.float64),
               flags=flags.cpu().numpy().reshape(-1), err=err, ws=ws, q=qd, pt=ptd, sl=sl)
    if out is not None:
        res["out"] = out.cpu().numpy().reshape(-1, wl.head_dim).astype(np.float64)
    return res


def oracle_pool(inp, k, v, outliers=False):
    wl = inp.wl
    c = oracle_cache(inp, outliers=outliers)
    rc = c.append(k, v, inp.page_table, np.zeros(wl.num_seqs, np.int32),
                  valid=np.array(inp.seq_lens, np.int32))
    assert rc == 0
    return c


def compare_outputs(out, ref):
    err = np.abs(out - ref)
    rel = np.linalg.norm(out - ref) / max(np.linalg.norm(ref), 1e-300)
    return float(err.max()), float(rel)


def record_margin(label, out, ref, **extra):
    """Append the observed output margin against the oracle (max-abs, relative
    L2, the worst row and its largest |output|) to the JSON-lines file named
    by KVQ_MARGIN_LOG, when that variable is set."""
    path = os.environ.get("KVQ_MARGIN_LOG")
    if not path:
        return
    err = np.abs(out - ref).max(axis=-1)
    row = int(err.argmax())
    rec = dict(label=label, max_abs=float(err.max()),
               rel_l2=float(np.linalg.norm(out - ref) / max(np.linalg.norm(ref), 1e-300)),
               worst_row=row, worst_row_max_abs_out=float(np.abs(ref[row]).max()),
               rows=int(err.size), **extra)
    with open(path, "a") as f:
        f.write(json.dumps(rec) + "\n")


def compare_flags(gflags, oflags, obound, tau):
    """Flags must agree except queries whose oracle bound is within the tie band of tau."""
    if math.isinf(tau):
        return int((gflags != 0).sum()), 0
    tie = np.abs(obound - tau) <= TIE_BAND * abs(tau)
    bad = (gflags.astype(bool) != oflags.astype(bool)) & ~tie
    return int(bad.sum()), int(tie.sum())
