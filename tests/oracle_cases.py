"""Oracle-sized versions of the five workloads (same recipe, smaller shapes) and a
helper that runs the oracle end to end on one of them.  Test helper only."""

import math

import numpy as np

import oracle
from quantized_decode_attention_kvq_b200 import inputs as synth

# name -> overrides; each keeps the workload's recipe, spans several pages and
# leaves a ragged last page
SMALL = {
    "tiny": {},
    "llama8b": dict(num_seqs=2, num_q_heads=8, num_kv_heads=2, ctx=300),
    "long128k": dict(num_seqs=1, num_q_heads=8, num_kv_heads=2, ctx=1500),
    "rotated": dict(num_seqs=2, num_q_heads=8, num_kv_heads=2, ctx=300),
    "serving": dict(num_seqs=6, num_q_heads=8, num_kv_heads=2, ctx=200, ctx_min=20,
                    spike_seq_frac=0.2),
}


def small(name, seed=0, **kw):
    ov = dict(SMALL[name])
    ov.update(kw)
    return synth.make(name, seed, **ov)


def oracle_cache(inp, outliers=False):
    wl = inp.wl
    return oracle.Cache(wl.head_dim, wl.num_kv_heads, inp.num_pages, k_bits=wl.k_bits,
                        k_group=wl.k_group, k_rotate=wl.k_rotate, rot_signs=inp.rot_signs,
                        outliers=outliers)


def device_pool(c):
    """The oracle cache's pool (logical stripe order) in the library's device
    layout, as include/kvq.h documents it: with d = 128 and 8-bit keys, the
    16-byte chunk q of the 128-byte key row of token slot s sits at chunk
    q ^ (s % 8).  Every other layout is the same in both."""
    pool = np.asarray(c.pool)
    if not (c.cfg.d == 128 and c.cfg.kbits == 8):
        return pool
    blocks = pool.reshape(-1, c.block_bytes).copy()
    k = blocks[:, :16 * 128].reshape(-1, 16, 8, 16)
    out = np.empty_like(k)
    for s in range(16):
        out[:, s, [q ^ (s % 8) for q in range(8)], :] = k[:, s, :, :]
    blocks[:, :16 * 128] = out.reshape(-1, 16 * 128)
    return blocks.reshape(-1)


def run_oracle(inp, tau=None):
    """Append the whole context, decode every row, and compute dense attention."""
    wl = inp.wl
    k, v = inp.kv()
    q = inp.q()
    c = oracle_cache(inp)
    rc = c.append(k, v, inp.page_table, np.zeros(wl.num_seqs, np.int32),
                  valid=np.array(inp.seq_lens, np.int32))
    assert rc == 0
    tau = wl.tau if tau is None else tau
    o_hat, bound, flags, diag = c.decode(q, inp.page_table, inp.seq_lens, tau=tau)
    o_dense = oracle.dense(q, k, v, inp.seq_lens)
    return dict(q=q, k=k, v=v, cache=c, o_hat=o_hat, bound=bound, flags=flags, diag=diag,
                o_dense=o_dense, tau=tau)


def max_err(a, b):
    return np.abs(np.asarray(a, np.float64) - np.asarray(b, np.float64)).max(axis=-1)


def rel_l2(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


INF = math.inf
