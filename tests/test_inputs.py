"""The seeded input generator: determinism, shapes, recipe features."""

import numpy as np
import torch

from quantized_decode_attention_kvq_b200 import inputs as synth


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(10000).astype(np.float32) * 37,
                        np.array([1.00390625, 1.01171875, -2.5e-39, 3.0e38], np.float32)])
    ours = synth.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    assert np.array_equal(synth.bf16_bits_to_f32(ours),
                          torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_deterministic_and_lazy():
    a = synth.make("llama8b", 1, num_seqs=3, ctx=100)
    b = synth.make("llama8b", 1, num_seqs=3, ctx=100)
    assert np.array_equal(a.q(), b.q())
    ka, va = a.kv()
    k1, v1 = b.kv_seq(1)
    assert np.array_equal(ka[1], k1) and np.array_equal(va[1], v1)
    assert np.array_equal(a.page_table, b.page_table)
    c = synth.make("llama8b", 2, num_seqs=3, ctx=100)
    assert not np.array_equal(a.q(), c.q())


def test_page_table_is_a_permutation():
    inp = synth.make("serving", 0, num_seqs=10, ctx=500, ctx_min=10)
    used = np.concatenate([inp.page_table[b, :n] for b, n in enumerate(inp.pages_per_seq)])
    assert sorted(used.tolist()) == list(range(inp.num_pages))
    assert (inp.page_table[inp.page_table >= 0] < inp.num_pages).all()
    assert min(inp.seq_lens) >= 10 and max(inp.seq_lens) <= 500


def test_outliers_and_spikes():
    inp = synth.make("llama8b", 0, num_seqs=2, ctx=64)
    assert inp.outlier_channels.shape == (8, 3)
    k = inp.as_f32(inp.kv()[0])
    ch = inp.outlier_channels[0]
    others = np.setdiff1d(np.arange(128), ch)
    assert np.abs(k[:, 0][..., ch]).mean() > 10 * np.abs(k[:, 0][..., others]).mean()
    sv = synth.make("serving", 0, num_seqs=8, ctx=400, ctx_min=200, spike_seq_frac=0.01)
    assert len(sv.spike_seqs) == 1
    b = sv.spike_seqs[0]
    k, v = (sv.as_f32(x) for x in sv.kv_seq(b))
    assert (np.abs(k) == 50).sum() >= 8 and (np.abs(v) == 50).sum() >= 8


def test_full_size_metadata():
    for name, wl in synth.WORKLOADS.items():
        inp = synth.Inputs(wl, 0)
        assert len(inp.seq_lens) == wl.num_seqs
        assert inp.page_table.shape == (wl.num_seqs, wl.max_pages_per_seq)
    sv = synth.make("serving", 0)
    assert 1024 <= min(sv.seq_lens) and max(sv.seq_lens) <= 32768
    assert synth.make("rotated", 0).rot_signs.shape == (128,)
