"""The C-ABI library: it loads without a GPU, exports every symbol include/kvq.h
declares, and its host-side validation answers before any CUDA call."""

import math
import os
import re
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kvq.h")


@pytest.fixture(scope="module")
def kvq():
    from quantized_decode_attention_kvq_b200 import build
    build.build()
    from quantized_decode_attention_kvq_b200 import kvq as k
    return k


def _declared():
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"KVQ_API\s+[\w\s\*]+?\b(kvq_\w+)\s*\(", txt)))


def test_header_declares_the_four_calls():
    names = _declared()
    for fn in ("kvq_quantize_append", "kvq_decode_attention", "kvq_error_bound",
               "kvq_fallback_exact"):
        assert fn in names
    assert len(names) == 18


def test_library_exports_every_declared_symbol(kvq):
    out = subprocess.run(["nm", "-D", "--defined-only", kvq.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s(kvq_\w+)", out))
    assert set(_declared()) <= exported
    assert set(kvq.EXPORTED) == set(_declared())
    for name in _declared():
        getattr(kvq.lib(), name)


def _desc(kvq, **kw):
    a = dict(num_kv_heads=8, head_dim=128, page_size=16, num_pages=10, k_bits=8, k_group=128,
             k_rotate=0, v_bits=4, v_group=32, pool=0x1000, v_eta=0x2000, rot_signs=None,
             error_word=None)
    a.update(kw)
    return kvq.kvq_cache(**a)


def test_block_bytes_match_the_layout(kvq):
    # 210, 152, 108 bytes per token and kv head (K codes + V codes + scales + meta)
    assert kvq.kvq_block_bytes(_desc(kvq)) == 16 * 210
    assert kvq.kvq_block_bytes(_desc(kvq, k_bits=4, k_group=32)) == 16 * 152
    assert kvq.kvq_block_bytes(_desc(kvq, head_dim=64, k_group=32)) == 16 * 108
    assert kvq.kvq_pool_bytes(_desc(kvq)) == 16 * 210 * 10 * 8
    assert kvq.kvq_block_bytes(_desc(kvq, head_dim=96)) == 0
    assert kvq.kvq_block_bytes(_desc(kvq, v_group=64)) == 0
    assert kvq.kvq_block_bytes(_desc(kvq, k_group=48)) == 0


def test_outlier_section_size_and_checks(kvq):
    # the outlier section: 16 + 16 chunk indices, 16 x 4 fp16 values for K and for V
    for kw in ({}, dict(k_bits=4, k_group=32), dict(head_dim=64, k_group=32)):
        plain = kvq.kvq_block_bytes(_desc(kvq, **kw))
        ext = kvq.kvq_block_bytes(_desc(kvq, outliers=1, **kw))
        assert ext == plain + 288 and ext % 16 == 0
    assert kvq.kvq_block_bytes(_desc(kvq, outliers=2)) == 0
    # the adaptive-precision ladder reads caches with and without extraction
    assert kvq.kvq_adaptive_work_size(_desc(kvq), 2, 1, 32, 4) > 0
    assert kvq.kvq_adaptive_work_size(_desc(kvq, outliers=1), 2, 1, 32, 4) > 0


def test_kqv_block_size_and_checks(kvq):
    kqv = dict(codec=kvq.KVQ_CODEC_KQV, k_bits=4, v_bits=3, k_rotate=1, rot_signs=0x3000,
               qjl=0x4000)
    # codes 16 x d/2 + 16 x d/2, sketch 16 x d/8, four fp32 per token, the range
    assert kvq.kvq_block_bytes(_desc(kvq, k_group=128, v_group=128, **kqv)) == 2592
    assert kvq.kvq_block_bytes(_desc(kvq, head_dim=64, k_group=64, v_group=64, **kqv)) == 1424
    assert kvq.kvq_block_bytes(_desc(kvq, k_group=32, v_group=128, **kqv)) == 0
    assert kvq.kvq_block_bytes(_desc(kvq, k_group=128, v_group=128, codec=7)) == 0
    d = _desc(kvq, k_group=128, v_group=128, **kqv)
    assert kvq.kvq_adaptive_work_size(d, 2, 1, 32, 4) == 0


def test_hqmq_block_size_and_checks(kvq):
    hq = dict(codec=kvq.KVQ_CODEC_HQMQ, k_bits=6, v_bits=6, k_group=4, v_group=4,
              hq_sec=0x5000, hq_s=32)
    # u16 code + e4m3 radius per chunk for K and V (24 d per block), |k| and
    # eps per token, the range
    assert kvq.kvq_block_bytes(_desc(kvq, **hq)) == 24 * 128 + 128 + 32 == 3232
    assert kvq.kvq_block_bytes(_desc(kvq, head_dim=64, **hq)) == 24 * 64 + 128 + 16 == 1680
    assert kvq.kvq_block_bytes(_desc(kvq, **{**hq, "k_bits": 8})) == 0
    # Med3x over the HQMQ codec: the same 288-byte outlier section
    assert kvq.kvq_block_bytes(_desc(kvq, outliers=1, **hq)) == 3232 + 288
    assert kvq.kvq_block_bytes(_desc(kvq, head_dim=64, outliers=1, **hq)) == 1680 + 288
    assert kvq.kvq_block_bytes(_desc(kvq, k_rotate=1, rot_signs=0x3000, **hq)) == 0
    d = _desc(kvq, **hq)
    assert kvq.kvq_adaptive_work_size(d, 2, 1, 32, 4) == 0
    # hq_s beyond the decode's shared-memory tables, or no secondary units
    assert _decode(kvq, _desc(kvq, **{**hq, "hq_s": 65})) == kvq.KVQ_ERR_UNSUPPORTED
    assert _decode(kvq, _desc(kvq, **{**hq, "hq_s": 0})) == kvq.KVQ_ERR_UNSUPPORTED
    assert _decode(kvq, _desc(kvq, **{**hq, "hq_sec": None})) == kvq.KVQ_ERR_INVALID_ARG


def test_status_strings(kvq):
    assert kvq.status_string(0) == "KVQ_OK"
    assert kvq.status_string(-5) == "KVQ_ERR_TIMEOUT"
    assert kvq.status_string(99) == "KVQ_UNKNOWN_STATUS"


def _decode(kvq, desc, **kw):
    a = dict(q=0x10, q_dtype=kvq.KVQ_BF16, num_seqs=2, num_queries=1, num_q_heads=32,
             page_table=0x20, max_pages_per_seq=4, seq_lens=0x30, softmax_scale=0.0,
             tau=math.inf, out=0x40, bound=0x50, flags=0x60, workspace=0x70,
             workspace_bytes=1 << 20)
    a.update(kw)
    return kvq.kvq_decode_attention(desc, **a)


def test_validation_before_any_cuda_call(kvq):
    C = kvq
    assert kvq.lib().kvq_decode_attention(None, None, 0, 1, 1, 1, None, 1, None, 0.0, 0.0,
                                          None, None, None, None, 0, None) == C.KVQ_ERR_INVALID_ARG
    assert _decode(kvq, _desc(kvq, head_dim=96)) == C.KVQ_ERR_UNSUPPORTED
    assert _decode(kvq, _desc(kvq, page_size=32)) == C.KVQ_ERR_UNSUPPORTED
    assert _decode(kvq, _desc(kvq, k_rotate=1)) == C.KVQ_ERR_INVALID_ARG      # no signs
    assert _decode(kvq, _desc(kvq, pool=0x1004)) == C.KVQ_ERR_INVALID_ARG     # misaligned
    assert _decode(kvq, _desc(kvq, pool=None)) == C.KVQ_ERR_INVALID_ARG
    assert _decode(kvq, _desc(kvq), num_q_heads=30) == C.KVQ_ERR_INVALID_ARG  # not GQA
    assert _decode(kvq, _desc(kvq), num_queries=2) == C.KVQ_ERR_UNSUPPORTED   # 8 rows
    assert _decode(kvq, _desc(kvq), out=None) == C.KVQ_ERR_INVALID_ARG
    assert _decode(kvq, _desc(kvq), q_dtype=7) == C.KVQ_ERR_INVALID_ARG
    assert _decode(kvq, _desc(kvq), max_pages_per_seq=0) == C.KVQ_ERR_INVALID_ARG
    assert _decode(kvq, _desc(kvq), tau=math.nan) == C.KVQ_ERR_INVALID_ARG
    assert _decode(kvq, _desc(kvq), num_seqs=0) == C.KVQ_OK                  # nothing to do
    assert "num_queries" in kvq.last_error() or kvq.last_error() != ""
    d = _desc(kvq)
    assert kvq.kvq_quantize_append(d, 0x10, 0x20, 5, 0, 0, 0, 1, 1, None, 0x30, 0x40, 1) \
        == C.KVQ_ERR_INVALID_ARG
    assert kvq.kvq_quantize_append(d, None, 0x20, 1, 0, 0, 0, 1, 1, None, 0x30, 0x40, 1) \
        == C.KVQ_ERR_INVALID_ARG
    assert kvq.kvq_quantize_append(d, 0x10, 0x20, 1, -1, 0, 0, 1, 1, None, 0x30, 0x40, 1) \
        == C.KVQ_ERR_INVALID_ARG
    assert kvq.kvq_quantize_append(d, 0x10, 0x20, 1, 0, 0, 0, 0, 1, None, 0x30, 0x40, 1) \
        == C.KVQ_OK


def test_fallback_validation_and_staging_size(kvq):
    d = _desc(kvq)
    scratch = 48 * 8 * (128 + 2) * 4                  # merge scratch, a multiple of 256 B
    assert kvq.kvq_fallback_staging_size(d, kvq.KVQ_BF16, 1000) == scratch + 2 * 1000 * 128 * 2
    assert kvq.kvq_fallback_staging_size(d, kvq.KVQ_F32, 3) == scratch + 2 * 1536
    assert kvq.kvq_fallback_staging_size(d, kvq.KVQ_F32, 0) == scratch
    assert kvq.kvq_fallback_staging_size(d, 9, 10) == 0
    rc, n = kvq.kvq_fallback_exact(d, None, None, kvq.KVQ_BF16, 0, 0, 0x10, kvq.KVQ_BF16, 1, 1,
                                   32, None, 0.0, 0x20, 0x30, 0x40, 0x50, 1 << 20, 0, 0, 100)
    assert rc == kvq.KVQ_ERR_INVALID_ARG and n == 0
    rc, n = kvq.kvq_fallback_exact(d, 0x1, 0x1, 9, 0, 0, 0x10, kvq.KVQ_BF16, 1, 1, 32, 0x1,
                                   0.0, 0x20, 0x30, 0x40, 0x50, 1 << 20, 0, 0, 100)
    assert rc == kvq.KVQ_ERR_INVALID_ARG


def test_fallback_staging_checks_come_before_any_device_call(kvq):
    # (no GPU here: each call must fail on its arguments, not on the device)
    d = _desc(kvq)
    sl = np.array([10, 20], np.int32)
    need = kvq.kvq_fallback_staging_size(d, kvq.KVQ_BF16, 20)

    def call(lens, staging, nbytes):
        return kvq.kvq_fallback_exact(d, 0x100, 0x100, kvq.KVQ_BF16, 0, 0, 0x100, kvq.KVQ_BF16,
                                      2, 1, 32, lens.ctypes.data, 0.0, 0x100, 0x100, 0x100,
                                      staging, nbytes, 0, 0, 100)

    rc, n = call(sl, 0x108, need)
    assert rc == kvq.KVQ_ERR_INVALID_ARG and n == 0 and "aligned" in kvq.last_error()
    rc, n = call(sl, 0x100, need - 1)
    assert rc == kvq.KVQ_ERR_INVALID_ARG and "required" in kvq.last_error()
    rc, n = call(np.array([10, -1], np.int32), 0x100, need)
    assert rc == kvq.KVQ_ERR_INVALID_ARG and "seq_len" in kvq.last_error()
