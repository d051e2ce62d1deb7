"""Host-side pieces of bench.py that need no GPU: the DRAM traffic record is
reported only for the workload, launch and kernel source it was captured on,
and the CPU baseline (the oracle on the host's cores) reports what it ran."""

import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_traffic_record_only_for_its_capture(monkeypatch):
    assert bench._traffic_record("serving", False) is None
    assert bench._traffic_record("llama8b", True) is None
    # the committed record matches the current source
    v = bench._traffic_record("llama8b", False)
    assert v is None or v > 110e6
    # once the kernel source changes (here: another file hashed in its place),
    # the record is no longer used
    monkeypatch.setattr(bench, "DECODE_SRCS", [os.path.join(ROOT, "bench.py")])
    assert bench._traffic_record("llama8b", False) is None


def test_workload_variants():
    assert bench._variant("llama8b") == ("llama8b", "")
    assert bench._variant("llama8b+med3") == ("llama8b", "med3")
    assert bench._variant("llama8b+kqv") == ("llama8b", "kqv")
    assert bench._variant("llama8b+hqmq") == ("llama8b", "hqmq")
    assert "HQMQ" in bench._describe("llama8b+hqmq")
    assert bench._variant("llama8b+hqmq+med3") == ("llama8b", "hqmq+med3")
    assert "Med3x" in bench._describe("llama8b+hqmq+med3")
    assert "Med3x" in bench._describe("serving+med3")
    assert "KQV" in bench._describe("llama8b+kqv")
    for bad in ("llama8b+x", "nosuch", "nosuch+med3"):
        try:
            bench._variant(bad)
        except SystemExit:
            continue
        raise AssertionError(bad)


def test_cpu_baseline_reports_its_sample():
    r = bench.cpu_baseline("tiny", 0, 0.2)
    assert r["kind"] == "oracle" and r["unit"] == bench.UNIT
    assert r["cores"] == 1                       # one kv head: one process
    assert r["value"] > 0 and r["single_core_value"] > 0
    assert r["single_core_codec_value"] > 0 and r["single_core_dense_value"] > 0
    assert "tiny" in r["sample"]
