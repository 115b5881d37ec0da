"""The benchmark's use of the committed ncu records (profiles/traffic.json): a record
is reported only while it was taken on the current decode-kernel sources, and each
record is self-consistent (DRAM bytes within a few percent of the algorithmic bytes,
read + write adding up)."""
import json
import os

import pytest

import bench

RECORDS = os.path.join(os.path.dirname(os.path.dirname(__file__)), "profiles", "traffic.json")


class _Cfg:
    def __init__(self, name):
        self.name = name


def _records():
    with open(RECORDS) as f:
        return json.load(f)


def test_record_is_used_only_with_matching_kernel_sources(monkeypatch):
    rec = _records()["7b_bf16"]
    monkeypatch.setattr(bench, "kernel_sources_sha", lambda: rec["kernel_sources_sha256"])
    assert bench.recorded_traffic(_Cfg("7b_bf16")) == rec["traffic_bytes_per_launch"]
    assert bench.recorded_traffic(_Cfg("no_such_workload")) is None
    monkeypatch.setattr(bench, "kernel_sources_sha", lambda: "0" * 64)
    assert bench.recorded_traffic(_Cfg("7b_bf16")) is None


def test_kernel_hash_covers_the_decode_kernels_only(tmp_path, monkeypatch):
    csrc = tmp_path / "paged_kv_cache_342_b200" / "csrc"
    csrc.mkdir(parents=True)
    for name in ("decode_simt.cuh", "common.cuh", "decoder.cpp", "allocator.cpp"):
        (csrc / name).write_text("x")
    monkeypatch.setattr(bench, "HERE", str(tmp_path))
    h0 = bench.kernel_sources_sha()
    (csrc / "decoder.cpp").write_text("host code changed")
    (csrc / "allocator.cpp").write_text("host code changed")
    assert bench.kernel_sources_sha() == h0
    (csrc / "decode_simt.cuh").write_text("kernel changed")
    assert bench.kernel_sources_sha() != h0


@pytest.mark.parametrize("name", ["7b_bf16", "13b_fp16", "gqa_long_bf16", "prefix_cow_bf16",
                                  "gqa_long_bf16+fp8_cache"])
def test_records_are_consistent(name):
    rec = _records()[name]
    assert rec["read_bytes"] + rec["write_bytes"] > 0
    ratio = (rec["read_bytes"] + rec["write_bytes"]) / rec["algorithmic_bytes_of_capture"]
    assert ratio == pytest.approx(rec["traffic_over_algorithmic"], abs=1e-4)
    # no wasted re-reads; a little below 1 where the small inputs (q, tables, lengths)
    # were still in L2
    assert 0.99 <= ratio < 1.1
    if rec["captured_on"] == name:     # captured at full size
        assert rec["traffic_bytes_per_launch"] == rec["read_bytes"] + rec["write_bytes"]
    assert rec["kernels"]
