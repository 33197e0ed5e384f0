"""bench.py reports a kernel's DRAM traffic from its committed ncu record
only while the kernel's sources hash to the value stored beside it, and only
for the workload the record was captured on."""

from __future__ import annotations

import os
import shutil

import bench


def _copy_tree(tmp_path, record, sources):
    for rel in [record, *sources]:
        dst = tmp_path / rel
        dst.parent.mkdir(parents=True, exist_ok=True)
        shutil.copy(os.path.join(bench.ROOT, rel), dst)


def test_committed_records_match_the_sources():
    assert bench.recorded_traffic("l128k_h32_causal") is not None
    assert bench.recorded_traffic("l128k_h32_causal", bench.FP8_TRAFFIC_RECORD,
                                  bench.FP8_KERNEL_SOURCES) is not None


def test_other_workloads_get_no_traffic():
    assert bench.recorded_traffic("l32k_gqa4_causal") is None


def test_a_changed_source_voids_the_record(tmp_path, monkeypatch):
    for record, sources in ((bench.TRAFFIC_RECORD, bench.KERNEL_SOURCES),
                            (bench.FP8_TRAFFIC_RECORD, bench.FP8_KERNEL_SOURCES)):
        _copy_tree(tmp_path, record, sources)
        monkeypatch.setattr(bench, "ROOT", str(tmp_path))
        before = bench.recorded_traffic("l128k_h32_causal", record, sources)
        assert before is not None and before > 0
        with open(tmp_path / sources[0], "a") as f:
            f.write("\n// changed\n")
        assert bench.recorded_traffic("l128k_h32_causal", record, sources) is None
        monkeypatch.undo()


def test_a_missing_record_gives_none(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.recorded_traffic("l128k_h32_causal") is None
