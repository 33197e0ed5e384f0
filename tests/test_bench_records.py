"""bench.py reports a kernel's DRAM traffic from its committed ncu record
(profiles/traffic.json) only while the kernel's sources hash to the value
stored beside it, and only for the workload the record was captured on."""

from __future__ import annotations

import json
import os
import shutil

import bench


def _copy_tree(tmp_path, sources):
    for rel in [bench.TRAFFIC_RECORDS, *sources]:
        dst = tmp_path / rel
        dst.parent.mkdir(parents=True, exist_ok=True)
        shutil.copy(os.path.join(bench.ROOT, rel), dst)


def _write_record(tmp_path, kernel, workload, nbytes):
    path = tmp_path / bench.TRAFFIC_RECORDS
    recs = json.loads(path.read_text())
    recs[kernel] = {"workload": workload, "traffic_bytes_per_launch": nbytes,
                    "kernel_source_sha256": bench.sources_digest(bench.SOURCES_OF[kernel])}
    path.write_text(json.dumps(recs))


def test_records_parse_and_name_known_kernels():
    with open(os.path.join(bench.ROOT, bench.TRAFFIC_RECORDS)) as f:
        recs = json.load(f)
    for kernel, rec in recs.items():
        assert kernel in bench.SOURCES_OF
        assert int(rec["traffic_bytes_per_launch"]) > 0
        assert len(rec["kernel_source_sha256"]) == 64


def test_matching_sources_give_the_record_and_a_change_voids_it(tmp_path, monkeypatch):
    for kernel in (bench.KERNEL_FWD, bench.KERNEL_FP8):
        _copy_tree(tmp_path, bench.SOURCES_OF[kernel])
        monkeypatch.setattr(bench, "ROOT", str(tmp_path))
        _write_record(tmp_path, kernel, "l128k_h32_causal", 12345)
        assert bench.recorded_traffic("l128k_h32_causal", kernel) == 12345
        assert bench.recorded_traffic("l32k_gqa4_causal", kernel) is None
        with open(tmp_path / bench.SOURCES_OF[kernel][0], "a") as f:
            f.write("\n// changed\n")
        assert bench.recorded_traffic("l128k_h32_causal", kernel) is None
        monkeypatch.undo()


def test_a_missing_record_gives_none(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.recorded_traffic("l128k_h32_causal") is None
