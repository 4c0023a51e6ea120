"""The benchmark's DRAM-traffic records: a committed ncu figure is reported only while the kernel's source
files are the ones it was captured on (hash check), and the committed records match the current sources."""
import json
import os
import shutil
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


@pytest.mark.parametrize("workload", sorted(bench.TRAFFIC))
def test_committed_traffic_records_match_the_kernel_sources(workload):
    path, srcs = bench.TRAFFIC[workload]
    rec = json.load(open(os.path.join(ROOT, path)))
    assert rec["source_sha256"] == bench.source_hash(srcs), f"{path} was captured on other sources: re-capture"
    assert bench.kernel_traffic(path, srcs) == rec["dram_bytes_per_launch_full"]
    assert rec["dram_bytes_per_launch_full"] == rec["dram_bytes_read"] + rec["dram_bytes_write"]
    assert 0 < rec["dram_bytes_per_launch_full"] <= 1.5 * rec["algorithmic_bytes_per_launch"]


def test_traffic_is_dropped_when_the_sources_change(tmp_path, monkeypatch):
    path, srcs = bench.TRAFFIC["large"]
    # a copy of the repository's files with one source byte changed
    for rel in (path,) + tuple(srcs):
        dst = tmp_path / rel
        dst.parent.mkdir(parents=True, exist_ok=True)
        shutil.copy(os.path.join(ROOT, rel), dst)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.kernel_traffic(path, srcs) is not None
    with open(tmp_path / srcs[0], "ab") as f:
        f.write(b"\n// edited\n")
    assert bench.kernel_traffic(path, srcs) is None
