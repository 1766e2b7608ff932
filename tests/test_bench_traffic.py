"""The bench's attention-traffic lookup: the committed ncu figures are reported
only for the workloads they were captured on, and only while the attention
kernel's source is the one that was profiled."""

import hashlib
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _sha():
    src = os.path.join(ROOT, "block_sparse_attention_stem_b200", "csrc", "k_bsa.cu")
    return hashlib.sha256(open(src, "rb").read()).hexdigest()


def _write(tmp_path, sha):
    p = tmp_path / "traffic.txt"
    p.write_text("# comment\n"
                 "workload long128k\n"
                 f"source_sha256 {sha}\n"
                 "bytes_per_launch_full_workload 1000\n"
                 "bytes_per_launch long128k:fp8 600\n")
    return str(p)


def test_records_by_workload(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "TRAFFIC_FILE", _write(tmp_path, _sha()))
    assert bench.bsa_traffic_per_launch("long128k") == 1000.0
    assert bench.bsa_traffic_per_launch("long128k:fp8") == 600.0
    assert bench.bsa_traffic_per_launch("qwen32k") is None


def test_stale_source_gives_none(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "TRAFFIC_FILE", _write(tmp_path, "0" * 64))
    assert bench.bsa_traffic_per_launch("long128k") is None
    assert bench.bsa_traffic_per_launch("long128k:fp8") is None


def test_missing_file_gives_none(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(tmp_path / "absent.txt"))
    assert bench.bsa_traffic_per_launch("long128k") is None

