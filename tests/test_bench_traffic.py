"""Host logic of the bench's DRAM-traffic figure (CPU): the recorded ncu bytes are reported only
while the fused kernel's code hashes to the captured build, and the hash ignores comments and
whitespace."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _tree(tmp_path, text):
    d = tmp_path / "spatial_sparse_attention_b200" / "csrc"
    d.mkdir(parents=True, exist_ok=True)
    (d / "k.cu").write_text(text)
    return str(tmp_path)


def test_hash_ignores_comments_and_whitespace_only(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "KERNEL_SOURCES", ("k.cu",))
    monkeypatch.setattr(bench, "ROOT", _tree(tmp_path, "int f(int a) { return a + 1; }\n"))
    base = bench.kernel_sources_sha256()
    monkeypatch.setattr(bench, "ROOT", _tree(tmp_path, "// note\nint  f(int a)\n{\n  return a + 1;  // one more\n}\n"))
    assert bench.kernel_sources_sha256() == base
    monkeypatch.setattr(bench, "ROOT", _tree(tmp_path, "int f(int a) { return a + 2; }\n"))
    assert bench.kernel_sources_sha256() != base


def test_traffic_is_reported_only_for_the_captured_build(monkeypatch):
    current = bench.kernel_sources_sha256()
    rec = {"sources_sha256": current, "config": "pass3", "bytes_per_head": 1000.0}
    monkeypatch.setattr(bench, "KERNEL_TRAFFIC", rec)
    assert bench.kernel_traffic("pass3", 22) == 22000.0     # scaled by the heads of the launch
    assert bench.kernel_traffic("small", 22) is None        # another workload
    assert "scaled" in bench.traffic_source("pass3")
    monkeypatch.setattr(bench, "KERNEL_TRAFFIC", dict(rec, sources_sha256="0" * 64))
    assert bench.kernel_traffic("pass3", 22) is None        # the kernel changed since the capture
    assert bench.traffic_source("pass3").startswith("null")
    monkeypatch.setattr(bench, "KERNEL_TRAFFIC", dict(rec, bytes_per_head=None))
    assert bench.kernel_traffic("pass3", 22) is None
