"""The ncu traffic record behind bench.py's roofline `traffic` field (host logic only)."""
import json
import os

import bench


def test_record_is_ignored_once_the_kernel_sources_change(tmp_path, monkeypatch):
    rec = tmp_path / "traffic_decode.json"
    monkeypatch.setattr(bench, "traffic_record_path", lambda workload: str(rec))
    assert bench.load_traffic("decode") is None  # no record
    rec.write_text(json.dumps({"dram_bytes_per_step": 123, "source_sha256": bench.source_digest("decode")}))
    assert bench.load_traffic("decode") == 123
    rec.write_text(json.dumps({"dram_bytes_per_step": 123, "source_sha256": "0" * 64}))
    assert bench.load_traffic("decode") is None


def test_digest_ignores_comments_and_layout_only():
    a = "int f(int x) {  // one\n  return x + 1; /* two\n lines */ }\n"
    b = "int f(int x) {\n    return x + 1;\n}  // edited comment\n"
    c = "int f(int x) { return x + 2; }"
    assert bench.code_only(a) == bench.code_only(b) != bench.code_only(c)


def test_every_recorded_source_exists():
    for files in bench.KERNEL_SOURCES.values():
        for f in files:
            assert os.path.exists(os.path.join(bench.ROOT, f)), f
