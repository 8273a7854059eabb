"""The ncu traffic record behind bench.py's roofline `traffic` field (host logic only)."""
import json

from weight_only_int4_06_b200 import ncu_traffic as T

CSV = '''==PROF== Connected to process 1
"ID","Process ID","Process Name","Host Name","Kernel Name","Context","Stream","Block Size","Grid Size","Device","CC","Section Name","Metric Name","Metric Unit","Metric Value"
"0","1","python","h","void at::fill(int)","1","7","(128, 1, 1)","(1, 1, 1)","0","10.0","Command line profiler metrics","dram__bytes_read.sum","byte","64"
"1","1","python","h","void w4::gemv_stream_kernel<1>(int)","1","7","(576, 1, 1)","(148, 1, 1)","0","10.0","Command line profiler metrics","dram__bytes_read.sum","Mbyte","8.5"
"1","1","python","h","void w4::gemv_stream_kernel<1>(int)","1","7","(576, 1, 1)","(148, 1, 1)","0","10.0","Command line profiler metrics","dram__bytes_write.sum","Kbyte","2"
"1","1","python","h","void w4::gemv_stream_kernel<1>(int)","1","7","(576, 1, 1)","(148, 1, 1)","0","10.0","Command line profiler metrics","gpu__time_duration.sum","nsecond","9,248"
"2","1","python","h","void w4::gemv_stream_kernel<1>(int)","1","7","(576, 1, 1)","(148, 1, 1)","0","10.0","Command line profiler metrics","dram__bytes_read.sum","byte","1,000"
"2","1","python","h","void w4::gemv_stream_kernel<1>(int)","1","7","(576, 1, 1)","(148, 1, 1)","0","10.0","Command line profiler metrics","dram__bytes_write.sum","byte","0"
'''


def test_parse_launches_filters_and_scales_units(tmp_path):
    p = tmp_path / "t.csv"
    p.write_text(CSV)
    got = T.parse_launches(str(p), "gemv_stream")
    assert [g[0] for g in got] == [1, 2]
    assert got[0][2]["dram__bytes_read.sum"] == 8.5e6
    assert got[0][2]["dram__bytes_write.sum"] == 2e3
    assert got[0][2]["gpu__time_duration.sum"] == 9248.0
    assert got[1][2]["dram__bytes_read.sum"] == 1000.0


def test_record_is_ignored_once_the_kernel_sources_change(tmp_path, monkeypatch):
    rec = tmp_path / "traffic_decode.json"
    monkeypatch.setattr(T, "record_path", lambda workload: str(rec))
    assert T.load_traffic("decode") is None  # no record
    rec.write_text(json.dumps({"dram_bytes_per_step": 123, "source_sha256": T.source_digest("decode")}))
    assert T.load_traffic("decode") == 123
    rec.write_text(json.dumps({"dram_bytes_per_step": 123, "source_sha256": "0" * 64}))
    assert T.load_traffic("decode") is None


def test_digest_ignores_comments_and_layout_only():
    a = "int f(int x) {  // one\n  return x + 1; /* two\n lines */ }\n"
    b = "int f(int x) {\n    return x + 1;\n}  // edited comment\n"
    c = "int f(int x) { return x + 2; }"
    assert T.code_only(a) == T.code_only(b) != T.code_only(c)
