"""DRAM-traffic records for bench.py's roofline line.

An ncu capture (``--metrics dram__bytes_read.sum,dram__bytes_write.sum,gpu__time_duration.sum``,
``--csv --log-file``) of ``bench.py`` gives the DRAM bytes of every launch.  This module sums the
first ``launches_per_step`` launches of the kernel family a workload times (one step) and writes
``profiles/traffic_<workload>.json`` together with a digest of that kernel's sources.  bench.py
reports the number only while the digest still matches, so a kernel edited after the capture
reports no traffic.

    python -m weight_only_int4_06_b200.ncu_traffic --workload decode --csv traffic.csv \\
        --kernel gemv_stream --launches-per-step 4 --command "<the ncu command line>"
"""
from __future__ import annotations

import argparse
import csv
import hashlib
import json
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# Kernel sources whose DRAM counters a traffic record belongs to.
KERNEL_SOURCES = {
    "decode": ["weight_only_int4_06_b200/csrc/gemv_stream.cu", "weight_only_int4_06_b200/csrc/sm100.cuh",
               "weight_only_int4_06_b200/csrc/common.cuh"],
    "prefill": ["weight_only_int4_06_b200/csrc/gemm_tc.cu", "weight_only_int4_06_b200/csrc/sm100.cuh",
                "weight_only_int4_06_b200/csrc/common.cuh"],
}


_COMMENT = re.compile(r"/\*.*?\*/|//[^\n]*", re.S)


def code_only(text: str) -> str:
    """C/C++ source without comments and with whitespace collapsed: what the compiler sees."""
    return " ".join(_COMMENT.sub(" ", text).split())


def source_digest(workload: str) -> str:
    """Digest of the kernel sources' code (comments and layout excluded, so a record stays valid
    across comment edits and goes stale on any change to the code)."""
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[workload]:
        with open(os.path.join(ROOT, f), encoding="utf-8") as fh:
            h.update(f.encode() + b"\0" + code_only(fh.read()).encode())
    return h.hexdigest()


def record_path(workload: str) -> str:
    return os.path.join(ROOT, "profiles", f"traffic_{workload}.json")


def load_traffic(workload: str):
    """DRAM bytes per step, or None (no record, or the kernel sources changed since)."""
    try:
        with open(record_path(workload)) as f:
            rec = json.load(f)
        if rec.get("source_sha256") != source_digest(workload):
            return None
        return int(rec["dram_bytes_per_step"])
    except (OSError, KeyError, ValueError):
        return None


def parse_launches(csv_path: str, kernel_regex: str):
    """[(id, name, {metric: value})] of the launches whose kernel name matches, in launch order."""
    with open(csv_path, newline="") as f:
        lines = [ln for ln in f if ln.startswith('"')]  # ncu prefixes the table with log lines
    rows = list(csv.reader(lines))
    hdr = rows[0]
    col = {k: hdr.index(k) for k in ("ID", "Kernel Name", "Metric Name", "Metric Unit", "Metric Value")}
    pat = re.compile(kernel_regex)
    out = {}
    for r in rows[1:]:
        if len(r) != len(hdr) or not pat.search(r[col["Kernel Name"]]):
            continue
        lid = int(r[col["ID"]])
        val = float(r[col["Metric Value"]].replace(",", ""))
        unit = r[col["Metric Unit"]].strip().lower()
        scale = {"byte": 1, "kbyte": 1e3, "mbyte": 1e6, "gbyte": 1e9}.get(unit, 1)
        if r[col["Metric Name"]].startswith("dram__bytes"):
            val *= scale
        out.setdefault(lid, (r[col["Kernel Name"]], {}))[1][r[col["Metric Name"]]] = val
    return [(k, v[0], v[1]) for k, v in sorted(out.items())]


def main():
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--workload", required=True, choices=sorted(KERNEL_SOURCES))
    ap.add_argument("--csv", required=True)
    ap.add_argument("--kernel", required=True, help="regex on the kernel name")
    ap.add_argument("--launches-per-step", type=int, required=True)
    ap.add_argument("--command", required=True, help="the ncu command line that wrote the CSV")
    a = ap.parse_args()
    launches = parse_launches(a.csv, a.kernel)[: a.launches_per_step]
    if len(launches) < a.launches_per_step:
        raise SystemExit(f"only {len(launches)} matching launches in {a.csv}")
    per = [{"id": i, "kernel": n, "dram_read": int(m["dram__bytes_read.sum"]),
            "dram_write": int(m["dram__bytes_write.sum"]),
            "duration_ns": m.get("gpu__time_duration.sum")} for i, n, m in launches]
    rec = {"workload": a.workload, "command": a.command,
           "dram_bytes_per_step": sum(p["dram_read"] + p["dram_write"] for p in per),
           "launches": per, "source_files": KERNEL_SOURCES[a.workload],
           "source_sha256": source_digest(a.workload)}
    with open(record_path(a.workload), "w") as f:
        json.dump(rec, f, indent=1)
    print(json.dumps({k: rec[k] for k in ("workload", "dram_bytes_per_step")}))


if __name__ == "__main__":
    main()
