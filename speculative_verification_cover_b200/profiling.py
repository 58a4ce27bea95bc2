"""Machine-written DRAM-traffic records from ncu captures.

    python -m speculative_verification_cover_b200.profiling RAW_CSV KERNEL WORKLOAD \
        --source csrc/FILE.cu --command "the ncu command that made RAW_CSV"

RAW_CSV is the output of `ncu -i <report> --page raw --csv` (one row per captured
launch). The record for KERNEL -- dram__bytes_read.sum + dram__bytes_write.sum per
launch, averaged over the captured launches of that kernel -- is written to
profiles/traffic.json together with the workload, the command and a hash of the
kernel's source code (comments and layout ignored), so that a reader (bench.py)
can tell whether the figure still describes the current kernel. Nothing here is
edited by hand.
"""
from __future__ import annotations

import argparse
import csv
import hashlib
import json
import os
import re

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
TRAFFIC_JSON = os.path.join(ROOT, "profiles", "traffic.json")

_UNITS = {"byte": 1.0, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9, "Tbyte": 1e12,
          "KB": 1e3, "MB": 1e6, "GB": 1e9}


def _code_only(text: str) -> str:
    """The source with comments removed and whitespace runs collapsed: what the
    compiler sees, so that an edit to a comment does not retire a measurement."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def source_hash(path: str) -> str:
    """Hash of a kernel source's code (comments and layout ignored)."""
    with open(path, encoding="utf-8") as f:
        return hashlib.sha256(_code_only(f.read()).encode()).hexdigest()[:16]


def dram_bytes_per_launch(raw_csv: str, kernel: str):
    """Mean dram read + write bytes of the launches whose name contains `kernel`."""
    with open(raw_csv, newline="") as f:
        rows = [r for r in csv.reader(f) if r]
    # skip ncu's own log lines before the header
    start = next(i for i, r in enumerate(rows) if "Kernel Name" in r)
    head, units, data = rows[start], rows[start + 1], rows[start + 2:]
    col = {name: i for i, name in enumerate(head)}
    name_i = col["Kernel Name"]
    total, n = 0.0, 0
    for r in data:
        if kernel not in r[name_i]:
            continue
        b = 0.0
        for metric in ("dram__bytes_read.sum", "dram__bytes_write.sum"):
            i = col[metric]
            b += float(r[i].replace(",", "")) * _UNITS.get(units[i], 1.0)
        total += b
        n += 1
    if n == 0:
        raise ValueError(f"no launch of {kernel} in {raw_csv}")
    return total / n, n


def record(raw_csv, kernel, workload, source, command, out=TRAFFIC_JSON):
    per_launch, n = dram_bytes_per_launch(raw_csv, kernel)
    src = source if os.path.isabs(source) else os.path.join(HERE, source)
    db = {}
    if os.path.exists(out):
        with open(out) as f:
            db = json.load(f)
    db[f"{kernel}@{workload}"] = {
        "kernel": kernel, "workload": workload, "dram_bytes_per_launch": per_launch,
        "launches": n, "source": os.path.relpath(src, ROOT),
        "source_sha256_16": source_hash(src), "command": command}
    with open(out, "w") as f:
        json.dump(db, f, indent=1, sort_keys=True)
        f.write("\n")
    return db[f"{kernel}@{workload}"]


def lookup(kernel, workload, path=TRAFFIC_JSON):
    """DRAM bytes per launch of `kernel` on `workload`, or None when there is no record
    or the kernel's source has changed since the capture."""
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f).get(f"{kernel}@{workload}")
    if not rec:
        return None
    src = os.path.join(ROOT, rec["source"])
    if not os.path.exists(src) or source_hash(src) != rec["source_sha256_16"]:
        return None
    return rec["dram_bytes_per_launch"]


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("raw_csv")
    ap.add_argument("kernel")
    ap.add_argument("workload")
    ap.add_argument("--source", required=True)
    ap.add_argument("--command", required=True)
    a = ap.parse_args()
    print(json.dumps(record(a.raw_csv, a.kernel, a.workload, a.source, a.command)))
