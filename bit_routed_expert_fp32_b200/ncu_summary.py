"""Summaries of ncu command-line captures for the profiles/ folder.

    python -m bit_routed_expert_fp32_b200.ncu_summary launches <launches.csv>
        per kernel: launches, total device time, share (markdown table on stdout)
    python -m bit_routed_expert_fp32_b200.ncu_summary traffic <traffic.csv> <workload> <path> <kernel regex>
        DRAM bytes per launch of the first launch whose name matches; prints the JSON
        record that profiles/traffic.json keeps under <workload> (tied to the current
        source hash of the path's kernel, so a later source change voids it)

The CSV files are what `ncu --metrics ... --csv --log-file F` writes: one row per
(launch, metric) with the metric's unit and value in the last three columns.
"""
from __future__ import annotations

import csv
import json
import re
import sys
from collections import OrderedDict


def _rows(path: str):
    with open(path, newline="") as f:
        lines = [ln for ln in f if ln.startswith('"')]
    rd = csv.reader(lines)
    header = next(rd)
    idx = {h: i for i, h in enumerate(header)}
    for r in rd:
        yield {"id": r[idx["ID"]], "kernel": r[idx["Kernel Name"]], "metric": r[idx["Metric Name"]],
               "unit": r[idx["Metric Unit"]], "value": float(r[idx["Metric Value"]].replace(",", ""))}


def _short(name: str) -> str:
    name = re.sub(r"^void ", "", name)
    name = re.sub(r"\(anonymous namespace\)::|<unnamed>::|unnamed>::|moe::", "", name)
    return re.sub(r"\(.*\)$", "", name).strip()


def _to_us(v: float, unit: str) -> float:
    return {"ns": 1e-3, "usecond": 1.0, "us": 1.0, "msecond": 1e3, "ms": 1e3, "nsecond": 1e-3}.get(unit, 1e-3) * v


def launches(path: str) -> str:
    per = OrderedDict()
    for r in _rows(path):
        if r["metric"] != "gpu__time_duration.sum":
            continue
        k = _short(r["kernel"])
        n, t = per.get(k, (0, 0.0))
        per[k] = (n + 1, t + _to_us(r["value"], r["unit"]))
    total = sum(t for _, t in per.values())
    out = ["| kernel | launches | total us | share | mean us / launch |", "|---|---|---|---|---|"]
    for k, (n, t) in sorted(per.items(), key=lambda kv: -kv[1][1]):
        out.append(f"| {k} | {n} | {t:,.0f} | {100 * t / total:.1f} % | {t / n:,.1f} |")
    return "\n".join(out)


def traffic(path: str, workload: str, which: str, regex: str) -> dict:
    import os
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    got = OrderedDict()
    for r in _rows(path):
        if not re.search(regex, r["kernel"]):
            continue
        got.setdefault(r["id"], {"kernel": _short(r["kernel"])})[r["metric"]] = r["value"]
    first = next(iter(got.values()))
    rd, wr = first["dram__bytes_read.sum"], first["dram__bytes_write.sum"]
    return {workload: {"kernel": first["kernel"], "kernel_hash": bench.kernel_hash(which),
                       "dram_bytes_per_launch": int(rd + wr), "read_bytes": int(rd), "write_bytes": int(wr),
                       "launch_us_under_ncu": _to_us(first.get("gpu__time_duration.sum", 0.0), "ns")}}


if __name__ == "__main__":
    if sys.argv[1] == "launches":
        print(launches(sys.argv[2]))
    else:
        print(json.dumps(traffic(sys.argv[2], sys.argv[3], sys.argv[4], sys.argv[5]), indent=1))
