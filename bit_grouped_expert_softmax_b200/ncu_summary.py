"""Summarise Nsight Compute output into short markdown tables.

    python -m bit_grouped_expert_softmax_b200.ncu_summary launches <launches.csv> [--skip-prefix at::]
    python -m bit_grouped_expert_softmax_b200.ncu_summary report <raw.csv>

`launches` reads a `--metrics gpu__time_duration.sum --csv` launch list and
prints, per kernel, the launch count, total and average device time and the
share of the total. `report` reads `ncu -i <rep> --page raw --csv` and prints
the counters used for the roofline (DRAM bytes and throughput, tensor-pipe
activity, issue activity, registers, the largest warp-stall reasons).
"""

from __future__ import annotations

import collections
import csv
import re
import sys

_UNITS = {"ns": 1e-3, "nsecond": 1e-3, "us": 1.0, "usecond": 1.0, "ms": 1e3, "msecond": 1e3, "s": 1e6, "second": 1e6}


def _rows(path):
    with open(path) as f:
        lines = [ln for ln in f if not ln.startswith("==")]
    return list(csv.reader(lines))


def _short(name: str) -> str:
    name = re.sub(r"\(.*$", "", name)
    name = name.replace("void ", "").replace("moe::", "").replace("<unnamed>::", "").replace("(anonymous namespace)::", "")
    return name.strip()


def launches(path: str, skip_prefix: tuple[str, ...] = ("at::",)) -> str:
    rows = _rows(path)
    hdr = next(i for i, r in enumerate(rows) if "Kernel Name" in r)
    h = rows[hdr]
    ki, vi, ui = h.index("Kernel Name"), h.index("Metric Value"), h.index("Metric Unit")
    agg = collections.defaultdict(list)
    for r in rows[hdr + 1:]:
        if len(r) <= vi or not r[vi]:
            continue
        name = _short(r[ki])
        if any(name.startswith(p) for p in skip_prefix):
            continue
        agg[name].append(float(r[vi].replace(",", "")) * _UNITS.get(r[ui], 1.0))
    tot = sum(sum(v) for v in agg.values()) or 1.0
    out = ["| kernel | launches | total us | avg us | share |", "|---|---:|---:|---:|---:|"]
    for k, v in sorted(agg.items(), key=lambda kv: -sum(kv[1])):
        out.append(f"| {k} | {len(v)} | {sum(v):.1f} | {sum(v) / len(v):.2f} | {sum(v) / tot:.3f} |")
    return "\n".join(out)


_KEYS = [
    "gpu__time_duration.sum",
    "dram__bytes_read.sum",
    "dram__bytes_write.sum",
    "gpu__dram_throughput.avg.pct_of_peak_sustained_elapsed",
    "sm__pipe_tensor_cycles_active.avg.pct_of_peak_sustained_active",
    "sm__inst_executed_pipe_tensor.avg.pct_of_peak_sustained_active",
    "sm__issue_active.avg.pct_of_peak_sustained_elapsed",
    "sm__warps_active.avg.pct_of_peak_sustained_active",
    "lts__throughput.avg.pct_of_peak_sustained_elapsed",
    "l1tex__data_bank_conflicts_pipe_lsu_mem_shared.sum",
    "launch__registers_per_thread",
    "launch__grid_size",
    "launch__block_size",
]


def report(path: str, top_stalls: int = 6) -> str:
    rows = _rows(path)
    h, units, data = rows[0], rows[1], rows[2:]
    out = []
    for d in data:
        out.append(f"### {_short(d[h.index('Kernel Name')])}")
        out.append("| counter | value |")
        out.append("|---|---:|")
        for k in _KEYS:
            if k in h:
                i = h.index(k)
                out.append(f"| {k} | {d[i]} {units[i]} |")
        st = []
        for i, k in enumerate(h):
            if k.startswith("smsp__average_warps_issue_stalled") and k.endswith("_per_issue_active.ratio"):
                try:
                    st.append((float(d[i].replace(",", "")), k))
                except ValueError:
                    pass
        for v, k in sorted(st, reverse=True)[:top_stalls]:
            out.append(f"| {k} | {v:.3f} |")
        out.append("")
    return "\n".join(out)


if __name__ == "__main__":
    if len(sys.argv) < 3 or sys.argv[1] not in ("launches", "report"):
        print(__doc__)
        sys.exit(2)
    print(launches(sys.argv[2]) if sys.argv[1] == "launches" else report(sys.argv[2]))
