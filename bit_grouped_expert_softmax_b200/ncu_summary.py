"""Summarise Nsight Compute output into short markdown tables.

    python -m bit_grouped_expert_softmax_b200.ncu_summary launches <launches.csv>
    python -m bit_grouped_expert_softmax_b200.ncu_summary report <raw.csv>
    python -m bit_grouped_expert_softmax_b200.ncu_summary record <raw.csv> <kernel-regex> <name> <workload> <summary.md> <source>...

`launches` reads a `--metrics gpu__time_duration.sum --csv` launch list and
prints, per kernel, the launch count, total and average device time and the
share of the total. `report` reads `ncu -i <rep> --page raw --csv` and prints
the counters used for the roofline (DRAM bytes and throughput, tensor-pipe
activity, issue activity, registers, the largest warp-stall reasons).
`record` stores one kernel's DRAM bytes per launch (read + write, averaged over
the captured launches) in profiles/traffic.json under <name>, with the hash of
the listed source files: bench.py reports the figure only while those sources
are unchanged.
"""

from __future__ import annotations

import collections
import csv
import hashlib
import json
import os
import re
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

_UNITS = {"ns": 1e-3, "nsecond": 1e-3, "us": 1.0, "usecond": 1.0, "ms": 1e3, "msecond": 1e3, "s": 1e6, "second": 1e6}


def _rows(path):
    with open(path) as f:
        lines = [ln for ln in f if not ln.startswith("==")]
    return list(csv.reader(lines))


def _short(name: str) -> str:
    name = re.sub(r"\(.*$", "", name)
    name = name.replace("void ", "").replace("moe::", "").replace("<unnamed>::", "").replace("(anonymous namespace)::", "")
    return name.strip()


# torch's own kernels (fills, the spin kernel that holds a stream while the
# benchmark enqueues its profiled steps) are not the library's
TORCH_PREFIXES = ("at::", "native::", "cuda::spin_kernel")


def launches(path: str, skip_prefix: tuple[str, ...] = TORCH_PREFIXES) -> str:
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


def _num(v: str) -> float:
    return float(v.replace(",", ""))


_BYTES = {"byte": 1.0, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9}


def record(path: str, kernel_re: str, name: str, workload: str, summary: str, sources: list[str]) -> dict:
    rows = _rows(path)
    h, units, data = rows[0], rows[1], rows[2:]
    ki = h.index("Kernel Name")
    ri, wi = h.index("dram__bytes_read.sum"), h.index("dram__bytes_write.sum")
    per = [_num(d[ri]) * _BYTES[units[ri]] + _num(d[wi]) * _BYTES[units[wi]]
           for d in data if re.search(kernel_re, d[ki])]
    if not per:
        raise SystemExit(f"no launch of {kernel_re} in {path}")
    hs = hashlib.sha256()
    for src in sources:
        with open(os.path.join(ROOT, src), "rb") as f:
            hs.update(f.read())
    tpath = os.path.join(ROOT, "profiles", "traffic.json")
    rec = json.load(open(tpath)) if os.path.exists(tpath) else {}
    rec[name] = {"workload": workload, "dram_bytes_per_launch": int(round(sum(per) / len(per))),
                 "sources": sources, "sha": hs.hexdigest()[:16], "from": summary}
    with open(tpath, "w") as f:
        json.dump(rec, f, indent=1)
        f.write("\n")
    return rec[name]


if __name__ == "__main__":
    if len(sys.argv) < 3 or sys.argv[1] not in ("launches", "report", "record"):
        print(__doc__)
        sys.exit(2)
    if sys.argv[1] == "record":
        print(record(sys.argv[2], sys.argv[3], sys.argv[4], sys.argv[5], sys.argv[6], sys.argv[7:]))
    else:
        print(launches(sys.argv[2]) if sys.argv[1] == "launches" else report(sys.argv[2]))
