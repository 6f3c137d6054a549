"""The Nsight Compute summary tool: launch shares and the traffic record bench.py reads (CPU only)."""

import json
import os

import pytest

from bit_grouped_expert_softmax_b200 import ncu_summary


def _write(path, rows):
    with open(path, "w") as f:
        for r in rows:
            f.write(",".join(f'"{v}"' for v in r) + "\n")


def test_launch_list_shares(tmp_path):
    p = tmp_path / "launches.csv"
    _write(p, [["ID", "Kernel Name", "Metric Name", "Metric Unit", "Metric Value"],
               ["0", "void moe::k1(int)", "gpu__time_duration.sum", "us", "30"],
               ["1", "void moe::k2(int)", "gpu__time_duration.sum", "ns", "10000"],
               ["2", "void moe::k1(int)", "gpu__time_duration.sum", "us", "30"],
               ["3", "at::fill_kernel", "gpu__time_duration.sum", "us", "999"]])
    table = ncu_summary.launches(str(p))
    assert "| k1 | 2 | 60.0 | 30.00 | 0.857 |" in table
    assert "| k2 | 1 | 10.0 | 10.00 | 0.143 |" in table
    assert "fill" not in table


def test_record_averages_launches_and_hashes_sources(tmp_path, monkeypatch):
    root = tmp_path
    os.makedirs(root / "profiles")
    src = root / "k.cu"
    src.write_text("kernel source")
    raw = root / "raw.csv"
    _write(raw, [["Kernel Name", "dram__bytes_read.sum", "dram__bytes_write.sum"],
                 ["", "Mbyte", "Kbyte"],
                 ["moe::gemm_x(a)", "2.0", "500"],
                 ["moe::other(a)", "9.0", "9"],
                 ["moe::gemm_x(a)", "4.0", "1500"]])
    monkeypatch.setattr(ncu_summary, "ROOT", str(root))
    rec = ncu_summary.record(str(raw), "gemm_x", "gx", "zipf", "profiles/x.md", ["k.cu"])
    assert rec["dram_bytes_per_launch"] == int((2.0e6 + 0.5e6 + 4.0e6 + 1.5e6) / 2)
    stored = json.load(open(root / "profiles" / "traffic.json"))["gx"]
    assert stored == rec and stored["workload"] == "zipf" and stored["sources"] == ["k.cu"]
    # the hash follows the sources: bench.py reads the figure only while they are unchanged
    src.write_text("kernel source, changed")
    rec2 = ncu_summary.record(str(raw), "gemm_x", "gx", "zipf", "profiles/x.md", ["k.cu"])
    assert rec2["sha"] != rec["sha"]


def test_record_rejects_a_missing_kernel(tmp_path, monkeypatch):
    raw = tmp_path / "raw.csv"
    _write(raw, [["Kernel Name", "dram__bytes_read.sum", "dram__bytes_write.sum"], ["", "byte", "byte"],
                 ["moe::a(x)", "1", "1"]])
    monkeypatch.setattr(ncu_summary, "ROOT", str(tmp_path))
    with pytest.raises(SystemExit):
        ncu_summary.record(str(raw), "gemm_x", "gx", "zipf", "x.md", [])
