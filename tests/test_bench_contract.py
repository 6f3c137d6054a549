"""bench.py's JSON contract and roofline arithmetic, on CPU (the reference arm only runs the oracle)."""

import json
import os
import subprocess
import sys

import numpy as np
import pytest

import bench
import oracle
from bit_grouped_expert_softmax_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PEAKS = {"hbm_gbs": 6558.4, "bf16_tflops": 1653.4}


@pytest.mark.parametrize("name", ["tiny", "decode"])
def test_touched_experts_follow_the_routing_definition(name):
    inp = synth.make_workload(name)
    ids = oracle.route(inp.logits, inp.k)[0]
    assert bench.touched_experts(inp) == len(np.unique(ids)) + 1


def test_roofline_of_an_hbm_bound_kernel():
    inp = synth.make_workload("decode")
    rf = bench.roofline_numbers(inp, PEAKS)
    assert rf["bound"] == "hbm" and rf["touched"] == 9
    assert rf["weight_bytes"] == 9 * synth.expert_bytes(2048, 512) == 15925248
    r = {"rf": rf, "prof": {"small_t": (20.0, 1000)}, "workload": "decode"}  # ms over launches: 20 us each
    o = bench.roofline_obj(r, PEAKS, "measured")
    assert o["bound"] == "hbm" and o["unit"] == "GB/s" and o["kernel"] == "small_t"
    assert o["achieved"] == pytest.approx(15925248 / 20e-6 / 1e9, rel=1e-3)
    assert o["frac"] == pytest.approx(o["achieved"] / PEAKS["hbm_gbs"], rel=1e-3)
    assert set(o) >= {"bound", "achieved", "peak", "unit", "frac", "traffic"}


def test_roofline_of_a_tensor_bound_kernel_takes_its_share_of_the_flops():
    inp = synth.make_workload("zipf")
    rf = bench.roofline_numbers(inp, PEAKS)
    assert rf["bound"] == "tensor"
    # the gate/up GEMM does two of the expert's three matrix products
    r = {"rf": rf, "prof": {"gate_up": (0.230, 1), "down": (0.170, 1)}, "workload": "zipf"}  # ms, launches
    o = bench.roofline_obj(r, PEAKS, "measured")
    assert o["kernel"] == "gate_up" and o["unit"] == "TFLOP/s"
    assert o["achieved"] == pytest.approx(rf["flops"] * 2 / 3 / 230e-6 / 1e12, rel=1e-3)


def test_one_launch_step_takes_the_graph_timed_step_as_the_kernel_time():
    """A step of one launch: the graph-timed step bounds the kernel's own time,
    so the roofline uses it even where eager event times are longer."""
    inp = synth.make_workload("decode")
    rf = bench.roofline_numbers(inp, PEAKS)
    r = {"rf": rf, "prof": {"small_t": (23.0, 1000)}, "workload": "decode", "launches_per_step": 1,
         "ms_per_step": 0.0125}
    o = bench.roofline_obj(r, PEAKS, "measured")
    assert o["kernel_avg_us"] == pytest.approx(12.5)
    assert o["achieved"] == pytest.approx(rf["weight_bytes"] / 12.5e-6 / 1e9, rel=1e-3)
    assert "graph" in o["kernel_timing"]


def test_stack_roofline_is_per_layer_launch():
    """The stack's totals cover all its layers; one gate/up launch is one layer's."""
    inp = synth.make_workload("zipf")
    rf = dict(bench.roofline_numbers(inp, PEAKS))
    rf["flops"] *= 40
    rf["weight_bytes"] *= 40
    r = {"rf": rf, "prof": {"gate_up": (0.230 * 40, 40), "down": (0.17 * 40, 40)}, "workload": "stack",
         "layers": 40, "launches_per_step": 280, "ms_per_step": 20.0}
    o = bench.roofline_obj(r, PEAKS, "measured")
    assert o["algorithmic_per_launch"]["flops"] == pytest.approx(rf["flops"] / 40 * 2 / 3)
    assert o["kernel_avg_us"] == pytest.approx(230.0)


def _run(args, env_extra=None):
    env = dict(os.environ)
    env.update(env_extra or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True,
                          text=True, env=env, timeout=600, cwd=ROOT)


def test_reference_arm_prints_one_contract_line():
    p = _run(["--impl", "reference", "--workload", "tiny", "--steps", "2", "--warmup", "3"])
    assert p.returncode == 0, p.stderr
    lines = [ln for ln in p.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 2 and d["warmup"] == 3 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    assert d["config"]["workload"].startswith("tiny")


def test_reference_arm_other_ranks_exit_quietly():
    p = _run(["--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "3"],
             {"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert p.returncode == 0, p.stderr
    assert not [ln for ln in p.stdout.splitlines() if ln.startswith("{")]
