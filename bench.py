"""Benchmark of the routed int4 MoE layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl b200|reference]
                    [--workload decode|prefill|zipf|tiny|stack] [--no-extra]
                    [--regions R] [--region-ms MS]

One step = one MoE layer (routing, gate/up, down, combine) over one batch of
synthetic inputs already resident in HBM. The headline workload is the decode
layer (T=1, H=2048, E=256, top-8, I=Is=512); the prefill (T=512) and uneven
Zipf (T=4096) layers and the 40-layer T=8192 stack are measured the same way
and reported under "extra" (a stack step is one pass over all 40 layers).
Weights rotate over device replicas whose touched bytes exceed 4x the L2, so
every step reads its weights from HBM.

Timing: a CUDA graph of consecutive steps is replayed until one timed region
holds at least K steps and --region-ms of device time; R regions are timed
with CUDA events on the launching stream and the median is reported
("steps" = steps per region).

Multi-GPU: one process per GPU; each rank runs its own batch (tokens are
independent), no collective on the data path; value = all ranks' tokens over
the slowest rank's time ("scaling": "weak").

--impl reference times the fp64 CPU oracle on bounded samples of the same
workload, on the host cores.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from bit_grouped_expert_softmax_b200 import synth  # noqa: E402

METRIC = "MoE-layer tokens/s"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def reduce_max(value: float, world: int, device=None) -> float:
    """Maximum of a per-rank value over all ranks (device time: the slowest rank)."""
    if world <= 1:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_tokens_s(tokens_per_rank: int, world: int, ms_per_step: float) -> float:
    """Tokens all ranks processed per second, timed by the slowest rank."""
    return tokens_per_rank * world / (ms_per_step * 1e-3)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


# ----------------------------------------------------------------------------
# clocks sampling during the timed region
# ----------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------
# workloads
# ----------------------------------------------------------------------------

def touched_experts(inp):
    """Distinct routed experts the batch touches (+1 for the shared expert).

    Counted from the logits with a stable argsort, the generator's own view of
    which experts a token's largest logits select."""
    order = np.argsort(-inp.logits, axis=1, kind="stable")[:, :inp.k]
    return len(np.unique(order)) + 1


# Layers whose logits come from a router weight (the router scores computed by
# the library ahead of the routing), on the sizes and seeds of a base workload.
ROUTER_WORKLOADS = {"decode_router": "decode", "prefill_router": "prefill"}


def make_inputs(name):
    """(LayerInputs, router weight or None) of a benchmark workload."""
    if name in ROUTER_WORKLOADS:
        wl = synth.WORKLOADS[ROUTER_WORKLOADS[name]]
        return synth.make_router_layer(wl.T, wl.H, wl.E, wl.k, wl.I, wl.Is, wl.seed, wl.logit_std)
    return synth.make_workload(name), None


def roofline_numbers(inp, peaks, router_w=None):
    ex = touched_experts(inp)
    wbytes = ex * synth.expert_bytes(inp.H, inp.I)
    flops = synth.layer_flops(inp.T, inp.H, inp.k, inp.I)
    if router_w is not None:  # the router weight is read once, its scores are a dense product
        wbytes += router_w.size * 2
        flops += 2.0 * inp.T * inp.E * inp.H
    t_hbm = wbytes / (peaks["hbm_gbs"] * 1e9)
    t_tc = flops / (peaks["bf16_tflops"] * 1e12)
    return dict(touched=ex, weight_bytes=wbytes, flops=flops, t_hbm=t_hbm, t_tc=t_tc,
                bound="hbm" if t_hbm >= t_tc else "tensor")


def median_region_ms(run_region, regions, world, dev, stream, clk=None):
    """Median over ``regions`` timed regions of one region's device time (CUDA
    events on the launching stream, barrier + synchronize on both sides),
    then the maximum of that median over the ranks."""
    import torch
    times = []
    for _ in range(regions):
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        run_region()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        times.append(e0.elapsed_time(e1))
    return reduce_max(statistics.median(times), world, dev), times


def profile_kernels(api, plan, step, n_steps, stream, launches_per_step):
    """Per-kernel device times of n_steps eager steps. The stream is first held
    by a spin kernel long enough for the host to enqueue every step, so the
    library's per-kernel CUDA events measure the kernels back to back on the
    device and not the host's launch latency."""
    import torch
    api.moe_profile_enable(plan.handle, launches_per_step * n_steps + 8)
    torch.cuda.synchronize()
    torch.cuda._sleep(int(2e8))  # ~0.1 s at 2 GHz, on the current (launching) stream
    for i in range(n_steps):
        step(i)
    prof = api.moe_profile_read(plan.handle, stream)
    api.moe_profile_enable(plan.handle, 0)
    return prof


def run_gpu(args, rank, world, local_rank):
    import torch
    from bit_grouped_expert_softmax_b200 import api

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    peaks, peaks_kind = load_peaks()
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size

    def measure_stack(steps, warmup):
        """One step = the whole stack of layers over one T-token chunk (x reset
        from a device copy first, since the stack updates x in place)."""
        wl = synth.WORKLOADS["stack"]
        layers, logits, rfs = [], [], []
        for l in range(wl.layers):
            inp = synth.make_stack_layer(wl, l)
            layers.append(api.DeviceLayer.from_inputs(inp, dev))
            logits.append(inp.logits)
            rfs.append(roofline_numbers(inp, peaks))
            del inp
        rf = dict(rfs[0])
        rf["weight_bytes"] = sum(r["weight_bytes"] for r in rfs)
        rf["flops"] = sum(r["flops"] for r in rfs)
        rf["t_hbm"] = rf["weight_bytes"] / (peaks["hbm_gbs"] * 1e9)
        rf["t_tc"] = rf["flops"] / (peaks["bf16_tflops"] * 1e12)
        rf["bound"] = "hbm" if rf["t_hbm"] >= rf["t_tc"] else "tensor"
        x0 = torch.from_numpy(synth.make_stack_x(wl).view(np.int16)).to(dev)
        x = x0.clone()
        dlog = torch.from_numpy(np.stack(logits)).to(dev)
        del logits
        plan = api.Plan(wl.T, wl.H, wl.E, wl.k, wl.I, wl.Is)
        stream = torch.cuda.Stream(dev)
        torch.cuda.set_stream(stream)

        def step(i):
            x.copy_(x0)
            api.moe_stack_forward(plan.handle, wl.layers, wl.T, x, dlog, layers, stream)

        for i in range(warmup):
            step(i)
        plan.status_sync(stream)
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        step(0)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        per = max(e0.elapsed_time(e1), 1e-3)
        n_steps = max(steps, int(np.ceil(args.region_ms / per)))

        def region():
            for i in range(n_steps):
                step(i)

        with ClockSampler(local_rank) as clk:
            ms_region, all_regions = median_region_ms(region, args.regions, world, dev, stream)
        plan.status_sync(stream)
        ms_step = ms_region / n_steps
        prof = profile_kernels(api, plan, step, 1, stream, 7 * wl.layers)
        plan.status_sync(stream)
        res = dict(workload="stack", T=wl.T, ms_per_step=ms_step, tokens_s=whole_job_tokens_s(wl.T, world, ms_step),
                   rf=rf, achieved_gbs=rf["weight_bytes"] / (ms_step * 1e-3) / 1e9,
                   achieved_tflops=rf["flops"] / (ms_step * 1e-3) / 1e12, n_rep=1, graph=False,
                   timed_steps=n_steps, regions=[round(t, 4) for t in all_regions], clocks=clk.summary(),
                   e2e_tokens_s=None, h2d=0, d2h=0, launches=7 * wl.layers * n_steps, inp=None, prof=prof,
                   layers=wl.layers, launches_per_step=7 * wl.layers)
        plan.close()
        del layers, dlog
        torch.cuda.empty_cache()
        return res

    def measure(name, steps, warmup):
        if name == "stack":
            return measure_stack(steps, warmup)
        inp, router_w = make_inputs(name)
        base = api.DeviceLayer.from_inputs(inp, dev)
        x = torch.from_numpy(inp.x.view(np.int16)).to(dev)
        plan = api.Plan(inp.T, inp.H, inp.E, inp.k, inp.I, inp.Is)
        wr = None
        if router_w is not None:
            # the touched experts follow the library's own scores
            wr = torch.from_numpy(router_w.view(np.int16)).to(dev)
            lg = torch.empty((inp.T, inp.E), dtype=torch.float32, device=dev)
            api.moe_router_logits(plan.handle, inp.T, x, wr, lg)
            plan.status_sync()
            inp.logits = lg.cpu().numpy()
        rf = roofline_numbers(inp, peaks, router_w)
        layer_bytes = sum(t.numel() * t.element_size() for t in base.args())
        touched = max(rf["weight_bytes"], 1)
        n_rep = int(min(32, max(2, -(-4 * l2 // touched))))
        n_rep = int(min(n_rep, max(2, (40 << 30) // layer_bytes)))
        if args.replicas:
            n_rep = args.replicas
        reps = [base] + [api.DeviceLayer(*[t.clone() for t in base.args()]) for _ in range(n_rep - 1)]
        rep_ptrs = [[t.data_ptr() for t in r.args()] for r in reps]
        logits = torch.from_numpy(inp.logits).to(dev)
        out = torch.empty_like(x)
        stream = torch.cuda.Stream(dev)  # graphs cannot be captured on the default stream
        torch.cuda.set_stream(stream)

        def step(i):
            if wr is None:
                api.moe_forward(plan.handle, inp.T, x, logits, *rep_ptrs[i % n_rep], out, stream)
            else:
                api.moe_forward_router(plan.handle, inp.T, x, wr, *rep_ptrs[i % n_rep], out, stream)

        for i in range(warmup):
            step(i)
        plan.status_sync(stream)
        # per-kernel device times (and the number of launches one step makes)
        prof = profile_kernels(api, plan, step, max(n_rep, 8), stream, 8)
        plan.status_sync(stream)
        launches_per_step = max(1, round(sum(n for _, n in prof.values()) / max(n_rep, 8)))
        # CUDA graph of n_rep consecutive steps (one pass over the replicas)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(n_rep):
                step(i)
        g.replay()
        torch.cuda.synchronize(dev)
        plan.status_sync(stream)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(4):
            g.replay()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        per_replay = max(e0.elapsed_time(e1) / 4, 1e-4)
        replays = max(-(-steps // n_rep), int(np.ceil(args.region_ms / per_replay)))
        if world > 1:  # every rank replays the same number of times
            replays = int(reduce_max(float(replays), world, dev))
        timed_steps = replays * n_rep

        def region():
            for _ in range(replays):
                g.replay()

        with ClockSampler(local_rank) as clk:
            ms_region, all_regions = median_region_ms(region, args.regions, world, dev, stream)
        plan.status_sync(stream)
        ms_step = ms_region / timed_steps
        tokens_s = whole_job_tokens_s(inp.T, world, ms_step)
        e2e_tok_s = None
        if wr is None:
            e2e_tok_s = measure_e2e(inp, plan, rep_ptrs, n_rep, stream, ms_step)
        achieved_gbs = rf["weight_bytes"] / (ms_step * 1e-3) / 1e9
        achieved_tf = rf["flops"] / (ms_step * 1e-3) / 1e12
        res = dict(workload=name, T=inp.T, ms_per_step=ms_step, tokens_s=tokens_s, rf=rf,
                   achieved_gbs=achieved_gbs, achieved_tflops=achieved_tf, n_rep=n_rep,
                   graph=True, timed_steps=timed_steps, regions=[round(t, 4) for t in all_regions],
                   clocks=clk.summary(), e2e_tokens_s=e2e_tok_s,
                   h2d=inp.T * inp.H * 2 + inp.T * inp.E * 4, d2h=inp.T * inp.H * 2,
                   launches=launches_per_step * timed_steps, inp=inp, prof=prof,
                   launches_per_step=launches_per_step)
        del g
        plan.close()
        del reps, base
        torch.cuda.empty_cache()
        return res

    def measure_e2e(inp, plan, rep_ptrs, n_rep, stream, ms_step):
        """End to end through the host-buffer entry point (pinned host memory)."""
        xh = torch.from_numpy(inp.x.view(np.int16)).pin_memory()
        lh = torch.from_numpy(inp.logits).pin_memory()
        oh = torch.empty_like(xh).pin_memory()
        xp, lp, op = xh.data_ptr(), lh.data_ptr(), oh.data_ptr()
        # two passes over the weight replicas: the library captures each call's
        # graph on its second occurrence, so the timed calls replay graphs
        for i in range(max(3, 2 * n_rep)):
            api.moe_forward_host(plan.handle, inp.T, xp, lp, *rep_ptrs[i % n_rep], op, stream)
        n_e2e = max(50, min(2000, int(0.2 / max(ms_step * 1e-3, 1e-6))))
        torch.cuda.synchronize(dev)
        t0 = time.perf_counter()
        for i in range(n_e2e):
            api.moe_forward_host(plan.handle, inp.T, xp, lp, *rep_ptrs[i % n_rep], op, stream)
        e2e_s = (time.perf_counter() - t0) / n_e2e
        e2e_s = reduce_max(e2e_s, world, dev)
        plan.status_sync(stream)
        return inp.T * world / e2e_s

    main = measure(args.workload, args.steps, args.warmup)
    extra = {}
    if not args.no_extra and world == 1:
        for name in ("prefill", "zipf", "stack", "decode_router"):
            if name != args.workload:
                r = measure(name, 1 if name == "stack" else max(10, args.steps // 4), args.warmup)
                extra[name] = summarize_extra(r, peaks, peaks_kind)
    return main, extra, peaks, peaks_kind


KERNEL_SHARE = {"small_t": (1.0, 1.0), "gate_up": (2 / 3, 2 / 3), "down": (1 / 3, 1 / 3)}
# (the small-T kernel does the whole layer, the router's share included)


def measured_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu capture of this kernel and
    workload, or None if there is none or the kernel's sources changed since."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f).get(kernel)
    if not rec or rec.get("workload") != workload:
        return None
    h = hashlib.sha256()
    for src in rec["sources"]:
        if not os.path.exists(os.path.join(ROOT, src)):
            return None
        with open(os.path.join(ROOT, src), "rb") as f:
            h.update(f.read())
    return rec["dram_bytes_per_launch"] if h.hexdigest()[:16] == rec["sha"] else None


def kernel_table(r):
    prof = r["prof"]
    tot = sum(v[0] for v in prof.values()) or 1.0
    return {k: {"launches": n, "avg_us": round(1e3 * ms / max(n, 1), 3), "share": round(ms / tot, 4)}
            for k, (ms, n) in sorted(prof.items(), key=lambda kv: -kv[1][0])}


def roofline_obj(r, peaks, peaks_kind):
    """Roofline of the dominant kernel: its algorithmic bytes or FLOPs per launch
    over its average launch duration.

    A step of one launch (the small-batch kernel) takes the graph-timed step as
    that duration, an upper bound of the kernel's own time. Otherwise the
    duration is the library's per-kernel CUDA events on the launching stream,
    recorded while the stream was pre-filled, so no host launch gap is counted."""
    rf = r["rf"]
    prof = r["prof"]
    name = max(prof, key=lambda k: prof[k][0])
    ms, n = prof[name]
    avg_s = ms * 1e-3 / max(n, 1)
    timing = "per-kernel CUDA events on the pre-filled launching stream"
    if r.get("launches_per_step") == 1:
        avg_s = r["ms_per_step"] * 1e-3
        timing = "CUDA-graph step time (one launch per step), median of the timed regions"
    fb, ff = KERNEL_SHARE.get(name, (0.0, 0.0))
    per_launch = 1.0 / r.get("layers", 1)  # the stack's totals cover every layer; a launch is one layer
    kbytes, kflops = rf["weight_bytes"] * fb * per_launch, rf["flops"] * ff * per_launch
    t_hbm = kbytes / (peaks["hbm_gbs"] * 1e9)
    t_tc = kflops / (peaks["bf16_tflops"] * 1e12)
    if t_hbm >= t_tc:
        a, p, unit, bound = kbytes / avg_s / 1e9, peaks["hbm_gbs"], "GB/s", "hbm"
    else:
        a, p, unit, bound = kflops / avg_s / 1e12, peaks["bf16_tflops"], "TFLOP/s", "tensor"
    return {"bound": bound, "achieved": round(a, 2), "peak": p, "unit": unit, "frac": round(a / p, 4),
            "traffic": measured_traffic(name, r["workload"]), "traffic_unit": "bytes per launch (ncu)",
            "peak_source": peaks_kind, "kernel": name, "kernel_avg_us": round(avg_s * 1e6, 3),
            "kernel_timing": timing,
            "algorithmic_per_launch": {"weight_bytes": int(kbytes), "flops": kflops,
                                       "touched_experts_incl_shared": rf["touched"]}}


def summarize_extra(r, peaks, peaks_kind):
    return {"T": r["T"], "tokens_s": round(r["tokens_s"], 1), "ms_per_step": round(r["ms_per_step"], 6),
            "steps": r["timed_steps"], "region_ms": r["regions"], "effective_tflops": round(r["achieved_tflops"], 2), "achieved_weight_gbs": round(r["achieved_gbs"], 1),
            "roofline": roofline_obj(r, peaks, peaks_kind), "kernels": kernel_table(r), "graph": r["graph"],
            "clocks": r["clocks"],
            "e2e_tokens_s": None if r["e2e_tokens_s"] is None else round(r["e2e_tokens_s"], 1)}


def cpu_baseline(name, budget_s=15.0):
    """fp64 oracle on a bounded sample of the workload's tokens, on the host cores."""
    import oracle
    inp = synth.make_workload(name)
    cores = oracle.max_threads()

    def rows(n):  # the workload's first n token rows, repeated if T is smaller
        xs = np.resize(inp.x, (n, inp.H)) if n > inp.T else inp.x[:n]
        ls = np.resize(inp.logits, (n, inp.E)) if n > inp.T else inp.logits[:n]
        return np.ascontiguousarray(xs), np.ascontiguousarray(ls)

    # grow the sample until one run takes about the budget (each call dequantises
    # its touched experts once, so small samples cost more per token)
    n2, dt = max(4 * cores, 8), 0.0
    cap = max(inp.T, 1) if inp.T > 1 else 1 << 20
    for _ in range(6):
        n2 = min(n2, cap)
        xs, ls = rows(n2)
        t0 = time.perf_counter()
        oracle.moe_forward(inp, x=xs, logits=ls)
        dt = time.perf_counter() - t0
        if dt >= 0.5 * budget_s or n2 >= cap:
            break
        n2 = int(n2 * min(8.0, budget_s / max(dt, 1e-3)))
    out = {"value": round(n2 / dt, 3), "unit": "tokens/s", "cores": cores, "kind": "oracle",
           "sample": f"{n2} tokens of the {name} layer (token rows repeated if T is smaller), fp64, "
                     f"{dt:.1f} s wall"}
    if inp.T <= 512:
        # the same rows on one core, sized to about a quarter of the budget
        n1 = int(max(1, min(n2, budget_s / 4 / max(dt * cores / n2, 1e-9))))
        t0 = time.perf_counter()
        oracle.moe_forward(inp, nthreads=1, x=np.ascontiguousarray(xs[:n1]), logits=np.ascontiguousarray(ls[:n1]))
        dt1 = time.perf_counter() - t0
        out["single_core"] = {"value": round(n1 / dt1, 3), "unit": "tokens/s", "cores": 1,
                              "sample": f"first {n1} of those tokens, {dt1:.1f} s wall"}
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="b200", choices=["b200", "reference"])
    ap.add_argument("--workload", default="decode",
                    choices=["decode", "prefill", "zipf", "tiny", "stack", *ROUTER_WORKLOADS])
    ap.add_argument("--no-extra", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--regions", type=int, default=5, help="timed regions; the median is reported")
    ap.add_argument("--region-ms", type=float, default=100.0, help="minimum device time of one timed region")
    ap.add_argument("--replicas", type=int, default=0,
                    help="weight replicas to rotate over (default: enough to exceed 4x L2); for profiling runs")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    wl = synth.WORKLOADS[ROUTER_WORKLOADS.get(args.workload, args.workload)]
    config = {"workload": f"{wl.name}: T={wl.T} H={wl.H} E={wl.E} top_k={wl.k} I={wl.I} Is={wl.Is}, "
                          f"int4 g64 affine weights, seed {wl.seed}",
              "T": wl.T, "H": wl.H, "E": wl.E, "top_k": wl.k, "I": wl.I, "Is": wl.Is,
              "tokens_per_rank": wl.T, "parallelism": f"token-dp{args.gpus}"}

    if args.impl == "reference":
        if rank != 0:
            return
        import oracle
        steps = []
        inp = synth.make_workload(args.workload)
        n = min(inp.T, max(1, oracle.max_threads()))
        xs, ls = inp.x[:n], inp.logits[:n]
        if inp.T < n:
            xs, ls = np.resize(inp.x, (n, inp.H)), np.resize(inp.logits, (n, inp.E))
        for i in range(args.warmup + args.steps):
            t0 = time.perf_counter()
            oracle.moe_forward(inp, x=np.ascontiguousarray(xs), logits=np.ascontiguousarray(ls))
            if i >= args.warmup:
                steps.append(time.perf_counter() - t0)
        tot = sum(steps)
        val = n * len(steps) / tot
        line = {"impl": "reference", "metric": METRIC, "value": round(val, 3), "unit": "tokens/s",
                "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": round(1e3 * tot / len(steps), 3), "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config,
                "cpu_baseline": {"kind": "oracle", "cores": oracle.max_threads(), "value": round(val, 3),
                                 "unit": "tokens/s",
                                 "sample": f"{n} tokens of the {args.workload} layer per step"},
                "e2e": {"value": round(val, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return

    if world > 1:
        import torch
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    main_r, extra, peaks, peaks_kind = run_gpu(args, rank, world, local_rank)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(args.workload)
    if rank == 0:
        r = main_r
        line = {"metric": METRIC, "value": round(r["tokens_s"], 1), "unit": "tokens/s", "n_gpus": args.gpus,
                "steps": r["timed_steps"], "warmup": args.warmup, "ms_per_step": round(r["ms_per_step"], 6),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
                "data": "synthetic", "config": dict(config, l2=(
                    f"weights rotate over {r['n_rep']} device replicas "
                    f"({r['n_rep']} x {r['rf']['weight_bytes'] / 1e6:.1f} MB touched > 4 x L2)"),
                    graph=r["graph"], timed_regions=len(r["regions"]),
                    timing=f"median of {len(r['regions'])} CUDA-graph regions of {r['timed_steps']} steps each"),
                "region_ms": r["regions"],
                "roofline": roofline_obj(r, peaks, peaks_kind),
                "kernels": kernel_table(r),
                "effective_tflops": round(r["achieved_tflops"], 3),
                "cpu_baseline": cpu,
                "e2e": {"value": None if r["e2e_tokens_s"] is None else round(r["e2e_tokens_s"], 1), "unit": "tokens/s",
                        "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"]},
                "gpu_launches": r["launches"], "clocks": r["clocks"], "extra": extra}
        print(json.dumps(line))
    if world > 1:
        import torch
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
