"""CUDA path against the fp64 oracle, through the C ABI (needs a B200)."""

import numpy as np
import pytest

import oracle
from bit_grouped_expert_softmax_b200 import api, synth
from helpers import check_output, to_device

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _layer(inp):
    return api.DeviceLayer.from_inputs(inp)


def _plan(inp, T_max=None, flags=0):
    return api.Plan(T_max or max(1, inp.T), inp.H, inp.E, inp.k, inp.I, inp.Is, flags)


def _forward(plan, inp, layer=None):
    layer = layer or _layer(inp)
    x, logits = to_device(inp)
    out = plan.forward(x, logits, layer)
    plan.status_sync()
    return out.cpu().numpy()


_INPUT_CACHE = {}


def workload(name):
    if name not in _INPUT_CACHE:
        _INPUT_CACHE[name] = synth.make_workload(name)
    return _INPUT_CACHE[name]


def stack_logits(layer, T=None):
    w = synth.WORKLOADS["stack"]
    rng = np.random.default_rng([w.seed, layer])
    return synth.draw_logits(rng, w.T if T is None else T, w.E, w.k, w.logit_std, w.zipf_s)


# ----------------------------------------------------------------------------
# routing: ids, offsets and permutation bit-exact; weights to fp32 rounding
# ----------------------------------------------------------------------------

def _check_route(logits, k, plan):
    ids, w, offsets, perm = plan.route(torch.from_numpy(logits).cuda())
    plan.status_sync()
    r_ids, r_w, _, r_off, r_perm = oracle.route(logits, k)
    assert np.array_equal(ids.cpu().numpy(), r_ids)
    assert np.array_equal(offsets.cpu().numpy(), r_off)
    assert np.array_equal(perm.cpu().numpy(), r_perm)
    np.testing.assert_allclose(w.cpu().numpy(), r_w, rtol=2e-6, atol=1e-7)


@pytest.mark.parametrize("name", ["tiny", "decode", "prefill", "zipf"])
def test_route_bit_exact(name):
    wl = synth.WORKLOADS[name]
    rng = np.random.default_rng(wl.seed)
    _ = rng.standard_normal((wl.T, wl.H), dtype=np.float32)  # x is drawn first
    logits = synth.draw_logits(rng, wl.T, wl.E, wl.k, wl.logit_std, wl.zipf_s)
    assert np.array_equal(logits, workload(name).logits) if name in ("tiny", "decode") else True
    plan = api.Plan(wl.T, wl.H, wl.E, wl.k, wl.I, wl.Is)
    _check_route(logits, wl.k, plan)


@pytest.mark.parametrize("layer", [0, 39])
def test_route_bit_exact_stack_chunk(layer):
    wl = synth.WORKLOADS["stack"]
    plan = api.Plan(wl.T, wl.H, wl.E, wl.k, wl.I, wl.Is)
    _check_route(stack_logits(layer), wl.k, plan)


def test_route_ties_and_extremes():
    E, k, T = 64, 8, 40
    rng = np.random.default_rng(5)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    logits[0] = 1.0                       # all equal: ids 0..7
    logits[1, ::2] = 3.0                  # ties among the top
    logits[2] = -1e30                     # huge negative values
    logits[2, 5] = 0.0
    logits[3, 10] = 1e30                  # one dominant expert
    plan = api.Plan(T, 256, E, k, 128, 128)
    _check_route(logits, k, plan)


# ----------------------------------------------------------------------------
# whole layer
# ----------------------------------------------------------------------------

def test_forward_tiny():
    inp = workload("tiny")
    check_output(_forward(_plan(inp), inp), oracle.moe_forward(inp), "tiny")


def test_forward_decode():
    inp = workload("decode")
    check_output(_forward(_plan(inp), inp), oracle.moe_forward(inp), "decode")


def test_forward_mid_size_ragged():
    """Several n-tiles per expert with ragged tails, several m-blocks, Is != I."""
    inp = synth.make_layer(300, 512, 32, 4, 256, 384, seed=21, logit_std=1.0)
    check_output(_forward(_plan(inp), inp), oracle.moe_forward(inp), "mid")


@pytest.mark.parametrize("T", [256, 257])
def test_gate_up_tile_choice_boundary(T):
    """The gate/up GEMM takes 32-row tiles while the groups average at most 32
    rows (T*k <= 32*E) and 128-row tiles above: both sides of the boundary,
    with ragged groups of both sizes."""
    inp = synth.make_layer(T, 512, 32, 4, 256, 384, seed=40 + T, logit_std=1.5)
    check_output(_forward(_plan(inp), inp), oracle.moe_forward(inp), f"T={T}")


@pytest.mark.parametrize("name", ["prefill", "zipf"])
def test_forward_full_size_every_row(name):
    """Every token row of the full-size layer against the oracle (the by-expert
    form of the same definition). At Zipf T=4096 this covers the tail experts
    whose few tokens fill ragged, mostly empty tiles."""
    inp = workload(name)
    got = _forward(_plan(inp), inp)
    check_output(got, oracle.moe_forward_by_expert(inp), name)


def test_zipf_tail_experts_have_ragged_groups():
    """The Zipf layer does route some experts only a handful of tokens (the
    ragged tiles the previous test covers) and leaves others untouched."""
    inp = workload("zipf")
    counts = oracle.route(inp.logits, inp.k)[2]
    assert (counts == 0).sum() > 100 and ((counts > 0) & (counts < 16)).sum() >= 3


@pytest.mark.parametrize("T", [1, 2, 3, 5, 8, 9])
@pytest.mark.parametrize("flags", [0, api.MOE_FLAG_FORCE_GROUPED])
def test_forward_small_batches(T, flags):
    inp = synth.make_layer(T, 2048, 256, 8, 512, 512, seed=100 + T, logit_std=2.0)
    check_output(_forward(_plan(inp, flags=flags), inp), oracle.moe_forward(inp), f"T={T} flags={flags}")


@pytest.mark.parametrize("T,flags", [(1, 0), (4, 0), (4, api.MOE_FLAG_FORCE_GROUPED), (40, 0)])
def test_shared_expert_narrower_than_routed(T, flags):
    """Is < I on both paths (the small-batch kernel sizes its stages by the wider of the two)."""
    inp = synth.make_layer(T, 512, 32, 4, 384, 128, seed=200 + T, logit_std=1.0)
    check_output(_forward(_plan(inp, flags=flags), inp), oracle.moe_forward(inp), f"Is<I T={T} flags={flags}")


@pytest.mark.parametrize("H", [256, 512, 1280])
@pytest.mark.parametrize("T", [1, 3])
def test_small_batch_hidden_sizes(H, T):
    """Hidden sizes whose per-warp K slices of the small-batch kernel are 1, 2 and 5 blocks of 128."""
    inp = synth.make_layer(T, H, 16, 2, 128, 256, seed=300 + H + T, logit_std=1.0)
    check_output(_forward(_plan(inp), inp), oracle.moe_forward(inp), f"H={H} T={T}")


@pytest.mark.parametrize("H", [256, 512])
def test_small_batch_many_units_per_block(H):
    """T=8 over 256 experts: up to 65 distinct experts, so each CTA of the
    small-batch kernel takes many 16-row units and recycles both rings; at
    these hidden sizes a round could hold more units than ring stages."""
    inp = synth.make_layer(8, H, 256, 8, 512, 512, seed=400 + H, logit_std=2.0)
    check_output(_forward(_plan(inp), inp), oracle.moe_forward(inp), f"many units H={H}")


def test_one_expert_takes_every_token():
    inp = synth.make_layer(150, 256, 16, 2, 128, 128, seed=31)
    inp.logits[:, 3] += 100.0  # expert 3 is everyone's first choice; most experts get nothing
    check_output(_forward(_plan(inp), inp), oracle.moe_forward(inp), "hot expert")


def test_deterministic_reruns():
    inp = workload("prefill")
    plan = _plan(inp)
    layer = _layer(inp)
    a = _forward(plan, inp, layer)
    b = _forward(plan, inp, layer)
    assert np.array_equal(a, b)


@pytest.mark.parametrize("name", ["tiny", "decode"])
def test_forward_host_matches_device_call(name):
    """Host buffers: the first call runs eagerly, a repeat of it is captured
    into a graph, later repeats replay the graph; all equal the device call."""
    inp = workload(name)
    plan = _plan(inp)
    layer = _layer(inp)
    dev = _forward(plan, inp, layer)
    x = torch.from_numpy(inp.x.view(np.int16)).pin_memory()
    lg = torch.from_numpy(inp.logits).pin_memory()
    out = torch.empty_like(x).pin_memory()
    for call in range(4):
        out.fill_(0x7FC0)
        api.moe_forward_host(plan.handle, inp.T, x, lg, *layer.args(), out)
        assert np.array_equal(out.numpy(), dev), f"call {call}"
    plan.status_sync()
    # pageable buffers take the eager path
    xp, lp, op = inp.x.copy(), inp.logits.copy(), np.empty_like(inp.x)
    for call in range(2):
        api.moe_forward_host(plan.handle, inp.T, xp, lp, *layer.args(), op)
        assert np.array_equal(op.view(np.int16), dev), f"pageable call {call}"


def test_forward_host_unaligned_pinned_buffers():
    """Pinned host buffers at addresses that are not 16-byte aligned: the
    call stages them into aligned device buffers and gives the device call's
    result, eagerly and from its captured graph."""
    inp = workload("decode")
    plan = _plan(inp)
    layer = _layer(inp)
    dev = _forward(plan, inp, layer)
    n = inp.x.size
    xb = torch.empty(n + 2, dtype=torch.int16).pin_memory()
    xb[2:] = torch.from_numpy(inp.x.view(np.int16).ravel())
    lb = torch.empty(inp.logits.size + 1, dtype=torch.float32).pin_memory()
    lb[1:] = torch.from_numpy(inp.logits.ravel())
    ob = torch.empty(n + 2, dtype=torch.int16).pin_memory()
    for call in range(3):
        ob.fill_(0x7FC0)
        api.moe_forward_host(plan.handle, inp.T, xb.data_ptr() + 4, lb.data_ptr() + 4, *layer.args(),
                             ob.data_ptr() + 4)
        assert np.array_equal(ob[2:].numpy().reshape(dev.shape), dev), f"call {call}"
    plan.status_sync()


def test_output_canaries_untouched():
    inp = workload("tiny")
    plan = _plan(inp)
    x, logits = to_device(inp)
    guard = 4096
    buf = torch.full((inp.T * inp.H + 2 * guard,), 0x5A5A, dtype=torch.int16, device="cuda")
    out = buf[guard:guard + inp.T * inp.H].view(inp.T, inp.H)
    api.moe_forward(plan.handle, inp.T, x, logits, *_layer(inp).args(), out)
    plan.status_sync()
    b = buf.cpu().numpy()
    assert np.all(b[:guard] == 0x5A5A) and np.all(b[-guard:] == 0x5A5A)


def test_empty_batch_is_a_no_op():
    inp = workload("tiny")
    plan = _plan(inp)
    x, logits = to_device(inp)
    api.moe_forward(plan.handle, 0, x, logits, *_layer(inp).args(), torch.empty_like(x))
    plan.status_sync()


def test_invalid_arguments_enqueue_nothing():
    inp = workload("tiny")
    plan = _plan(inp)
    x, logits = to_device(inp)
    with pytest.raises(api.MoEError) as ei:
        api.moe_forward(plan.handle, inp.T + 1, x, logits, *_layer(inp).args(), torch.empty_like(x))
    assert ei.value.status == -1
    with pytest.raises(api.MoEError):
        api.moe_forward(plan.handle, inp.T, x, logits, *_layer(inp).args(), x)  # out aliases x
    plan.status_sync()


# ----------------------------------------------------------------------------
# MOE_FLAG_DEBUG range checks and the bounded waits
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("case", ["tiny", "mid", "zipf", "decode"])
def test_debug_range_checks_pass_on_valid_runs(case):
    """With every work item and inverse-permutation entry range-checked on the
    device, a valid layer reports no error and still matches the oracle."""
    if case == "mid":
        inp = synth.make_layer(300, 512, 32, 4, 256, 384, seed=21, logit_std=1.0)
    else:
        inp = workload(case)
    plan = _plan(inp, flags=api.MOE_FLAG_DEBUG | (api.MOE_FLAG_FORCE_GROUPED if case == "decode" else 0))
    got = _forward(plan, inp)  # status_sync raises on any recorded error
    ref = oracle.moe_forward_by_expert(inp) if inp.T > 64 else oracle.moe_forward(inp)
    check_output(got, ref, f"debug {case}")


@pytest.mark.parametrize("T", [1, 3])
def test_small_batch_launches_read_only_their_own_swiglu_outputs(T):
    """The small-batch kernel hands each SwiGLU output between CTAs as a word
    tagged with its launch. Two inputs alternated on one plan and one layer
    (T = 1: the readers poll whole rows together; T = 3: each lane polls its
    own words) give each input its own result, bit for bit on every launch
    and within tolerance of the oracle: no launch uses words an earlier one
    left in the scratch."""
    import dataclasses
    a = synth.make_layer(T, 2048, 256, 8, 512, 512, seed=611, logit_std=2.0)
    rng = np.random.default_rng(612)
    b = dataclasses.replace(a, x=synth.bf16_rne(rng.standard_normal((T, 2048), dtype=np.float32)),
                            logits=synth.draw_logits(rng, T, 256, 8, 2.0, None))
    layer = _layer(a)
    plan = _plan(a)
    ra, rb = _forward(plan, a, layer), _forward(plan, b, layer)
    check_output(ra, oracle.moe_forward(a), f"T={T} input a")
    check_output(rb, oracle.moe_forward(b), f"T={T} input b")
    for rep in range(3):
        assert np.array_equal(_forward(plan, a, layer), ra), f"T={T} input a, repeat {rep}"
        assert np.array_equal(_forward(plan, b, layer), rb), f"T={T} input b, repeat {rep}"


def test_bounded_wait_runs_out_and_the_plan_recovers():
    """The test flag makes one wait of the plan's first small-T launch run out
    (row block 0 of the shared expert never announces its output) under a
    2 ms budget: nothing faults, every other wait is bounded, the launch ends
    and moe_status_sync reports the timeout. The next launch on the same plan
    runs normally and matches the oracle."""
    inp = synth.make_layer(1, 2048, 256, 8, 512, 512, seed=601, logit_std=2.0)
    layer = _layer(inp)
    plan = _plan(inp, flags=api.MOE_FLAG_TEST_WAIT_TIMEOUT)
    x, logits = to_device(inp)
    plan.forward(x, logits, layer)
    with pytest.raises(api.MoEError) as ei:
        plan.status_sync()
    assert ei.value.status == -4 and "wait ran out" in str(ei.value)
    for _ in range(2):
        out = plan.forward(x, logits, layer)
        plan.status_sync()
        check_output(out.cpu().numpy(), oracle.moe_forward(inp), "after the timeout")


@pytest.mark.parametrize("T", [300, 3])
def test_programmatic_dependent_launch_gives_identical_results(T):
    """Three stacked layers, with the default programmatic dependent launch and
    in plain stream order: bit-identical outputs. T = 300 takes the grouped
    path; T = 3 the small-batch kernel, whose next layer's CTAs request the
    shared expert's weights before the layer ahead has finished."""
    inp = synth.make_layer(T, 512, 32, 4, 256, 384, seed=23, logit_std=1.0)
    layer = _layer(inp)
    rng = np.random.default_rng(5)
    logits = np.stack([synth.draw_logits(rng, inp.T, inp.E, inp.k, 1.0, None) for _ in range(3)])
    dlog = torch.from_numpy(logits).cuda()
    outs = []
    for flags in (0, api.MOE_FLAG_NO_PDL):
        plan = _plan(inp, flags=flags)
        x = torch.from_numpy(inp.x.view(np.int16)).cuda()
        torch.cuda.synchronize()
        plan.stack_forward(x, dlog, [layer] * 3)
        plan.status_sync()
        outs.append(x.cpu().numpy())
        plan.close()
    assert np.array_equal(outs[0], outs[1])
