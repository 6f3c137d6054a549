"""The stacked layers, x <- bf16(x + moe_l(x)), against the oracle (needs a B200).

The stack has no normalisation, so activations grow by orders of magnitude per
layer and leave bfloat16's range after a few layers. Each layer is checked
teacher-forced: the oracle recomputes layer l from the GPU's own bf16 input
x_l on every token row of the first four layers and on a fixed sample of 256
rows of each later layer. Rows whose reference stays well inside
the float range are held to the usual tolerance; rows whose reference
exceeds bfloat16's largest value must come out non-finite, and once an input
row is non-finite it is no longer compared.
"""

import numpy as np
import pytest

import oracle
from bit_grouped_expert_softmax_b200 import api, synth
from helpers import ROW_MAX, REL_L1, bf16_bits_to_f64

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

# The smallest magnitude that rounds to infinity in bfloat16 (round to nearest
# even): halfway between the largest finite value (2 - 2^-7) * 2^127 and 2^128.
# Values between the largest finite value and this one round to the largest
# finite value.
BF16_OVERFLOW = (2.0 - 2.0 ** -8) * 2.0 ** 127
N_ROWS = 256      # sampled token rows per layer from layer FULL_LAYERS on
FULL_LAYERS = 4   # layers whose every row is compared


def _layers(wl, n):
    """Device weights and float32 logits of the stack's first n layers (host arrays dropped)."""
    layers, logits = [], []
    for l in range(n):
        inp = synth.make_stack_layer(wl, l)
        layers.append(api.DeviceLayer.from_inputs(inp))
        logits.append(inp.logits)
    return layers, np.stack(logits)


def test_stack_forward_matches_layer_by_layer_and_oracle():
    wl = synth.WORKLOADS["stack"]
    L = wl.layers
    layers, logits = _layers(wl, L)
    x0 = synth.make_stack_x(wl)
    dev_logits = torch.from_numpy(logits).cuda()
    plan = api.Plan(wl.T, wl.H, wl.E, wl.k, wl.I, wl.Is)

    # whole stack in one call
    x_full = torch.from_numpy(x0.view(np.int16)).cuda()
    plan.stack_forward(x_full, dev_logits, layers)
    plan.status_sync()

    # the same call captured into a CUDA graph and replayed
    stream = torch.cuda.Stream()
    x_graph = torch.from_numpy(x0.view(np.int16)).cuda()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        api.moe_stack_forward(plan.handle, L, wl.T, x_graph, dev_logits, layers, stream)
    x_graph.copy_(torch.from_numpy(x0.view(np.int16)).cuda())
    g.replay()
    torch.cuda.synchronize()
    plan.status_sync()
    assert torch.equal(x_graph, x_full)
    del g

    # layer by layer, keeping each layer's input for the teacher-forced check
    rng = np.random.default_rng(77)
    sampled = np.sort(rng.choice(wl.T, N_ROWS, replace=False))
    x = torch.from_numpy(x0.view(np.int16)).cuda()
    n_checked, n_overflow = 0, 0
    for l in range(L):
        rows = np.arange(wl.T) if l < FULL_LAYERS else sampled
        x_in = x[torch.from_numpy(rows).cuda()].cpu().numpy()
        api.moe_stack_forward(plan.handle, 1, wl.T, x, dev_logits[l:l + 1], layers[l:l + 1])
        plan.status_sync()
        x_out = bf16_bits_to_f64(x[torch.from_numpy(rows).cuda()].cpu().numpy())
        xin64 = bf16_bits_to_f64(x_in)
        finite_in = np.all(np.isfinite(xin64), axis=1)
        if not finite_in.any():
            continue
        inp = synth.make_stack_layer(wl, l)
        r = np.nonzero(finite_in)[0]
        ref = xin64[r] + oracle.moe_forward_by_expert(inp, x=np.ascontiguousarray(x_in[r]).view(np.uint16),
                                                      logits=inp.logits[rows[r]])
        got = x_out[r]
        amax = np.abs(ref).max(axis=1)
        safe = amax < 1e37
        huge = ~np.isfinite(ref).all(axis=1) | (amax > BF16_OVERFLOW)
        if safe.any():
            d = np.abs(got[safe] - ref[safe])
            assert np.all(np.isfinite(got[safe])), f"layer {l}: non-finite output on a finite row"
            rel = d.sum() / np.abs(ref[safe]).sum()
            row = (d.max(axis=1) / np.abs(ref[safe]).max(axis=1)).max()
            assert rel <= REL_L1 and row <= ROW_MAX, f"layer {l}: rel-L1 {rel:.3e}, row-max {row:.3e}"
            n_checked += int(safe.sum())
        if huge.any():
            # where the exact value rounds to infinity by more than the row
            # tolerance (ROW_MAX of the row's largest magnitude), the output
            # cannot be finite
            rh, gh = ref[huge], got[huge]
            bound = BF16_OVERFLOW + ROW_MAX * np.abs(rh).max(axis=1, keepdims=True)
            big = np.abs(rh) > bound
            assert np.all(~np.isfinite(gh[big])), f"layer {l}: finite output where the value overflows"
            n_overflow += int(huge.sum())
    assert n_checked >= 2 * wl.T  # at least the first layers are compared on every row
    # the layer-by-layer run is the same computation as the single call
    assert torch.equal(x, x_full)
    plan.close()
