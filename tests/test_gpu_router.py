"""The router scores computed on the GPU (logits = x . W_router^T) and the layer
that computes its own routing from them, against the fp64 oracle (needs a B200).

The selection compares float32 scores: where a token's k-th and (k+1)-th
exact scores are closer than the float32 accumulation error, either order is
a correct result. Tokens whose two scores are at least 1e-3 apart (all but a
few) must match the oracle; the others are left out of the comparison.
"""

import numpy as np
import pytest

import oracle
from bit_grouped_expert_softmax_b200 import api, synth
from helpers import check_output

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

MARGIN = 1e-3


def _dev(a, dt):
    return torch.from_numpy(np.ascontiguousarray(a).view(dt)).cuda()


def _margins(logits64, k):
    s = -np.sort(-logits64, axis=1)
    return s[:, k - 1] - s[:, k]


@pytest.mark.parametrize("T,H,E", [(300, 512, 256), (130, 2048, 20), (1, 2048, 256), (8, 256, 16)])
def test_router_scores_match_oracle(T, H, E):
    inp, w = synth.make_router_layer(T, H, E, 2, 128, 128, seed=700 + T + E)
    plan = api.Plan(T, H, E, 2, 128, 128)
    out = torch.full((T, E), float("nan"), dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()
    api.moe_router_logits(plan.handle, T, _dev(inp.x, np.int16), _dev(w, np.int16), out)
    plan.status_sync()
    got = out.cpu().numpy().astype(np.float64)
    ref = oracle.router_logits(inp.x, w)
    # float32 accumulation of bf16 products: bounded by a few ulps of the sum of |products|
    scale = np.abs(oracle.bf16_to_f64(inp.x)) @ np.abs(oracle.bf16_to_f64(w)).T
    assert np.all(np.isfinite(got))
    assert np.all(np.abs(got - ref) <= 1e-5 * scale + 1e-30)


@pytest.mark.parametrize("T,flags", [(1, 0), (3, 0), (8, 0), (5, api.MOE_FLAG_FORCE_GROUPED), (300, 0), (512, 0)])
def test_layer_with_router_matches_oracle(T, flags):
    H, E, k, I = (2048, 256, 8, 512) if T in (1, 8, 512) else (512, 64, 4, 256)
    inp, w = synth.make_router_layer(T, H, E, k, I, I, seed=800 + T, logit_std=2.0)
    clear = _margins(oracle.router_logits(inp.x, w), k) >= MARGIN
    assert clear.mean() >= 0.95
    layer = api.DeviceLayer.from_inputs(inp)
    plan = api.Plan(T, H, E, k, I, I, flags)
    x = _dev(inp.x, np.int16)
    out = torch.empty_like(x)
    torch.cuda.synchronize()
    api.moe_forward_router(plan.handle, T, x, _dev(w, np.int16), *layer.args(), out)
    plan.status_sync()
    ref = oracle.moe_forward_router(inp, w, by_expert=T > 64)
    check_output(out.cpu().numpy()[clear], ref[clear], f"router T={T} flags={flags}")


def test_layer_with_router_equals_layer_on_its_scores():
    """The router path on T > 8 is the router kernel followed by moe_forward on
    its scores: bit-identical outputs."""
    T, H, E, k, I = 300, 512, 64, 4, 256
    inp, w = synth.make_router_layer(T, H, E, k, I, I, seed=901)
    layer = api.DeviceLayer.from_inputs(inp)
    plan = api.Plan(T, H, E, k, I, I)
    x, wd = _dev(inp.x, np.int16), _dev(w, np.int16)
    logits = torch.empty((T, E), dtype=torch.float32, device="cuda")
    a, b = torch.empty_like(x), torch.empty_like(x)
    torch.cuda.synchronize()
    api.moe_router_logits(plan.handle, T, x, wd, logits)
    api.moe_forward(plan.handle, T, x, logits, *layer.args(), a)
    api.moe_forward_router(plan.handle, T, x, wd, *layer.args(), b)
    plan.status_sync()
    assert torch.equal(a, b)
