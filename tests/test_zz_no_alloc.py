"""The allocation-free small-T entry point against the plan-based one.

moe_forward_small_t_noalloc serves callers that cannot call cudaMalloc (an
allocator callback, a pool that owns all device memory, a runtime that
reserves every byte up front): it takes its scratch from a static device
array inside the library. Both entry points run the same deterministic
kernel on the same inputs, so its output must equal moe_forward's bit for
bit (which implies the tests' tolerance), on two calls in a row, whether this
file runs alone in a fresh process or after the rest of the suite.
"""

import ctypes

import numpy as np
import pytest

from bit_grouped_expert_softmax_b200 import api, synth
from helpers import REL_L1, ROW_MAX, bf16_bits_to_f64, to_device

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _noalloc(lib, inp, x, logits, layer, out, status, stream):
    f = lib.moe_forward_small_t_noalloc
    f.argtypes = [ctypes.c_int] * 6 + [ctypes.c_void_p] * 11
    f.restype = ctypes.c_int
    return f(inp.T, inp.H, inp.E, inp.k, inp.I, inp.Is, x.data_ptr(), logits.data_ptr(),
             *[t.data_ptr() for t in layer.args()], out.data_ptr(), status.data_ptr(), stream.cuda_stream)


def _close(got_bits, ref_bits):
    got, ref = bf16_bits_to_f64(got_bits), bf16_bits_to_f64(ref_bits)
    d = np.abs(got - ref)
    rel = d.sum() / np.abs(ref).sum()
    row = (d.max(axis=1) / np.abs(ref).max(axis=1)).max()
    return rel <= REL_L1 and row <= ROW_MAX, rel, row


def test_noalloc_matches_plan_entry_point_twice():
    lib = api.load()
    stream = torch.cuda.Stream()
    cases = [synth.make_layer(1, 2048, 256, 8, 512, 512, seed=501, logit_std=2.0),
             synth.make_layer(5, 2048, 256, 8, 512, 512, seed=502, logit_std=2.0)]
    for inp in cases:
        layer = api.DeviceLayer.from_inputs(inp)
        x, logits = to_device(inp)
        plan = api.Plan(inp.T, inp.H, inp.E, inp.k, inp.I, inp.Is)
        ref = torch.empty_like(x)
        torch.cuda.synchronize()  # inputs were made on the default stream
        api.moe_forward(plan.handle, inp.T, x, logits, *layer.args(), ref, stream)
        plan.status_sync(stream)
        for call in range(2):
            out = torch.full_like(x, 0x7FC0)  # NaN pattern: every element must be written
            status = torch.full((4,), -1, dtype=torch.int32, device="cuda")
            torch.cuda.synchronize()  # the fills run on the default stream, the call on `stream`
            rc = _noalloc(lib, inp, x, logits, layer, out, status, stream)
            assert rc == 0, api.moe_last_error()
            stream.synchronize()
            assert status.cpu().numpy()[0] == 0, "device status reports an error"
            got, want = out.cpu().numpy(), ref.cpu().numpy()
            ok, rel, row = _close(got, want)
            assert ok, f"T={inp.T} call {call}: rel-L1 {rel:.3e}, row-max {row:.3e}"
            assert np.array_equal(got, want), f"T={inp.T} call {call}: not bit-identical to moe_forward"
        plan.close()


def test_noalloc_rejects_sizes_beyond_its_scratch():
    lib = api.load()
    f = lib.moe_forward_small_t_noalloc
    f.argtypes = [ctypes.c_int] * 6 + [ctypes.c_void_p] * 11
    f.restype = ctypes.c_int
    # 8 * (16 + 1) * 8192 * 4 bytes of tagged outputs > 512 KiB
    rc = f(1, 2048, 64, 16, 8192, 512, *([None] * 11))
    assert rc == -2 and "512 KiB" in api.moe_last_error()
    rc = f(9, 2048, 256, 8, 512, 512, *([None] * 11))
    assert rc == -1
    rc = f(1, 384, 16, 2, 128, 128, *([None] * 11))  # hidden must be a multiple of 256
    assert rc == -1 and "256" in api.moe_last_error()


def test_noalloc_empty_batch_writes_an_ok_status():
    lib = api.load()
    f = lib.moe_forward_small_t_noalloc
    f.argtypes = [ctypes.c_int] * 6 + [ctypes.c_void_p] * 11
    f.restype = ctypes.c_int
    status = torch.full((4,), -1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    rc = f(0, 2048, 256, 8, 512, 512, *([None] * 9), status.data_ptr(), stream.cuda_stream)
    assert rc == 0, api.moe_last_error()
    stream.synchronize()
    assert status.cpu().numpy().tolist() == [0, 0, 0, 0]
