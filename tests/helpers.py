"""Shared helpers of the GPU tests: device copies and the acceptance checks."""

import numpy as np

from bit_grouped_expert_softmax_b200 import synth

# Acceptance bounds of the layer output against the fp64 oracle:
#   relative L1 over the whole output  sum|gpu - ref| / sum|ref|        <= 2e-3
#   per token row                      max_h|gpu - ref| <= 1e-2 * max_h|ref|
REL_L1 = 2e-3
ROW_MAX = 1e-2


def to_device(inp, device="cuda"):
    import torch
    x = torch.from_numpy(np.ascontiguousarray(inp.x).view(np.int16)).to(device)
    logits = torch.from_numpy(np.ascontiguousarray(inp.logits)).to(device)
    return x, logits


def bf16_bits_to_f64(bits):
    return synth.bf16_to_f32(np.asarray(bits).view(np.uint16)).astype(np.float64)


def check_output(gpu_bits, ref, what=""):
    """gpu_bits: uint16/int16 bf16 patterns [T, H]; ref: fp64 [T, H]."""
    got = bf16_bits_to_f64(gpu_bits)
    assert got.shape == ref.shape
    assert np.all(np.isfinite(got)), f"{what}: non-finite outputs"
    d = np.abs(got - ref)
    rel_l1 = d.sum() / max(np.abs(ref).sum(), 1e-300)
    row_ratio = d.max(axis=1) / np.maximum(np.abs(ref).max(axis=1), 1e-300)
    assert rel_l1 <= REL_L1, f"{what}: relative L1 {rel_l1:.3e} > {REL_L1}"
    worst = int(np.argmax(row_ratio))
    assert row_ratio.max() <= ROW_MAX, f"{what}: row {worst} max-ratio {row_ratio.max():.3e} > {ROW_MAX}"
    return rel_l1, float(row_ratio.max())
