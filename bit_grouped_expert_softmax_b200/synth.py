"""Seeded synthetic inputs for the routed int4 MoE layer.

This module only draws random numbers and lays them out in the layer's input
format. It holds none of the layer's arithmetic: no softmax, no top-k
selection, no dequantisation, no matrix products. Both the CPU oracle's tests
and the CUDA path's tests/benchmark take their inputs from here, so that the
two sides see the same bytes.

Workloads follow the model layout described on the pages ("Perplexity open
sources Lily", section "Requirements and model layout"): a router that scores
256 experts and picks eight, one shared expert that sees every token, and
groupwise-affine 4-bit weights where every group of 64 weights shares one
bfloat16 scale and one bfloat16 bias. Hidden sizes are not on the pages;
H=2048 and I=512 are assumed.

Input format (shared with the C ABI):

* ``x``       : uint16 [T, H], bfloat16 bit patterns.
* ``logits``  : float32 [T, E].
* ``packed``  : uint32 [E, 3*I*H/8] = per expert [gate (I rows x H/8 words) |
                up (I x H/8) | down (H rows x I/8 words)], K contiguous.
                Word w of a row holds K elements 8w..8w+7, element 8w+j in
                bits 4j..4j+3 (low nibble first).
* ``scales`` / ``biases`` : uint16 [E, 3*I*H/64] bfloat16 bit patterns,
                per expert [gate (I x H/64) | up (I x H/64) | down (H x I/64)];
                group g of a row covers K in [64g, 64g+64).
* ``sh_*``    : the same for the one shared expert, with intermediate Is.

Draw order for one layer, all from one ``numpy.random.default_rng``:

1. x  = bf16_rne(standard_normal((T, H), float32))          (unless given)
2. logits = standard_normal((T, E), float32) * std (+ Zipf bias), then every
   row whose k-th and (k+1)-th largest logits differ by less than the margin
   is redrawn, in row order, until it satisfies the margin.
3. for e in 0..E-1, then the shared expert, for each of gate [I,H], up [I,H],
   down [H,I] (N rows, K columns):
     words = integers(0, 2**32, (N, K/8), uint32)  -- eight independent
             uniform nibbles 0..15 per word, already in packed form
     s = bf16_rne(|standard_normal((N, K/64), float32)| * 0.02)
     b = bf16_rne(-7.5 * s + standard_normal((N, K/64), float32) * 0.002)
"""

from __future__ import annotations

import dataclasses
import math

import numpy as np

GROUP = 64          # weights per scale/bias group (pages: groups of 64)
NIBBLES = 8         # 4-bit codes per uint32 word
TOPK_MARGIN = 1e-3  # minimum gap between the k-th and (k+1)-th logit


# ----------------------------------------------------------------------------
# workloads
# ----------------------------------------------------------------------------

@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int
    H: int
    E: int
    k: int
    I: int
    Is: int
    logit_std: float
    zipf_s: float | None
    seed: int
    layers: int = 1

    @property
    def dims(self):
        return dict(T=self.T, H=self.H, E=self.E, k=self.k, I=self.I, Is=self.Is)


WORKLOADS = {
    # tiny MoE layer: T16 H256 E16 top-2 I=Is=128, logits N(0,1), seed 0
    "tiny": Workload("tiny", 16, 256, 16, 2, 128, 128, 1.0, None, 0),
    # Qwen3.6-35B-A3B-shaped layer at decode: T1 H2048 E256 top-8 I=Is=512
    "decode": Workload("decode", 1, 2048, 256, 8, 512, 512, 2.0, None, 1),
    # same layer at prefill, the pages' 512-token ablation prompt
    "prefill": Workload("prefill", 512, 2048, 256, 8, 512, 512, 2.0, None, 2),
    # prefill with uneven expert groups: N(0,1) + 3 ln(Zipf(1.1) weight)
    "zipf": Workload("zipf", 4096, 2048, 256, 8, 512, 512, 1.0, 1.1, 3),
    # 40 stacked layers, T=8192 prefill chunk, N(0,2) logits per layer
    "stack": Workload("stack", 8192, 2048, 256, 8, 512, 512, 2.0, None, 4, 40),
}


# ----------------------------------------------------------------------------
# format helpers (bit layout only)
# ----------------------------------------------------------------------------

def bf16_rne(a: np.ndarray) -> np.ndarray:
    """float32 array -> uint16 bfloat16 bit patterns, round to nearest even."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    """uint16 bfloat16 bit patterns -> float32 (exact)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def pack_nibbles(q: np.ndarray) -> np.ndarray:
    """uint8 codes [N, K] (values 0..15) -> uint32 words [N, K/8], low nibble first."""
    q = np.asarray(q)
    n, kdim = q.shape
    assert kdim % NIBBLES == 0 and q.max(initial=0) < 16
    q = q.reshape(n, kdim // NIBBLES, NIBBLES).astype(np.uint32)
    shifts = (4 * np.arange(NIBBLES, dtype=np.uint32))
    return np.bitwise_or.reduce(q << shifts, axis=2).astype(np.uint32)


def zipf_bias(E: int, s: float) -> np.ndarray:
    """Per-expert logit bias 3*ln(p_rank), rank(e) = e+1, p_r = r^-s / sum_r' r'^-s."""
    r = np.arange(1, E + 1, dtype=np.float64)
    p = r ** (-s)
    p /= p.sum()
    return (3.0 * np.log(p)).astype(np.float32)


# ----------------------------------------------------------------------------
# draws
# ----------------------------------------------------------------------------

def _margin_ok(rows: np.ndarray, k: int, margin: float) -> np.ndarray:
    """True where the k-th largest value exceeds the (k+1)-th by >= margin."""
    if rows.shape[1] <= k:
        return np.ones(rows.shape[0], dtype=bool)
    part = -np.partition(-rows, k, axis=1)[:, : k + 1]
    part = -np.sort(-part, axis=1)
    return (part[:, k - 1] - part[:, k]) >= np.float32(margin)


def draw_logits(rng, T: int, E: int, k: int, std: float, zipf_s: float | None,
                margin: float = TOPK_MARGIN) -> np.ndarray:
    bias = zipf_bias(E, zipf_s) if zipf_s is not None else None

    def row_draw(shape):
        z = rng.standard_normal(shape, dtype=np.float32) * np.float32(std)
        if bias is not None:
            z = z + bias
        return z.astype(np.float32)

    logits = row_draw((T, E))
    bad = np.nonzero(~_margin_ok(logits, k, margin))[0]
    for t in bad:  # redraw violating rows in row order from the same stream
        while True:
            row = row_draw((1, E))
            if _margin_ok(row, k, margin)[0]:
                logits[t] = row[0]
                break
    return logits


def draw_matrix(rng, N: int, K: int):
    """One int4 weight matrix [N, K]: packed words, bf16 scales, bf16 biases."""
    words = rng.integers(0, 2 ** 32, size=(N, K // NIBBLES), dtype=np.uint32)
    s = bf16_rne(np.abs(rng.standard_normal((N, K // GROUP), dtype=np.float32)) * np.float32(0.02))
    s32 = bf16_to_f32(s)
    b = bf16_rne(np.float32(-7.5) * s32
                 + rng.standard_normal((N, K // GROUP), dtype=np.float32) * np.float32(0.002))
    return words, s, b


def draw_expert(rng, H: int, I: int):
    """gate [I,H], up [I,H], down [H,I] concatenated in the packed layout."""
    parts = [draw_matrix(rng, I, H), draw_matrix(rng, I, H), draw_matrix(rng, H, I)]
    words = np.concatenate([p[0].ravel() for p in parts])
    s = np.concatenate([p[1].ravel() for p in parts])
    b = np.concatenate([p[2].ravel() for p in parts])
    return words, s, b


@dataclasses.dataclass
class LayerInputs:
    T: int
    H: int
    E: int
    k: int
    I: int
    Is: int
    x: np.ndarray        # uint16 [T, H]
    logits: np.ndarray   # float32 [T, E]
    packed: np.ndarray   # uint32 [E, 3*I*H/8]
    scales: np.ndarray   # uint16 [E, 3*I*H/64]
    biases: np.ndarray   # uint16 [E, 3*I*H/64]
    sh_packed: np.ndarray  # uint32 [3*Is*H/8]
    sh_scales: np.ndarray  # uint16 [3*Is*H/64]
    sh_biases: np.ndarray  # uint16 [3*Is*H/64]


def draw_weights(rng, H, E, I, Is):
    wpe, gpe = 3 * I * H // NIBBLES, 3 * I * H // GROUP
    packed = np.empty((E, wpe), dtype=np.uint32)
    scales = np.empty((E, gpe), dtype=np.uint16)
    biases = np.empty((E, gpe), dtype=np.uint16)
    for e in range(E):
        packed[e], scales[e], biases[e] = draw_expert(rng, H, I)
    shp, shs, shb = draw_expert(rng, H, Is)
    return packed, scales, biases, shp, shs, shb


def make_layer(T, H, E, k, I, Is, seed, logit_std=1.0, zipf_s=None,
               x: np.ndarray | None = None) -> LayerInputs:
    """Draw one layer's inputs. ``seed`` may be an int or a sequence (numpy SeedSequence)."""
    for name, v in (("H", H), ("I", I), ("Is", Is)):
        if v % GROUP:
            raise ValueError(f"{name}={v} must be a multiple of {GROUP}")
    rng = np.random.default_rng(seed)
    if x is None:
        x = bf16_rne(rng.standard_normal((T, H), dtype=np.float32))
    logits = draw_logits(rng, T, E, k, logit_std, zipf_s)
    packed, scales, biases, shp, shs, shb = draw_weights(rng, H, E, I, Is)
    return LayerInputs(T, H, E, k, I, Is, np.ascontiguousarray(x), logits,
                       packed, scales, biases, shp, shs, shb)


def draw_router(rng, E: int, H: int, logit_std: float) -> np.ndarray:
    """Router weight [E, H] as bf16 bit patterns, N(0, 1) * logit_std / sqrt(H):
    with x ~ N(0, 1) the router scores have standard deviation ~logit_std."""
    w = rng.standard_normal((E, H), dtype=np.float32) * np.float32(logit_std / math.sqrt(H))
    return bf16_rne(w)


def make_router_layer(T, H, E, k, I, Is, seed, logit_std=2.0):
    """A layer whose logits come from a router weight instead of being given:
    draws x, then the router weight [E, H], then the experts (``logits`` is
    left empty: the method computes it). Returns (LayerInputs, router_w)."""
    rng = np.random.default_rng(seed)
    x = bf16_rne(rng.standard_normal((T, H), dtype=np.float32))
    router_w = draw_router(rng, E, H, logit_std)
    packed, scales, biases, shp, shs, shb = draw_weights(rng, H, E, I, Is)
    inp = LayerInputs(T, H, E, k, I, Is, x, np.zeros((T, E), np.float32), packed, scales, biases, shp, shs, shb)
    return inp, router_w


def make_workload(name: str, T: int | None = None) -> LayerInputs:
    """Inputs of a single-layer workload (``T`` overrides the token count)."""
    w = WORKLOADS[name]
    if w.layers != 1:
        raise ValueError("use make_stack_layer for the stacked workload")
    return make_layer(w.T if T is None else T, w.H, w.E, w.k, w.I, w.Is, w.seed,
                      w.logit_std, w.zipf_s)


def make_stack_x(w: Workload, T: int | None = None) -> np.ndarray:
    """Stack input activations: default_rng(seed) draws x first."""
    rng = np.random.default_rng(w.seed)
    return bf16_rne(rng.standard_normal((w.T if T is None else T, w.H), dtype=np.float32))


def make_stack_layer(w: Workload, layer: int, T: int | None = None) -> LayerInputs:
    """Layer ``layer`` of the stack: default_rng([seed, layer]) draws logits, then weights."""
    T = w.T if T is None else T
    rng = np.random.default_rng([w.seed, layer])
    logits = draw_logits(rng, T, w.E, w.k, w.logit_std, w.zipf_s)
    packed, scales, biases, shp, shs, shb = draw_weights(rng, w.H, w.E, w.I, w.Is)
    return LayerInputs(T, w.H, w.E, w.k, w.I, w.Is, None, logits, packed, scales,
                       biases, shp, shs, shb)


def expert_bytes(H: int, I: int) -> int:
    """HBM bytes of one expert: packed nibbles plus bf16 scale and bias."""
    return 3 * H * I // 2 + 3 * H * I // GROUP * 4


def layer_flops(T: int, H: int, k: int, I: int) -> float:
    """Effective FLOPs of one layer, 2*T*(k+1)*3*H*I."""
    return 2.0 * T * (k + 1) * 3 * H * I


def log2_ceil(n: int) -> int:
    return int(math.ceil(math.log2(max(1, n))))
