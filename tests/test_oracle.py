"""Pins of the fp64 CPU oracle against what the pages and the mathematics fix.

None of these checks re-types the oracle's own code: the expected values come
from hand-worked fixtures under tests/golden/, from independent numpy
restatements (argsort routing, dense dequantised matmuls), from closed forms
and from invariants.
"""

import math
import os

import numpy as np
import pytest

import oracle
from bit_grouped_expert_softmax_b200 import synth


# ----------------------------------------------------------------------------
# fixture readers
# ----------------------------------------------------------------------------

def _rows(path):
    with open(path) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield line.split()


def _routing_cases(golden_dir):
    cases, cur = [], None
    for tok in _rows(os.path.join(golden_dir, "routing_cases.txt")):
        if tok[0] == "case":
            cur = {"name": tok[1], "k": int(tok[2])}
            cases.append(cur)
        elif tok[0] == "logits":
            cur["logits"] = np.array([float(v) for v in tok[1:]], np.float32)
        elif tok[0] == "ids":
            cur["ids"] = [int(v) for v in tok[1:]]
        elif tok[0] == "w":
            cur["w"] = [eval(v, {"exp": math.exp}) for v in tok[1:]]
    return cases


# ----------------------------------------------------------------------------
# independent numpy restatements used as brute-force references
# ----------------------------------------------------------------------------

def np_dequant(words, scales, biases, N, K):
    """Dense weights by numpy bit operations (not the oracle's code)."""
    words = np.asarray(words, np.uint32).reshape(N, K // 8)
    codes = (words[:, :, None] >> (4 * np.arange(8, dtype=np.uint32))) & 0xF
    codes = codes.reshape(N, K).astype(np.float64)
    s = synth.bf16_to_f32(np.asarray(scales).reshape(N, K // 64)).astype(np.float64)
    b = synth.bf16_to_f32(np.asarray(biases).reshape(N, K // 64)).astype(np.float64)
    return codes * np.repeat(s, 64, axis=1) + np.repeat(b, 64, axis=1)


def np_expert_mats(words, scales, biases, H, I):
    n1, g1 = I * H // 8, I * H // 64
    G = np_dequant(words[:n1], scales[:g1], biases[:g1], I, H)
    U = np_dequant(words[n1:2 * n1], scales[g1:2 * g1], biases[g1:2 * g1], I, H)
    D = np_dequant(words[2 * n1:], scales[2 * g1:], biases[2 * g1:], H, I)
    return G, U, D


def np_swiglu_mlp(G, U, D, X):
    """Dense SwiGLU MLP on rows of X with numpy matmuls."""
    g = X @ G.T
    u = X @ U.T
    return (g * (1.0 / (1.0 + np.exp(-g))) * u) @ D.T


def np_route_dense(logits, k):
    """Routing matrix R [T, E] via a full stable argsort of each row."""
    T, E = logits.shape
    order = np.argsort(-logits.astype(np.float64), axis=1, kind="stable")[:, :k]
    sel = np.take_along_axis(logits.astype(np.float64), order, axis=1)
    ex = np.exp(sel - sel.max(axis=1, keepdims=True))
    wts = ex / ex.sum(axis=1, keepdims=True)   # softmax over the chosen k
    R = np.zeros((T, E))
    np.put_along_axis(R, order, wts, axis=1)
    return order, wts, R


# ----------------------------------------------------------------------------
# dequantisation
# ----------------------------------------------------------------------------

def test_nibble_layout_golden(golden_dir):
    for tok in _rows(os.path.join(golden_dir, "nibble_layout.txt")):
        word = np.array([int(tok[0], 16)], np.uint32)
        want = [int(v) for v in tok[1:]]
        got = [oracle.code(word, j) for j in range(8)]
        assert got == want, tok[0]


def test_dequant_golden(golden_dir):
    for tok in _rows(os.path.join(golden_dir, "dequant_cases.txt")):
        q, sbits, bbits, want = int(tok[0]), int(tok[1], 16), int(tok[2], 16), float(tok[3])
        # one 1 x 64 matrix, element 0 carries code q, all others code 0
        words = np.zeros(8, np.uint32)
        words[0] = q
        w = oracle.dequant_matrix(words, np.array([sbits], np.uint16),
                                  np.array([bbits], np.uint16), 1, 64)
        assert w[0, 0] == want
        assert np.all(w[0, 1:] == oracle.bf16_value(bbits))  # q = 0 gives the bias


def test_pack_unpack_roundtrip():
    rng = np.random.default_rng(123)
    q = rng.integers(0, 16, size=(5, 128), dtype=np.uint8)
    words = synth.pack_nibbles(q)
    for n in range(5):
        got = [oracle.code(words[n], kk) for kk in range(128)]
        assert got == q[n].tolist()


def test_single_code_position_and_group_axis():
    """One nonzero code at (n0, k0): only that weight moves off its group's bias,
    and the bias/scale group is the one along K that contains k0."""
    N, K = 3, 192
    for n0, k0 in [(0, 0), (1, 63), (2, 64), (1, 130), (2, 191)]:
        q = np.zeros((N, K), np.uint8)
        q[n0, k0] = 9
        words = synth.pack_nibbles(q)
        s = (np.arange(N * K // 64, dtype=np.uint16) + 0x3c00).astype(np.uint16)  # distinct per group
        b = (np.arange(N * K // 64, dtype=np.uint16) + 0xbc00).astype(np.uint16)
        W = oracle.dequant_matrix(words, s, b, N, K)
        bias = synth.bf16_to_f32(b).astype(np.float64).reshape(N, K // 64)
        scale = synth.bf16_to_f32(s).astype(np.float64).reshape(N, K // 64)
        want = np.repeat(bias, 64, axis=1)
        want[n0, k0] += 9 * scale[n0, k0 // 64]
        assert np.array_equal(W, want)


def test_dequant_matches_numpy_on_random_matrix():
    rng = np.random.default_rng(7)
    words, s, b = synth.draw_matrix(rng, 16, 256)
    assert np.array_equal(oracle.dequant_matrix(words, s, b, 16, 256),
                          np_dequant(words, s, b, 16, 256))


# ----------------------------------------------------------------------------
# routing
# ----------------------------------------------------------------------------

def test_routing_golden(golden_dir):
    for c in _routing_cases(golden_dir):
        ids, w, counts, offsets, perm = oracle.route(c["logits"][None, :], c["k"])
        assert ids[0].tolist() == c["ids"], c["name"]
        np.testing.assert_allclose(w[0], c["w"], rtol=1e-14, atol=0, err_msg=c["name"])


def test_permutation_golden(golden_dir):
    f = {t[0]: [int(v) for v in t[1:]] for t in _rows(os.path.join(golden_dir, "permutation_case.txt"))}
    T, E, k = f["T"][0], f["E"][0], f["k"][0]
    ids = np.array(f["ids"]).reshape(T, k)
    logits = np.zeros((T, E), np.float32)
    for t in range(T):
        for j in range(k):
            logits[t, ids[t, j]] = 3.0 - j   # slot 0 largest, slot 1 next
    got_ids, _, counts, offsets, perm = oracle.route(logits, k)
    assert np.array_equal(got_ids, ids)
    assert counts.tolist() == f["counts"]
    assert offsets.tolist() == f["offsets"]
    assert perm.tolist() == f["perm"]


@pytest.mark.parametrize("name", ["tiny", "decode", "prefill", "zipf"])
def test_routing_invariants_and_bruteforce(name):
    w_ = synth.WORKLOADS[name]
    rng = np.random.default_rng(w_.seed)
    T = min(w_.T, 1024)
    logits = synth.draw_logits(rng, T, w_.E, w_.k, w_.logit_std, w_.zipf_s)
    ids, w, counts, offsets, perm = oracle.route(logits, w_.k)
    k, E = w_.k, w_.E
    # exactly k distinct experts per token
    assert all(len(set(r)) == k for r in ids.tolist())
    # weights sum to one and are positive
    np.testing.assert_allclose(w.sum(axis=1), 1.0, rtol=0, atol=1e-12)
    assert np.all(w > 0)
    # brute force: stable argsort of the negated logits picks the same ids in the same order,
    # and the softmax over just the chosen logits equals the renormalised full softmax
    order, wts, _ = np_route_dense(logits, k)
    assert np.array_equal(ids, order)
    np.testing.assert_allclose(w, wts, rtol=1e-12, atol=0)
    # histogram and offsets
    assert np.array_equal(counts, np.bincount(ids.ravel(), minlength=E))
    assert offsets[0] == 0 and offsets[-1] == T * k
    assert np.all(np.diff(offsets) == counts)
    # perm is a bijection on [0, T*k), grouped by expert, stable in token order
    assert np.array_equal(np.sort(perm), np.arange(T * k))
    flat = ids.ravel()
    for e in range(E):
        seg = perm[offsets[e]:offsets[e + 1]]
        assert np.all(flat[seg] == e)
        assert np.all(np.diff(seg // k) > 0)


def test_routing_selection_uses_float32_logits():
    """Two logits that differ only in float32's last place are ordered by that bit."""
    a = np.float32(1.0)
    b = np.nextafter(a, np.float32(2.0))
    logits = np.array([[a, b, 0.0, -1.0]], np.float32)
    ids, w, *_ = oracle.route(logits, 2)
    assert ids[0].tolist() == [1, 0]


# ----------------------------------------------------------------------------
# the layer
# ----------------------------------------------------------------------------

def _tiny_inputs(E=16, k=2, T=16, H=256, I=128, Is=128, seed=0, std=1.0):
    return synth.make_layer(T, H, E, k, I, Is, seed, std)


def test_layer_matches_dense_brute_force_tiny():
    """out = sum_e R[:, e] * SwiGLU_e(x) + SwiGLU_shared(x), all experts dense."""
    inp = synth.make_workload("tiny")
    out = oracle.moe_forward(inp)
    X = synth.bf16_to_f32(inp.x).astype(np.float64)
    _, _, R = np_route_dense(inp.logits, inp.k)
    want = np_swiglu_mlp(*np_expert_mats(inp.sh_packed, inp.sh_scales, inp.sh_biases, inp.H, inp.Is), X)
    for e in range(inp.E):
        Y = np_swiglu_mlp(*np_expert_mats(inp.packed[e], inp.scales[e], inp.biases[e], inp.H, inp.I), X)
        want += R[:, e:e + 1] * Y
    np.testing.assert_allclose(out, want, rtol=1e-10, atol=1e-10 * np.abs(want).max())


def test_single_expert_reduces_to_dense_swiglu():
    """E=1, k=1: the routed expert has weight 1 -> two dense SwiGLU MLPs summed."""
    inp = _tiny_inputs(E=1, k=1, T=5, seed=11)
    out = oracle.moe_forward(inp)
    X = synth.bf16_to_f32(inp.x).astype(np.float64)
    want = np_swiglu_mlp(*np_expert_mats(inp.packed[0], inp.scales[0], inp.biases[0], inp.H, inp.I), X)
    want += np_swiglu_mlp(*np_expert_mats(inp.sh_packed, inp.sh_scales, inp.sh_biases, inp.H, inp.Is), X)
    np.testing.assert_allclose(out, want, rtol=1e-10, atol=1e-10 * np.abs(want).max())


def test_all_scales_zero_closed_form():
    """scale = 0 everywhere -> W is constant per (row, group):
    gate_i = sum_g b_ig * sum_{k in g} x_k, and the same for up and down."""
    inp = _tiny_inputs(E=4, k=2, T=3, H=256, I=128, Is=192, seed=5)
    inp.scales[:] = 0
    inp.sh_scales[:] = 0
    out = oracle.moe_forward(inp)
    X = synth.bf16_to_f32(inp.x).astype(np.float64)
    ids, w, *_ = oracle.route(inp.logits, inp.k)

    def closed(biases, I):
        H = inp.H
        g1 = I * H // 64
        bg = synth.bf16_to_f32(biases[:g1]).astype(np.float64).reshape(I, H // 64)
        bu = synth.bf16_to_f32(biases[g1:2 * g1]).astype(np.float64).reshape(I, H // 64)
        bd = synth.bf16_to_f32(biases[2 * g1:]).astype(np.float64).reshape(H, I // 64)
        xg = X.reshape(X.shape[0], H // 64, 64).sum(axis=2)      # group sums of x
        g = xg @ bg.T
        u = xg @ bu.T
        a = g / (1 + np.exp(-g)) * u
        ag = a.reshape(a.shape[0], I // 64, 64).sum(axis=2)      # group sums of a
        return ag @ bd.T

    want = closed(inp.sh_biases, inp.Is)
    for e in range(inp.E):
        Ye = closed(inp.biases[e], inp.I)
        for t in range(inp.T):
            for j in range(inp.k):
                if ids[t, j] == e:
                    want[t] += w[t, j] * Ye[t]
    np.testing.assert_allclose(out, want, rtol=1e-10, atol=1e-10 * np.abs(want).max())


def test_one_hot_input_picks_weight_columns():
    """x = e_i: gate = W_gate[:, i] and up = W_up[:, i]; with k=1 the layer output is
    D @ (silu(Wg[:, i]) * Wu[:, i]) for the chosen expert plus the shared one."""
    inp = _tiny_inputs(E=3, k=1, T=1, H=128, I=64, Is=64, seed=9)
    for i in (0, 5, 63, 64, 127):
        x = np.zeros((1, inp.H), np.float32)
        x[0, i] = 1.0
        xb = synth.bf16_rne(x)
        out = oracle.moe_forward(inp, x=xb)
        e = int(np.argmax(inp.logits[0]))
        want = np.zeros(inp.H)
        for (P, S, B) in ((inp.packed[e], inp.scales[e], inp.biases[e]),
                          (inp.sh_packed, inp.sh_scales, inp.sh_biases)):
            G, U, D = np_expert_mats(P, S, B, inp.H, 64)
            g, u = G[:, i], U[:, i]
            want += D @ (g / (1 + np.exp(-g)) * u)
        np.testing.assert_allclose(out[0], want, rtol=1e-12, atol=1e-12)


def test_tokens_are_independent():
    """Running a subset of rows gives the same rows (sampled-row parity relies on it)."""
    inp = synth.make_workload("tiny")
    full = oracle.moe_forward(inp)
    rows = np.array([0, 3, 7, 15])
    sub = oracle.moe_forward(inp, x=inp.x[rows], logits=inp.logits[rows])
    assert np.array_equal(sub, full[rows])


def test_thread_count_does_not_change_result():
    inp = synth.make_workload("tiny")
    assert np.array_equal(oracle.moe_forward(inp, nthreads=1), oracle.moe_forward(inp, nthreads=4))


def test_empty_batch():
    inp = synth.make_workload("tiny", T=0)
    assert oracle.moe_forward(inp).shape == (0, inp.H)


# ----------------------------------------------------------------------------
# the by-expert form of the same layer (used to check every row at full size)
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("T,H,E,k,I,Is,chunk", [
    (16, 256, 16, 2, 128, 128, 2048),   # the tiny layer, one chunk
    (70, 512, 32, 4, 256, 384, 24),     # Is != I, several chunks with a ragged last one
    (9, 256, 8, 8, 128, 64, 4),         # every expert routed (k = E), narrow shared expert
])
def test_by_expert_form_matches_per_token_oracle(T, H, E, k, I, Is, chunk):
    inp = synth.make_layer(T, H, E, k, I, Is, seed=T + E, logit_std=1.0)
    a = oracle.moe_forward(inp)
    b = oracle.moe_forward_by_expert(inp, chunk=chunk)
    scale = np.abs(a).max(axis=1, keepdims=True)
    assert np.all(np.abs(a - b) <= 1e-12 * scale)


def test_by_expert_form_matches_dense_brute_force_tiny():
    inp = synth.make_workload("tiny")
    out = oracle.moe_forward_by_expert(inp, chunk=5)
    X = synth.bf16_to_f32(inp.x).astype(np.float64)
    _, _, R = np_route_dense(inp.logits, inp.k)
    want = np_swiglu_mlp(*np_expert_mats(inp.sh_packed, inp.sh_scales, inp.sh_biases, inp.H, inp.Is), X)
    for e in range(inp.E):
        Y = np_swiglu_mlp(*np_expert_mats(inp.packed[e], inp.scales[e], inp.biases[e], inp.H, inp.I), X)
        want += R[:, e:e + 1] * Y
    np.testing.assert_allclose(out, want, rtol=1e-10, atol=1e-10 * np.abs(want).max())


# ----------------------------------------------------------------------------
# the router scores (logits = x . W_router^T)
# ----------------------------------------------------------------------------

def test_router_logits_match_numpy_matmul():
    inp, w = synth.make_router_layer(6, 512, 32, 4, 128, 128, seed=12)
    got = oracle.router_logits(inp.x, w)
    want = synth.bf16_to_f32(inp.x).astype(np.float64) @ synth.bf16_to_f32(w).astype(np.float64).T
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())


def test_router_logits_of_one_hot_input_are_a_weight_column():
    _, w = synth.make_router_layer(1, 256, 16, 2, 128, 128, seed=13)
    for h in (0, 63, 64, 255):
        x = np.zeros((1, 256), np.float32)
        x[0, h] = 1.0
        got = oracle.router_logits(synth.bf16_rne(x), w)[0]
        assert np.array_equal(got, synth.bf16_to_f32(w[:, h]).astype(np.float64))


def test_router_logits_scale_exactly_with_a_power_of_two():
    inp, w = synth.make_router_layer(3, 256, 16, 2, 128, 128, seed=14)
    x2 = synth.bf16_rne(synth.bf16_to_f32(inp.x) * np.float32(4.0))  # exact in bf16
    assert np.array_equal(oracle.router_logits(x2, w), 4.0 * oracle.router_logits(inp.x, w))


def test_layer_with_router_is_the_layer_on_its_rounded_scores():
    inp, w = synth.make_router_layer(5, 256, 16, 2, 128, 128, seed=15)
    logits = oracle.router_logits(inp.x, w).astype(np.float32)
    assert np.array_equal(oracle.moe_forward_router(inp, w), oracle.moe_forward(inp, logits=logits))
    assert np.allclose(oracle.moe_forward_router(inp, w, by_expert=True), oracle.moe_forward(inp, logits=logits),
                       rtol=1e-12, atol=1e-12)
