"""fp64 CPU oracle of the routed int4 MoE layer (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package. The CUDA library never links, loads or calls it,
and it shares no code with the CUDA library.

The arithmetic lives in ``moe_oracle.c`` (plain C, fp64, OpenMP over tokens);
this module compiles it with gcc and marshals numpy arrays to it.
``moe_forward_by_expert`` computes the same layer with the C routing and
dequantisation and numpy's fp64 matrix products, so that every row of a
full-size batch can be checked in seconds.
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile moe_oracle.c into liboracle.so next to it (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-std=c11", "-O2", "-fopenmp", "-fPIC", "-shared", "-Wall",
               "-o", _LIB + ".tmp", _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i = ctypes.c_int
        lib.oracle_route.argtypes = [i, i, i, P, P, P, P, P, P]
        lib.oracle_route.restype = i
        lib.oracle_moe_forward.argtypes = [i, i, i, i, i, i, P, P, P, P, P, P, P, P, P, i]
        lib.oracle_moe_forward.restype = i
        lib.oracle_dequant_matrix.argtypes = [P, P, P, i, i, P]
        lib.oracle_dequant_matrix.restype = None
        lib.oracle_expert.argtypes = [i, i, P, P, P, P, P, P]
        lib.oracle_expert.restype = None
        lib.oracle_bf16_value.argtypes = [ctypes.c_uint16]
        lib.oracle_bf16_value.restype = ctypes.c_double
        lib.oracle_code.argtypes = [P, i]
        lib.oracle_code.restype = i
        lib.oracle_router_logits.argtypes = [i, i, i, P, P, P]
        lib.oracle_router_logits.restype = None
        lib.oracle_max_threads.argtypes = []
        lib.oracle_max_threads.restype = i
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def max_threads() -> int:
    return _load().oracle_max_threads()


def bf16_value(bits: int) -> float:
    return _load().oracle_bf16_value(int(bits))


def code(words: np.ndarray, kk: int) -> int:
    """4-bit code of element kk of one packed row."""
    words = _c(words, np.uint32)
    return _load().oracle_code(_ptr(words), int(kk))


def route(logits: np.ndarray, k: int):
    """Routing of T tokens: (ids i32 [T,k], w f64 [T,k], counts i32 [E], offsets i32 [E+1], perm i32 [T*k])."""
    logits = _c(logits, np.float32)
    T, E = logits.shape
    ids = np.zeros((T, k), np.int32)
    w = np.zeros((T, k), np.float64)
    counts = np.zeros(E, np.int32)
    offsets = np.zeros(E + 1, np.int32)
    perm = np.zeros(T * k, np.int32)
    rc = _load().oracle_route(T, E, k, _ptr(logits), _ptr(ids), _ptr(w), _ptr(counts),
                              _ptr(offsets), _ptr(perm))
    if rc:
        raise ValueError("oracle_route: bad arguments")
    return ids, w, counts, offsets, perm


def dequant_matrix(words: np.ndarray, scales: np.ndarray, biases: np.ndarray, N: int, K: int) -> np.ndarray:
    """Dense fp64 [N, K] weights of one packed matrix."""
    words, scales, biases = _c(words, np.uint32), _c(scales, np.uint16), _c(biases, np.uint16)
    assert words.size == N * K // 8 and scales.size == N * K // 64 == biases.size
    out = np.empty((N, K), np.float64)
    _load().oracle_dequant_matrix(_ptr(words), _ptr(scales), _ptr(biases), N, K, _ptr(out))
    return out


def expert(H: int, I: int, words, scales, biases, x: np.ndarray) -> np.ndarray:
    """One SwiGLU expert applied to one fp64 vector x [H]."""
    words, scales, biases = _c(words, np.uint32), _c(scales, np.uint16), _c(biases, np.uint16)
    x = _c(x, np.float64)
    y = np.empty(H, np.float64)
    a = np.empty(I, np.float64)
    _load().oracle_expert(H, I, _ptr(words), _ptr(scales), _ptr(biases), _ptr(x), _ptr(y), _ptr(a))
    return y


def moe_forward(inp, nthreads: int = 0, x: np.ndarray | None = None,
                logits: np.ndarray | None = None) -> np.ndarray:
    """fp64 output [T, H] of the layer for a ``synth.LayerInputs`` (x/logits may be overridden)."""
    x = _c(inp.x if x is None else x, np.uint16)
    logits = _c(inp.logits if logits is None else logits, np.float32)
    T = x.shape[0]
    assert logits.shape == (T, inp.E) and x.shape == (T, inp.H)
    out = np.empty((T, inp.H), np.float64)
    args = [_c(inp.packed, np.uint32), _c(inp.scales, np.uint16), _c(inp.biases, np.uint16),
            _c(inp.sh_packed, np.uint32), _c(inp.sh_scales, np.uint16), _c(inp.sh_biases, np.uint16)]
    rc = _load().oracle_moe_forward(T, inp.H, inp.E, inp.k, inp.I, inp.Is, _ptr(x), _ptr(logits),
                                    *[_ptr(a) for a in args], _ptr(out), int(nthreads))
    if rc:
        raise ValueError("oracle_moe_forward: bad arguments")
    return out


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns -> exact float64 (the bits are the top half of a float32)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def moe_forward_by_expert(inp, x: np.ndarray | None = None, logits: np.ndarray | None = None,
                          chunk: int = 2048) -> np.ndarray:
    """The layer of ``moe_forward``, computed expert by expert (same definition).

    Routing is the C oracle's. Each touched expert is dequantised once per
    chunk of tokens into dense fp64 matrices (C ``oracle_dequant_matrix``:
    w = q * scale + bias) and applied with fp64 matrix products to the tokens
    routed to it: g = X Wg^T, u = X Wu^T, h = silu(g) * u, y = h Wd^T. Each
    token's output is then summed in the fixed order j = 0..k-1 with its
    renormalised routing weights, then the shared expert with weight 1. Only
    the order of the additions inside a dot product differs from the per-token
    C loop (the matrix product is a library routine), so the two agree to fp64
    rounding.
    """
    x = _c(inp.x if x is None else x, np.uint16)
    logits = _c(inp.logits if logits is None else logits, np.float32)
    T, H, E, k, I, Is = x.shape[0], inp.H, inp.E, inp.k, inp.I, inp.Is
    assert logits.shape == (T, E) and x.shape == (T, H)
    out = np.empty((T, H), np.float64)
    ids_all, w_all, _, _, _ = route(logits, k)

    def expert_mats(words, scales, biases, Ie):
        n1, g1 = Ie * H // 8, Ie * H // 64
        wg = dequant_matrix(words[:n1], scales[:g1], biases[:g1], Ie, H)
        wu = dequant_matrix(words[n1:2 * n1], scales[g1:2 * g1], biases[g1:2 * g1], Ie, H)
        wd = dequant_matrix(words[2 * n1:], scales[2 * g1:], biases[2 * g1:], H, Ie)
        return wg, wu, wd

    def apply(mats, xs):
        wg, wu, wd = mats
        g = xs @ wg.T
        u = xs @ wu.T
        with np.errstate(over="ignore"):  # exp(-g) = inf for very negative g: silu -> 0
            h = g / (1.0 + np.exp(-g)) * u  # silu(gate) * up
        return h @ wd.T

    for c0 in range(0, T, chunk):
        c1 = min(T, c0 + chunk)
        xs = bf16_to_f64(x[c0:c1])
        ids, w = ids_all[c0:c1], w_all[c0:c1]
        y = np.zeros((c1 - c0, k + 1, H), np.float64)  # per (token, slot) expert outputs
        for e in np.unique(ids):
            rows, slots = np.nonzero(ids == e)
            mats = expert_mats(inp.packed[e], inp.scales[e], inp.biases[e], I)
            y[rows, slots] = apply(mats, xs[rows])
        y[:, k] = apply(expert_mats(inp.sh_packed, inp.sh_scales, inp.sh_biases, Is), xs)
        o = np.zeros((c1 - c0, H), np.float64)
        for j in range(k):
            o += w[:, j:j + 1] * y[:, j]
        o += y[:, k]  # shared expert, weight 1
        out[c0:c1] = o
    return out


def router_logits(x: np.ndarray, router_w: np.ndarray) -> np.ndarray:
    """fp64 router scores [T, E] = x [T, H] . router_w [E, H]^T from bf16 bit patterns."""
    x, router_w = _c(x, np.uint16), _c(router_w, np.uint16)
    T, H = x.shape
    E = router_w.shape[0]
    assert router_w.shape == (E, H)
    out = np.empty((T, E), np.float64)
    _load().oracle_router_logits(T, E, H, _ptr(x), _ptr(router_w), _ptr(out))
    return out


def router_logits_f32(x: np.ndarray, router_w: np.ndarray) -> np.ndarray:
    """The router scores rounded once to float32, the precision in which the
    top-k selection compares them (the layer's routing takes float32 logits)."""
    return router_logits(x, router_w).astype(np.float32)


def moe_forward_router(inp, router_w: np.ndarray, x: np.ndarray | None = None, by_expert: bool = False):
    """The layer with its router: logits = float32(x . router_w^T), then the
    layer of ``moe_forward`` (or of ``moe_forward_by_expert``) on those logits."""
    x = _c(inp.x if x is None else x, np.uint16)
    logits = router_logits_f32(x, router_w)
    if by_expert:
        return moe_forward_by_expert(inp, x=x, logits=logits)
    return moe_forward(inp, x=x, logits=logits)
