"""ctypes binding of libmoe_b200.so with the C ABI's names.

Argument marshalling only: tensors become device pointers, streams become
cudaStream_t handles. Every step of the layer runs in the CUDA library; there
is no Python or CPU fallback, and importing a function whose library is
missing raises.
"""

from __future__ import annotations

import ctypes
import dataclasses
import os

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoe_b200.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "moe_b200.h")

MOE_OK = 0
STATUS_NAMES = {0: "MOE_OK", -1: "MOE_ERR_INVALID_ARG", -2: "MOE_ERR_UNSUPPORTED", -3: "MOE_ERR_CUDA",
                -4: "MOE_ERR_DEVICE_TIMEOUT", -5: "MOE_ERR_DEVICE_BOUNDS", -6: "MOE_ERR_NO_DEVICE"}
MOE_FLAG_NONE = 0
MOE_FLAG_FORCE_GROUPED = 1
MOE_FLAG_FORCE_SMALL_T = 2
MOE_FLAG_DEBUG = 4
MOE_FLAG_TEST_WAIT_TIMEOUT = 8
MOE_FLAG_NO_PDL = 16

_lib = None


class MoEError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


class moe_layer_weights(ctypes.Structure):
    _fields_ = [("packed_w", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("biases", ctypes.c_void_p),
                ("shared_packed_w", ctypes.c_void_p), ("shared_scales", ctypes.c_void_p),
                ("shared_biases", ctypes.c_void_p)]


def load():
    """Load the CUDA library; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m bit_grouped_expert_softmax_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, L = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
    lib.moe_plan.argtypes = [I, I, I, I, I, I, I, ctypes.POINTER(P)]
    lib.moe_plan_destroy.argtypes = [P]
    lib.moe_plan_workspace_bytes.argtypes = [P]
    lib.moe_plan_workspace_bytes.restype = L
    lib.moe_forward.argtypes = [P, I, P, P, P, P, P, P, P, P, P, P]
    lib.moe_forward_host.argtypes = [P, I, P, P, P, P, P, P, P, P, P, P]
    lib.moe_forward_router.argtypes = [P, I, P, P, P, P, P, P, P, P, P, P]
    lib.moe_router_logits.argtypes = [P, I, P, P, P, P]
    lib.moe_stack_forward.argtypes = [P, I, I, P, P, ctypes.POINTER(moe_layer_weights), P]
    lib.moe_route.argtypes = [P, I, P, P, P, P, P, P]
    lib.moe_status_sync.argtypes = [P, P]
    lib.moe_profile_enable.argtypes = [P, I]
    lib.moe_profile_read.argtypes = [P, P, P, P]
    lib.moe_last_error.restype = ctypes.c_char_p
    lib.moe_version.restype = ctypes.c_char_p
    for name in ("moe_plan", "moe_plan_destroy", "moe_forward", "moe_forward_host", "moe_forward_router",
                 "moe_router_logits", "moe_stack_forward",
                 "moe_route", "moe_status_sync", "moe_profile_enable", "moe_profile_read"):
        getattr(lib, name).restype = I
    _lib = lib
    return lib


def _check(status: int):
    if status != MOE_OK:
        raise MoEError(status, load().moe_last_error().decode())


def _ptr(t) -> int | None:
    """Device or host address of a torch tensor / numpy array, or an int address as given."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if isinstance(t, np.ndarray):
        return t.ctypes.data
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def moe_version() -> str:
    return load().moe_version().decode()


def moe_last_error() -> str:
    return load().moe_last_error().decode()


def moe_plan(T_max, hidden, n_experts, top_k, inter, shared_inter, flags=MOE_FLAG_NONE) -> int:
    p = ctypes.c_void_p()
    _check(load().moe_plan(T_max, hidden, n_experts, top_k, inter, shared_inter, flags, ctypes.byref(p)))
    return p.value


def moe_plan_destroy(plan: int):
    _check(load().moe_plan_destroy(plan))


def moe_plan_workspace_bytes(plan: int) -> int:
    return load().moe_plan_workspace_bytes(plan)


def moe_forward(plan, T, x, logits, packed_w, scales, biases, shared_packed_w, shared_scales, shared_biases,
                out, stream=None):
    _check(load().moe_forward(plan, T, _ptr(x), _ptr(logits), _ptr(packed_w), _ptr(scales), _ptr(biases),
                              _ptr(shared_packed_w), _ptr(shared_scales), _ptr(shared_biases), _ptr(out),
                              _stream(stream)))


def moe_forward_router(plan, T, x, router_w, packed_w, scales, biases, shared_packed_w, shared_scales,
                       shared_biases, out, stream=None):
    _check(load().moe_forward_router(plan, T, _ptr(x), _ptr(router_w), _ptr(packed_w), _ptr(scales), _ptr(biases),
                                     _ptr(shared_packed_w), _ptr(shared_scales), _ptr(shared_biases), _ptr(out),
                                     _stream(stream)))


def moe_router_logits(plan, T, x, router_w, logits_out, stream=None):
    _check(load().moe_router_logits(plan, T, _ptr(x), _ptr(router_w), _ptr(logits_out), _stream(stream)))


def moe_forward_host(plan, T, x_host, logits_host, packed_w, scales, biases, shared_packed_w, shared_scales,
                     shared_biases, out_host, stream=None):
    _check(load().moe_forward_host(plan, T, _ptr(x_host), _ptr(logits_host), _ptr(packed_w), _ptr(scales),
                                   _ptr(biases), _ptr(shared_packed_w), _ptr(shared_scales), _ptr(shared_biases),
                                   _ptr(out_host), _stream(stream)))


def moe_stack_forward(plan, n_layers, T, x_inout, logits, layers, stream=None):
    """layers: sequence of DeviceLayer (or anything with the six weight tensors)."""
    arr = (moe_layer_weights * max(1, n_layers))()
    for i, L in enumerate(layers[:n_layers]):
        arr[i] = moe_layer_weights(_ptr(L.packed), _ptr(L.scales), _ptr(L.biases), _ptr(L.sh_packed),
                                   _ptr(L.sh_scales), _ptr(L.sh_biases))
    _check(load().moe_stack_forward(plan, n_layers, T, _ptr(x_inout), _ptr(logits), arr, _stream(stream)))


def moe_route(plan, T, logits, ids=None, w=None, offsets=None, perm=None, stream=None):
    _check(load().moe_route(plan, T, _ptr(logits), _ptr(ids), _ptr(w), _ptr(offsets), _ptr(perm),
                            _stream(stream)))


def moe_status_sync(plan, stream=None):
    _check(load().moe_status_sync(plan, _stream(stream)))


KERNEL_NAMES = ["route_topk", "route_scan", "route_scatter", "gather", "gate_up", "down", "combine", "small_t",
                "router"]


def moe_profile_enable(plan, max_launches):
    _check(load().moe_profile_enable(plan, max_launches))


def moe_profile_read(plan, stream=None):
    """{kernel name: (total ms, launches)} since the last read."""
    ms = (ctypes.c_double * len(KERNEL_NAMES))()
    n = (ctypes.c_int32 * len(KERNEL_NAMES))()
    _check(load().moe_profile_read(plan, _stream(stream), ms, n))
    return {name: (ms[i], n[i]) for i, name in enumerate(KERNEL_NAMES) if n[i]}


# ----------------------------------------------------------------------------
# device copies of the generator's arrays (plumbing for tests and benchmark)
# ----------------------------------------------------------------------------

@dataclasses.dataclass
class DeviceLayer:
    packed: "torch.Tensor"
    scales: "torch.Tensor"
    biases: "torch.Tensor"
    sh_packed: "torch.Tensor"
    sh_scales: "torch.Tensor"
    sh_biases: "torch.Tensor"

    @classmethod
    def from_inputs(cls, inp, device="cuda"):
        import torch

        def up(a, dt):
            return torch.from_numpy(np.ascontiguousarray(a).view(dt)).to(device)

        return cls(up(inp.packed, np.int32), up(inp.scales, np.int16), up(inp.biases, np.int16),
                   up(inp.sh_packed, np.int32), up(inp.sh_scales, np.int16), up(inp.sh_biases, np.int16))

    def args(self):
        return (self.packed, self.scales, self.biases, self.sh_packed, self.sh_scales, self.sh_biases)


class Plan:
    """Owning wrapper of a moe_plan handle."""

    def __init__(self, T_max, hidden, n_experts, top_k, inter, shared_inter, flags=MOE_FLAG_NONE):
        self.handle = moe_plan(T_max, hidden, n_experts, top_k, inter, shared_inter, flags)
        self.dims = dict(T_max=T_max, H=hidden, E=n_experts, k=top_k, I=inter, Is=shared_inter)

    def close(self):
        if self.handle:
            moe_plan_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def forward(self, x, logits, layer: DeviceLayer, out=None, stream=None):
        import torch
        T = x.shape[0]
        if out is None:
            out = torch.empty_like(x)
        moe_forward(self.handle, T, x, logits, *layer.args(), out, stream)
        return out

    def route(self, logits, stream=None):
        import torch
        T, E = logits.shape
        k = self.dims["k"]
        dev = logits.device
        ids = torch.empty((T, k), dtype=torch.int32, device=dev)
        w = torch.empty((T, k), dtype=torch.float32, device=dev)
        offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
        perm = torch.empty(T * k, dtype=torch.int32, device=dev)
        moe_route(self.handle, T, logits, ids, w, offsets, perm, stream)
        return ids, w, offsets, perm

    def stack_forward(self, x, logits, layers, stream=None):
        n_layers = logits.shape[0]
        moe_stack_forward(self.handle, n_layers, x.shape[0], x, logits, layers, stream)
        return x

    def status_sync(self, stream=None):
        moe_status_sync(self.handle, stream)
