"""The C ABI on the host: the library loads, exports every declared symbol, and
rejects bad arguments before touching a GPU."""

import ctypes
import re

import pytest

from bit_grouped_expert_softmax_b200 import api


def declared_functions():
    text = open(api.HEADER_PATH).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_]+)\s*\(", text)))


def test_library_exports_every_declared_function():
    lib = api.load()
    names = declared_functions()
    assert {"moe_plan", "moe_forward", "moe_stack_forward", "moe_route"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def test_version_string():
    assert "sm_100a" in api.moe_version()


@pytest.mark.parametrize("args, fragment", [
    ((16, 250, 16, 2, 128, 128), "hidden"),
    ((16, 256, 16, 2, 96, 128), "inter"),
    ((16, 256, 16, 2, 128, 100), "shared_inter"),
    ((16, 256, 0, 1, 128, 128), "n_experts"),
    ((16, 256, 300, 8, 128, 128), "n_experts"),
    ((16, 256, 16, 0, 128, 128), "top_k"),
    ((16, 256, 4, 5, 128, 128), "top_k"),
    ((16, 256, 64, 17, 128, 128), "top_k"),
    ((0, 256, 16, 2, 128, 128), "T_max"),
])
def test_plan_rejects_bad_sizes(args, fragment):
    with pytest.raises(api.MoEError) as ei:
        api.moe_plan(*args)
    assert ei.value.status == -1
    assert fragment in str(ei.value)


def test_plan_rejects_conflicting_flags():
    with pytest.raises(api.MoEError) as ei:
        api.moe_plan(16, 256, 16, 2, 128, 128, api.MOE_FLAG_FORCE_GROUPED | api.MOE_FLAG_FORCE_SMALL_T)
    assert ei.value.status == -1


def test_calls_reject_null_plan():
    lib = api.load()
    assert lib.moe_forward(None, 1, None, None, None, None, None, None, None, None, None, None) == -1
    assert lib.moe_route(None, 1, None, None, None, None, None, None) == -1
    assert lib.moe_status_sync(None, None) == -1
    assert lib.moe_plan_destroy(None) == -1
    assert b"plan is NULL" in lib.moe_last_error()


def test_valid_plan_without_gpu_reports_no_device():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    with pytest.raises(api.MoEError) as ei:
        api.moe_plan(16, 256, 16, 2, 128, 128)
    assert ei.value.status == -6


@pytest.mark.parametrize("args, rc, fragment", [
    ((9, 2048, 256, 8, 512, 512), -1, "T must be"),
    ((1, 384, 16, 2, 128, 128), -1, "hidden"),
    ((1, 2048, 256, 8, 200, 512), -1, "inter"),
    ((1, 2048, 256, 8, 512, 100), -1, "inter"),
    ((1, 2048, 300, 8, 512, 512), -1, "n_experts"),
    ((1, 2048, 256, 17, 512, 512), -1, "top_k"),
    # the SwiGLU outputs take 8 * (top_k + 1) * max(I, Is) * 4 bytes (fp16 pairs with
    # a 4-byte launch tag) of the 512 KiB scratch less its 1280-byte header
    ((1, 2048, 256, 8, 1920, 512), -2, "512 KiB"),    # 552,960 bytes: too large
    ((1, 2048, 256, 8, 1792, 512), -1, "pointers"),   # 516,096 bytes: fits, stops at the NULL tensors
])
def test_noalloc_rejects_bad_arguments_before_touching_a_gpu(args, rc, fragment):
    lib = api.load()
    f = lib.moe_forward_small_t_noalloc
    f.argtypes = [ctypes.c_int] * 6 + [ctypes.c_void_p] * 11
    f.restype = ctypes.c_int
    assert f(*args, *([None] * 11)) == rc
    assert fragment in api.moe_last_error()


def test_noalloc_empty_batch_without_status_does_nothing():
    lib = api.load()
    f = lib.moe_forward_small_t_noalloc
    f.argtypes = [ctypes.c_int] * 6 + [ctypes.c_void_p] * 11
    f.restype = ctypes.c_int
    assert f(0, 2048, 256, 8, 512, 512, *([None] * 11)) == 0
