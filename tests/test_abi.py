"""C ABI checks that need no GPU: the library builds/loads, exports every
entry point include/moe.h declares, and rejects bad arguments with a status
(never a crash) before touching the device."""
import ctypes
import os
import re

import pytest

from routed_expert_ffn_forward_b200 import build, moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return moe.lib()


def declared_entry_points():
    text = open(os.path.join(ROOT, "include", "moe.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_]+)\s*\(", text)))


def test_header_and_binding_agree():
    assert declared_entry_points() == sorted(moe.EXPORTS)


def test_kernel_kinds_match_the_header():
    text = open(os.path.join(ROOT, "include", "moe.h")).read()
    kinds = {int(v): n.lower() for n, v in re.findall(r"\bMOE_K_([A-Z_]+)\s*=\s*(\d+)", text)}
    count = kinds.pop(max(kinds))
    assert count == "count" and len(moe.KERNELS) == max(kinds) + 1
    assert all(moe.KERNELS[v] == n for v, n in kinds.items())


def test_every_declared_symbol_is_exported(lib):
    for name in declared_entry_points():
        assert hasattr(lib, name), name


def test_expert_bytes():
    assert moe.moe_expert_bytes(7168, 2048) == 24_772_608
    assert moe.moe_expert_bytes(256, 128) == 2 * 128 * 144 + 256 * 1 * 144
    assert moe.moe_expert_bytes(256, 100) == 2 * 128 * 144 + 256 * 1 * 144   # rows padded to 64
    assert moe.moe_expert_bytes(300, 128) == 0          # hidden not a multiple of 256
    assert moe.moe_expert_bytes(256, 128, 2) == 0       # not Q4_K


@pytest.mark.parametrize("args,status", [
    ((255, 128, 16, 2, 0, moe.MOE_Q4_K), moe.MOE_ERR_INVALID_ARG),
    ((256, 0, 16, 2, 0, moe.MOE_Q4_K), moe.MOE_ERR_INVALID_ARG),
    ((256, 128, 0, 1, 0, moe.MOE_Q4_K), moe.MOE_ERR_INVALID_ARG),
    ((256, 128, 16, 17, 0, moe.MOE_Q4_K), moe.MOE_ERR_INVALID_ARG),
    ((256, 128, 64, 33, 0, moe.MOE_Q4_K), moe.MOE_ERR_INVALID_ARG),
    ((256, 128, 16, 2, 9, moe.MOE_Q4_K), moe.MOE_ERR_INVALID_ARG),
    ((256, 128, 16, 2, 0, 2), moe.MOE_ERR_UNSUPPORTED),
])
def test_create_rejects_bad_shapes(lib, args, status):
    h = ctypes.c_void_p()
    assert lib.moe_layer_create(*args, ctypes.byref(h)) == status
    assert h.value is None
    assert lib.moe_last_error()


def test_null_arguments(lib):
    assert lib.moe_layer_create(256, 128, 16, 2, 0, 12, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_forward(None, None, None, 1, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_set_router(None, None, None, 0) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_set_experts(None, None, None, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_get_stats(None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_layer_destroy(None) == moe.MOE_OK


def test_process_wide_settings_validate_on_the_host(lib):
    for bad in (-2, 65):
        assert lib.moe_set_few_row_tiles(bad) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_set_cache_policy(7) == moe.MOE_ERR_INVALID_ARG
    for ok in (0, 64, -1):
        assert lib.moe_set_few_row_tiles(ok) == moe.MOE_OK


def test_stats_without_gpu():
    moe.moe_reset_stats()
    s = moe.moe_get_stats()
    assert s["forwards"] == 0 and s["h2d_bytes"] == 0


def test_error_is_a_status_not_a_crash_without_gpu(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("GPU present")
    h = ctypes.c_void_p()
    st = lib.moe_layer_create(256, 128, 16, 2, 0, 12, ctypes.byref(h))
    assert st in (moe.MOE_ERR_CUDA, moe.MOE_ERR_OOM)
    assert h.value is None
