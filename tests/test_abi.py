"""The C-ABI library builds, loads without a GPU and exports what its header declares."""
import ctypes
import os
import re

import pytest

from nvfp4_expert_layer_b200 import _lib, build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")


def _declared():
    names = set()
    for fn in os.listdir(HEADER):
        if fn.endswith(".h"):
            src = open(os.path.join(HEADER, fn)).read()
            names |= set(re.findall(r"MOE_FP4_API\s+[\w\s\*]+?\b(moe_fp4_\w+)\s*\(", src))
    return names


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def test_header_declares_the_api():
    names = _declared()
    assert {"moe_fp4_create", "moe_fp4_load_experts", "moe_fp4_forward", "moe_fp4_destroy",
            "moe_fp4_forward_ex", "moe_fp4_reserve", "moe_fp4_status_string"} <= names


def test_every_declared_symbol_is_exported(lib):
    for name in _declared():
        assert hasattr(lib, name), name
        assert name in _lib.SIGNATURES, f"binding lacks {name}"


def test_status_enum_matches_header():
    src = open(os.path.join(HEADER, "moe_fp4.h")).read()
    enum = dict((n, int(v)) for n, v in re.findall(r"(MOE_FP4_\w+)\s*=\s*(\d+)", src))
    assert enum == _lib.STATUS_CODE


def test_status_strings(lib):
    for code in _lib.STATUS:
        assert lib.moe_fp4_status_string(code)
    assert lib.moe_fp4_status_string(999) == b"unknown status"


def test_shape_checks_precede_any_cuda_call(lib):
    h = ctypes.c_void_p()
    bad = [(0, 1, 128, 128), (2000, 1, 128, 128), (8, 0, 128, 128), (8, 9, 128, 128),
           (8, 2, 100, 128), (8, 2, 128, 64), (8, 2, 32768, 128)]
    for E, k, d, f in bad:
        assert lib.moe_fp4_create(E, k, d, f, ctypes.byref(h)) == _lib.STATUS_CODE["MOE_FP4_ERR_UNSUPPORTED"]
        assert h.value is None
    assert lib.moe_fp4_create(8, 2, 128, 128, None) == _lib.STATUS_CODE["MOE_FP4_ERR_INVALID_ARG"]


def test_null_handle_calls_are_rejected(lib):
    inv = _lib.STATUS_CODE["MOE_FP4_ERR_INVALID_ARG"]
    assert lib.moe_fp4_forward(None, None, 1, None, None, None) == inv
    assert lib.moe_fp4_reserve(None, 4) == inv
    assert lib.moe_fp4_set_dense_threshold(None, 4) == inv
    assert lib.moe_fp4_load_experts(None, None) == inv
    code = ctypes.c_int()
    assert lib.moe_fp4_get_device_error(None, ctypes.byref(code)) == inv
    lib.moe_fp4_destroy(None)


def test_create_without_a_device_reports_cuda_error(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    h = ctypes.c_void_p()
    assert lib.moe_fp4_create(8, 2, 512, 256, ctypes.byref(h)) == _lib.STATUS_CODE["MOE_FP4_ERR_CUDA"]


def test_new_calls_reject_null_handles_and_bad_values(lib):
    inv = _lib.STATUS_CODE["MOE_FP4_ERR_INVALID_ARG"]
    assert lib.moe_fp4_set_expert_norm(None, 1, 1e-6) == inv
    assert lib.moe_fp4_set_act_scale(None, 1) == inv
    assert lib.moe_fp4_set_residual(None, 1) == inv
    assert lib.moe_fp4_set_resident_classes(None, 1, 1) == inv
    assert lib.moe_fp4_set_wait_timeout_ms(None, 5) == inv
    assert lib.moe_fp4_set_unreachable_wait(None, 1) == inv
    assert lib.moe_fp4_route(None, None, 1, None, None, None) == inv
    assert lib.moe_fp4_forward_routed(None, None, 1, None, None, None) == inv
    assert lib.moe_fp4_forward_layers(None, 1, None, 1, None, None, None) == inv
    # handle-free calls check their sizes before touching any pointer
    assert lib.moe_fp4_gather_rows(None, 4, 100, None, 4, 1, None, None) == inv      # d % 8
    assert lib.moe_fp4_gather_rows(None, 0, 128, None, 0, 1, None, None) == 0        # nothing to do
    assert lib.moe_fp4_combine_rows(None, None, None, -1, 1, 128, None, None) == inv
    assert lib.moe_fp4_combine_rows(None, None, None, 0, 1, 128, None, None) == 0
    import ctypes as C
    wb, sb = C.c_size_t(1), C.c_size_t(1)
    assert lib.moe_fp4_device_bytes(None, C.byref(wb), C.byref(sb)) == inv
    assert lib.moe_fp4_last_error_detail() is not None
