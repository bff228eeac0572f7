"""Host-side checks of libconvrot.so that need no GPU: the library loads, it
exports every entry point include/convrot.h declares, the ctypes table covers
them, and argument validation rejects bad calls before any CUDA work."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "convrot.h")


@pytest.fixture(scope="module")
def lib():
    from w8a8_int8_quantized_rmsnorm_b200 import build, _capi
    build.build()
    return _capi.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(convrot_\w+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ["convrot_quantize_weight", "convrot_quantize_weight_w4", "convrot_rotate_quant_act",
              "convrot_int8_linear", "convrot_w4a8_linear", "convrot_smoothquant_calibrate",
              "convrot_int8_gemm_s32", "convrot_w4a8_gemm_s32", "convrot_device_status",
              "convrot_status_string", "convrot_linear_workspace_bytes", "convrot_version"]:
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    from w8a8_int8_quantized_rmsnorm_b200 import _capi
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert name in _capi.SIGNATURES, name


def test_version_and_status_strings(lib):
    assert lib.convrot_version() >> 16 == 1
    for code, name in __import__("w8a8_int8_quantized_rmsnorm_b200._capi",
                                 fromlist=["STATUS"]).STATUS.items():
        assert lib.convrot_status_string(code).decode().startswith(name)


def _p(v):
    return ctypes.c_void_p(v)


def test_validation_before_any_launch(lib):
    # fake but aligned device addresses: validation must reject before launching
    A = _p(0x10000)
    # unsupported group
    assert lib.convrot_rotate_quant_act(A, 4, 512, 128, None, 1e-6, A, A, None) == 4
    # K not a multiple of the group
    assert lib.convrot_rotate_quant_act(A, 4, 384, 256, None, 1e-6, A, A, None) == 2
    # K not a multiple of 16 with group 0 or 16
    assert lib.convrot_rotate_quant_act(A, 4, 40, 0, None, 1e-6, A, A, None) == 2
    assert lib.convrot_rotate_quant_act(A, 4, 40, 16, None, 1e-6, A, A, None) == 2
    # int4 weights need K % 32 also with group 16
    assert lib.convrot_quantize_weight_w4(A, 4, 4304, 16, None, 0.8, 1.0, 21, A, A, None) == 2
    # null pointers
    assert lib.convrot_rotate_quant_act(None, 4, 512, 256, None, 1e-6, A, A, None) == 1
    assert lib.convrot_quantize_weight(A, 4, 512, 256, None, None, A, None) == 1
    # misaligned matrix
    assert lib.convrot_rotate_quant_act(_p(0x10008), 4, 512, 256, None, 1e-6, A, A, None) == 3
    # misaligned norm weight
    assert lib.convrot_rotate_quant_act(A, 4, 512, 256, _p(0x10004), 1e-6, A, A, None) == 3
    # M = 0 is a no-op
    assert lib.convrot_rotate_quant_act(None, 0, 512, 256, None, 1e-6, None, None, None) == 0
    assert lib.convrot_int8_linear(None, None, None, None, 0, 256, 512, None, None, 0, None) == 0
    # GEMM shape rules
    assert lib.convrot_int8_linear(A, A, A, A, 4, 12, 512, A, None, 0, None) == 2   # N % 8
    assert lib.convrot_int8_linear(A, A, A, A, 4, 16, 40, A, None, 0, None) == 2    # K % 16
    assert lib.convrot_w4a8_linear(A, A, A, A, 4, 16, 48, A, None, 0, None) == 2    # K % 32
    assert lib.convrot_int8_linear(A, A, A, A, 4, 16, 131072 + 16, A, None, 0, None) == 2
    assert lib.convrot_int8_gemm_s32(None, A, 4, 16, 512, A, None, 0, None) == 1
    # int4 clip grid
    assert lib.convrot_quantize_weight_w4(A, 4, 512, 256, None, 0.8, 1.0, 0, A, A, None) == 2
    assert lib.convrot_quantize_weight_w4(A, 4, 512, 256, None, 1.0, 0.8, 21, A, A, None) == 2
    # the wait-timeout self-test validates its bound before launching
    assert lib.convrot_selftest_wait_timeout(0, None) == 2
    assert lib.convrot_selftest_wait_timeout(999, None) == 2
    assert lib.convrot_selftest_wait_timeout(100000001, None) == 2
    # calibration may not fold in place
    assert lib.convrot_smoothquant_calibrate(A, 4, 512, A, 1e-6, A, 8, 0.5, A, A, None) == 4
    # weight-only path: shapes, pointers and alignment before any device query
    assert lib.convrot_weight_only_linear(A, A, A, 4, 12, 512, A, None, 0, None) == 2   # N % 8
    assert lib.convrot_weight_only_linear(A, A, A, 4, 16, 40, A, None, 0, None) == 2    # K % 16
    assert lib.convrot_weight_only_linear(A, A, None, 4, 16, 512, A, None, 0, None) == 1  # s_row
    assert lib.convrot_weight_only_gemm_f32(A, A, 4, 16, 512, None, None, 0, None) == 1
    assert lib.convrot_weight_only_linear(_p(0x10008), A, A, 4, 16, 512, A, None, 0, None) == 3
    assert lib.convrot_weight_only_linear(None, None, None, 0, 16, 512, None, None, 0, None) == 0
    assert lib.convrot_weight_only_workspace_bytes(4, 12, 512) == 0  # invalid shape: no size


def test_binding_refuses_cpu_tensors():
    import torch
    import w8a8_int8_quantized_rmsnorm_b200 as cr
    with pytest.raises(ValueError):
        cr.convrot_rotate_quant_act(torch.zeros(4, 256, dtype=torch.bfloat16))
