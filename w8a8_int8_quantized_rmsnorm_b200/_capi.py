"""ctypes declarations of libconvrot.so (the C ABI in include/convrot.h).

Loading the library needs no GPU; calling a compute entry point does.  There
is no fallback: if the library is missing, every call raises.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libconvrot.so")

c_int = ctypes.c_int
c_float = ctypes.c_float
c_size_t = ctypes.c_size_t
c_void_p = ctypes.c_void_p
c_char_p = ctypes.c_char_p
c_uint32_p = ctypes.POINTER(ctypes.c_uint32)

STATUS = {
    0: "CONVROT_OK",
    1: "CONVROT_ERR_NULL",
    2: "CONVROT_ERR_SHAPE",
    3: "CONVROT_ERR_ALIGN",
    4: "CONVROT_ERR_UNSUPPORTED",
    5: "CONVROT_ERR_CUDA",
    6: "CONVROT_ERR_DEVICE_TIMEOUT",
    7: "CONVROT_ERR_WORKSPACE",
}

# name -> (restype, argtypes); every symbol include/convrot.h declares
SIGNATURES = {
    "convrot_version": (c_int, []),
    "convrot_status_string": (c_char_p, [c_int]),
    "convrot_device_status": (c_int, [c_void_p, c_uint32_p]),
    "convrot_selftest_wait_timeout": (c_int, [ctypes.c_uint32, c_void_p]),
    "convrot_quantize_weight": (c_int, [c_void_p, c_int, c_int, c_int, c_void_p, c_void_p,
                                        c_void_p, c_void_p]),
    "convrot_quantize_weight_w4": (c_int, [c_void_p, c_int, c_int, c_int, c_void_p, c_float,
                                           c_float, c_int, c_void_p, c_void_p, c_void_p]),
    "convrot_smoothquant_calibrate": (c_int, [c_void_p, c_int, c_int, c_void_p, c_float,
                                              c_void_p, c_int, c_float, c_void_p, c_void_p,
                                              c_void_p]),
    "convrot_rotate_quant_act": (c_int, [c_void_p, c_int, c_int, c_int, c_void_p, c_float,
                                         c_void_p, c_void_p, c_void_p]),
    "convrot_linear_workspace_bytes": (c_size_t, [c_int, c_int, c_int, c_int]),
    "convrot_int8_linear": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_int, c_int,
                                    c_void_p, c_void_p, c_size_t, c_void_p]),
    "convrot_w4a8_linear": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_int, c_int,
                                    c_void_p, c_void_p, c_size_t, c_void_p]),
    "convrot_swiglu_workspace_bytes": (c_size_t, [c_int, c_int, c_int, c_int]),
    "convrot_int8_linear_swiglu": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_int, c_int,
                                           c_void_p, c_void_p, c_size_t, c_void_p]),
    "convrot_w4a8_linear_swiglu": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_int, c_int,
                                           c_void_p, c_void_p, c_size_t, c_void_p]),
    "convrot_interleave_gate_up": (c_int, [c_void_p, c_void_p, c_int, c_size_t, c_void_p, c_void_p]),
    "convrot_fold_row_scales": (c_int, [c_void_p, c_void_p, c_int, c_void_p]),
    "convrot_rotate_act_bf16": (c_int, [c_void_p, c_int, c_int, c_int, c_void_p, c_float, c_void_p,
                                        c_void_p]),
    "convrot_weight_only_workspace_bytes": (c_size_t, [c_int, c_int, c_int]),
    "convrot_weight_only_linear": (c_int, [c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_void_p,
                                           c_void_p, c_size_t, c_void_p]),
    "convrot_weight_only_gemm_f32": (c_int, [c_void_p, c_void_p, c_int, c_int, c_int, c_void_p,
                                             c_void_p, c_size_t, c_void_p]),
    "convrot_int8_linear_noalloc": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_int,
                                            c_int, c_void_p, c_void_p]),
    "convrot_int8_gemm_s32": (c_int, [c_void_p, c_void_p, c_int, c_int, c_int, c_void_p,
                                      c_void_p, c_size_t, c_void_p]),
    "convrot_w4a8_gemm_s32": (c_int, [c_void_p, c_void_p, c_int, c_int, c_int, c_void_p,
                                      c_void_p, c_size_t, c_void_p]),
}

_lib = None


def load(path: str = LIB_PATH):
    """Loads libconvrot.so and declares its signatures (cached)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} is missing: build it with `python -m w8a8_int8_quantized_rmsnorm_b200.build`"
            " (there is no CPU or library fallback)")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib
