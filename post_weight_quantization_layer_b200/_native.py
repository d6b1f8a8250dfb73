"""ctypes loader for the native library ``lib/libgptq.so``.

The library is loaded on first use and never replaced by anything else: if it
is missing or fails to load, every call raises.  There is no CPU fallback.
"""

from __future__ import annotations

import ctypes
import os
import re
import threading

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "lib", "libgptq.so")
HEADER = os.path.join(os.path.dirname(PKG), "include", "gptq.h")

_lock = threading.Lock()
_lib = None

c_i64 = ctypes.c_int64
c_int = ctypes.c_int
c_float = ctypes.c_float
c_void_p = ctypes.c_void_p


class GptqStats(ctypes.Structure):
    _fields_ = [
        ("damped_loss", ctypes.c_double),
        ("ms_prepare", ctypes.c_float),
        ("ms_factor", ctypes.c_float),
        ("ms_sweep", ctypes.c_float),
        ("ms_pack", ctypes.c_float),
        ("panel_width", ctypes.c_int32),
        ("outer_width", ctypes.c_int32),
    ]


_SIGNATURES = {
    "gptq_accumulate_hessian": (c_int, [c_void_p, c_int, c_i64, c_i64, c_void_p, c_void_p]),
    "gptq_quantize_layer": (c_int, [c_void_p, c_int, c_i64, c_i64, c_void_p, c_int, c_int, c_float, c_int,
                                    c_int, c_int, c_int, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                    ctypes.POINTER(GptqStats)]),
    "gptq_factor_hessian": (c_int, [c_void_p, c_i64, c_float, c_int, c_void_p, c_void_p, c_void_p]),
    "gptq_factor_hessians": (c_int, [c_int, ctypes.POINTER(c_void_p), ctypes.POINTER(c_i64), c_float, c_int,
                                     ctypes.POINTER(c_void_p), ctypes.POINTER(c_void_p), c_void_p,
                                     ctypes.POINTER(c_int)]),
    "gptq_quantize_layer_factored": (c_int, [c_void_p, c_int, c_i64, c_i64, c_void_p, c_void_p, c_int, c_int,
                                             c_int, c_int, c_int, c_void_p, c_void_p, c_void_p, c_void_p,
                                             c_void_p, ctypes.POINTER(GptqStats)]),
    "gptq_quantize_linears": (c_int, [c_int, ctypes.POINTER(c_void_p), ctypes.POINTER(c_i64), c_float, c_int,
                                      ctypes.POINTER(c_void_p), ctypes.POINTER(c_void_p), c_int,
                                      ctypes.POINTER(c_void_p), c_int, ctypes.POINTER(c_i64), ctypes.POINTER(c_int),
                                      c_int, c_int, c_int, c_int, c_int, ctypes.POINTER(c_void_p),
                                      ctypes.POINTER(c_void_p), ctypes.POINTER(c_void_p), ctypes.POINTER(c_void_p),
                                      ctypes.POINTER(c_void_p), c_void_p, ctypes.POINTER(c_int)]),
    "gptq_export_layer": (c_int, [c_void_p, c_void_p, c_i64, c_i64, c_int, c_void_p, c_void_p, c_void_p]),
    "gptq_dequantize_weight": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_i64, c_i64, c_i64, c_int, c_int,
                                       c_void_p, c_void_p]),
    "gptq_quantized_linear": (c_int, [c_void_p, c_int, c_i64, c_i64, c_void_p, c_void_p, c_void_p, c_void_p,
                                      c_void_p, c_i64, c_i64, c_int, c_void_p, c_void_p]),
    "gptq_reorder_act_order": (c_int, [c_void_p, c_void_p, c_i64, c_i64, c_i64, c_int, c_void_p, c_void_p, c_void_p,
                                       c_void_p]),
    "gptq_test_wait_expiry": (c_int, [c_int, ctypes.c_uint32]),
    "gptq_rmsnorm": (c_int, [c_void_p, c_int, c_i64, c_i64, c_void_p, c_float, c_void_p, c_void_p]),
    "gptq_rope": (c_int, [c_void_p, c_int, c_i64, c_int, c_int, c_int, ctypes.c_double, c_void_p]),
    "gptq_attention": (c_int, [c_void_p, c_void_p, c_void_p, c_int, c_i64, c_int, c_int, c_int, c_void_p, c_void_p]),
    "gptq_silu_mul": (c_int, [c_void_p, c_void_p, c_int, c_i64, c_void_p, c_void_p]),
    "gptq_add": (c_int, [c_void_p, c_void_p, c_int, c_i64, c_void_p, c_void_p]),
    "gptq_device_status": (c_int, [c_void_p, c_int]),
    "gptq_trim_workspace": (c_int, []),
    "gptq_status_string": (ctypes.c_char_p, [c_int]),
    "gptq_launch_count": (ctypes.c_uint64, []),
    "gptq_version": (c_int, []),
}


def lib():
    """The loaded native library (raises RuntimeError if it is not built)."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"native GPTQ library missing at {LIB_PATH}; build it with "
                    "`python -m post_weight_quantization_layer_b200.build`")
            handle = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in _SIGNATURES.items():
                fn = getattr(handle, name)
                fn.restype = res
                fn.argtypes = args
            _lib = handle
    return _lib


def declared_symbols():
    """Names of the functions declared in include/gptq.h."""
    with open(HEADER) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gptq_[a-z_]+)\s*\(", text)))
