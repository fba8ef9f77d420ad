"""ctypes loader for libmoe_b200.so (the C ABI in include/moe_b200.h).

Loading fails loudly when the library is missing: there is no fallback path.
"""

from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

_c_int, _c_void_p, _c_float_p, _c_int_p = ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p

# name -> (restype, argtypes); pointers are passed as integers (c_void_p)
SIGNATURES = {
    "moe_create": (_c_int, [_c_int, _c_int, _c_int, _c_int, _c_int, ctypes.POINTER(ctypes.c_void_p)]),
    "moe_destroy": (_c_int, [_c_void_p]),
    "moe_load_weights": (_c_int, [_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p]),
    "moe_load_weights_fp8": (_c_int, [_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p]),
    "moe_load_weights_mixed": (_c_int, [_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p]),
    "moe_load_weights_shard": (_c_int, [_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_int, _c_int, _c_int,
                                        _c_void_p]),
    "moe_reserve": (_c_int, [_c_void_p, _c_int, _c_void_p]),
    "moe_forward": (_c_int, [_c_void_p, _c_void_p, _c_void_p, _c_int, _c_void_p, _c_void_p]),
    "moe_forward_noalloc": (_c_int, [_c_void_p, _c_void_p, _c_void_p, _c_int, _c_void_p, _c_void_p]),
    "moe_forward_host": (_c_int, [_c_void_p, _c_void_p, _c_void_p, _c_int, _c_void_p, _c_void_p]),
    "moe_status_string": (ctypes.c_char_p, [_c_int]),
    "moe_get_device_error": (_c_int, [_c_void_p, ctypes.POINTER(ctypes.c_int)]),
    "moe_last_launch_count": (_c_int, [_c_void_p]),
    "moe_last_gemm_pairs": (_c_int, [_c_void_p]),
    "moe_set_fused_decode": (_c_int, [_c_void_p, _c_int]),
    "moe_set_gemv_max_tokens": (_c_int, [_c_void_p, _c_int]),
    "moe_profile_enable": (_c_int, [_c_void_p, _c_int]),
    "moe_profile_read": (_c_int, [_c_void_p, _c_void_p, _c_void_p]),
    "moe_debug_routing": (_c_int, [_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p,
                                   _c_void_p, ctypes.POINTER(ctypes.c_int)]),
    "moe_debug_activations": (_c_int, [_c_void_p, _c_void_p, _c_void_p]),
    "moe_debug_weights": (_c_int, [_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p]),
    "moe_inv_rope_fp8_quant": (_c_int, [_c_void_p, _c_void_p, _c_void_p, _c_int, _c_int, _c_int, _c_int, _c_int,
                                        _c_int, _c_void_p, _c_void_p, _c_void_p]),
}

_lib = None


def load_library(path: str | None = None):
    """Load the library once and declare every entry point's signature."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(f"{p} is missing: build it with `python -m mixture_experts_layer_sort_b200.build` "
                           "(there is no CPU fallback)")
    lib = ctypes.CDLL(p)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if path is None:
        _lib = lib
    return lib


def status_string(code: int) -> str:
    return load_library().moe_status_string(code).decode()
