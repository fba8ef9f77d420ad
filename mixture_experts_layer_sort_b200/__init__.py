"""B200-native fused Mixture-of-Experts layer (sm_100a).

The compute lives in ``libmoe_b200.so`` (hand-written CUDA for sm_100a behind
a C ABI declared in ``include/moe_b200.h``); this package is a thin ctypes
binding over it plus seeded input generators. Importing the package does not
load the library: ``MoELayer`` does, and raises if it is missing.
"""

__all__ = ["MoELayer", "load_library", "MoEError", "inv_rope_fp8_quant"]


def __getattr__(name):
    if name in ("MoELayer", "MoEError", "inv_rope_fp8_quant"):
        from . import layer
        return getattr(layer, name)
    if name == "load_library":
        from ._lib import load_library
        return load_library
    raise AttributeError(name)
