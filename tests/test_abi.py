"""CPU checks of the C ABI: the library loads, exports every entry point that
include/moe_b200.h declares, and rejects bad arguments before touching a GPU."""

import ctypes
import os
import re

import pytest

from mixture_experts_layer_sort_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_b200.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(_lib.LIB_PATH):
        from mixture_experts_layer_sort_b200 import build
        build.build()
    return _lib.load_library()


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("moe_create", "moe_load_weights", "moe_forward", "moe_destroy", "moe_status_string"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} not exported"
        assert name in _lib.SIGNATURES, f"{name} has no Python signature"


def test_only_declared_symbols_are_exported(lib):
    import subprocess
    r = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True, text=True)
    if r.returncode != 0:
        pytest.skip("nm unavailable")
    exported = {l.split()[-1] for l in r.stdout.splitlines() if " T " in l and l.split()[-1].startswith("moe_")}
    assert exported == set(declared_functions())


def test_status_strings(lib):
    assert lib.moe_status_string(0) == b"ok"
    assert lib.moe_status_string(-1) == b"invalid argument"
    assert lib.moe_status_string(-6) == b"device wait timed out"
    assert lib.moe_status_string(12345) == b"unknown status"


@pytest.mark.parametrize("E,k,H,I,dt", [
    (0, 1, 256, 256, 0), (513, 8, 256, 256, 0), (8, 0, 256, 256, 0), (8, 9, 256, 256, 0),
    (8, 17, 256, 256, 0), (32, 17, 256, 256, 0), (8, 2, 200, 256, 0), (8, 2, 256, 100, 0),
    (8, 2, 0, 256, 0), (8, 2, 256, 256, 4), (8, 2, 256, 256, -1), (8, 2, 32768, 256, 0)])
def test_create_rejects_bad_shapes_without_a_gpu(lib, E, k, H, I, dt):
    h = ctypes.c_void_p()
    assert lib.moe_create(E, k, H, I, dt, ctypes.byref(h)) == -1
    assert h.value is None


def test_null_handles_are_rejected(lib):
    assert lib.moe_create(8, 2, 256, 256, 0, None) == -1
    assert lib.moe_forward(None, None, None, 4, None, None) == -1
    assert lib.moe_load_weights(None, None, None, None, None) == -1
    assert lib.moe_destroy(None) == -1
    assert lib.moe_reserve(None, 4, None) == -1
    assert lib.moe_get_device_error(None, None) == -1
    assert lib.moe_last_launch_count(None) == 0
    assert lib.moe_last_gemm_pairs(None) == 0


def test_every_entry_point_rejects_a_null_handle(lib):
    # each returns MOE_ERR_INVALID_ARG before any CUDA call
    assert lib.moe_forward_host(None, None, None, 4, None, None) == -1
    assert lib.moe_forward_noalloc(None, None, None, 4, None, None) == -1
    assert lib.moe_load_weights_fp8(None, None, None, None, None, None) == -1
    assert lib.moe_set_fused_decode(None, 1) == -1
    assert lib.moe_set_gemv_max_tokens(None, 1) == -1
    assert lib.moe_profile_enable(None, 1) == -1
    assert lib.moe_profile_read(None, None, None) == -1
    assert lib.moe_debug_routing(None, None, None, None, None, None, None, None) == -1
    assert lib.moe_debug_activations(None, None, None) == -1
    assert lib.moe_debug_weights(None, None, None, None, None) == -1


@pytest.mark.parametrize("max_pos,T,NH,D,inter,fmt", [
    (16, -1, 4, 128, 0, 1), (16, 4, 0, 128, 0, 1), (0, 4, 4, 128, 0, 1), (16, 4, 4, 96, 0, 1),
    (16, 4, 4, 512, 0, 1), (16, 4, 4, 128, 2, 1), (16, 4, 4, 128, 0, 0), (16, 4, 4, 128, 0, 3)])
def test_inv_rope_rejects_bad_arguments_without_a_gpu(lib, max_pos, T, NH, D, inter, fmt):
    # every check happens before any CUDA call
    assert lib.moe_inv_rope_fp8_quant(16, 16, 16, max_pos, T, NH, D, inter, fmt, 16, 16, None) == -1


def test_inv_rope_rejects_null_or_misaligned_pointers(lib):
    assert lib.moe_inv_rope_fp8_quant(None, 16, 16, 16, 4, 4, 128, 0, 1, 16, 16, None) == -1
    assert lib.moe_inv_rope_fp8_quant(24, 16, 16, 16, 4, 4, 128, 0, 1, 16, 16, None) == -1   # x not 16-aligned
    assert lib.moe_inv_rope_fp8_quant(16, 16, 16, 16, 0, 4, 128, 0, 1, None, None, None) == 0   # no tokens: no-op
