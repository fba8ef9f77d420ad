"""GPU parity of the single-launch decode path (moe_set_fused_decode): the whole
forward of up to 64 tokens in one cooperative kernel, bf16 and FP8 (e4m3, e5m2),
against the CPU oracle, with the same routing/permutation checks as the kernel
chain, and s_x bit-exact for FP8."""

import numpy as np
import pytest
import torch

from mixture_experts_layer_sort_b200 import synth
from oracle import moe_oracle as O
from tests.parity_helpers import Case, check_output, check_routing, tokens

pytestmark = pytest.mark.gpu

FMT = {"bf16": "e4m3", "fp8": "e4m3", "fp8_e5m2": "e5m2"}
TOLKEY = {"bf16": "bf16", "fp8": "fp8", "fp8_e5m2": "fp8"}


def _case(E, k, H, I, dtype, w_std=0.02):
    c = Case(E, k, H, I, dtype, w_std=w_std)
    c.layer.set_fused_decode(True)
    c.cache = {}
    return c


@pytest.fixture(scope="module", params=["bf16", "fp8", "fp8_e5m2"])
def tiny_fused(request):
    c = _case(8, 2, 256, 512, request.param)
    yield c
    c.close()


@pytest.fixture(scope="module", params=["bf16", "fp8"])
def decode_fused(request):
    wl = synth.WORKLOADS["decode"]
    c = _case(wl.E, wl.k, wl.H, wl.I, request.param, wl.w_std)
    yield c
    c.close()


def _oracle(c, x, logits):
    fp8 = c.dtype != "bf16"
    return O.moe_forward(x.float().cpu().numpy(), logits.cpu().numpy(), c.k, provider=c.provider, fp8=fp8,
                         fp8_format=FMT[c.dtype], weight_cache=c.cache if fp8 else None,
                         return_intermediates=True)


def _check(c, x, logits, M, out):
    dbg, _ = check_routing(c, logits, M)
    ref, inter = _oracle(c, x, logits)
    if c.dtype != "bf16":
        assert np.float32(dbg["s_x"]) == inter["s_x"], "s_x differs"
    check_output(out, ref, TOLKEY[c.dtype])


@pytest.mark.parametrize("M", [1, 3, 16, 37, 64])
def test_fused_tiny(tiny_fused, M):
    x, logits = tokens(tiny_fused.E, tiny_fused.H, M, seed=300 + M)
    out = tiny_fused.run(x, logits)
    assert tiny_fused.layer.last_launch_count == 1
    _check(tiny_fused, x, logits, M, out)
    assert tiny_fused.layer.device_error() == 0


@pytest.mark.parametrize("M", [1, 4, 8, 16, 32, 64])
def test_fused_decode_layer(decode_fused, M):
    x, logits = tokens(decode_fused.E, decode_fused.H, M, seed=M)
    out = decode_fused.run(x, logits)
    assert decode_fused.layer.last_launch_count == 1
    _check(decode_fused, x, logits, M, out)


def test_fused_repeated_and_skewed(tiny_fused):
    # back-to-back launches reuse the counters; all tokens on two experts
    x, logits = tokens(tiny_fused.E, tiny_fused.H, 48, seed=9)
    logits[:, 1] += 50.0
    logits[:, 6] += 40.0
    ref, _ = _oracle(tiny_fused, x, logits)
    for _ in range(3):
        out = tiny_fused.run(x, logits)
        check_output(out, ref, TOLKEY[tiny_fused.dtype])
    assert tiny_fused.layer.device_error() == 0


def test_fused_and_chain_alternate_on_one_handle(tiny_fused):
    # the two paths share the handle's workspace and must leave it clean for each other
    for i, (fused, M) in enumerate([(True, 5), (False, 5), (True, 20), (False, 64), (True, 64)]):
        tiny_fused.layer.set_fused_decode(fused)
        x, logits = tokens(tiny_fused.E, tiny_fused.H, M, seed=700 + i)
        out = tiny_fused.run(x, logits)
        assert (tiny_fused.layer.last_launch_count == 1) == fused
        ref, _ = _oracle(tiny_fused, x, logits)
        check_output(out, ref, TOLKEY[tiny_fused.dtype])
    tiny_fused.layer.set_fused_decode(True)
    assert tiny_fused.layer.device_error() == 0


def test_large_batches_keep_the_chain(tiny_fused):
    x, logits = tokens(tiny_fused.E, tiny_fused.H, 300, seed=10)
    out = tiny_fused.run(x, logits)
    assert tiny_fused.layer.last_launch_count >= 6
    ref, _ = _oracle(tiny_fused, x, logits)
    check_output(out, ref, TOLKEY[tiny_fused.dtype])
