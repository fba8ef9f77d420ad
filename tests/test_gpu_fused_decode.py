"""GPU parity of the single-launch decode path (moe_set_fused_decode): the whole bf16
forward of up to 64 tokens in one cooperative kernel, against the CPU oracle, with
the same routing/permutation checks as the kernel chain."""

import pytest
import torch

from mixture_experts_layer_sort_b200 import synth
from oracle import moe_oracle as O
from tests.parity_helpers import Case, check_output, check_routing, tokens

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tiny_fused():
    c = Case(8, 2, 256, 512, "bf16", w_std=0.02)
    c.layer.set_fused_decode(True)
    yield c
    c.close()


@pytest.fixture(scope="module")
def decode_fused():
    wl = synth.WORKLOADS["decode"]
    c = Case(wl.E, wl.k, wl.H, wl.I, "bf16", w_std=wl.w_std)
    c.layer.set_fused_decode(True)
    yield c
    c.close()


@pytest.mark.parametrize("M", [1, 3, 16, 37, 64])
def test_fused_tiny(tiny_fused, M):
    x, logits = tokens(tiny_fused.E, tiny_fused.H, M, seed=300 + M)
    out = tiny_fused.run(x, logits)
    assert tiny_fused.layer.last_launch_count == 1
    check_routing(tiny_fused, logits, M)
    ref = O.moe_forward(x.float().cpu().numpy(), logits.cpu().numpy(), tiny_fused.k, provider=tiny_fused.provider)
    check_output(out, ref, "bf16")


@pytest.mark.parametrize("M", [1, 4, 16, 64])
def test_fused_decode_layer(decode_fused, M):
    x, logits = tokens(decode_fused.E, decode_fused.H, M, seed=M)
    out = decode_fused.run(x, logits)
    assert decode_fused.layer.last_launch_count == 1
    check_routing(decode_fused, logits, M)
    ref = O.moe_forward(x.float().cpu().numpy(), logits.cpu().numpy(), decode_fused.k, provider=decode_fused.provider)
    check_output(out, ref, "bf16")


def test_fused_repeated_and_skewed(tiny_fused):
    # back-to-back launches reuse the counters; all tokens on two experts
    x, logits = tokens(tiny_fused.E, tiny_fused.H, 48, seed=9)
    logits[:, 1] += 50.0
    logits[:, 6] += 40.0
    ref = O.moe_forward(x.float().cpu().numpy(), logits.cpu().numpy(), tiny_fused.k, provider=tiny_fused.provider)
    for _ in range(3):
        out = tiny_fused.run(x, logits)
        check_output(out, ref, "bf16")
    assert tiny_fused.layer.device_error() == 0


def test_large_batches_keep_the_chain(tiny_fused):
    x, logits = tokens(tiny_fused.E, tiny_fused.H, 300, seed=10)
    out = tiny_fused.run(x, logits)
    assert tiny_fused.layer.last_launch_count == 6
    ref = O.moe_forward(x.float().cpu().numpy(), logits.cpu().numpy(), tiny_fused.k, provider=tiny_fused.provider)
    check_output(out, ref, "bf16")
