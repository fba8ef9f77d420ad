"""GPU parity of the host-buffer entry point (moe_forward_host): copies in, the
forward and the copy out on one stream. Pinned buffers replay a captured graph per
(M, buffers); pageable buffers take the eager path; both must match the oracle, and
a graph must notice new weights and a grown workspace."""

import numpy as np
import pytest
import torch

from mixture_experts_layer_sort_b200 import synth
from oracle import moe_oracle as O
from tests.parity_helpers import Case, check_output

pytestmark = pytest.mark.gpu


def host_tokens(E, H, M, seed, pinned):
    x, logits = synth.make_tokens(E, H, M, seed=seed, device="cpu")
    out = torch.empty((M, H), dtype=torch.bfloat16)
    if pinned:
        x, logits, out = x.pin_memory(), logits.pin_memory(), out.pin_memory()
    return x, logits, out


@pytest.mark.parametrize("dtype", ["bf16", "fp8"])
@pytest.mark.parametrize("pinned", [True, False])
def test_forward_host_matches_oracle(dtype, pinned):
    c = Case(8, 2, 256, 512, dtype, w_std=0.02)
    try:
        for M in (1, 16, 37, 16, 300):       # 16 twice: the second call replays the cached graph
            x, logits, out = host_tokens(c.E, c.H, M, seed=M, pinned=pinned)
            for _ in range(2):
                out.fill_(0)
                c.layer.forward_host(x, logits, out)
                ref = O.moe_forward(x.float().numpy(), logits.numpy(), c.k, provider=c.provider,
                                    fp8=(dtype == "fp8"))
                check_output(out, ref, dtype)
        assert c.layer.device_error() == 0
    finally:
        c.close()


def test_forward_host_graph_sees_new_weights():
    c = Case(8, 2, 256, 512, "bf16", w_std=0.02)
    try:
        M = 24
        x, logits, out = host_tokens(c.E, c.H, M, seed=3, pinned=True)
        c.layer.forward_host(x, logits, out)
        first = out.float().clone()
        # doubled down-projection weights double the output (exactly, up to bf16 rounding)
        c.layer.load_weights(c.wg, c.wu, (c.wd.float() * 2).to(torch.bfloat16))
        c.layer.forward_host(x, logits, out)
        assert torch.allclose(out.float(), 2 * first, rtol=2e-2, atol=1e-3)
        # a larger batch grows the workspace; the smaller batch's graph must be re-made
        xb, lb, ob = host_tokens(c.E, c.H, 3000, seed=4, pinned=True)
        c.layer.forward_host(xb, lb, ob)
        c.layer.forward_host(x, logits, out)
        assert torch.allclose(out.float(), 2 * first, rtol=2e-2, atol=1e-3)
    finally:
        c.close()
