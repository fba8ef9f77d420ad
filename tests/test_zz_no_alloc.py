"""moe_forward_noalloc: the forward pass for callers that cannot allocate device
memory (a runtime that owns all of HBM, a stream being captured into a CUDA graph,
a loop that cannot take cudaMalloc's synchronisation). It takes its per-call
scratch from the library's fixed 32 MiB device array instead of allocating.

Checked through the C ABI against moe_forward on the same inputs, at the parity
tolerance of the other GPU tests, on two calls in a row (the second call must not
be disturbed by what the first left in the shared array). This file is collected
last on purpose, and it builds everything it needs itself, so it passes alone in a
fresh process as well as after the other tests.
"""

import ctypes

import pytest
import torch

from mixture_experts_layer_sort_b200 import MoELayer, synth

pytestmark = pytest.mark.gpu

TOL = {"bf16": (1e-2, 1e-3), "fp8": (4e-2, 2e-3)}


def _noalloc(layer, x, logits, out):
    stream = torch.cuda.current_stream().cuda_stream
    return layer.lib.moe_forward_noalloc(layer.handle, x.data_ptr(), logits.data_ptr(), x.shape[0],
                                         out.data_ptr(), stream)


def _close(a, b, dtype):
    rtol, atol = TOL[dtype]
    a = a.float()
    b = b.float()
    err = torch.max(torch.abs(a - b)).item()
    bound = rtol * torch.max(torch.abs(b)).item() + atol
    assert torch.isfinite(a).all()
    assert err <= bound, f"max abs err {err:.3e} > {bound:.3e}"


@pytest.mark.parametrize("E,k,H,I,dtype,Ms", [
    (8, 2, 256, 512, "bf16", (37, 16)),       # the carve shifts between the two calls
    (8, 2, 256, 512, "fp8", (16, 16)),
    (128, 8, 2048, 768, "bf16", (64, 64)),    # the decode layer at its largest decode batch
    (128, 8, 2048, 768, "fp8", (1, 64)),
])
def test_noalloc_matches_moe_forward_twice(E, k, H, I, dtype, Ms):
    wg, wu, wd = synth.make_weights(E, H, I, 0.02, seed=3, device="cuda")
    layer = MoELayer(E, k, H, I, dtype)
    layer.load_weights(wg, wu, wd)
    for call, M in enumerate(Ms):
        x, logits = synth.make_tokens(E, H, M, seed=10 + call, device="cuda")
        ref = layer.forward(x, logits)
        out = torch.full((M, H), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert _noalloc(layer, x, logits, out) == 0
        torch.cuda.synchronize()
        _close(out, ref, dtype)
    layer.close()


def test_noalloc_rejects_batches_beyond_the_static_scratch():
    E, k, H, I = 128, 8, 2048, 768
    wg, wu, wd = synth.make_weights(E, H, I, 0.02, seed=3, device="cuda")
    layer = MoELayer(E, k, H, I, "bf16")
    layer.load_weights(wg, wu, wd)
    M = 512
    x, logits = synth.make_tokens(E, H, M, seed=1, device="cuda")
    out = torch.zeros((M, H), dtype=torch.bfloat16, device="cuda")
    assert _noalloc(layer, x, logits, out) == -1          # MOE_ERR_INVALID_ARG, nothing launched
    torch.cuda.synchronize()
    assert torch.count_nonzero(out).item() == 0
    # M = 0 is a no-op, like moe_forward
    assert layer.lib.moe_forward_noalloc(layer.handle, None, None, 0, None, None) == 0
    layer.close()
