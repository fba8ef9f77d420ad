"""moe_forward_noalloc: the forward pass for callers that cannot allocate device
memory (a serving runtime that owns all of HBM and forbids later allocations, or a
loop that cannot take the device-wide synchronisation of cudaMalloc/cudaFree). It
takes its per-call scratch from the library's fixed 32 MiB device array instead of
allocating.

Checked through the C ABI against moe_forward on the same inputs and against the
CPU oracle, at the parity tolerance of the other GPU tests, on two calls in a row
(the second call must not be disturbed by what the first left in the shared
array). The tiny-layer batch of 8400 pairs takes the one-block align for more than
8192 pairs, which moe_forward never uses (it switches to the multi-block align
there). This file is collected last on purpose, and it builds everything it needs
itself, so it passes alone in a fresh process as well as after the other tests.
"""

import numpy as np
import pytest
import torch

from mixture_experts_layer_sort_b200 import MoELayer, synth
from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu

TOL = {"bf16": (1e-2, 1e-3), "fp8": (4e-2, 2e-3), "fp8_e5m2": (4e-2, 2e-3)}


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


def _close_oracle(out, ref, dtype):
    rtol, atol = TOL[dtype]
    g = out.float().cpu().numpy().astype(np.float64)
    err = float(np.max(np.abs(g - ref)))
    bound = rtol * float(np.max(np.abs(ref))) + atol
    assert np.all(np.isfinite(g))
    assert err <= bound, f"max abs err vs oracle {err:.3e} > {bound:.3e}"


@pytest.mark.parametrize("E,k,H,I,dtype,Ms", [
    (8, 2, 256, 512, "bf16", (37, 16)),       # the carve shifts between the two calls
    (8, 2, 256, 512, "fp8", (16, 16)),
    (8, 2, 256, 512, "fp8_e5m2", (300, 5)),
    (8, 2, 256, 512, "bf16", (4200, 7)),      # 8400 pairs: one-block align above 8192 pairs
    (128, 8, 2048, 768, "bf16", (64, 64)),    # the decode layer at its largest decode batch
    (128, 8, 2048, 768, "fp8", (1, 64)),
])
def test_noalloc_matches_moe_forward_and_oracle_twice(E, k, H, I, dtype, Ms):
    wg, wu, wd = synth.make_weights(E, H, I, 0.02, seed=3, device="cuda")
    host = [synth.bf16_to_f32_numpy(w) for w in (wg, wu, wd)]
    layer = MoELayer(E, k, H, I, dtype)
    layer.load_weights(wg, wu, wd)
    fp8 = dtype != "bf16"
    for call, M in enumerate(Ms):
        x, logits = synth.make_tokens(E, H, M, seed=10 + call, device="cuda")
        ref = layer.forward(x, logits)
        out = torch.full((M, H), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert _noalloc(layer, x, logits, out) == 0
        torch.cuda.synchronize()
        _close(out, ref, dtype)
        oracle = O.moe_forward(x.float().cpu().numpy(), logits.cpu().numpy(), k, *host, fp8=fp8,
                               fp8_format="e5m2" if dtype == "fp8_e5m2" else "e4m3")
        _close_oracle(out, oracle, dtype)
    assert layer.device_error() == 0
    layer.close()


def test_noalloc_leaves_free_device_memory_unchanged():
    # the first call on a device may load the module that holds the static array;
    # after it, calls neither allocate nor free device memory
    E, k, H, I = 8, 2, 256, 512
    wg, wu, wd = synth.make_weights(E, H, I, 0.02, seed=4, device="cuda")
    layer = MoELayer(E, k, H, I, "bf16")
    layer.load_weights(wg, wu, wd)
    x, logits = synth.make_tokens(E, H, 200, seed=5, device="cuda")
    out = torch.empty((200, H), dtype=torch.bfloat16, device="cuda")
    assert _noalloc(layer, x, logits, out) == 0
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for M in (200, 1, 150):
        assert _noalloc(layer, x[:M], logits[:M], out[:M]) == 0
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
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
