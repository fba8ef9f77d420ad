"""GPU parity of the thin-batch path (kernels_gemv.cu): route + plan, then gate_up and
down as streams of warp-level tensor-core products, three launches, `out` written by
down.

Against the oracle at the layer's tolerances, with the routing, the padded
permutation, s_x and the FP8 x codes bit-exact, in bf16, e4m3 and e5m2; at the tiny,
decode and size-limit shapes; through ties and rows of -inf logits, zero input,
forwards queued without synchronisation, and alternation with the tensor-core chain on
one handle (they share the workspace and the FP8 amax words).
"""

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from tests.parity_helpers import Case, check_output, check_routing, tokens

pytestmark = pytest.mark.gpu

TOLKEY = {"bf16": "bf16", "fp8": "fp8", "fp8_e5m2": "fp8"}


def oracle(c, x, logits, **kw):
    fp8 = c.dtype != "bf16"
    return O.moe_forward(x.float().cpu().numpy(), logits.cpu().numpy(), c.k, provider=c.provider, fp8=fp8,
                         fp8_format="e5m2" if c.dtype == "fp8_e5m2" else "e4m3",
                         weight_cache=c.cache if fp8 else None, **kw)


def check(c, M, seed, x=None, logits=None, gemv=True):
    if x is None:
        x, logits = tokens(c.E, c.H, M, seed=seed)
    out = c.run(x, logits)
    assert (c.layer.last_launch_count == 3) == gemv, c.layer.last_launch_count
    dbg, padded = check_routing(c, logits, M)
    ref, inter = oracle(c, x, logits, return_intermediates=True)
    if c.dtype != "bf16":
        assert np.float32(dbg["s_x"]) == inter["s_x"], "s_x differs"
        xp, _ = c.layer.debug_activations(len(padded))
        valid = padded < M * c.k
        assert np.array_equal(xp.cpu().numpy()[valid], inter["x_codes"][padded[valid] // c.k]), "x codes differ"
    check_output(out, ref, TOLKEY[c.dtype])
    return out


@pytest.fixture(scope="module", params=["bf16", "fp8", "fp8_e5m2"])
def tiny(request):
    c = Case(8, 2, 256, 512, request.param, w_std=0.02)
    c.cache = {}
    c.layer.set_gemv_max_tokens(16)
    yield c
    c.close()


@pytest.mark.parametrize("M", [1, 2, 3, 5, 8, 13, 16])
def test_tiny(tiny, M):
    check(tiny, M, 300 + M)


def test_tiny_ties_and_infinite_logits(tiny):
    M = 12
    x, logits = tokens(tiny.E, tiny.H, M, seed=31)
    logits = torch.round(logits)              # many exact ties
    logits[0] = 0.0
    logits[1, :] = -float("inf")
    logits[1, 5] = 1.0
    logits[2, :] = -float("inf")              # no finite logit: weight 1/k each
    check(tiny, M, 0, x, logits)


def test_tiny_zero_input(tiny):
    x, logits = tokens(tiny.E, tiny.H, 6, seed=32)
    x.zero_()
    out = tiny.run(x, logits)
    assert tiny.layer.last_launch_count == 3
    assert torch.count_nonzero(out).item() == 0
    if tiny.dtype != "bf16":
        dbg = tiny.layer.debug_routing(6)
        assert dbg["s_x"] == 1.0 and dbg["s_h"] == 1.0


def test_tiny_alternating_with_the_chain(tiny):
    # thin batches, chain batches and the chain at a thin size, on one handle, in turn
    for i, (M, gemv) in enumerate([(4, True), (40, False), (16, True), (4, False), (1, True), (300, False),
                                   (2, True)]):
        tiny.layer.set_gemv_max_tokens(16 if gemv else 0)
        check(tiny, M, 400 + i, gemv=gemv and M <= 16)
    tiny.layer.set_gemv_max_tokens(16)


def test_tiny_queued_forwards(tiny):
    xs = [tokens(tiny.E, tiny.H, 7, seed=500 + i) for i in range(6)]
    outs = [tiny.layer.forward(x, l) for x, l in xs]
    torch.cuda.synchronize()
    for (x, l), out in zip(xs, outs):
        check_output(out, oracle(tiny, x, l), TOLKEY[tiny.dtype])
    assert tiny.layer.device_error() == 0


@pytest.mark.parametrize("dtype,Ms", [("bf16", (1, 4, 9, 16)), ("fp8", (1, 8, 16)), ("fp8_e5m2", (1, 8))])
def test_decode_layer(dtype, Ms):
    c = Case(128, 8, 2048, 768, dtype, w_std=0.02)
    c.cache = {}
    c.layer.set_gemv_max_tokens(16)
    try:
        for M in Ms:
            check(c, M, 600 + M)
    finally:
        c.close()


@pytest.mark.parametrize("dtype", ["bf16", "fp8"])
def test_size_limits(dtype):
    # E = 512 experts and k = 16 slots (the largest of the layer), 16 tokens
    c = Case(512, 16, 2048, 1024, dtype, w_std=0.02)
    c.cache = {}
    c.layer.set_gemv_max_tokens(16)
    try:
        for M in (1, 16):
            check(c, M, 700 + M)
    finally:
        c.close()


def test_default_thresholds():
    # new handles take the path up to 8 tokens
    for dtype, top in (("bf16", 8), ("fp8", 8)):
        c = Case(8, 2, 256, 512, dtype, w_std=0.02)
        c.cache = {}
        try:
            for M in (top, top + 1):
                check(c, M, 800 + M, gemv=M <= top)
        finally:
            c.close()
