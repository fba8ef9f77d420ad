"""GPU parity of the small-batch path (batches of up to 64 tokens): route -> gate_up
-> down for bf16, route -> quant_x -> gate_up -> quant_h -> down for FP8, the GEMMs
building the batch's schedule themselves, gate_up reading token rows directly and down
finishing token rows itself. Against the oracle, with the routing and the padded
permutation bit-exact, through back-to-back calls and alternating with the full chain
(larger batches) on one handle, which share the workspace, the fp32 accumulator and
the FP8 amax words."""

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from tests.parity_helpers import Case, check_output, check_routing, tokens

pytestmark = pytest.mark.gpu

LAUNCHES = {"bf16": 3, "fp8": 5, "fp8_e5m2": 5}
TOLKEY = {"bf16": "bf16", "fp8": "fp8", "fp8_e5m2": "fp8"}


@pytest.fixture(scope="module", params=["bf16", "fp8", "fp8_e5m2"])
def tiny(request):
    c = Case(8, 2, 256, 512, request.param, w_std=0.02)
    c.cache = {}
    yield c
    c.close()


def _check(c, M, seed):
    x, logits = tokens(c.E, c.H, M, seed=seed)
    out = c.run(x, logits)
    dbg, _ = check_routing(c, logits, M)
    fp8 = c.dtype != "bf16"
    ref, inter = O.moe_forward(x.float().cpu().numpy(), logits.cpu().numpy(), c.k, provider=c.provider, fp8=fp8,
                               fp8_format="e5m2" if c.dtype == "fp8_e5m2" else "e4m3",
                               weight_cache=c.cache if fp8 else None, return_intermediates=True)
    if fp8:
        assert np.float32(dbg["s_x"]) == inter["s_x"], "s_x differs"
    check_output(out, ref, TOLKEY[c.dtype])
    return c.layer.last_launch_count


def test_small_batches_take_the_short_chain(tiny):
    for M in (1, 2, 16, 33, 64):
        assert _check(tiny, M, seed=900 + M) == LAUNCHES[tiny.dtype]
    assert tiny.layer.device_error() == 0


def test_small_and_full_chain_alternate(tiny):
    # M <= 64 takes the small-batch path, M = 65 and 300 the full chain
    for i, M in enumerate((5, 300, 64, 65, 1, 300, 16)):
        n = _check(tiny, M, seed=950 + i)
        assert (n == LAUNCHES[tiny.dtype]) == (M <= 64)
    assert tiny.layer.device_error() == 0


def test_back_to_back_without_synchronisation(tiny):
    # five forwards queued on one stream before anyone reads: the token counters, the
    # accumulator and the amax words must be clean for each next forward
    xs = [tokens(tiny.E, tiny.H, 16, seed=970 + i) for i in range(5)]
    outs = [tiny.layer.forward(x, l) for x, l in xs]
    torch.cuda.synchronize()
    fp8 = tiny.dtype != "bf16"
    for (x, l), out in zip(xs, outs):
        ref = O.moe_forward(x.float().cpu().numpy(), l.cpu().numpy(), tiny.k, provider=tiny.provider, fp8=fp8,
                            fp8_format="e5m2" if tiny.dtype == "fp8_e5m2" else "e4m3",
                            weight_cache=tiny.cache if fp8 else None)
        check_output(out, ref, TOLKEY[tiny.dtype])
