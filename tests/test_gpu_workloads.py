"""GPU parity at the workload shapes: decode (E=128 top-8, H=2048, I=768) in bf16
and FP8 at every decode batch size, the Zipf-skewed large decode layer (E=256,
H=7168, I=2048) and prefill (M=4096) on sampled tokens, in the launch
configuration bench.py times."""

import numpy as np
import pytest
import torch

from mixture_experts_layer_sort_b200 import synth
from oracle import moe_oracle as O
from tests.parity_helpers import Case, check_output, check_routing, tokens

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def decode():
    wl = synth.WORKLOADS["decode"]
    c = Case(wl.E, wl.k, wl.H, wl.I, "bf16", w_std=wl.w_std)
    yield c
    c.close()


@pytest.fixture(scope="module")
def decode_fp8():
    wl = synth.WORKLOADS["decode_fp8"]
    c = Case(wl.E, wl.k, wl.H, wl.I, "fp8", w_std=wl.w_std)
    c.cache = {}
    yield c
    c.close()


@pytest.mark.parametrize("M", [1, 4, 16, 64])
def test_decode_bf16(decode, M):
    x, logits = tokens(decode.E, decode.H, M, seed=0)
    out = decode.run(x, logits)
    check_routing(decode, logits, M)
    ref = O.moe_forward(x.float().cpu().numpy(), logits.cpu().numpy(), decode.k, provider=decode.provider)
    check_output(out, ref, "bf16")


@pytest.mark.parametrize("M", [1, 8, 32, 64])
def test_decode_fp8(decode_fp8, M):
    c = decode_fp8
    x, logits = tokens(c.E, c.H, M, seed=0)
    out = c.run(x, logits)
    dbg, padded = check_routing(c, logits, M)
    ref, inter = O.moe_forward(x.float().cpu().numpy(), logits.cpu().numpy(), c.k, provider=c.provider,
                               fp8=True, weight_cache=c.cache, return_intermediates=True)
    assert np.float32(dbg["s_x"]) == inter["s_x"]
    check_output(out, ref, "fp8")


@pytest.fixture(scope="module")
def large():
    wl = synth.WORKLOADS["large_decode"]
    c = Case(wl.E, wl.k, wl.H, wl.I, "bf16", w_std=wl.w_std)
    yield c
    c.close()


@pytest.mark.slow
@pytest.mark.parametrize("M", [1, 32, 64, 128])
def test_large_decode_bf16_zipf(large, M):
    wl = synth.WORKLOADS["large_decode"]
    x, logits = tokens(large.E, large.H, M, seed=0, zipf_s=wl.zipf_s)
    out = large.run(x, logits)
    dbg, _ = check_routing(large, logits, M)
    if M == 128:
        assert int(dbg["counts"].max()) > 64   # the skew puts most tokens on one expert
    ref = O.moe_forward(x.float().cpu().numpy(), logits.cpu().numpy(), large.k, provider=large.provider)
    check_output(out, ref, "bf16")


@pytest.mark.slow
def test_prefill_bf16_sampled(large):
    # same E/H/I as the large decode layer; uniform router logits, M = 4096
    M = 4096
    x, logits = tokens(large.E, large.H, M, seed=0)
    out = large.run(x, logits)
    check_routing(large, logits, M)
    rows = sorted(np.random.default_rng(0).choice(M, size=48, replace=False).tolist())
    ref = O.moe_forward(x.float().cpu().numpy(), logits.cpu().numpy(), large.k, provider=large.provider,
                        tokens=rows)
    check_output(out, ref, "bf16", rows=rows)


@pytest.mark.slow
def test_prefill_fp8_sampled(large):
    # the prefill layer quantised to e4m3 from the same bf16 weights; s_x and s_h are
    # per-tensor over the whole batch, so the oracle still evaluates every pair's h
    from mixture_experts_layer_sort_b200 import MoELayer
    M = 4096
    layer = MoELayer(large.E, large.k, large.H, large.I, "fp8")
    try:
        layer.load_weights(large.wg, large.wu, large.wd)
        x, logits = tokens(large.E, large.H, M, seed=1)
        out = layer.forward(x, logits)
        torch.cuda.synchronize()
        dbg = layer.debug_routing(M)
        rows = sorted(np.random.default_rng(1).choice(M, size=32, replace=False).tolist())
        ref, inter = O.moe_forward(x.float().cpu().numpy(), logits.cpu().numpy(), large.k,
                                   provider=large.provider, fp8=True, tokens=rows, return_intermediates=True)
        assert np.array_equal(dbg["ids"].cpu().numpy(), inter["ids"]), "expert ids differ"
        assert np.float32(dbg["s_x"]) == inter["s_x"], "s_x differs"
        check_output(out, ref, "fp8", rows=rows)
    finally:
        layer.close()
