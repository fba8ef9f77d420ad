"""GPU parity of the tensor-parallel split over the intermediate dimension
(moe_load_weights_shard): G shard handles on one GPU, each loading its slice from the
full weights in the library's load kernels, each running its forward; their outputs
summed (here, in fp32, standing in for the all-reduce of TensorParallelMoE) must match
the oracle's tensor-parallel layer at the bf16 and FP8 tolerances. The bf16 sum is
also checked against the unsharded oracle (the same value in exact arithmetic)."""

import numpy as np
import pytest
import torch

from mixture_experts_layer_sort_b200 import MoELayer, synth
from oracle import moe_oracle as O
from tests.parity_helpers import check_output, tokens

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mid_weights():
    E, k, H, I = 32, 4, 1024, 1024
    w = synth.make_weights(E, H, I, 0.02, seed=21, device="cuda")
    host = [synth.bf16_to_f32_numpy(t) for t in w]
    return (E, k, H, I), w, host


def _shard_sum(dims, w, G, dtype, x, logits):
    E, k, H, I = dims
    total = torch.zeros((x.shape[0], H), dtype=torch.float32, device="cuda")
    for g in range(G):
        layer = MoELayer(E, k, H, I // G, dtype)
        layer.load_weights_shard(*w, g, G)
        total += layer.forward(x, logits).float()
        torch.cuda.synchronize()
        assert layer.device_error() == 0
        layer.close()
    return total


@pytest.mark.parametrize("G", [2, 4, 8])
@pytest.mark.parametrize("dtype", ["bf16", "fp8"])
@pytest.mark.parametrize("M", [1, 16, 100])
def test_shards_sum_to_the_oracle(mid_weights, G, dtype, M):
    dims, w, host = mid_weights
    E, k, H, I = dims
    x, logits = tokens(E, H, M, seed=40 + M)
    got = _shard_sum(dims, w, G, dtype, x, logits)
    xs, ls = x.float().cpu().numpy(), logits.cpu().numpy()
    ref = O.moe_forward_tp(xs, ls, k, *host, num_shards=G, fp8=dtype == "fp8")
    check_output(got, ref, dtype)
    if dtype == "bf16":
        check_output(got, O.moe_forward(xs, ls, k, *host), "bf16")


def test_decode_layer_split_three_and_six_ways():
    wl = synth.WORKLOADS["decode"]
    w = synth.make_weights(wl.E, wl.H, wl.I, wl.w_std, seed=0, device="cuda")
    cache = {}

    def provider(e):
        if e not in cache:
            cache[e] = tuple(synth.bf16_to_f32_numpy(t[e]) for t in w)
        return cache[e]

    x, logits = tokens(wl.E, wl.H, 4, seed=3)
    xs, ls = x.float().cpu().numpy(), logits.cpu().numpy()
    for G in (3, 6):                              # 256 and 128 intermediate features per shard
        for dtype in ("bf16", "fp8"):
            got = _shard_sum((wl.E, wl.k, wl.H, wl.I), w, G, dtype, x, logits)
            ref = O.moe_forward_tp(xs, ls, wl.k, num_shards=G, provider=provider, fp8=dtype == "fp8")
            check_output(got, ref, dtype)


def test_bad_shard_arguments_are_rejected(mid_weights):
    dims, w, _ = mid_weights
    E, k, H, I = dims
    layer = MoELayer(E, k, H, I // 4, "bf16")
    lib, hnd = layer.lib, layer.handle
    p = [t.data_ptr() for t in w]
    assert lib.moe_load_weights_shard(hnd, *p, I, 4, 4, None) == -1      # shard out of range
    assert lib.moe_load_weights_shard(hnd, *p, I, 0, 2, None) == -1      # I * 2 != I_full
    assert lib.moe_load_weights_shard(hnd, *p, I, -1, 4, None) == -1
    assert lib.moe_load_weights_shard(hnd, *p, I, 3, 4, None) == 0
    layer.close()
