"""GPU parity of a layer with a precision per expert (MOE_DTYPE_MIXED_E4M3,
moe_load_weights_mixed) against the oracle's per-expert reading: FP8 experts take the
e4m3 path (s_x over all of x, s_h over the FP8 experts' h rows only), the others bf16.
Routing and the padded permutation bit-exact, s_x bit-exact, the output within the FP8
tolerance (bf16 when no expert is FP8)."""

import numpy as np
import pytest
import torch

from mixture_experts_layer_sort_b200 import MoELayer, synth
from oracle import moe_oracle as O
from tests.parity_helpers import check_output, check_routing, tokens

pytestmark = pytest.mark.gpu


class MixedCase:
    def __init__(self, E, k, H, I, flags, w_std=0.02, seed=0):
        self.E, self.k, self.H, self.I, self.flags = E, k, H, I, np.asarray(flags, dtype=bool)
        self.wg, self.wu, self.wd = synth.make_weights(E, H, I, w_std, seed=seed, device="cuda")
        self.layer = MoELayer(E, k, H, I, "mixed")
        self.layer.load_weights_mixed(self.wg, self.wu, self.wd, self.flags)
        torch.cuda.synchronize()
        self._cache = {}

    def provider(self, e):
        if e not in self._cache:
            self._cache[e] = tuple(synth.bf16_to_f32_numpy(w[e]) for w in (self.wg, self.wu, self.wd))
        return self._cache[e]

    def check(self, M, seed):
        x, logits = tokens(self.E, self.H, M, seed=seed)
        out = self.layer.forward(x, logits)
        torch.cuda.synchronize()
        assert self.layer.last_launch_count == 9
        dbg, _ = check_routing(self, logits, M)
        ref, inter = O.moe_forward(x.float().cpu().numpy(), logits.cpu().numpy(), self.k, provider=self.provider,
                                   expert_fp8=self.flags, return_intermediates=True)
        if self.flags.any():
            assert np.float32(dbg["s_x"]) == inter["s_x"], "s_x differs"
        check_output(out, ref, "fp8" if self.flags.any() else "bf16")
        assert self.layer.device_error() == 0

    def close(self):
        self.layer.close()


TINY_FLAGS = {
    "alternate": [1, 0, 1, 0, 1, 0, 1, 0],
    "one_fp8": [0, 0, 0, 1, 0, 0, 0, 0],
    "all_fp8": [1] * 8,
    "all_bf16": [0] * 8,
}


@pytest.mark.parametrize("name", list(TINY_FLAGS))
@pytest.mark.parametrize("M", [1, 16, 37, 300])
def test_mixed_tiny(name, M):
    c = MixedCase(8, 2, 256, 512, TINY_FLAGS[name], seed=5)
    try:
        c.check(M, seed=500 + M)
    finally:
        c.close()


@pytest.mark.parametrize("M", [4, 64])
def test_mixed_decode_layer_half_fp8(M):
    wl = synth.WORKLOADS["decode"]
    flags = np.random.default_rng(7).random(wl.E) < 0.5
    c = MixedCase(wl.E, wl.k, wl.H, wl.I, flags, w_std=wl.w_std)
    try:
        c.check(M, seed=M)
        c.check(M, seed=M + 1)          # a second call on the same workspace
    finally:
        c.close()


def test_mixed_layer_rejects_the_uniform_loaders():
    E, k, H, I = 8, 2, 256, 512
    wg, wu, wd = synth.make_weights(E, H, I, 0.02, seed=1, device="cuda")
    layer = MoELayer(E, k, H, I, "mixed")
    lib, h = layer.lib, layer.handle
    assert lib.moe_load_weights(h, wg.data_ptr(), wu.data_ptr(), wd.data_ptr(), None) == -1
    assert lib.moe_load_weights_shard(h, wg.data_ptr(), wu.data_ptr(), wd.data_ptr(), I, 0, 1, None) == -1
    layer.load_weights_mixed(wg, wu, wd, [1, 0] * 4)
    x, logits = tokens(E, H, 4, seed=2)
    out = torch.empty((4, H), dtype=torch.bfloat16, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    assert lib.moe_forward_noalloc(h, x.data_ptr(), logits.data_ptr(), 4, out.data_ptr(), stream) == -5
    layer.close()
