"""Shared helpers of the GPU parity tests: seeded inputs, one GPU forward through
the C ABI, the oracle on the same inputs, and the comparison rule.

Tolerance (applied to the whole [M, H] output of one run):
  bf16: max|gpu - oracle| <= 1e-2 * max|oracle| + 1e-3
  FP8:  max|gpu - oracle| <= 4e-2 * max|oracle| + 2e-3
Routing ids and the padded permutation must be bit-exact; routing weights within
1e-6; FP8 weight codes, s_x and the x codes bit-exact.
"""

from __future__ import annotations

import numpy as np
import torch

from mixture_experts_layer_sort_b200 import synth
from oracle import moe_oracle as O

TOL = {"bf16": (1e-2, 1e-3), "fp8": (4e-2, 2e-3)}
PAD = 16


class Case:
    """Weights + a layer for one (E, k, H, I, dtype) shape, reusable across M."""

    def __init__(self, E, k, H, I, dtype="bf16", w_std=0.02, seed=0):
        from mixture_experts_layer_sort_b200 import MoELayer
        self.E, self.k, self.H, self.I, self.dtype, self.seed = E, k, H, I, dtype, seed
        self.wg, self.wu, self.wd = synth.make_weights(E, H, I, w_std, seed=seed, device="cuda")
        self.layer = MoELayer(E, k, H, I, dtype)
        self.layer.load_weights(self.wg, self.wu, self.wd)
        torch.cuda.synchronize()
        self._host_cache = {}

    def provider(self, e):
        if e not in self._host_cache:
            self._host_cache[e] = tuple(synth.bf16_to_f32_numpy(w[e]) for w in (self.wg, self.wu, self.wd))
            if len(self._host_cache) > 64:
                self._host_cache.pop(next(iter(self._host_cache)))
        return self._host_cache[e]

    def run(self, x, logits):
        out = self.layer.forward(x, logits)
        torch.cuda.synchronize()
        return out

    def close(self):
        self.layer.close()
        del self.wg, self.wu, self.wd
        torch.cuda.empty_cache()


def tokens(E, H, M, seed=0, zipf_s=0.0):
    return synth.make_tokens(E, H, M, seed=seed, device="cuda", zipf_s=zipf_s)


def check_output(gpu_out, ref, dtype, rows=None):
    g = gpu_out.float().cpu().numpy().astype(np.float64)
    if rows is not None:
        g = g[rows]
        ref = ref[rows]
    rtol, atol = TOL[dtype]
    err = float(np.max(np.abs(g - ref))) if g.size else 0.0
    bound = rtol * float(np.max(np.abs(ref))) + atol if ref.size else atol
    assert np.all(np.isfinite(g)), "non-finite GPU output"
    assert err <= bound, f"max abs err {err:.3e} > bound {bound:.3e}"
    return err, bound


def check_routing(case, logits, M, inter=None):
    """ids bit-exact, weights within 1e-6, counts and the padded permutation bit-exact."""
    dbg = case.layer.debug_routing(M)
    lg = logits.cpu().numpy()
    ids, w = O.route(lg, case.k)
    counts, _, sorted_pairs = O.permute(ids, case.E)
    poff, padded = O.pad_permutation(counts, sorted_pairs, dbg["tile_rows"], sentinel=M * case.k)
    assert np.array_equal(dbg["ids"].cpu().numpy(), ids), "expert ids differ"
    assert np.max(np.abs(dbg["w"].cpu().numpy() - w)) <= 1e-6, "routing weights differ"
    assert np.array_equal(dbg["counts"].cpu().numpy(), counts), "expert counts differ"
    assert np.array_equal(dbg["padded_offsets"].cpu().numpy(), poff), "padded offsets differ"
    assert np.array_equal(dbg["padded_pairs"].cpu().numpy(), padded), "padded permutation differs"
    return dbg, padded
