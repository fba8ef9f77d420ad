"""Pins for the oracle's per-expert precision choice (CPU only).

- all experts bf16 / all experts FP8 reproduce the uniform paths exactly;
- a mixed layer matches an independent dense emulation: FP8 experts through torch's
  e4m3 cast (x, weights and h quantised, s_h over the FP8 experts' h rows only),
  bf16 experts in plain fp64;
- planted mistakes (the flags ignored either way, s_h over every expert's rows) fail.
"""

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from tests.test_oracle_layer import rand_layer, torch_q, torch_scale


@pytest.mark.parametrize("fp8", [False, True])
def test_uniform_flags_are_the_uniform_paths(fp8):
    x, logits, wg, wu, wd = rand_layer(9, 6, 2, 32, 16, seed=31)
    flags = np.full(6, fp8)
    assert np.array_equal(O.moe_forward(x, logits, 2, wg, wu, wd, expert_fp8=flags),
                          O.moe_forward(x, logits, 2, wg, wu, wd, fp8=fp8))


def emulate_mixed(x, logits, k, wg, wu, wd, flags):
    """Dense evaluation of every (token, selected expert), each expert in its own precision."""
    M, H = x.shape
    E = logits.shape[1]
    ids, w = O.route(logits, k)            # routing itself is pinned in test_oracle_routing.py
    xq = torch_q(x, torch_scale(x))
    x64 = torch.as_tensor(x, dtype=torch.float64)
    W = {}
    for e in range(E):
        if flags[e]:
            W[e] = tuple(torch_q(t[e], torch_scale(t[e])) for t in (wg, wu, wd))
        else:
            W[e] = tuple(torch.as_tensor(t[e], dtype=torch.float64) for t in (wg, wu, wd))
    hs = {}
    for t in range(M):
        for j in range(k):
            e = int(ids[t, j])
            g, u, _ = W[e]
            xi = xq[t] if flags[e] else x64[t]
            hs[(t, j)] = torch.nn.functional.silu(xi @ g.T) * (xi @ u.T)
    f8_rows = [v for (t, j), v in hs.items() if flags[int(ids[t, j])]]
    amax = max((float(v.to(torch.float32).abs().max()) for v in f8_rows), default=0.0)
    s_h = np.float32(1.0) if amax == 0 else np.float32(np.float32(amax) / np.float32(448.0))
    out = np.zeros((M, H))
    for t in range(M):
        for j in range(k):
            e = int(ids[t, j])
            h = hs[(t, j)]
            if flags[e]:
                h = torch_q(h.to(torch.float32).numpy(), s_h)
            out[t] += w[t, j] * (h @ W[e][2].T).numpy()
    return out, s_h


@pytest.mark.parametrize("seed", [32, 33])
def test_mixed_layer_matches_independent_emulation(seed):
    M, E, k, H, I = 10, 6, 2, 32, 16
    x, logits, wg, wu, wd = rand_layer(M, E, k, H, I, seed=seed)
    flags = np.array([True, False, True, False, False, True])
    out, inter = O.moe_forward(x, logits, k, wg, wu, wd, expert_fp8=flags, return_intermediates=True)
    ref, s_h = emulate_mixed(x, logits, k, wg, wu, wd, flags)
    assert inter["s_h"] == s_h
    np.testing.assert_allclose(out, ref, rtol=1e-11, atol=1e-13)


def _pin_fails():
    with pytest.raises(AssertionError):
        test_mixed_layer_matches_independent_emulation(32)


def test_flags_ignored_as_all_fp8_is_caught(monkeypatch):
    real = O.moe_forward
    monkeypatch.setattr(O, "moe_forward", lambda *a, expert_fp8=None, **kw: real(*a, fp8=True, **kw))
    _pin_fails()


def test_flags_ignored_as_all_bf16_is_caught(monkeypatch):
    real = O.moe_forward

    def all_bf16(*a, expert_fp8=None, return_intermediates=False, **kw):
        out = real(*a, **kw)
        return (out, {"s_h": np.float32(1.0)}) if return_intermediates else out

    monkeypatch.setattr(O, "moe_forward", all_bf16)
    _pin_fails()


def test_s_h_over_every_expert_is_caught(monkeypatch):
    # an oracle whose s_h also covered the bf16 experts' h rows: emulate it by
    # patching the scale of the FP8 experts' h to the all-rows amax
    real = O.moe_forward

    def wide_s_h(x, logits, k, wg, wu, wd, expert_fp8=None, return_intermediates=False, **kw):
        _, inter_all = real(x, logits, k, wg, wu, wd, fp8=True, return_intermediates=True)
        out, inter = real(x, logits, k, wg, wu, wd, expert_fp8=expert_fp8, return_intermediates=True)
        inter["s_h"] = inter_all["s_h"]
        return (out, inter) if return_intermediates else out

    monkeypatch.setattr(O, "moe_forward", wide_s_h)
    _pin_fails()
