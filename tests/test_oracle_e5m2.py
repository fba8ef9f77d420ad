"""Pins for the oracle's e5m2 codec and its per-tensor quantiser (CPU only).

The codec is written from the format definition; here it is checked against
torch's independent float8_e5m2 conversion (exhaustively over every code and
every bf16 input), against hand-worked anchors in tests/golden, and through the
layer: an FP8 forward in e5m2 against an independent emulation with torch casts.
"""

import os

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "e5m2_anchors.txt")


def torch_codes(v32: np.ndarray) -> np.ndarray:
    """torch's RNE cast; it overflows to infinity, so clamp to the finite range first."""
    t = torch.from_numpy(np.asarray(v32, dtype=np.float32)).clamp(-57344.0, 57344.0)
    return t.to(torch.float8_e5m2).view(torch.uint8).numpy()


def test_decode_every_code_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    mine = O.e5m2_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e5m2).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(mine), nan)
    assert nan.sum() == 6                                   # 0x7d-0x7f, 0xfd-0xff
    assert np.array_equal(mine[~nan], ref[~nan])            # +-inf at 0x7c / 0xfc included


def test_encode_every_bf16_matches_torch():
    bits = np.arange(65536, dtype=np.uint32) << 16
    v = bits.view(np.float32)
    finite = np.isfinite(v)
    assert np.array_equal(O.e5m2_encode(v[finite]), torch_codes(v[finite]))


def test_encode_random_fp32_matches_torch():
    rng = np.random.default_rng(12)
    mant = rng.integers(0, 1 << 23, size=400_000, dtype=np.uint32)
    expo = rng.integers(127 - 20, 127 + 17, size=400_000, dtype=np.uint32)
    sign = rng.integers(0, 2, size=400_000, dtype=np.uint32)
    v = ((sign << 31) | (expo << 23) | mant).view(np.float32)
    assert np.array_equal(O.e5m2_encode(v), torch_codes(v))


def test_encode_saturates_and_keeps_nan():
    v = np.array([np.inf, -np.inf, 1e30, -1e30, 61440.0, np.nan], dtype=np.float32)
    c = O.e5m2_encode(v)
    assert c[:5].tolist() == [0x7B, 0xFB, 0x7B, 0xFB, 0x7B]
    assert (c[5] & 0x7F) == 0x7F


def test_golden_anchors():
    rows = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                val, code = line.split()
                rows.append((float(val), int(code, 16)))
    assert len(rows) >= 20
    vals = np.array([r[0] for r in rows], dtype=np.float32)
    assert O.e5m2_encode(vals).tolist() == [r[1] for r in rows]


def test_roundtrip_of_every_finite_code():
    codes = np.arange(256, dtype=np.uint8)
    vals = O.e5m2_decode(codes)
    finite = np.isfinite(vals)
    assert finite.sum() == 248
    again = O.e5m2_encode(vals[finite].astype(np.float32))
    assert np.array_equal(again, codes[finite])


@pytest.mark.parametrize("shape", [(3, 64, 32), (2, 17, 5)])
def test_expert_weight_quantiser_matches_torch(shape):
    g = torch.Generator().manual_seed(5)
    W = (torch.randn(shape, generator=g) * 0.02).to(torch.bfloat16).to(torch.float32)
    scales, codes = O.quantize_expert_weights(W.numpy(), "e5m2")
    for e in range(shape[0]):
        s = (W[e].abs().amax() / torch.tensor(57344.0)).to(torch.float32)
        assert np.float32(s.item()) == scales[e]
        ref = (W[e] / s).clamp(-57344, 57344).to(torch.float8_e5m2).view(torch.uint8).numpy()
        assert np.array_equal(codes[e], ref)
        assert np.max(codes[e] & 0x7F) == 0x7B              # the largest magnitude is the top code


def test_e5m2_layer_matches_torch_emulation():
    # the whole FP8 forward in e5m2 against an emulation built from torch casts only
    rng = np.random.default_rng(3)
    E, k, H, I, M = 4, 2, 32, 24, 6
    x = torch.from_numpy(rng.standard_normal((M, H)).astype(np.float32)).to(torch.bfloat16).float()
    logits = rng.standard_normal((M, E)).astype(np.float32)
    Wg = (torch.randn(E, I, H, generator=torch.Generator().manual_seed(1)) * 0.1).to(torch.bfloat16).float()
    Wu = (torch.randn(E, I, H, generator=torch.Generator().manual_seed(2)) * 0.1).to(torch.bfloat16).float()
    Wd = (torch.randn(E, H, I, generator=torch.Generator().manual_seed(3)) * 0.1).to(torch.bfloat16).float()
    out = O.moe_forward(x.numpy(), logits, k, Wg.numpy(), Wu.numpy(), Wd.numpy(), fp8=True, fp8_format="e5m2")

    def q(t):
        s = (t.abs().amax() / 57344.0).to(torch.float32)
        if s == 0:
            s = torch.tensor(1.0)
        c = (t / s).clamp(-57344, 57344).to(torch.float8_e5m2)
        return c.to(torch.float64) * s.double()

    xq = q(x)
    ids, w = O.route(logits, k)
    hs = {}
    for t in range(M):
        for j in range(k):
            e = int(ids[t, j])
            g = q(Wg[e]) @ xq[t]
            u = q(Wu[e]) @ xq[t]
            hs[(t, j)] = g / (1 + torch.exp(-g)) * u
    hall = torch.stack(list(hs.values()))
    s_h = (hall.float().abs().amax() / 57344.0).to(torch.float32)
    ref = np.zeros((M, H))
    for t in range(M):
        for j in range(k):
            e = int(ids[t, j])
            hq = (hs[(t, j)].float() / s_h).clamp(-57344, 57344).to(torch.float8_e5m2).double() * s_h.double()
            ref[t] += w[t, j] * (q(Wd[e]) @ hq).numpy()
    assert np.max(np.abs(out - ref)) <= 1e-9 * np.max(np.abs(ref)) + 1e-12
