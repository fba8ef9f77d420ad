"""Pins for the oracle's e4m3 codec and per-tensor quantiser (CPU only).

The codec is written from the format definition; here it is checked against
torch's independent float8_e4m3fn conversion (exhaustively over every code and
every bf16 input), and against hand-worked anchors in tests/golden.
"""

import os

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "e4m3_anchors.txt")


def torch_codes(v32: np.ndarray) -> np.ndarray:
    """torch's RNE cast; it does not saturate, so clamp to the finite range first."""
    t = torch.from_numpy(np.asarray(v32, dtype=np.float32)).clamp(-448.0, 448.0)
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_decode_every_code_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    mine = O.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(mine), nan)
    assert nan.sum() == 2                                   # 0x7f and 0xff
    assert np.array_equal(mine[~nan], ref[~nan])


def test_encode_every_bf16_matches_torch():
    bits = np.arange(65536, dtype=np.uint32) << 16
    v = bits.view(np.float32)
    finite = np.isfinite(v)
    mine = O.e4m3_encode(v[finite])
    ref = torch_codes(v[finite])
    # torch maps -0.0 and tiny negatives that round to zero to 0x80 as well
    assert np.array_equal(mine, ref)


def test_encode_random_fp32_matches_torch():
    rng = np.random.default_rng(11)
    mant = rng.integers(0, 1 << 23, size=400_000, dtype=np.uint32)
    expo = rng.integers(127 - 14, 127 + 10, size=400_000, dtype=np.uint32)
    sign = rng.integers(0, 2, size=400_000, dtype=np.uint32)
    v = ((sign << 31) | (expo << 23) | mant).view(np.float32)
    assert np.array_equal(O.e4m3_encode(v), torch_codes(v))


def test_encode_saturates_and_keeps_nan():
    v = np.array([np.inf, -np.inf, 1e30, -1e30, 479.0, np.nan], dtype=np.float32)
    c = O.e4m3_encode(v)
    assert c[:5].tolist() == [0x7E, 0xFE, 0x7E, 0xFE, 0x7E]
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
    codes = O.e4m3_encode(vals)
    assert codes.tolist() == [r[1] for r in rows]
    # decode(encode(v)) == v for the exactly representable anchors
    back = O.e4m3_decode(codes)
    for (v, _), b in zip(rows, back):
        if abs(v) <= 448 and v in (1.0, -1.0, 0.5, 1.5, 3.0, 240.0, 256.0, 448.0, -448.0,
                                   0.015625, 0.013671875, 0.001953125, 0.0):
            assert b == v


def test_roundtrip_of_every_code():
    codes = np.arange(256, dtype=np.uint8)
    vals = O.e4m3_decode(codes)
    finite = ~np.isnan(vals)
    again = O.e4m3_encode(vals[finite].astype(np.float32))
    assert np.array_equal(again, codes[finite])


@pytest.mark.parametrize("shape", [(3, 64, 32), (2, 17, 5)])
def test_expert_weight_quantiser_matches_torch(shape):
    g = torch.Generator().manual_seed(4)
    W = (torch.randn(shape, generator=g) * 0.02).to(torch.bfloat16).to(torch.float32)
    W[0, 0, 0] = 0.0
    scales, codes = O.quantize_expert_weights(W.numpy())
    for e in range(shape[0]):
        s = (W[e].abs().amax() / torch.tensor(448.0)).to(torch.float32)
        assert np.float32(s.item()) == scales[e]
        ref = (W[e] / s).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        assert np.array_equal(codes[e], ref)
        # the largest magnitude lands exactly on the top code
        assert np.max(codes[e] & 0x7F) == 0x7E


def test_zero_tensor_scale_is_one():
    assert O.per_tensor_scale(np.zeros((4, 4), np.float32)) == np.float32(1.0)
    assert np.all(O.quantize(np.zeros(8, np.float32), np.float32(1.0)) == 0)
