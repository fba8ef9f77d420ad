"""The pins catch plausible mistakes: each test plants one in the oracle (on the
CPU, through monkeypatching) and checks that an independent pin then fails."""

import numpy as np
import pytest

from oracle import moe_oracle as O
from tests.test_oracle_layer import dense_brute, rand_layer


def _brute_disagrees():
    x, logits, wg, wu, wd = rand_layer(4, 4, 2, 6, 8, seed=99)
    out = O.moe_forward(x, logits, 2, wg, wu, wd)
    ref = dense_brute(x, logits, 2, wg, wu, wd)
    return not np.allclose(out, ref, rtol=1e-9, atol=1e-12)


def test_sigmoid_instead_of_silu_is_caught(monkeypatch):
    monkeypatch.setattr(O, "silu", lambda z: 1.0 / (1.0 + np.exp(-np.asarray(z, np.float64))))
    assert _brute_disagrees()


def test_missing_renormalisation_is_caught(monkeypatch):
    real = O.route

    def no_renorm(logits, k):
        ids, _ = real(logits, k)
        l64 = np.asarray(logits, np.float64)
        p = np.exp(l64 - l64.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        return ids, np.take_along_axis(p, ids.astype(np.int64), axis=1)

    monkeypatch.setattr(O, "route", no_renorm)
    assert _brute_disagrees()


def test_wrong_tie_break_is_caught(monkeypatch):
    def highest_id_first(logits, k):
        l = np.asarray(logits, np.float32)
        order = np.argsort(-l[:, ::-1], axis=1, kind="stable")
        ids = (l.shape[1] - 1 - order)[:, :k].astype(np.int32)
        w = np.full(ids.shape, 1.0 / k)
        return ids, w

    monkeypatch.setattr(O, "route", highest_id_first)
    from tests.test_oracle_routing import brute_route
    logits = np.zeros((3, 5), np.float32)
    ids, _ = O.route(logits, 2)
    assert not np.array_equal(ids, brute_route(logits, 2)[0])


def test_transposed_down_projection_is_caught(monkeypatch):
    real = O._Weights.get
    monkeypatch.setattr(O._Weights, "get", lambda self, e: (lambda g, u, d: (g, u, d.T))(*real(self, e)))
    x, logits, wg, wu, wd = rand_layer(4, 4, 2, 8, 8, seed=98)   # H == I keeps the shapes valid
    out = O.moe_forward(x, logits, 2, wg, wu, wd)
    assert not np.allclose(out, dense_brute(x, logits, 2, wg, wu, wd), rtol=1e-9, atol=1e-12)


def test_rounding_half_away_from_zero_is_caught(monkeypatch):
    monkeypatch.setattr(O.np, "rint", lambda a: np.floor(np.asarray(a) + 0.5))
    from tests.test_oracle_e4m3 import torch_codes
    bits = np.arange(65536, dtype=np.uint32) << 16
    v = bits.view(np.float32)
    v = v[np.isfinite(v)]
    assert not np.array_equal(O.e4m3_encode(v), torch_codes(v))


def test_e5m2_wrong_bias_is_caught(monkeypatch):
    # an e5m2 decode with exponent bias 16 instead of 15 disagrees with torch's decode
    real = O.e5m2_decode
    monkeypatch.setattr(O, "e5m2_decode", lambda c: real(c) * 0.5)
    from tests.test_oracle_e5m2 import test_decode_every_code_matches_torch
    with pytest.raises(AssertionError):
        test_decode_every_code_matches_torch()


def test_e5m2_scale_with_the_e4m3_maximum_is_caught(monkeypatch):
    # a quantiser that divides amax by 448 for e5m2 too fails the torch-based weight pin
    monkeypatch.setitem(O.FP8_FORMATS, "e5m2", (O.e5m2_encode, O.e5m2_decode, O.E4M3_MAX))
    from tests.test_oracle_e5m2 import test_expert_weight_quantiser_matches_torch
    with pytest.raises(AssertionError):
        test_expert_weight_quantiser_matches_torch((3, 64, 32))
