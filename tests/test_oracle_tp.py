"""Pins for the oracle's tensor-parallel reading (CPU only): the slices partition the
intermediate dimension, the sum of the bf16 shards is the unsharded layer (an exact
identity of the arithmetic: SwiGLU acts per feature and the down projection sums over
features), one shard is the plain layer, and a planted slicing mistake is caught."""

import numpy as np
import pytest

from oracle import moe_oracle as O
from tests.test_oracle_layer import rand_layer


def test_slices_partition_the_intermediate_dimension():
    _, _, wg, wu, wd = rand_layer(2, 6, 2, 16, 24, seed=1)
    parts = [O.shard_weights(wg, wu, wd, g, 4) for g in range(4)]
    assert np.array_equal(np.concatenate([p[0] for p in parts], axis=1), wg)
    assert np.array_equal(np.concatenate([p[1] for p in parts], axis=1), wu)
    assert np.array_equal(np.concatenate([p[2] for p in parts], axis=2), wd)


@pytest.mark.parametrize("G", [2, 3, 4, 8])
def test_sum_of_bf16_shards_is_the_layer(G):
    x, logits, wg, wu, wd = rand_layer(9, 6, 2, 16, 24, seed=G)
    full = O.moe_forward(x, logits, 2, wg, wu, wd)
    tp = O.moe_forward_tp(x, logits, 2, wg, wu, wd, num_shards=G)
    np.testing.assert_allclose(tp, full, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("fp8", [False, True])
def test_one_shard_is_the_plain_layer(fp8):
    x, logits, wg, wu, wd = rand_layer(5, 6, 2, 16, 24, seed=11)
    assert np.array_equal(O.moe_forward_tp(x, logits, 2, wg, wu, wd, num_shards=1, fp8=fp8),
                          O.moe_forward(x, logits, 2, wg, wu, wd, fp8=fp8))


def test_fp8_shards_are_fp8_layers_of_their_slices():
    # each rank quantises its own slice and its own h: the sum of FP8 layers over
    # slices taken here by plain indexing (not through shard_weights)
    x, logits, wg, wu, wd = rand_layer(12, 8, 2, 32, 64, seed=12)
    want = sum(O.moe_forward(x, logits, 2, wg[:, 16 * g:16 * g + 16], wu[:, 16 * g:16 * g + 16],
                             wd[:, :, 16 * g:16 * g + 16], fp8=True) for g in range(4))
    assert np.array_equal(O.moe_forward_tp(x, logits, 2, wg, wu, wd, num_shards=4, fp8=True), want)


def test_overlapping_slices_are_caught(monkeypatch):
    real = O.shard_weights

    def overlapping(w_gate, w_up, w_down, shard, num_shards):
        g, u, d = real(w_gate, w_up, w_down, shard, num_shards)
        return g, u, np.asarray(w_down)[:, :, : d.shape[2]]      # always the first columns of W_down

    monkeypatch.setattr(O, "shard_weights", overlapping)
    with pytest.raises(AssertionError):
        test_sum_of_bf16_shards_is_the_layer(2)


def test_provider_form_matches_the_array_form():
    x, logits, wg, wu, wd = rand_layer(7, 6, 2, 16, 24, seed=13)
    a = O.moe_forward_tp(x, logits, 2, wg, wu, wd, num_shards=3, fp8=True)
    b = O.moe_forward_tp(x, logits, 2, num_shards=3, provider=lambda e: (wg[e], wu[e], wd[e]), fp8=True)
    assert np.array_equal(a, b)
