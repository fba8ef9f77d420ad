"""Pins for the oracle's routing and permutation (CPU only).

Each check is independent of the oracle's own code: a full Python sort per
token, closed forms for k = 1 and k = 2, and an O(P*E) scan for the grouping.
"""

import math

import numpy as np
import pytest

from oracle import moe_oracle as O


def brute_route(logits, k):
    ids, ws = [], []
    for row in logits.tolist():
        ranked = sorted(range(len(row)), key=lambda e: (-row[e], e))
        S = ranked[:k]
        m = max(row)
        p = [math.exp(v - m) if v != -math.inf else 0.0 for v in row]
        Z = sum(p)
        p = [v / Z for v in p]
        ps = sum(p[e] for e in S)
        ids.append(S)
        ws.append([p[e] / ps for e in S])
    return np.array(ids), np.array(ws)


@pytest.mark.parametrize("M,E,k", [(7, 8, 2), (33, 16, 4), (5, 128, 8), (3, 6, 6), (4, 9, 1)])
def test_route_matches_full_sort(M, E, k):
    rng = np.random.default_rng(M * 1000 + E)
    logits = rng.standard_normal((M, E)).astype(np.float32)
    ids, w = O.route(logits, k)
    bi, bw = brute_route(logits, k)
    assert np.array_equal(ids, bi)
    np.testing.assert_allclose(w, bw, rtol=1e-12, atol=1e-15)


def test_route_ties_go_to_lowest_id():
    # integer-valued logits force many exact ties, plus signed zeros
    rng = np.random.default_rng(3)
    logits = rng.integers(-2, 3, size=(64, 16)).astype(np.float32)
    logits[0, :] = 0.0
    logits[0, 5] = -0.0
    ids, w = O.route(logits, 4)
    bi, bw = brute_route(logits, 4)
    assert np.array_equal(ids, bi)
    assert list(ids[0]) == [0, 1, 2, 3]          # all equal: ids ascending
    np.testing.assert_allclose(w[0], 0.25, rtol=1e-15)
    for t in range(64):                          # slot order: logit desc, id asc
        keys = [(-logits[t, e], e) for e in ids[t]]
        assert keys == sorted(keys)


def test_route_k1_weight_is_one_and_k2_closed_form():
    rng = np.random.default_rng(5)
    logits = rng.standard_normal((50, 12)).astype(np.float32) * 3
    _, w1 = O.route(logits, 1)
    assert np.all(w1 == 1.0)
    ids, w2 = O.route(logits, 2)
    l1 = logits[np.arange(50), ids[:, 0]].astype(np.float64)
    l2 = logits[np.arange(50), ids[:, 1]].astype(np.float64)
    expect = 1.0 / (1.0 + np.exp(l2 - l1))
    np.testing.assert_allclose(w2[:, 0], expect, rtol=1e-14)
    np.testing.assert_allclose(w2[:, 1], 1.0 - expect, rtol=1e-12)


def test_route_weights_sum_to_one_and_are_ordered():
    rng = np.random.default_rng(6)
    logits = rng.standard_normal((200, 128)).astype(np.float32)
    _, w = O.route(logits, 8)
    assert np.max(np.abs(w.sum(axis=1) - 1.0)) < 1e-12
    assert np.all(np.diff(w, axis=1) <= 0)       # descending logits -> descending weights


def test_route_negative_infinity_logits():
    logits = np.full((2, 6), -np.inf, dtype=np.float32)
    logits[0, [1, 4]] = [0.5, 2.0]
    logits[1, [0, 2, 5]] = [1.0, 1.0, -1.0]
    ids, w = O.route(logits, 3)
    assert list(ids[0]) == [4, 1, 0]               # third pick is the lowest -inf id
    assert w[0, 2] == 0.0
    np.testing.assert_allclose(w[0, :2].sum(), 1.0, rtol=1e-15)
    assert list(ids[1]) == [0, 2, 5]


def test_route_row_of_only_negative_infinity_is_the_equal_logit_limit():
    # no finite softmax exists; the row must equal the limit of a row of equal
    # finite logits: the k lowest ids, each with weight 1/k
    logits = np.full((3, 6), -np.inf, dtype=np.float32)
    logits[1] = np.float32(-3.0e38)
    logits[2, 4] = 0.0
    ids, w = O.route(logits, 4)
    assert list(ids[0]) == [0, 1, 2, 3]
    np.testing.assert_array_equal(ids[0], ids[1])
    np.testing.assert_allclose(w[0], np.full(4, 0.25), rtol=0, atol=0)
    np.testing.assert_allclose(w[0], w[1], rtol=0, atol=1e-15)
    assert np.all(np.isfinite(w))
    assert list(ids[2]) == [4, 0, 1, 2] and w[2, 0] == 1.0 and np.all(w[2, 1:] == 0.0)


def brute_permute(ids, E):
    flat = ids.ravel().tolist()
    counts, order = [], []
    for e in range(E):
        grp = [p for p in range(len(flat)) if flat[p] == e]
        counts.append(len(grp))
        order.extend(grp)
    return counts, order


@pytest.mark.parametrize("M,E,k", [(16, 8, 2), (64, 128, 8), (1, 128, 8), (37, 5, 3)])
def test_permute_matches_scan(M, E, k):
    rng = np.random.default_rng(M + E)
    logits = rng.standard_normal((M, E)).astype(np.float32)
    ids, _ = O.route(logits, k)
    counts, offsets, sp = O.permute(ids, E)
    bc, bo = brute_permute(ids, E)
    assert counts.tolist() == bc
    assert sp.tolist() == bo
    assert offsets[0] == 0 and offsets[-1] == M * k
    assert sorted(sp.tolist()) == list(range(M * k))   # a bijection
    for e in range(E):                                  # stable inside an expert
        grp = sp[offsets[e]:offsets[e + 1]]
        assert np.all(np.diff(grp) > 0)
        assert np.all(ids.ravel()[grp] == e)


def test_permute_all_tokens_one_expert():
    ids = np.zeros((10, 1), dtype=np.int32)
    counts, offsets, sp = O.permute(ids, 4)
    assert counts.tolist() == [10, 0, 0, 0]
    assert sp.tolist() == list(range(10))


@pytest.mark.parametrize("BT", [1, 8, 16, 128])
def test_pad_permutation(BT):
    rng = np.random.default_rng(BT)
    ids = rng.integers(0, 6, size=(20, 3)).astype(np.int32)
    counts, offsets, sp = O.permute(ids, 6)
    P = ids.size
    poff, padded = O.pad_permutation(counts, sp, BT, sentinel=P)
    assert np.all(np.diff(poff) % BT == 0)
    assert np.all(np.diff(poff) - counts >= 0) and np.all(np.diff(poff) - counts < BT)
    unpadded = padded[padded != P]
    assert np.array_equal(unpadded, sp)
    for e in range(6):
        seg = padded[poff[e]:poff[e + 1]]
        assert np.all(seg[:counts[e]] == sp[offsets[e]:offsets[e + 1]])
        assert np.all(seg[counts[e]:] == P)
