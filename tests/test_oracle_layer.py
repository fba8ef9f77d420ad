"""Pins for the oracle's full layer (CPU only).

- a dense brute force in pure Python loops (every expert on every token, a
  dense gate matrix that is zero off the selected set): an independent code
  path from the oracle's grouped, permuted evaluation;
- topk = E with identical experts reduces to one dense SwiGLU FFN;
- E = 1, k = 1 reduces to torch's fp64 silu / matmul;
- token-permutation equivariance, x = 0, exact scaling by 2;
- the FP8 path against an independent emulation built on torch's e4m3 cast.
"""

import math

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O


def rand_layer(M, E, k, H, I, seed, std=0.3):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, H)).astype(np.float32)
    logits = rng.standard_normal((M, E)).astype(np.float32)
    wg = (rng.standard_normal((E, I, H)) * std).astype(np.float32)
    wu = (rng.standard_normal((E, I, H)) * std).astype(np.float32)
    wd = (rng.standard_normal((E, H, I)) * std).astype(np.float32)
    return x, logits, wg, wu, wd


def dense_brute(x, logits, k, wg, wu, wd):
    M, H = x.shape
    E = logits.shape[1]
    I = wg.shape[1]
    x, logits, wg, wu, wd = (a.tolist() for a in (x, logits, wg, wu, wd))
    out = [[0.0] * H for _ in range(M)]
    for t in range(M):
        row = logits[t]
        S = sorted(range(E), key=lambda e: (-row[e], e))[:k]
        m = max(row)
        p = [math.exp(v - m) for v in row]
        Z = sum(p)
        ps = sum(p[e] / Z for e in S)
        gate = [(p[e] / Z) / ps if e in S else 0.0 for e in range(E)]
        for e in range(E):
            hv = []
            for i in range(I):
                g = sum(wg[e][i][j] * x[t][j] for j in range(H))
                u = sum(wu[e][i][j] * x[t][j] for j in range(H))
                hv.append(g / (1.0 + math.exp(-g)) * u)
            for o in range(H):
                out[t][o] += gate[e] * sum(wd[e][o][i] * hv[i] for i in range(I))
    return np.array(out)


@pytest.mark.parametrize("M,E,k,H,I", [(5, 4, 2, 8, 16), (3, 6, 3, 4, 8), (4, 3, 1, 6, 4)])
def test_layer_matches_dense_brute_force(M, E, k, H, I):
    x, logits, wg, wu, wd = rand_layer(M, E, k, H, I, seed=M * 7 + E)
    out = O.moe_forward(x, logits, k, wg, wu, wd)
    ref = dense_brute(x, logits, k, wg, wu, wd)
    np.testing.assert_allclose(out, ref, rtol=1e-11, atol=1e-13)


def swiglu_ffn(x, g, u, d):
    x = torch.from_numpy(np.asarray(x, np.float64))
    g, u, d = (torch.from_numpy(np.asarray(a, np.float64)) for a in (g, u, d))
    return (torch.nn.functional.silu(x @ g.T) * (x @ u.T) @ d.T).numpy()


def test_topk_equals_E_with_identical_experts_is_a_dense_ffn():
    M, E, H, I = 9, 5, 16, 24
    x, logits, wg, wu, wd = rand_layer(M, E, E, H, I, seed=21)
    wg[:] = wg[0]
    wu[:] = wu[0]
    wd[:] = wd[0]
    out = O.moe_forward(x, logits, E, wg, wu, wd)
    np.testing.assert_allclose(out, swiglu_ffn(x, wg[0], wu[0], wd[0]), rtol=1e-12, atol=1e-13)


def test_single_expert_is_textbook_swiglu():
    x, logits, wg, wu, wd = rand_layer(11, 1, 1, 32, 48, seed=2)
    out = O.moe_forward(x, logits, 1, wg, wu, wd)
    np.testing.assert_allclose(out, swiglu_ffn(x, wg[0], wu[0], wd[0]), rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("fp8", [False, True])
def test_token_permutation_equivariance(fp8):
    x, logits, wg, wu, wd = rand_layer(12, 6, 2, 16, 32, seed=8)
    out = O.moe_forward(x, logits, 2, wg, wu, wd, fp8=fp8)
    perm = np.random.default_rng(1).permutation(12)
    out_p = O.moe_forward(x[perm], logits[perm], 2, wg, wu, wd, fp8=fp8)
    np.testing.assert_allclose(out_p, out[perm], rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("fp8", [False, True])
def test_zero_input_and_exact_doubling(fp8):
    x, logits, wg, wu, wd = rand_layer(7, 4, 2, 8, 16, seed=9)
    z = O.moe_forward(np.zeros_like(x), logits, 2, wg, wu, wd, fp8=fp8)
    assert np.all(z == 0.0)
    out = O.moe_forward(x, logits, 2, wg, wu, wd, fp8=fp8)
    out2 = O.moe_forward(x, logits, 2, wg, wu, 2 * wd, fp8=fp8)
    assert np.array_equal(out2, 2 * out)


@pytest.mark.parametrize("fp8", [False, True])
def test_token_subset_equals_full_rows(fp8):
    x, logits, wg, wu, wd = rand_layer(20, 8, 3, 16, 16, seed=10)
    full = O.moe_forward(x, logits, 3, wg, wu, wd, fp8=fp8)
    toks = [0, 5, 19]
    sub = O.moe_forward(x, logits, 3, wg, wu, wd, fp8=fp8, tokens=toks)
    np.testing.assert_allclose(sub[toks], full[toks], rtol=1e-12, atol=1e-14)
    assert np.all(np.isnan(np.delete(sub, toks, axis=0)))


def torch_q(t, s):
    """Independent quantise -> dequantise through torch's e4m3 cast (fp32 division)."""
    t = torch.as_tensor(np.asarray(t, np.float32))
    q = (t / torch.tensor(s, dtype=torch.float32)).clamp(-448, 448).to(torch.float8_e4m3fn)
    return q.to(torch.float64) * float(s)


def torch_scale(t):
    a = torch.as_tensor(np.asarray(t, np.float32)).abs().amax()
    return np.float32(1.0) if a.item() == 0 else np.float32((a / torch.tensor(448.0)).item())


def test_fp8_layer_matches_independent_emulation():
    M, E, k, H, I = 10, 6, 2, 32, 16
    x, logits, wg, wu, wd = rand_layer(M, E, k, H, I, seed=12)
    out, inter = O.moe_forward(x, logits, k, wg, wu, wd, fp8=True, return_intermediates=True)
    # independent: dense over every (token, selected expert), torch casts, fp64 math
    ids, w = O.route(logits, k)   # routing itself is pinned in test_oracle_routing.py
    s_x = torch_scale(x)
    xq = torch_q(x, s_x)
    deq = {}
    for e in range(E):
        deq[e] = tuple(torch_q(W[e], torch_scale(W[e])) for W in (wg, wu, wd))
    hs = {}
    for t in range(M):
        for j in range(k):
            g, u, _ = deq[int(ids[t, j])]
            hs[(t, j)] = torch.nn.functional.silu(xq[t] @ g.T) * (xq[t] @ u.T)
    amax = max(float(v.to(torch.float32).abs().max()) for v in hs.values())
    s_h = np.float32(np.float32(amax) / np.float32(448.0))
    assert s_h == inter["s_h"] and s_x == inter["s_x"]
    ref = np.zeros((M, H))
    for t in range(M):
        for j in range(k):
            d = deq[int(ids[t, j])][2]
            ref[t] += w[t, j] * (torch_q(hs[(t, j)].to(torch.float32).numpy(), s_h) @ d.T).numpy()
    np.testing.assert_allclose(out, ref, rtol=1e-11, atol=1e-13)


def test_fp8_identical_experts_topk_E_is_quantised_ffn():
    M, E, H, I = 6, 4, 16, 16
    x, logits, wg, wu, wd = rand_layer(M, E, E, H, I, seed=13)
    wg[:] = wg[0]
    wu[:] = wu[0]
    wd[:] = wd[0]
    out = O.moe_forward(x, logits, E, wg, wu, wd, fp8=True)
    xq = torch_q(x, torch_scale(x))
    g, u, d = (torch_q(W[0], torch_scale(W[0])) for W in (wg, wu, wd))
    h = torch.nn.functional.silu(xq @ g.T) * (xq @ u.T)
    s_h = torch_scale(h.to(torch.float32).numpy())
    ref = (torch_q(h.to(torch.float32).numpy(), s_h) @ d.T).numpy()
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-13)


def test_provider_matches_arrays():
    x, logits, wg, wu, wd = rand_layer(8, 4, 2, 8, 8, seed=15)
    a = O.moe_forward(x, logits, 2, wg, wu, wd)
    b = O.moe_forward(x, logits, 2, provider=lambda e: (wg[e], wu[e], wd[e]))
    assert np.array_equal(a, b)
