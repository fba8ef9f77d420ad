"""GPU parity of the fused MoE layer against the CPU oracle, through the C ABI.

Sizes span several tiles, ragged tails, split tiles, one and several 256-row token
blocks per expert, the single-block and multi-block align paths, in bf16 and FP8,
plus edge cases and the size limits.
"""

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from tests.parity_helpers import Case, check_output, check_routing, tokens

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tiny():
    c = Case(8, 2, 256, 512, "bf16", w_std=0.02)
    yield c
    c.close()


@pytest.fixture(scope="module")
def tiny_fp8():
    c = Case(8, 2, 256, 512, "fp8", w_std=0.02)
    yield c
    c.close()


def oracle_full(case, x, logits, fp8):
    return O.moe_forward(x.float().cpu().numpy(), logits.cpu().numpy(), case.k,
                         provider=case.provider, fp8=fp8, return_intermediates=True)


@pytest.mark.parametrize("M", [16, 1, 3, 37, 100, 300, 700])
def test_tiny_bf16(tiny, M):
    # M=16: the tiny workload; the others cross one and several token blocks per
    # expert, split tiles and ragged tails
    x, logits = tokens(tiny.E, tiny.H, M, seed=M)
    out = tiny.run(x, logits)
    check_routing(tiny, logits, M)
    ref, _ = oracle_full(tiny, x, logits, fp8=False)
    check_output(out, ref, "bf16")


@pytest.mark.parametrize("M", [16, 1, 37, 300])
def test_tiny_fp8(tiny_fp8, M):
    x, logits = tokens(tiny_fp8.E, tiny_fp8.H, M, seed=100 + M)
    out = tiny_fp8.run(x, logits)
    dbg, padded = check_routing(tiny_fp8, logits, M)
    ref, inter = oracle_full(tiny_fp8, x, logits, fp8=True)
    assert np.float32(dbg["s_x"]) == inter["s_x"], "s_x differs"
    # x codes of every valid permuted row are bit-exact
    xp, _ = tiny_fp8.layer.debug_activations(len(padded))
    xp = xp.cpu().numpy()
    valid = padded < M * tiny_fp8.k
    tok = padded[valid] // tiny_fp8.k
    assert np.array_equal(xp[valid], inter["x_codes"][tok]), "x codes differ"
    check_output(out, ref, "fp8")


@pytest.mark.parametrize("M", [1, 3, 8, 16])
@pytest.mark.parametrize("dtype", ["bf16", "fp8"])
def test_tiny_chain_small_batches(tiny, tiny_fp8, dtype, M):
    # the tensor-core chain at the sizes that the thin-batch path takes by default
    c = tiny if dtype == "bf16" else tiny_fp8
    c.layer.set_gemv_max_tokens(0)
    try:
        x, logits = tokens(c.E, c.H, M, seed=200 + M)
        out = c.run(x, logits)
        assert c.layer.last_launch_count >= 5
        check_routing(c, logits, M)
        ref, _ = oracle_full(c, x, logits, fp8=dtype == "fp8")
        check_output(out, ref, dtype)
    finally:
        c.layer.set_gemv_max_tokens(-1)


def test_fp8_weight_codes_bit_exact(tiny_fp8):
    g, u, d, sc = tiny_fp8.layer.debug_weights()
    for e in range(tiny_fp8.E):
        wg, wu, wd = tiny_fp8.provider(e)
        for j, (W, Q) in enumerate(((wg, g), (wu, u), (wd, d))):
            s = O.per_tensor_scale(W)
            assert np.float32(sc[e, j].item()) == s
            assert np.array_equal(Q[e].cpu().numpy(), O.quantize(W, s))


def test_m_zero_is_a_no_op(tiny):
    x, logits = tokens(tiny.E, tiny.H, 4)
    out = torch.full((0, tiny.H), 7.0, dtype=torch.bfloat16, device="cuda")
    tiny.layer.forward(x[:0], logits[:0], out=out)
    assert tiny.layer.last_launch_count == 0


def test_all_tokens_to_one_expert(tiny):
    M = 200
    x, logits = tokens(tiny.E, tiny.H, M, seed=5)
    logits[:, 3] += 100.0
    logits[:, 6] += 50.0
    out = tiny.run(x, logits)
    dbg, _ = check_routing(tiny, logits, M)
    assert int(dbg["counts"][3]) == M and int(dbg["counts"][6]) == M
    ref, _ = oracle_full(tiny, x, logits, fp8=False)
    check_output(out, ref, "bf16")


def test_tied_and_negative_infinite_logits(tiny):
    M = 40
    x, logits = tokens(tiny.E, tiny.H, M, seed=6)
    logits = torch.round(logits)              # many exact ties
    logits[0] = 0.0
    logits[1, :] = -float("inf")
    logits[1, 5] = 1.0
    logits[1, 2] = 1.0
    logits[2, :] = -float("inf")              # no finite logit: weight 1/k each
    out = tiny.run(x, logits)
    check_routing(tiny, logits, M)
    ref, _ = oracle_full(tiny, x, logits, fp8=False)
    check_output(out, ref, "bf16")


def test_zero_input_gives_zero(tiny_fp8):
    x, logits = tokens(tiny_fp8.E, tiny_fp8.H, 24, seed=7)
    x.zero_()
    out = tiny_fp8.run(x, logits)
    assert torch.count_nonzero(out).item() == 0
    dbg = tiny_fp8.layer.debug_routing(24)
    assert dbg["s_x"] == 1.0 and dbg["s_h"] == 1.0


def test_repeated_calls_are_stable(tiny):
    x, logits = tokens(tiny.E, tiny.H, 64, seed=8)
    a = tiny.run(x, logits).float()
    b = tiny.run(x, logits).float()
    # scatter-add order may differ between calls: compare within bf16 rounding
    assert torch.max(torch.abs(a - b)).item() <= 1e-2 * torch.max(torch.abs(a)).item()
    assert tiny.layer.device_error() == 0


def test_tiny_many_token_blocks(tiny):
    # ~625 tokens per expert: three 256-row token blocks per expert, one TMEM buffer
    M = 2500
    x, logits = tokens(tiny.E, tiny.H, M, seed=2500)
    out = tiny.run(x, logits)
    check_routing(tiny, logits, M)
    ref, _ = oracle_full(tiny, x, logits, fp8=False)
    check_output(out, ref, "bf16")


def test_topk_equals_E():
    # every token routed to every expert: P = M*E pairs, each expert sees all tokens
    c = Case(8, 8, 256, 512, "bf16", w_std=0.02)
    try:
        for M in (1, 33):
            x, logits = tokens(c.E, c.H, M, seed=40 + M)
            out = c.run(x, logits)
            dbg, _ = check_routing(c, logits, M)
            assert np.all(dbg["counts"].cpu().numpy() == M)
            ref, _ = oracle_full(c, x, logits, fp8=False)
            check_output(out, ref, "bf16")
    finally:
        c.close()


@pytest.mark.parametrize("E,k,H,I,dtype,Ms", [
    (512, 16, 128, 128, "bf16", (1, 37, 130)),    # the largest E and topk, the smallest H and I
    (512, 16, 128, 128, "fp8", (37,)),
    (4, 2, 16384, 128, "bf16", (5,)),             # the largest H (256 K blocks of gate_up)
    (2, 1, 128, 16384, "bf16", (3, 20)),          # the largest I (128 gate_up row blocks, 256 K blocks of down)
    (2, 1, 128, 16384, "fp8", (20,)),
])
def test_size_limits(E, k, H, I, dtype, Ms):
    c = Case(E, k, H, I, dtype, w_std=0.02)
    try:
        for M in Ms:
            x, logits = tokens(c.E, c.H, M, seed=M + E)
            out = c.run(x, logits)
            check_routing(c, logits, M)
            ref, _ = oracle_full(c, x, logits, fp8=(dtype == "fp8"))
            check_output(out, ref, dtype)
        assert c.layer.device_error() == 0
    finally:
        c.close()


@pytest.mark.parametrize("E,k,M", [(8, 2, 5000), (64, 8, 1100), (200, 6, 2000)])
def test_multi_block_align(E, k, M):
    # more than 8192 pairs: per-chunk counts, the plan block and the per-chunk
    # placement; the padded permutation must still be the stable one, bit for bit
    c = Case(E, k, 256, 256, "bf16", w_std=0.02)
    try:
        x, logits = tokens(c.E, c.H, M, seed=E + M)
        out = c.run(x, logits)
        check_routing(c, logits, M)
        ref, _ = oracle_full(c, x, logits, fp8=False)
        check_output(out, ref, "bf16")
    finally:
        c.close()


@pytest.mark.parametrize("dtype", ["fp8", "fp8_e5m2"])
def test_fp8_multi_block_x_codes(dtype):
    # more than 8192 pairs: x is quantised once per token and the gather copies the
    # codes; every valid row of x_perm must still hold the oracle's codes bit for bit
    fmt = "e5m2" if dtype == "fp8_e5m2" else "e4m3"
    c = Case(8, 2, 256, 512, dtype, w_std=0.02)
    try:
        M = 5000
        x, logits = tokens(c.E, c.H, M, seed=77)
        out = c.run(x, logits)
        dbg, padded = check_routing(c, logits, M)
        ref, inter = O.moe_forward(x.float().cpu().numpy(), logits.cpu().numpy(), c.k, provider=c.provider,
                                   fp8=True, fp8_format=fmt, return_intermediates=True)
        assert np.float32(dbg["s_x"]) == inter["s_x"], "s_x differs"
        xp, _ = c.layer.debug_activations(len(padded))
        valid = padded < M * c.k
        assert np.array_equal(xp.cpu().numpy()[valid], inter["x_codes"][padded[valid] // c.k]), "x codes differ"
        check_output(out, ref, "fp8")
    finally:
        c.close()
