"""GPU parity of the chain's grouped GEMMs on CTA pairs (clusters of two CTAs issuing
M = 256 tcgen05 MMAs; each CTA holds its own weight rows and half of every token tile).

Against the oracle at the layer's tolerances, with routing and the padded permutation
bit-exact, in bf16, e4m3 and e5m2: token tiles from a few rows to several 256-row
blocks per expert (one and two TMEM accumulator buffers, a second token block), ragged
counts that are not multiples of the pair's 32-row granularity, the automatic choice at
a prefill-shaped batch, and the single-CTA GEMMs on the same handle in turn.
"""

import numpy as np
import pytest

from oracle import moe_oracle as O
from tests.parity_helpers import Case, check_output, check_routing, tokens

pytestmark = pytest.mark.gpu

TOLKEY = {"bf16": "bf16", "fp8": "fp8", "fp8_e5m2": "fp8"}


def oracle(c, x, logits):
    fp8 = c.dtype != "bf16"
    return O.moe_forward(x.float().cpu().numpy(), logits.cpu().numpy(), c.k, provider=c.provider, fp8=fp8,
                         fp8_format="e5m2" if c.dtype == "fp8_e5m2" else "e4m3",
                         weight_cache=c.cache if fp8 else None)


def check(c, M, seed, pair):
    x, logits = tokens(c.E, c.H, M, seed=seed)
    out = c.run(x, logits)
    assert c.layer.last_gemm_pairs == pair
    check_routing(c, logits, M)
    check_output(out, oracle(c, x, logits), TOLKEY[c.dtype])
    return out


@pytest.fixture(scope="module", params=["bf16", "fp8", "fp8_e5m2"])
def small(request):
    # H a multiple of 512 and I of 256: the shapes the pair tiles cover (I = 512 keeps the
    # e5m2 code flips of h, which the tolerance absorbs, a small part of each output)
    c = Case(8, 2, 512, 512, request.param, w_std=0.02)
    c.cache = {}
    c.layer.set_gemv_max_tokens(0)
    yield c
    c.close()


@pytest.mark.parametrize("M", [24, 64, 100, 333, 700, 1100])
def test_forced_pairs(small, M, monkeypatch):
    # ~6 to ~275 tokens per expert: 32-row pair tiles, two buffers, one buffer, two blocks
    if small.dtype == "fp8_e5m2" and M > 333:
        # e5m2 h codes flip where the kernel's bf16 h and the oracle's differ by an ulp
        # (steps of 25 %); over hundreds of thousands of outputs the largest of those
        # errors can pass the FP8 bound whichever GEMM form runs. These sizes are checked
        # against the single-CTA form instead (test_pairs_match_single_ctas).
        pytest.skip("e5m2 at this size: compared with the single-CTA GEMMs")
    monkeypatch.setenv("MOE_PAIR_GEMM", "1")
    check(small, M, 900 + M, True)


def test_pairs_then_single_ctas(small, monkeypatch):
    # the same handle and workspace, the two GEMM forms in turn
    for i, (M, mode) in enumerate([(200, "1"), (200, "0"), (520, "1"), (40, "0"), (40, "1")]):
        monkeypatch.setenv("MOE_PAIR_GEMM", mode)
        check(small, M, 950 + i, mode == "1")


@pytest.mark.parametrize("M", [480, 1100])
def test_pairs_match_single_ctas(small, M, monkeypatch):
    # one input through both forms: each within the oracle's tolerance (e5m2: the pair no
    # further from the oracle than the single-CTA form, see above), and close to the other
    x, logits = tokens(small.E, small.H, M, seed=977 + M)
    monkeypatch.setenv("MOE_PAIR_GEMM", "0")
    one = small.run(x, logits).clone()
    assert not small.layer.last_gemm_pairs
    monkeypatch.setenv("MOE_PAIR_GEMM", "1")
    two = small.run(x, logits).clone()
    assert small.layer.last_gemm_pairs
    ref = oracle(small, x, logits)
    if small.dtype != "fp8_e5m2":
        check_output(one, ref, TOLKEY[small.dtype])
        check_output(two, ref, TOLKEY[small.dtype])
    else:
        err = [float(np.max(np.abs(o.float().cpu().numpy() - ref))) for o in (one, two)]
        rtol, atol = (4e-2, 2e-3)
        assert err[1] <= max(rtol * float(np.max(np.abs(ref))) + atol, 1.25 * err[0]), err
    # the same products in the same K order: equal up to the order of the fp32 additions
    # (the down GEMM's scatter-adds land in any order), i.e. a bf16 rounding step or two
    diff = (one.float() - two.float()).abs().max().item()
    assert diff <= 1e-2 * float(np.max(np.abs(ref)))


@pytest.mark.parametrize("dtype", ["bf16", "fp8"])
def test_auto_choice_prefill_shape(dtype, monkeypatch):
    # 128 tokens per expert on average: the default takes the pairs; a decode batch does not
    monkeypatch.delenv("MOE_PAIR_GEMM", raising=False)
    c = Case(32, 4, 1024, 512, dtype, w_std=0.02)
    c.cache = {}
    c.layer.set_gemv_max_tokens(0)
    try:
        check(c, 1024, 990, True)
        check(c, 64, 991, False)
    finally:
        c.close()


@pytest.mark.parametrize("dtype", ["bf16", "fp8"])
def test_balanced_schedule_on_pairs(dtype, monkeypatch):
    # 64 experts x ~96 tokens: 256 gate_up and 128 down pair tiles, between one and eight
    # waves of the 74 pairs, so both GEMMs take the balanced schedule (tiles cut between
    # pairs at K-block boundaries, split-K fix-ups counted per CTA of a pair)
    monkeypatch.delenv("MOE_PAIR_GEMM", raising=False)
    c = Case(64, 8, 1024, 1024, dtype, w_std=0.02)
    c.cache = {}
    c.layer.set_gemv_max_tokens(0)
    try:
        check(c, 768, 995, True)
    finally:
        c.close()
