"""GPU parity of the chain with the combine folded into the down GEMM (opt-in,
MOE_FOLD_FINALIZE=1): the epilogue that adds a token's last K block writes its output
row and clears its accumulator row, and the last CTA to finish writes the forward's FP8
scales and clears the amax words (no finalize launch).

Against the oracle at the layer's tolerances (s_x bit-exact, s_h within rounding), in
bf16, e4m3 and e5m2, through a single-block and a multi-block align; one launch fewer
than with the finalize kernel; and the two forms in turn on one handle, which needs the
per-token counts and the CTA count back at zero after every forward.
"""

import numpy as np
import pytest

from oracle import moe_oracle as O
from tests.parity_helpers import Case, check_output, check_routing, tokens

pytestmark = pytest.mark.gpu

TOLKEY = {"bf16": "bf16", "fp8": "fp8", "fp8_e5m2": "fp8"}


@pytest.fixture(scope="module", params=["bf16", "fp8", "fp8_e5m2"])
def tiny(request):
    c = Case(8, 2, 256, 512, request.param, w_std=0.02)
    c.cache = {}
    c.layer.set_gemv_max_tokens(0)
    yield c
    c.close()


def run_checked(c, M, seed):
    x, logits = tokens(c.E, c.H, M, seed=seed)
    out = c.run(x, logits)
    dbg, _ = check_routing(c, logits, M)
    fp8 = c.dtype != "bf16"
    ref, inter = O.moe_forward(x.float().cpu().numpy(), logits.cpu().numpy(), c.k, provider=c.provider, fp8=fp8,
                               fp8_format="e5m2" if c.dtype == "fp8_e5m2" else "e4m3",
                               weight_cache=c.cache if fp8 else None, return_intermediates=True)
    check_output(out, ref, TOLKEY[c.dtype])
    if fp8:
        assert np.float32(dbg["s_x"]) == inter["s_x"], "s_x differs"
        assert abs(dbg["s_h"] - float(inter["s_h"])) <= 1e-2 * float(inter["s_h"]), "s_h differs"
    return c.layer.last_launch_count


@pytest.mark.parametrize("M", [20, 300, 5000])
def test_folded_combine(tiny, M, monkeypatch):
    monkeypatch.setenv("MOE_FOLD_FINALIZE", "1")
    folded = run_checked(tiny, M, 1100 + M)
    monkeypatch.delenv("MOE_FOLD_FINALIZE", raising=False)
    separate = run_checked(tiny, M, 1100 + M)
    assert folded == separate - 1


def test_forms_in_turn(tiny, monkeypatch):
    # counts left non-zero by one forward would corrupt the next one's rows
    for i, (M, mode) in enumerate([(64, "1"), (64, "1"), (200, "0"), (17, "1"), (900, "1"), (33, "0"), (33, "1")]):
        monkeypatch.setenv("MOE_FOLD_FINALIZE", mode)
        run_checked(tiny, M, 1200 + i)
    assert tiny.layer.device_error() == 0
