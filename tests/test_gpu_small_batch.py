"""GPU parity of the small-batch path (MOE_SMALL_BATCH=1, read once per process, so
the checks run in a child process): batches of up to 64 tokens take route -> gate_up
-> down for bf16 and route -> quant_x -> gate_up -> quant_h -> down for FP8, the GEMMs
building the batch's schedule themselves, gate_up reading token rows directly and down
finishing token rows itself. Against the oracle, with the routing and the padded
permutation bit-exact, through back-to-back calls queued without synchronisation, and
alternating with the full chain (larger batches) on one handle, which share the
workspace, the fp32 accumulator and the FP8 amax words."""

import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import sys
sys.path.insert(0, sys.argv[1])
import numpy as np
import torch
from oracle import moe_oracle as O
from tests.parity_helpers import Case, check_output, check_routing, tokens

LAUNCHES = {"bf16": 3, "fp8": 5, "fp8_e5m2": 5}
TOLKEY = {"bf16": "bf16", "fp8": "fp8", "fp8_e5m2": "fp8"}

def oracle(c, x, l, **kw):
    fp8 = c.dtype != "bf16"
    return O.moe_forward(x.float().cpu().numpy(), l.cpu().numpy(), c.k, provider=c.provider, fp8=fp8,
                         fp8_format="e5m2" if c.dtype == "fp8_e5m2" else "e4m3",
                         weight_cache=c.cache if fp8 else None, **kw)

def check(c, M, seed):
    x, logits = tokens(c.E, c.H, M, seed=seed)
    out = c.run(x, logits)
    dbg, _ = check_routing(c, logits, M)
    ref, inter = oracle(c, x, logits, return_intermediates=True)
    if c.dtype != "bf16":
        assert np.float32(dbg["s_x"]) == inter["s_x"], "s_x differs"
    check_output(out, ref, TOLKEY[c.dtype])
    return c.layer.last_launch_count

for dtype in ("bf16", "fp8", "fp8_e5m2"):
    c = Case(8, 2, 256, 512, dtype, w_std=0.02)
    c.cache = {}
    for M in (1, 2, 16, 33, 64):
        assert check(c, M, 900 + M) == LAUNCHES[dtype]
    # M <= 64 takes the small-batch path, M = 65 and 300 the full chain
    for i, M in enumerate((5, 300, 64, 65, 1, 300, 16)):
        assert (check(c, M, 950 + i) == LAUNCHES[dtype]) == (M <= 64)
    # forwards queued back to back before anyone reads
    xs = [tokens(c.E, c.H, 16, seed=970 + i) for i in range(5)]
    outs = [c.layer.forward(x, l) for x, l in xs]
    torch.cuda.synchronize()
    for (x, l), out in zip(xs, outs):
        check_output(out, oracle(c, x, l), TOLKEY[dtype])
    assert c.layer.device_error() == 0
    c.close()
# the decode layer, both dtypes
for dtype in ("bf16", "fp8"):
    c = Case(128, 8, 2048, 768, dtype, w_std=0.02)
    c.cache = {}
    for M in (1, 4, 16, 64):
        assert check(c, M, M) == LAUNCHES[dtype]
    c.close()
print("SMALL_BATCH_OK")
"""


def test_small_batch_path_parity():
    r = subprocess.run([sys.executable, "-c", CHILD, ROOT], env={**os.environ, "MOE_SMALL_BATCH": "1"},
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0 and "SMALL_BATCH_OK" in r.stdout, r.stdout[-2000:] + r.stderr[-4000:]
