"""Failure detection without a GPU fault, in a child process of its own.

1. The GEMMs' pipeline waits are bounded; MOE_WAIT_BUDGET_CYCLES shrinks the bound
   so far that the waits give up on purpose (a wait that nothing completes in time).
   The kernels then record a wait code in the device error word, drain what they
   issued and return; moe_get_device_error must report MOE_ERR_DEVICE_TIMEOUT with
   that code, and the context must stay usable: a fresh handle with the default
   budget passes parity against the oracle in the same process.
2. A host-side injected allocation failure (MOE_TEST_FAIL_WORKSPACE=1) makes
   moe_forward return MOE_ERR_OOM without touching the GPU; once it is lifted, the
   same handle runs normally.
No test here faults, traps or hangs the GPU: every wait involved is bounded."""

import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import ctypes, json, os, sys
sys.path.insert(0, {root!r})
import numpy as np, torch
from mixture_experts_layer_sort_b200 import MoELayer, synth
from oracle import moe_oracle as O
E, k, H, I, M = 8, 2, 256, 512, 64
wg, wu, wd = synth.make_weights(E, H, I, 0.02, seed=0, device="cuda")
x, logits = synth.make_tokens(E, H, M, seed=1, device="cuda")
res = {{}}

def forward_rc(layer, out):
    s = torch.cuda.current_stream().cuda_stream
    return layer.lib.moe_forward(layer.handle, x.data_ptr(), logits.data_ptr(), M, out.data_ptr(), s)

def device_error(layer):
    c = ctypes.c_int(0)
    rc = layer.lib.moe_get_device_error(layer.handle, ctypes.byref(c))
    return rc, c.value

# 1. waits that give up
for dtype in ("bf16", "fp8"):
    layer = MoELayer(E, k, H, I, dtype)
    layer.load_weights(wg, wu, wd)
    out = torch.empty((M, H), dtype=torch.bfloat16, device="cuda")
    os.environ["MOE_WAIT_BUDGET_CYCLES"] = "32"
    res[dtype + "_forward_rc"] = forward_rc(layer, out)
    torch.cuda.synchronize()
    del os.environ["MOE_WAIT_BUDGET_CYCLES"]
    res[dtype + "_timeout"] = device_error(layer)
    res[dtype + "_cleared"] = device_error(layer)
    layer.close()

# the context is still usable: a fresh handle, default budget, parity with the oracle
layer = MoELayer(E, k, H, I, "bf16")
layer.load_weights(wg, wu, wd)
got = layer.forward(x, logits).float().cpu().numpy()
ref = O.moe_forward(x.float().cpu().numpy(), logits.cpu().numpy(), k,
                    *[synth.bf16_to_f32_numpy(w) for w in (wg, wu, wd)])
res["after_err"] = float(np.max(np.abs(got - ref)))
res["after_bound"] = 1e-2 * float(np.max(np.abs(ref))) + 1e-3
res["after_device_error"] = device_error(layer)
layer.close()

# 2. an injected allocation failure on the host
layer = MoELayer(E, k, H, I, "bf16")
layer.load_weights(wg, wu, wd)
out = torch.empty((M, H), dtype=torch.bfloat16, device="cuda")
os.environ["MOE_TEST_FAIL_WORKSPACE"] = "1"
res["oom_rc"] = forward_rc(layer, out)
del os.environ["MOE_TEST_FAIL_WORKSPACE"]
res["after_oom_rc"] = forward_rc(layer, out)
torch.cuda.synchronize()
res["after_oom_device_error"] = device_error(layer)
layer.close()
print("RESULT " + json.dumps(res))
"""

WAIT_CODES = {0x101, 0x102, 0x103, 0x104, 0x106}


def test_bounded_waits_report_and_the_context_survives():
    r = subprocess.run([sys.executable, "-c", CHILD.format(root=ROOT)], capture_output=True, text=True,
                       timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-3000:]
    line = [l for l in r.stdout.splitlines() if l.startswith("RESULT ")][-1]
    res = json.loads(line[len("RESULT "):])
    for dtype in ("bf16", "fp8"):
        assert res[dtype + "_forward_rc"] == 0                 # launches succeed; the waits give up inside
        rc, code = res[dtype + "_timeout"]
        assert rc == -6, res                                   # MOE_ERR_DEVICE_TIMEOUT
        assert code in WAIT_CODES, hex(code)
        assert res[dtype + "_cleared"] == [0, 0]               # reading cleared the word
    assert res["after_err"] <= res["after_bound"], res
    assert res["after_device_error"] == [0, 0]
    assert res["oom_rc"] == -3                                 # MOE_ERR_OOM, nothing launched
    assert res["after_oom_rc"] == 0 and res["after_oom_device_error"] == [0, 0]
