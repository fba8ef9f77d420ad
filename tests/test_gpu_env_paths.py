"""GPU parity of the schedule and launch alternatives that environment variables
select (each read once per process, so every setting runs in a child process):

  MOE_UNIFORM_SPLITS=1     one split-K factor per GEMM from the cost model instead of
                           the balanced unit schedule
  MOE_DISABLE_PDL=1        plain stream order instead of programmatic dependent launch
  MOE_SMALL_BATCH=1        batches of up to 64 tokens take the small-batch GEMMs (no align,
                           gather or finalize) instead of the full chain
  MOE_DISABLE_DIRECT_X=1   small bf16 batches gather x instead of loading token rows
  MOE_MAX_STAGES1/2=2      the shallowest stage rings
  MOE_GEMV_MAX_M=n         batches of up to n tokens take the thin-batch (CUDA-core) path
                           (0: none; 16: FP8 layers too up to 16 tokens)
  MOE_GEMV_PREFETCH_KB=4   the thin-batch down kernel asks L2 for its first weight blocks
                           before it waits for gate_up

The shape (E=64, k=8, H=1024, I=1024) gives one to eight waves of tiles on a B200 at
M=64 (the balanced schedule's range) and fewer than one at M=1.
"""

import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import sys
sys.path.insert(0, sys.argv[1])
from oracle import moe_oracle as O
from tests.parity_helpers import Case, check_output, check_routing, tokens
for dtype in ("bf16", "fp8"):
    c = Case(64, 8, 1024, 1024, dtype, w_std=0.02)
    for M in (1, 5, 64):
        x, logits = tokens(c.E, c.H, M, seed=7 * M + (dtype == "fp8"))
        out = c.run(x, logits)
        check_routing(c, logits, M)
        ref = O.moe_forward(x.float().cpu().numpy(), logits.cpu().numpy(), c.k, provider=c.provider,
                            fp8=(dtype == "fp8"))
        check_output(out, ref, dtype)
    c.close()
print("PARITY_OK")
"""

# MOE_GEMV_MAX_M=0 keeps the small batches on the tensor-core chain, whose alternatives
# these are
SETTINGS = [
    {"MOE_UNIFORM_SPLITS": "1", "MOE_GEMV_MAX_M": "0"},
    {"MOE_DISABLE_PDL": "1"},
    {"MOE_DISABLE_PDL": "1", "MOE_GEMV_MAX_M": "0"},
    {"MOE_DISABLE_DIRECT_X": "1", "MOE_GEMV_MAX_M": "0"},
    {"MOE_SMALL_BATCH": "1"},
    {"MOE_SMALL_BATCH": "1", "MOE_UNIFORM_SPLITS": "1"},
    {"MOE_MAX_STAGES1": "2", "MOE_MAX_STAGES2": "2", "MOE_GEMV_MAX_M": "0"},
    {"MOE_GEMV_PREFETCH_KB": "4"},
    {"MOE_GEMV_MAX_M": "16"},
]


@pytest.mark.parametrize("env", SETTINGS, ids=lambda e: ",".join(f"{k}={v}" for k, v in e.items()))
def test_env_path_parity(env):
    r = subprocess.run([sys.executable, "-c", CHILD, ROOT], env={**os.environ, **env}, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0 and "PARITY_OK" in r.stdout, r.stdout[-2000:] + r.stderr[-4000:]
