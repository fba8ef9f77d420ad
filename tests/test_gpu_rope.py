"""GPU parity of the inverse-RoPE + per-head FP8 quantisation kernel
(moe_inv_rope_fp8_quant) against the CPU oracle, through the C ABI: codes and
scales bit-exact (both sides take every rounding in IEEE fp32 in the same order),
for both pair layouts, both FP8 formats, the three head sizes, token counts from 1
up (one kernel for every count), out-of-range positions and zero heads."""

import numpy as np
import pytest
import torch

from mixture_experts_layer_sort_b200 import inv_rope_fp8_quant
from oracle import rope_oracle as R

pytestmark = pytest.mark.gpu


def _run(T, NH, D, interleaved, fmt, max_pos=4096, seed=0, edit=None):
    g = torch.Generator(device="cpu").manual_seed(seed)
    x = torch.randn((T, NH, D), generator=g).to(torch.bfloat16)
    pos = torch.randint(0, max_pos, (T,), generator=g, dtype=torch.int32)
    table = torch.from_numpy(R.rope_cos_sin_table(max_pos, D))
    if edit is not None:
        edit(x, pos)
    codes, scales = inv_rope_fp8_quant(x.cuda(), pos.cuda(), table.cuda(), interleaved=interleaved, fmt=fmt)
    torch.cuda.synchronize()
    want_c, want_s = R.inv_rope_fp8_quant(x.float().numpy(), pos.numpy(), table.numpy(), interleaved, fmt)
    got_c, got_s = codes.cpu().numpy(), scales.cpu().numpy()
    assert np.array_equal(np.isnan(got_s), np.isnan(want_s)), "NaN scales differ"
    ok = ~np.isnan(want_s)
    assert np.array_equal(got_s[ok].view(np.uint32), want_s[ok].view(np.uint32)), "scales differ"
    diff = np.argwhere(got_c != want_c)
    assert diff.size == 0, f"{len(diff)} codes differ, first at {diff[:3].tolist()}"
    return got_c, got_s


@pytest.mark.parametrize("T,NH,D,interleaved,fmt", [
    (1, 16, 128, False, "e4m3"),
    (17, 8, 64, True, "e4m3"),
    (300, 4, 256, False, "e5m2"),
    (1000, 3, 128, True, "e5m2"),
    (4096, 16, 128, False, "e4m3"),
    (33, 5, 64, False, "e5m2"),
    (129, 7, 256, True, "e4m3"),
])
def test_matches_oracle_bit_exact(T, NH, D, interleaved, fmt):
    _run(T, NH, D, interleaved, fmt, seed=T + NH + D)


def test_every_token_count_uses_the_same_kernel():
    # token counts are run-time arguments: a sweep of counts, each bit-exact
    for T in (1, 2, 3, 5, 8, 13, 31, 64, 65, 127):
        _run(T, 4, 128, False, "e4m3", max_pos=256, seed=1000 + T)


def test_out_of_range_positions_and_zero_heads():
    def edit(x, pos):
        pos[0] = -1
        pos[5] = 4096
        x[3, 2].zero_()
        x[7].zero_()

    _, s = _run(12, 4, 128, False, "e4m3", edit=edit)
    assert np.all(np.isnan(s[0])) and np.all(np.isnan(s[5]))
    assert s[3, 2] == 1.0 and np.all(s[7] == 1.0)


def test_zero_tokens_is_a_no_op():
    x = torch.empty((0, 4, 128), dtype=torch.bfloat16, device="cuda")
    pos = torch.empty((0,), dtype=torch.int32, device="cuda")
    table = torch.zeros((8, 128), dtype=torch.float32, device="cuda")
    codes, scales = inv_rope_fp8_quant(x, pos, table)
    assert codes.shape == (0, 4, 128) and scales.shape == (0, 4)
