"""CPU oracle for the inverse-RoPE + per-head FP8 quantisation kernel.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import, call or
execute this module: only the tests, `__graft_entry__.smoke()` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it. It shares
no code, table or helper with the CUDA library and imports nothing from it.

What it computes
----------------
The pages name one kernel, ``_fused_inv_rope_fp8_quant_per_head``, that used to
be recompiled for every new token count until its variable-length parameters
were marked so that the compiler would not specialise on them (toolboxkart.tech,
"AWS SageMaker MoE kernel optimizations H200", section "3. Removing repeat
compilation can reduce first-token delay"; aib.vote, "AWS SageMaker MoE kernel
optimizations", fourth paragraph). The pages give only the name; this module
takes the plain reading of it:

1. inverse RoPE - every head vector of D values was rotated, pair by pair, by
   the angle of its token's position; undo that rotation. With (a', b') a
   rotated pair, c = cos(angle) and s = sin(angle):
       a = a' * c + b' * s
       b = b' * c - a' * s
   Pairs are (i, i + D/2) in the half-split ("NeoX") layout or (2i, 2i + 1)
   in the interleaved layout; pair i uses the i-th angle of the position's
   entry in a cos/sin table [max_pos, D] (cos in the first D/2 columns, sin in
   the last D/2).
2. per-head FP8 quantisation - one scale per (token, head) vector:
   s = amax(|y|) / F (F = 448 for e4m3, 57344 for e5m2; s = 1 for an all-zero
   vector), codes = round-to-nearest-even(y / s), saturated.

Precision: every step is taken in IEEE fp32 with one rounding per multiply,
add and divide, in the order written above, because the result is an integer
code and a code decision has to be taken in the kernel's precision. The fp64
rotation (``inv_rope_f64``) is kept for the pins.

Positions outside [0, max_pos) have no table entry: that head's scale is NaN
and its codes are 0.

Pinned by ``tests/test_oracle_rope.py`` (complex-number rotation, round trip
through a forward rotation, position 0, the half-split / interleaved
relation, closed-form scales); no function is "parity unpinned".
"""

from __future__ import annotations

import numpy as np

from oracle import moe_oracle as _fp8   # the FP8 codecs (pinned in tests/test_oracle_e4m3.py, _e5m2.py)


def _pair_index(D: int, interleaved: bool):
    """Element indices (first, second) of each of the D/2 pairs of a head vector."""
    i = np.arange(D // 2)
    if interleaved:
        return 2 * i, 2 * i + 1
    return i, i + D // 2


def inv_rope_f32(x: np.ndarray, positions: np.ndarray, cos_sin: np.ndarray, interleaved: bool = False):
    """Inverse rotation of x [T, NH, D] in fp32, one rounding per operation.

    Returns (y [T, NH, D] float32, valid [T] bool): rows whose position has no
    table entry come back as zeros with valid = False.
    """
    x = np.asarray(x, dtype=np.float32)
    T, NH, D = x.shape
    cs = np.asarray(cos_sin, dtype=np.float32)
    pos = np.asarray(positions, dtype=np.int64)
    valid = (pos >= 0) & (pos < cs.shape[0])
    safe = np.where(valid, pos, 0)
    c = cs[safe, : D // 2][:, None, :]        # [T, 1, D/2]
    s = cs[safe, D // 2:][:, None, :]
    ia, ib = _pair_index(D, interleaved)
    a, b = x[..., ia], x[..., ib]
    y = np.zeros_like(x)
    # each product and each sum rounded to fp32 (numpy float32 ops do exactly that)
    y[..., ia] = (a * c) + (b * s)
    y[..., ib] = (b * c) - (a * s)
    y[~valid] = 0.0
    return y, valid


def inv_rope_f64(x: np.ndarray, positions: np.ndarray, cos_sin: np.ndarray, interleaved: bool = False):
    """The same rotation in fp64 (for the pins)."""
    x = np.asarray(x, dtype=np.float64)
    T, NH, D = x.shape
    cs = np.asarray(cos_sin, dtype=np.float64)
    pos = np.asarray(positions, dtype=np.int64)
    c = cs[pos, : D // 2][:, None, :]
    s = cs[pos, D // 2:][:, None, :]
    ia, ib = _pair_index(D, interleaved)
    a, b = x[..., ia], x[..., ib]
    y = np.empty_like(x)
    y[..., ia] = a * c + b * s
    y[..., ib] = b * c - a * s
    return y


def quant_per_head(y: np.ndarray, valid: np.ndarray, fmt: str = "e4m3"):
    """Per-(token, head) FP8 codes and scales of y [T, NH, D] (fp32 values)."""
    y = np.asarray(y, dtype=np.float32)
    T, NH, D = y.shape
    enc, _, fmax = _fp8.FP8_FORMATS[fmt]
    amax = np.max(np.abs(y), axis=2)                               # exact in fp32
    scales = np.where(amax == 0, np.float32(1.0), amax / np.float32(fmax)).astype(np.float32)
    codes = enc((y / scales[..., None]).astype(np.float32))
    scales = np.where(valid[:, None], scales, np.float32(np.nan)).astype(np.float32)
    codes = np.where(valid[:, None, None], codes, np.uint8(0)).astype(np.uint8)
    return codes, scales


def inv_rope_fp8_quant(x, positions, cos_sin, interleaved: bool = False, fmt: str = "e4m3"):
    """The kernel's result: (codes [T, NH, D] uint8, scales [T, NH] float32)."""
    y, valid = inv_rope_f32(x, positions, cos_sin, interleaved)
    return quant_per_head(y, valid, fmt)


def rope_cos_sin_table(max_pos: int, D: int, base: float = 10000.0) -> np.ndarray:
    """A cos/sin table [max_pos, D] fp32 for the usual angle schedule
    angle(p, i) = p * base^(-2i/D), i < D/2 (the tests' input; the kernel takes any table)."""
    i = np.arange(D // 2, dtype=np.float64)
    inv_freq = base ** (-2.0 * i / D)
    ang = np.arange(max_pos, dtype=np.float64)[:, None] * inv_freq[None, :]
    return np.concatenate([np.cos(ang), np.sin(ang)], axis=1).astype(np.float32)
