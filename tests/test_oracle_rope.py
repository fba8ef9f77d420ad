"""Pins for the inverse-RoPE + per-head FP8 quantisation oracle (CPU only).

Each check stands apart from the oracle's own code: the rotation is compared with
complex-number arithmetic (a pair (a, b) is the number a + ib, rotating by an
angle is multiplying by e^(i*angle), undoing it is dividing), a forward rotation
followed by the oracle's inverse must give the input back, position 0 must be the
identity, the interleaved layout must equal the half-split one on permuted
columns, and the scales must be the closed form amax / F. The last tests plant
mistakes in the oracle and check that a pin catches each.
"""

import math

import numpy as np
import pytest

from oracle import moe_oracle as O
from oracle import rope_oracle as R


def _inputs(T=7, NH=3, D=64, max_pos=50, seed=0):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, NH, D)).astype(np.float32)
    pos = rng.integers(0, max_pos, size=T).astype(np.int32)
    table = R.rope_cos_sin_table(max_pos, D)
    return x, pos, table


def _complex_pairs(v, interleaved):
    D = v.shape[-1]
    if interleaved:
        return v[..., 0::2] + 1j * v[..., 1::2]
    return v[..., : D // 2] + 1j * v[..., D // 2:]


def _from_complex(z, interleaved):
    D = 2 * z.shape[-1]
    out = np.empty(z.shape[:-1] + (D,), dtype=np.float64)
    if interleaved:
        out[..., 0::2], out[..., 1::2] = z.real, z.imag
    else:
        out[..., : D // 2], out[..., D // 2:] = z.real, z.imag
    return out


def _unit(table, pos):
    D = table.shape[1]
    t = table.astype(np.float64)[pos]
    return (t[:, : D // 2] + 1j * t[:, D // 2:])[:, None, :]      # e^(i angle), [T, 1, D/2]


def test_cos_sin_table_matches_math():
    table = R.rope_cos_sin_table(40, 16, base=10000.0)
    for p in (0, 1, 17, 39):
        for i in (0, 3, 7):
            ang = p * 10000.0 ** (-2.0 * i / 16)
            assert abs(table[p, i] - math.cos(ang)) < 1e-6
            assert abs(table[p, 8 + i] - math.sin(ang)) < 1e-6


@pytest.mark.parametrize("interleaved", [False, True])
def test_inverse_rotation_is_complex_division(interleaved):
    x, pos, table = _inputs(seed=1)
    got = R.inv_rope_f64(x, pos, table, interleaved)
    want = _from_complex(_complex_pairs(x.astype(np.float64), interleaved) / _unit(table, pos), interleaved)
    # the table's cos^2 + sin^2 is 1 only to fp32 rounding: division and multiplication
    # by the conjugate differ by that much
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-5)
    want_conj = _from_complex(_complex_pairs(x.astype(np.float64), interleaved) * np.conj(_unit(table, pos)),
                              interleaved)
    np.testing.assert_allclose(got, want_conj, rtol=0, atol=1e-12)


@pytest.mark.parametrize("interleaved", [False, True])
def test_forward_then_inverse_is_identity(interleaved):
    v, pos, table = _inputs(seed=2)
    u = _unit(table, pos)
    u = u / np.abs(u)                                   # exact unit rotations
    rotated = _from_complex(_complex_pairs(v.astype(np.float64), interleaved) * u, interleaved)
    exact = np.concatenate([u.real, u.imag], axis=2)[:, 0, :]
    tab = np.zeros((pos.max() + 1, v.shape[2]))
    tab[pos] = exact
    back = R.inv_rope_f64(rotated, pos, tab, interleaved)
    np.testing.assert_allclose(back, v, rtol=0, atol=1e-12)


def test_fp32_rotation_is_the_fp64_one_rounded():
    x, pos, table = _inputs(seed=3)
    y32, valid = R.inv_rope_f32(x, pos, table)
    y64 = R.inv_rope_f64(x, pos, table)
    assert valid.all()
    # two roundings of products and one of the sum: a few fp32 ulps of the larger term
    scale = np.abs(x).max() * 4
    assert np.max(np.abs(y32 - y64)) <= scale * 2.0 ** -22


def test_position_zero_is_identity_and_quantises_x_itself():
    x, _, table = _inputs(seed=4)
    pos = np.zeros(x.shape[0], np.int32)
    y, valid = R.inv_rope_f32(x, pos, table)
    assert np.array_equal(y, x)
    codes, scales = R.inv_rope_fp8_quant(x, pos, table)
    for t in range(x.shape[0]):
        for h in range(x.shape[1]):
            s = O.per_tensor_scale(x[t, h])
            assert scales[t, h] == s
            assert np.array_equal(codes[t, h], O.quantize(x[t, h], s))


def test_interleaved_is_half_split_on_permuted_columns():
    x, pos, table = _inputs(seed=5)
    D = x.shape[2]
    perm = np.concatenate([np.arange(0, D, 2), np.arange(1, D, 2)])   # interleaved -> half-split
    y_int, _ = R.inv_rope_f32(x, pos, table, interleaved=True)
    y_half, _ = R.inv_rope_f32(x[..., perm], pos, table, interleaved=False)
    assert np.array_equal(y_int[..., perm], y_half)


@pytest.mark.parametrize("fmt,fmax,top", [("e4m3", 448.0, 0x7E), ("e5m2", 57344.0, 0x7B)])
def test_scales_are_amax_over_fmax_and_codes_round_to_nearest(fmt, fmax, top):
    x, pos, table = _inputs(seed=6)
    codes, scales = R.inv_rope_fp8_quant(x, pos, table, fmt=fmt)
    y, _ = R.inv_rope_f32(x, pos, table)
    dec = O.FP8_FORMATS[fmt][1]
    step = 2.0 ** (-3 if fmt == "e4m3" else -2)          # relative spacing of the normal codes
    for t in range(x.shape[0]):
        for h in range(x.shape[1]):
            amax = np.float32(np.max(np.abs(y[t, h])))
            assert scales[t, h] == np.float32(amax / np.float32(fmax))
            # the largest magnitude lands on the largest finite code
            j = int(np.argmax(np.abs(y[t, h])))
            assert codes[t, h, j] & 0x7F == top
            back = dec(codes[t, h]) * np.float64(scales[t, h])
            err = np.abs(back - y[t, h].astype(np.float64))
            tiny = scales[t, h] * (2.0 ** -9 if fmt == "e4m3" else 2.0 ** -16)
            assert np.all(err <= np.maximum(np.abs(y[t, h]) * step / 2 * (1 + 1e-6), tiny))


def test_zero_head_and_invalid_positions():
    x, pos, table = _inputs(T=4, seed=7)
    x[1, 2] = 0.0
    pos = pos.copy()
    pos[0] = -1
    pos[3] = table.shape[0]
    codes, scales = R.inv_rope_fp8_quant(x, pos, table)
    # a zero head rotates to signed zeros (0x00 or 0x80): every code decodes to 0
    assert scales[1, 2] == 1.0 and not (codes[1, 2] & 0x7F).any()
    assert np.all(np.isnan(scales[0])) and np.all(np.isnan(scales[3]))
    assert not codes[0].any() and not codes[3].any()
    assert np.all(np.isfinite(scales[1:3]))


# ----------------------------------------------------------------------------- planted mistakes
def test_forward_rotation_instead_of_inverse_is_caught(monkeypatch):
    real = R.inv_rope_f64

    def forward(x, positions, cos_sin, interleaved=False):
        t = np.asarray(cos_sin, np.float64).copy()
        D = t.shape[1]
        t[:, D // 2:] *= -1.0                               # sin -> -sin: rotates the other way
        return real(x, positions, t, interleaved)

    monkeypatch.setattr(R, "inv_rope_f64", forward)
    with pytest.raises(AssertionError):
        test_forward_then_inverse_is_identity(False)


def test_wrong_pairing_is_caught(monkeypatch):
    monkeypatch.setattr(R, "_pair_index", lambda D, interleaved: (np.arange(0, D, 2), np.arange(1, D, 2)))
    with pytest.raises(AssertionError):
        test_inverse_rotation_is_complex_division(False)


def test_scale_over_the_wrong_axis_is_caught(monkeypatch):
    real = R.quant_per_head

    def per_token(y, valid, fmt="e4m3"):
        y = np.asarray(y, np.float32)
        amax = np.max(np.abs(y), axis=(1, 2), keepdims=True)      # one scale per token
        yy = np.broadcast_to(amax, y.shape).copy()
        yy[..., 1:] = y[..., 1:]
        return real(y, valid, fmt)[0], np.broadcast_to(amax[..., 0] / 448.0, y.shape[:2]).astype(np.float32)

    monkeypatch.setattr(R, "quant_per_head", per_token)
    with pytest.raises(AssertionError):
        test_position_zero_is_identity_and_quantises_x_itself()
