"""Pins for the oracle's 8-bit latent cache (reading R16): the E4M3 rounding
against the format's own definition and torch's float8 cast, the bf16 and
half-precision roundings against torch's casts, and the per-token
quantization against its closed-form error bound and hand-worked values."""

import numpy as np
import pytest
import torch

from oracle import mla_oracle as om


def _e4m3_table():
    """All finite E4M3 values from the bit layout: sign, 4 exponent bits
    (bias 7), 3 mantissa bits; exponent field 0 is subnormal (m/8 * 2^-6);
    the pattern with all exponent and mantissa bits set is NaN."""
    vals = []
    for byte in range(256):
        sgn = -1.0 if byte & 0x80 else 1.0
        ef, mf = (byte >> 3) & 0xF, byte & 0x7
        if ef == 0xF and mf == 0x7:
            continue
        v = (mf / 8.0) * 2.0 ** -6 if ef == 0 else (1 + mf / 8.0) * 2.0 ** (ef - 7)
        vals.append((sgn * v, mf))
    return vals


def test_e4m3_values_are_fixed_points_and_max_is_448():
    tab = _e4m3_table()
    assert len(tab) == 254
    v = np.array([x for x, _ in tab])
    np.testing.assert_array_equal(om.e4m3_round(v), v)
    assert v.max() == 448.0 and om.E4M3_MAX == 448.0
    assert np.abs(v[v != 0]).min() == 2.0 ** -9


def test_e4m3_midpoints_round_to_even_and_saturate():
    pos = sorted({x for x, _ in _e4m3_table() if x >= 0})
    mant = {x: m for x, m in _e4m3_table() if x >= 0}
    for a, b in zip(pos[:-1], pos[1:]):
        mid = (a + b) / 2
        even = a if mant[a] % 2 == 0 else b
        assert om.e4m3_round(mid) == even, (a, b)
        assert om.e4m3_round(np.nextafter(mid, 0)) == a
        assert om.e4m3_round(np.nextafter(mid, 1e9)) == b
        assert om.e4m3_round(-mid) == -even
    assert om.e4m3_round(1e6) == 448.0 and om.e4m3_round(-500.0) == -448.0


def test_e4m3_matches_torch_float8_cast():
    rng = np.random.default_rng(40)
    x = np.concatenate([rng.standard_normal(20000) * s for s in (1e-3, 0.1, 1, 30, 200)])
    x = x[np.abs(x) <= 448]
    ref = torch.tensor(x, dtype=torch.float32).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    # the float32 step rounds x first; ties of the 8-bit grid are far from
    # float32 rounding, so the two agree exactly
    np.testing.assert_array_equal(om.e4m3_round(x.astype(np.float32).astype(np.float64)), ref)


def test_bf16_round_matches_torch_cast():
    rng = np.random.default_rng(41)
    x = (rng.standard_normal(50000) * 10.0 ** rng.integers(-20, 20, 50000)).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(om.bf16_round(x.astype(np.float64)), ref)


def test_f16_round_matches_torch_cast():
    rng = np.random.default_rng(44)
    x = (rng.standard_normal(50000) * 10.0 ** rng.integers(-9, 5, 50000)).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float16).to(torch.float64).numpy()
    np.testing.assert_array_equal(om.f16_round(x.astype(np.float64)), ref)


def test_quantize_latent_fp8_error_bound_and_worked_values():
    rng = np.random.default_rng(42)
    C = (rng.standard_normal((50, 512)) * rng.uniform(0.1, 10, (50, 1))).astype(np.float32)
    KR = rng.standard_normal((50, 64)).astype(np.float32)
    s, c8, kr8 = om.quantize_latent_fp8(C, KR)
    np.testing.assert_allclose(s, np.abs(C).max(1) / 448, rtol=2 ** -23)
    assert (np.abs(c8) <= 448).all() and (np.abs(c8).max(1) == 448).all()
    Cd, KRd = om.dequantize_fp8(s, c8, kr8)
    # nearest rounding of x = C/s: at most half a grid step, 2^(e-4) for |x|
    # in [2^e, 2^(e+1)), 2^-10 below 2^-6; plus the single-precision division
    xs = np.abs(C.astype(np.float64) / s[:, None])
    half = np.where(xs >= 2.0 ** -6, np.exp2(np.floor(np.log2(np.maximum(xs, 1e-300))) - 4),
                    2.0 ** -10)
    assert (np.abs(Cd - C) <= (half + xs * 2.0 ** -23) * s[:, None] * (1 + 1e-9)).all()
    # the RoPE key: half precision of KR / s (11 significant bits) times s
    assert (np.abs(KRd - KR) <= (2.0 ** -11 + 2.0 ** -23) * np.abs(KR) * (1 + 1e-9)).all()
    # hand-worked token: max |c| = 896, so s = 2; 3 / 2 = 1.5 (exact), 1.1 / 2
    # = 0.55 -> 0.5625 (grid step 1/16 in [0.5, 1)), -896 / 2 = -448; RoPE
    # parts / 2 in [1, 2) sit on a grid of 2^-10: 3 + 2^-9 -> 1.5 + 2^-10 is
    # kept, 3 + 2^-10 -> 1.5 + 2^-11, a tie, goes to the even neighbour 1.5
    s1, c1, k1 = om.quantize_latent_fp8(np.array([[3.0, 1.1, -896.0]]),
                                        np.array([[3.001953125, 3.0009765625]]))
    assert s1[0] == 2.0
    np.testing.assert_array_equal(c1[0], [1.5, 0.5625, -448.0])
    np.testing.assert_array_equal(k1[0], [1.5009765625, 1.5])
    # a RoPE key too large for half precision at the latent's scale sets s
    s2, c2, k2 = om.quantize_latent_fp8(np.array([[0.5, -0.25]]), np.array([[1.0e3, -2.0]]))
    assert s2[0] == np.float32(np.float32(1.0e3) / np.float32(65504.0))
    assert np.abs(k2).max() <= 65504.0
    # an all-zero row keeps scale 1
    s0, c0, k0 = om.quantize_latent_fp8(np.zeros((1, 4)), np.zeros((1, 2)))
    assert s0[0] == 1.0 and (c0 == 0).all() and (k0 == 0).all()


def test_planted_rounding_slips_are_caught(monkeypatch):
    """A truncating rounding or a wrong mantissa width planted in the
    oracle's grid rounding fails the definition's fixed points or torch."""
    rng = np.random.default_rng(43)
    x = rng.standard_normal(5000)
    ref = torch.tensor(x, dtype=torch.float32).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    orig = om.round_to_grid
    monkeypatch.setattr(om, "round_to_grid",
                        lambda v, mb, emin, mx: orig(v, mb + 1, emin, mx))
    assert np.abs(om.e4m3_round(x.astype(np.float32).astype(np.float64)) - ref).max() > 0
    monkeypatch.setattr(om, "round_to_grid", orig)
    monkeypatch.setattr(om.np, "round", np.trunc)
    try:
        assert np.abs(om.e4m3_round(x.astype(np.float32).astype(np.float64)) - ref).max() > 0
    finally:
        monkeypatch.undo()
