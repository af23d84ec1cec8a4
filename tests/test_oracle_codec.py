"""Pins of the oracle's FP4 / E4M3 codec against things other than itself.

- E2M1 and E4M3 decode tables against their closed-form definitions (golden file) and
  against torch's own float8_e4m3fn decode (a library routine);
- the E4M3 encoder against torch's float8_e4m3fn cast on every finite bf16 value
  inside the non-saturating range, and saturation above it;
- the block quantiser's two steps, exhaustively, against an exact threshold
  formulation (comparisons of exactly representable products, no division);
- the 448 x 6 = 2688 saturation point the pages print.
"""
import json
import os

import numpy as np
import pytest
import torch

from oracle import oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def all_bf16_finite_nonneg():
    bits = np.arange(0, 0x7F80, dtype=np.uint32)  # +0 .. largest finite
    return (bits << 16).view(np.float32).astype(np.float64)


def test_e2m1_table_matches_definition():
    g = _golden("e2m1_e4m3_formats.json")
    mags = g["e2m1_magnitudes_by_code"]
    for c in range(16):
        v = O.e2m1_value(c)
        expect = mags[c & 7] * (-1.0 if c & 8 else 1.0)
        assert v == expect and np.signbit(v) == bool(c & 8)


def test_e4m3_decode_matches_torch_all_256():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        v = O.e4m3_value(c)
        if np.isnan(ref[c]):
            assert np.isnan(v), c
        else:
            assert v == ref[c] and np.signbit(v) == np.signbit(ref[c]), c
    g = _golden("e2m1_e4m3_formats.json")
    assert O.e4m3_value(0x7E) == g["e4m3_max"]
    assert O.e4m3_value(0x01) == g["e4m3_min_subnormal"]
    assert all(np.isnan(O.e4m3_value(c)) for c in g["e4m3_nan_codes"])


def test_e4m3_encode_matches_torch_cast_on_all_bf16():
    v = all_bf16_finite_nonneg()
    v = np.concatenate([v, -v])
    inside = np.abs(v) < 464.0  # torch's cast is RNE below the saturation midpoint
    ours = O.e4m3_encode_many(v[inside])
    ref = torch.from_numpy(v[inside]).to(torch.float32).to(torch.float8_e4m3fn)
    ref = ref.view(torch.uint8).numpy()
    np.testing.assert_array_equal(ours, ref)
    sat = O.e4m3_encode_many(v[~inside])
    assert np.all((sat & 0x7F) == 0x7E)
    np.testing.assert_array_equal(sat >> 7, (v[~inside] < 0).astype(np.uint8))


def test_e4m3_round_trip_all_finite_codes():
    for c in range(256):
        if c in (0x7F, 0xFF):
            continue
        assert O.e4m3_encode(O.e4m3_value(c)) == c


# ---- exact threshold formulation (independent of the oracle's nearest-grid search) -----

E4M3_GRID = np.array([((m / 8.0) * 2.0 ** -6) if e == 0 else (1 + m / 8.0) * 2.0 ** (e - 7)
                      for e in range(16) for m in range(8)][:127])
E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def threshold_code(num, den, grid):
    """Code of num/den rounded to nearest-even on `grid`, saturating, decided only by
    comparisons 2*num vs (g_i + g_{i+1}) * den, which are exact in float64 here."""
    code = np.zeros(num.shape, np.int64)
    for i in range(len(grid) - 1):
        lhs = 2.0 * num
        rhs = (grid[i] + grid[i + 1]) * den
        above = lhs > rhs
        tie = lhs == rhs
        # past midpoint i -> at least code i+1; on the midpoint -> the even of (i, i+1)
        code = np.where(above | (tie & ((i + 1) % 2 == 0)), i + 1, code)
    return code


def test_scale_step_exhaustive_against_thresholds():
    amax = all_bf16_finite_nonneg()
    ours = O.fp4_scale_codes(amax).astype(np.int64)
    ref = threshold_code(amax, np.full_like(amax, 6.0), E4M3_GRID)
    np.testing.assert_array_equal(ours, ref)


def test_element_step_exhaustive_against_thresholds():
    mags = all_bf16_finite_nonneg()
    scales = E4M3_GRID[1:]  # every finite positive scale (126 of them)
    x = np.repeat(mags, scales.size)
    s = np.tile(scales, mags.size)
    for sign in (1.0, -1.0):
        ours = O.fp4_codes(sign * x, s).astype(np.int64)
        ref = threshold_code(x, s, E2M1_GRID) | (8 if sign < 0 else 0)
        np.testing.assert_array_equal(ours, ref)


def test_zero_scale_block_and_signed_zero():
    codes, sc = O.quantize_block16(np.array([1e-4, -1e-4] + [0.0] * 13 + [-0.0]))
    assert sc == 0  # 1e-4 / 6 is below half the smallest E4M3 subnormal
    assert list(codes[:2]) == [0x0, 0x8] and codes[15] == 0x8 and codes[2] == 0x0


def test_saturation_point_2688():
    g = _golden("pages_numbers.json")["fp4_max_magnitude"]
    assert g["factors"][0] * g["factors"][1] == g["value"]
    for big in (float(g["value"]), 3000.0, 1.0e6):
        x = np.zeros(16)
        x[3] = -big
        x[7] = big
        codes, sc = O.quantize_block16(x)
        assert sc == 0x7E and O.e4m3_value(sc) == g["factors"][0]
        assert codes[3] == 0xF and codes[7] == 0x7
        assert O.e2m1_value(codes[7]) * O.e4m3_value(sc) == min(big, g["value"])


def test_dequant_error_within_half_step():
    rng = np.random.default_rng(5)
    bits = torch.from_numpy(rng.standard_normal((64, 512)).astype(np.float32)).to(
        torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    codes, scales = O.quantize_entries(bits)
    x = O.bf16_array_to_f64(bits).reshape(64, 512)
    y = O.dequant_entries(codes, scales)
    s = np.repeat(O.e4m3_array_to_f64(scales), 16, axis=1)
    # the E2M1 grid step is at most 2 (between 4 and 6), so |x - y| <= 1 * s
    assert np.all(np.abs(x - y) <= 1.0 * s + 1e-300)
    # per-block maxima land exactly on 6*s or within a grid half-step of it
    assert np.all(np.abs(y) <= 6.0 * s)


def test_pack_order_low_nibble_first():
    grid = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]  # block max 6 -> scale exactly 1
    x = np.array([grid[i % 8] * (-1) ** (i // 8) for i in range(512)], dtype=np.float32)
    bits = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    codes, scales = O.quantize_entries(bits[None, :])
    y = O.dequant_entries(codes, scales)[0]
    np.testing.assert_array_equal(y, x.astype(np.float64))
    c0 = O.e2m1_encode(0.0 / O.e4m3_value(scales[0, 0]))
    c1 = O.e2m1_encode(0.5 / O.e4m3_value(scales[0, 0]))
    assert codes[0, 0] == (c0 | (c1 << 4))


def test_main_entry_is_288_bytes():
    assert O.main_entry_bytes(512) == 512 // 2 + 512 // 16 == 288
