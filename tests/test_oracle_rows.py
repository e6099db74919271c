"""Pins of the checkpoint-row oracle (oracle/rows.py) against what fixes it from outside:
the E4M3 and bf16 formats' definitions (every code, every rounding midpoint), PyTorch's own
fp32 -> float8_e4m3fn and fp32 -> bfloat16 conversions (library routines), and hand-worked
rows whose codes follow from the definitions by inspection."""

import numpy as np
import pytest
import torch

from oracle import rows as R


def test_e4m3_values_of_named_codes():
    # OCP FP8 E4M3: bias 7, 3 mantissa bits, no infinities, S.1111.111 NaN
    assert R.e4m3_value(0x00) == 0.0
    assert R.e4m3_value(0x01) == 2.0 ** -9          # smallest subnormal
    assert R.e4m3_value(0x07) == 7 * 2.0 ** -9      # largest subnormal
    assert R.e4m3_value(0x08) == 2.0 ** -6          # smallest normal
    assert R.e4m3_value(0x38) == 1.0
    assert R.e4m3_value(0x39) == 1.125
    assert R.e4m3_value(0x7E) == 448.0              # largest finite
    assert np.isnan(R.e4m3_value(0x7F)) and np.isnan(R.e4m3_value(0xFF))
    assert R.e4m3_value(0xB8) == -1.0
    vals = [R.e4m3_value(c) for c in range(127)]
    assert all(a < b for a, b in zip(vals, vals[1:]))  # codes 0..126 ascend


def test_e4m3_every_finite_code_round_trips():
    for c in list(range(0, 127)) + list(range(0x81, 0xFF)):
        assert R.e4m3_encode(R.e4m3_value(c)) == c, hex(c)
    assert R.e4m3_encode(-0.0) == 0x00  # a zero result is always +0


def test_e4m3_midpoints_round_to_the_even_code():
    for c in range(126):
        lo, hi = R.e4m3_value(c), R.e4m3_value(c + 1)
        mid = (lo + hi) / 2  # exact in double
        want = c if c % 2 == 0 else c + 1
        assert R.e4m3_encode(mid) == want, (c, mid)
        assert R.e4m3_encode(-mid) == (want | 0x80 if want else 0)
        assert R.e4m3_encode(np.nextafter(mid, 0.0)) == c
        assert R.e4m3_encode(np.nextafter(mid, 1e9)) == c + 1


def test_e4m3_saturates():
    for x in (448.0, 449.0, 463.9, 464.0, 500.0, 1e30):
        assert R.e4m3_encode(x) == 0x7E
        assert R.e4m3_encode(-x) == 0xFE


def test_e4m3_matches_torch_conversion():
    """PyTorch's fp32 -> float8_e4m3fn (round to nearest even) on 200k values in range;
    its overflow behaviour differs (NaN beyond the rounding range), so |x| < 464 here."""
    rng = np.random.default_rng(5)
    x = (rng.standard_normal(200_000) * rng.choice([1e-4, 1e-2, 1.0, 30.0, 150.0], 200_000))
    x = np.clip(x, -463.0, 463.0).astype(np.float32)
    ours = np.array([R.e4m3_encode(float(v)) for v in x], np.uint8)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ref = np.where((ref & 0x7F) == 0, 0, ref)  # canonical zero
    np.testing.assert_array_equal(ours, ref)


def test_bf16_matches_torch_conversion_and_rounds_ties_to_even():
    rng = np.random.default_rng(6)
    x = (rng.standard_normal(100_000) * 10.0 ** rng.integers(-30, 30, 100_000)).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(R.bf16_encode(x), ref)
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7: ties to the even code (1.0);
    # 1 + 3 * 2^-8 is halfway between 1 + 2^-7 and 1 + 2^-6: rounds up to the even one
    t = np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8], np.float32)
    np.testing.assert_array_equal(R.bf16_decode(R.bf16_encode(t)),
                                  np.array([1.0, 1 + 2.0 ** -6], np.float32))


def test_hand_worked_e4m3_row():
    """amax = 448 gives s = 1, so the codes are the values' own E4M3 codes."""
    row = np.array([[448.0, 1.0, -1.0, 0.5, 1.0625, -1.09375, 2.0 ** -10, -2.0 ** -12]],
                   np.float32)
    codes, scales = R.pack(row, "e4m3")
    assert scales[0] == np.float32(1.0)
    assert codes[0].tolist() == [0x7E, 0x38, 0xB8, 0x30, 0x38, 0xB9, 0x00, 0x00]
    back = R.unpack(codes, scales, "e4m3", 8)
    np.testing.assert_array_equal(back[0], [448, 1, -1, 0.5, 1, -1.125, 0, 0])


def test_hand_worked_int4_row():
    """amax = 7 gives s = 1: the codes are the rounded values, two per byte, the even element
    in the low nibble; 2.5 and -0.5 round to even (2 and -0)."""
    row = np.array([[7.0, -7.0, 2.5, -0.5, 1.4, -3.6, 0.0, 6.5]], np.float32)
    codes, scales = R.pack(row, "int4")
    assert scales[0] == np.float32(1.0)
    # nibbles: 7, -7=0x9, 2, 0, 1, -4=0xC, 0, 6
    assert codes[0].tolist() == [0x97, 0x02, 0xC1, 0x60]
    back = R.unpack(codes, scales, "int4", 8)
    np.testing.assert_array_equal(back[0], [7, -7, 2, 0, 1, -4, 0, 6])


def test_zero_row_has_zero_scale_and_codes():
    """All-zero rows, and rows so small that their scale would fall below the smallest
    normal fp32 (whose reciprocal would overflow), are stored as zero."""
    row = np.zeros((4, 8), np.float32)
    row[1, 3] = -0.0
    row[2, :] = np.float32(1e-38)
    row[3, 5] = np.float32(-5e-38)
    for fmt in ("e4m3", "int4"):
        codes, scales = R.pack(row, fmt)
        assert not codes.any() and not scales.any()
        assert not R.unpack(codes, scales, fmt, 8).any()


@pytest.mark.parametrize("fmt", ["e4m3", "int4"])
def test_round_trip_error_is_within_half_a_code_step(fmt):
    """|unpack(pack(x)) - x| is at most half the spacing of the code grid at x / s, times s
    (plus the fp32 roundings of 1 / s, x * (1 / s) and code * s), and the row's largest |x|
    comes back within the same roundings."""
    rng = np.random.default_rng(7)
    M = (rng.standard_normal((64, 32)) * 10.0 ** rng.integers(-3, 3, (64, 1))).astype(np.float32)
    codes, scales = R.pack(M, fmt)
    back = R.unpack(codes, scales, fmt, 32)
    s = scales[:, None].astype(np.float64)
    q = np.abs(M / s)
    if fmt == "int4":
        step = np.ones_like(q)
    else:
        grid = np.array([R.e4m3_value(c) for c in range(127)])
        i = np.clip(np.searchsorted(grid, q, side="right") - 1, 0, 125)
        step = grid[i + 1] - grid[i]
    err = np.abs(back.astype(np.float64) - M)
    assert np.all(err <= s * step / 2 + 5e-7 * np.abs(M) + 1e-30)
    amax = np.abs(M).max(axis=1)
    got = np.abs(back).max(axis=1)
    assert np.all(np.abs(got - amax) <= 5e-7 * amax)
