"""Pins for the oracle's FP8 window rows (no GPU).

Pinned against hand-worked rows (tests/golden/fp8_window_rows.txt), the
ml_dtypes and torch float8_e4m3fn conversions of x / s (independent library
routines for the element format), the scale definition and byte accounting.
"""

import os

import ml_dtypes
import numpy as np
import pytest
import torch

from oracle import fp8

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "fp8_window_rows.txt")


def _golden_rows():
    rows = []
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        name, xs, sc, codes, deq = [p.strip() for p in line.split("|")]
        rows.append((name, np.array([float(v) for v in xs.split()], dtype=np.float32), float(sc),
                     np.array([int(c, 16) for c in codes.split()], dtype=np.uint8),
                     np.array([float(v) for v in deq.split()], dtype=np.float64)))
    return rows


@pytest.mark.parametrize("row", _golden_rows(), ids=lambda r: r[0])
def test_hand_worked_rows(row):
    name, xs, sc, codes, deq = row
    x = np.zeros((1, 512), dtype=np.float32)
    x[0, :xs.shape[0]] = xs
    got_codes, got_s = fp8.quantize_window_fp8(x)
    assert float(got_s[0]) == sc, name
    np.testing.assert_array_equal(got_codes[0, :xs.shape[0]], codes, err_msg=name)
    assert np.all(got_codes[0, xs.shape[0]:] == 0)
    v = fp8.dequantize_window_fp8(got_codes, got_s)[0, :xs.shape[0]]
    np.testing.assert_array_equal(v, deq)
    np.testing.assert_array_equal(np.signbit(v), np.signbit(deq))


def _random_rows(seed, n=4000):
    rng = np.random.default_rng(seed)
    scale = np.exp2(rng.uniform(-40, 40, (n, 1)))
    x = rng.normal(0, 1, (n, 512)) * scale
    x[::7, ::3] = 0.0                                   # zeros and negative zeros mixed in
    x[1::7, ::5] = -0.0
    return torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).to(torch.float32).numpy()


def test_scale_is_the_rounded_amax_over_448():
    x = _random_rows(1)
    _, s = fp8.quantize_window_fp8(x)
    want = (np.max(np.abs(x), axis=1) / np.float32(448)).astype(np.float32)
    np.testing.assert_array_equal(s, want)


def test_codes_match_two_library_conversions():
    x = _random_rows(2)
    codes, s = fp8.quantize_window_fp8(x)
    y = (x / s[:, None]).astype(np.float32)
    y_clip = np.clip(y, -448, 448)                      # both libraries give NaN beyond 448
    ref_md = y_clip.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    ref_t = torch.from_numpy(y_clip).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(codes, ref_md)
    np.testing.assert_array_equal(codes, ref_t)
    # every non-zero row reaches the largest magnitude code
    nz = np.max(np.abs(x), axis=1) > 0
    assert np.all((codes[nz] & 0x7F).max(axis=1) == 0x7E)


def test_zero_row_keeps_signs():
    x = np.zeros((1, 512), dtype=np.float32)
    x[0, 1::2] = -0.0
    codes, s = fp8.quantize_window_fp8(x)
    assert s[0] == 0
    np.testing.assert_array_equal(codes[0, 0::2], 0x00)
    np.testing.assert_array_equal(codes[0, 1::2], 0x80)
    assert np.all(fp8.dequantize_window_fp8(codes, s) == 0)


def test_dequantisation_error_is_within_half_a_step():
    """|v - x| <= 2^-4 |x| for normal elements (three mantissa bits) and
    <= s * 2^-10 for subnormal ones (half the step 2^-9 s)."""
    x = _random_rows(3, n=500)
    codes, s = fp8.quantize_window_fp8(x)
    v = fp8.dequantize_window_fp8(codes, s)
    bound = np.maximum(np.abs(x) * 2.0 ** -4, s[:, None].astype(np.float64) * 2.0 ** -10) * (1 + 1e-6)
    assert np.all(np.abs(v - x) <= bound)


def test_row_bytes():
    """512 E4M3 codes and one float32 scale: 516 B per row against 1024 B of
    bf16 (about half, the FP8 side of the section's FP4/FP8 comparison)."""
    assert fp8.row_bytes() == 516
    assert fp8.row_bytes() / 1024 < 0.51
