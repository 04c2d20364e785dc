"""Pins for the oracle's FP4 encoder (no GPU).

Pinned against: hand-worked blocks (tests/golden/fp4_blocks.txt), the
ml_dtypes float4_e2m1fn / float8_e4m3fn and torch float8_e4m3fn
conversions (independent library routines for the two element formats),
exhaustive code round-trips and byte accounting.
"""

import os

import ml_dtypes
import numpy as np
import pytest
import torch

from oracle import fp4

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "fp4_blocks.txt")


def _golden_blocks():
    rows = []
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        name, xs, sc, codes, deq = [p.strip() for p in line.split("|")]
        rows.append((name,
                     np.array([float(v) for v in xs.split()], dtype=np.float32),
                     int(sc, 16),
                     np.array([int(c, 16) for c in codes.split()], dtype=np.uint8),
                     np.array([float(v) for v in deq.split()], dtype=np.float64)))
    return rows


@pytest.mark.parametrize("block", _golden_blocks(), ids=lambda b: b[0])
def test_hand_worked_blocks(block):
    name, x, scale, codes, deq = block
    assert x.shape == (16,)
    got_codes, got_scale = fp4.quantize_block_codes(x[None])
    assert int(got_scale[0]) == scale, name
    np.testing.assert_array_equal(got_codes[0], codes, err_msg=name)
    # dequantised values, including the sign of zeros
    got = fp4.e2m1_value(got_codes[0]) * fp4.e4m3_value(got_scale[0])
    np.testing.assert_array_equal(got, deq)
    np.testing.assert_array_equal(np.signbit(got), np.signbit(deq))


def test_golden_blocks_through_entry_packing():
    """The golden blocks laid into one 512-channel entry: nibble order and
    scale bytes of the packed 288-byte row."""
    blocks = _golden_blocks()
    x = np.zeros((1, 512), dtype=np.float32)
    for k, (_, xs, _, _, _) in enumerate(blocks):
        x[0, 16 * k:16 * k + 16] = xs
    row = fp4.quantize_kv_fp4(x)[0]
    assert row.shape == (288,)
    for k, (name, _, sc, codes, _) in enumerate(blocks):
        assert row[256 + k] == sc, name
        for i in range(16):
            c = 16 * k + i
            byte = row[c // 2]
            nib = byte & 0xF if c % 2 == 0 else byte >> 4
            assert nib == codes[i], (name, i)


def test_golden_entry_dequantises_to_the_golden_values():
    """The packed golden entry through unpack_codes and dequantize_kv_fp4:
    every channel equals the hand-worked dequantised value bit for bit,
    the sign of zero included (a swapped nibble order, a scale applied to
    the wrong block or a dropped sign fails here).  The blocks are placed
    in reverse order in the second row, so the block-to-scale pairing is
    tested at two different offsets."""
    blocks = _golden_blocks()
    n = len(blocks)
    x = np.zeros((2, 512), dtype=np.float32)
    want = np.zeros((2, 512), dtype=np.float64)
    want_codes = np.zeros((2, 512), dtype=np.uint8)
    want_scales = np.zeros((2, 32), dtype=np.uint8)
    for k, (_, xs, sc, codes, deq) in enumerate(blocks):
        for row, blk in ((0, k), (1, 31 - k)):
            x[row, 16 * blk:16 * blk + 16] = xs
            want[row, 16 * blk:16 * blk + 16] = deq
            want_codes[row, 16 * blk:16 * blk + 16] = codes
            want_scales[row, blk] = sc
    packed = fp4.quantize_kv_fp4(x)
    codes, scales = fp4.unpack_codes(packed)
    np.testing.assert_array_equal(codes, want_codes)
    np.testing.assert_array_equal(scales, want_scales)
    got = fp4.dequantize_kv_fp4(packed)
    assert got.dtype == np.float64 and got.shape == (2, 512)
    np.testing.assert_array_equal(got, want)
    np.testing.assert_array_equal(np.signbit(got), np.signbit(want))
    assert n >= 11 and np.signbit(want).any()


def test_e4m3_decode_matches_torch_for_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float32).numpy().astype(np.float64)
    got = fp4.e4m3_value(codes)
    nan = np.isnan(ref)
    assert list(np.nonzero(nan)[0]) == [0x7F, 0xFF]
    np.testing.assert_array_equal(np.isnan(got), nan)
    np.testing.assert_array_equal(got[~nan], ref[~nan])
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9


def test_e2m1_decode_matches_ml_dtypes_for_all_codes():
    codes = np.arange(16, dtype=np.uint8)
    ref = codes.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    np.testing.assert_array_equal(fp4.e2m1_value(codes), ref)
    np.testing.assert_array_equal(fp4.e2m1_value(np.arange(8)), [0, 0.5, 1, 1.5, 2, 3, 4, 6])


def _midpoints_and_neighbours(mags):
    """Every midpoint between adjacent grid values, each grid value, and
    their float32 neighbours one ulp either side."""
    mids = (mags[:-1] + mags[1:]) / 2
    pts = np.concatenate([mids, mags, mags[-1:] * 1.01]).astype(np.float32)
    up = np.nextafter(pts, np.float32(np.inf))
    dn = np.nextafter(pts, np.float32(0))
    return np.concatenate([pts, up, dn, -pts, -up, -dn])


def test_e2m1_encode_matches_ml_dtypes():
    rng = np.random.default_rng(1)
    grid = fp4.e2m1_value(np.arange(8))
    x = np.concatenate([
        _midpoints_and_neighbours(grid),
        rng.normal(0, 3, 200000).astype(np.float32),
        rng.uniform(-8, 8, 200000).astype(np.float32),
        np.array([0.0, -0.0, 100.0, -1e30, 1e-30, -1e-30], dtype=np.float32),
    ]).astype(np.float32)
    ref = x.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    np.testing.assert_array_equal(fp4.e2m1_encode(x), ref)


def test_e4m3_encode_matches_libraries_below_saturation():
    rng = np.random.default_rng(2)
    grid = fp4.e4m3_value(np.arange(0x7F))
    x = np.concatenate([
        _midpoints_and_neighbours(grid),
        np.exp2(rng.uniform(-14, 8.8, 300000)).astype(np.float32),
        np.abs(rng.normal(0, 1, 100000)).astype(np.float32) / np.float32(6),
    ]).astype(np.float32)
    x = x[np.abs(x) < 448]            # both libraries turn larger values into NaN
    ref_md = x.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    ref_t = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = fp4.e4m3_encode(x)
    np.testing.assert_array_equal(got, ref_md)
    np.testing.assert_array_equal(got, ref_t)


def test_e4m3_encode_saturates():
    x = np.array([448, 455, 463.99, 464, 465, 1e6, 3.0e38], dtype=np.float32)
    np.testing.assert_array_equal(fp4.e4m3_encode(x), 0x7E)


def test_code_round_trips_are_exhaustive():
    # every finite E4M3 code except -0 decodes and re-encodes to itself
    for c in range(256):
        if c in (0x7F, 0xFF):
            continue
        v = np.float32(fp4.e4m3_value(c))
        assert int(fp4.e4m3_encode(np.array([v]))[0]) == c, hex(c)
    for c in range(16):
        v = np.float32(fp4.e2m1_value(c))
        assert int(fp4.e2m1_encode(np.array([v]))[0]) == c, hex(c)


def test_block_quantiser_agrees_with_library_composition():
    """The block recipe rebuilt from library conversions: s = E4M3(min(sf,
    448)) by ml_dtypes, y = fp32(x / s), code = E2M1(y) by ml_dtypes."""
    rng = np.random.default_rng(3)
    n = 40000
    scale = np.exp2(rng.uniform(-20, 14, (n, 1)))
    x = (rng.normal(0, 1, (n, 16)) * scale)
    x = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).to(torch.float32).numpy()
    codes, sc = fp4.quantize_block_codes(x)
    sf = np.max(np.abs(x), axis=1) / np.float32(6)
    s_code = np.minimum(sf, np.float32(448)).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    np.testing.assert_array_equal(sc, s_code)
    s = s_code.view(ml_dtypes.float8_e4m3fn).astype(np.float32)[:, None]
    with np.errstate(divide="ignore", invalid="ignore"):
        y = np.where(s != 0, x / np.where(s != 0, s, 1), np.copysign(np.float32(0), x)).astype(np.float32)
    ref = y.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    np.testing.assert_array_equal(codes, ref)
    assert (sc == 0).any() and (sc == 0x7E).any()      # both ends of the scale range were hit


def test_dequantised_values_are_exact_in_bf16():
    rng = np.random.default_rng(4)
    x = torch.randn(64, 512, generator=torch.Generator().manual_seed(4)).to(torch.bfloat16).float().numpy()
    v = fp4.dequantize_kv_fp4(fp4.quantize_kv_fp4(x))
    vb = torch.from_numpy(v).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(v, vb)
    # quantisation error bound: |x - v| <= s/4*... at most half the E2M1 step
    # times the scale, or saturation of at most (amax - 6 s)
    assert np.max(np.abs(v - x)) < 0.6
    del rng


def test_idempotent_when_amax_is_six_times_a_scale():
    """Quantising a dequantised block reproduces its bytes when the block
    holds a saturated value 6*s (then amax/6 = s exactly)."""
    rng = np.random.default_rng(5)
    for _ in range(200):
        s_code = int(rng.integers(0x08, 0x76))     # normal scales
        codes = rng.integers(0, 16, 16).astype(np.uint8)
        codes[rng.integers(0, 16)] = 7 | (8 * int(rng.integers(0, 2)))
        x = (fp4.e2m1_value(codes) * fp4.e4m3_value(s_code)).astype(np.float32)
        c2, s2 = fp4.quantize_block_codes(x[None])
        assert int(s2[0]) == s_code
        # -0 and +0 are both zero; compare decoded values and non-zero codes
        np.testing.assert_array_equal(fp4.e2m1_value(c2[0]), fp4.e2m1_value(codes))


def test_byte_accounting():
    """Packed entry = 256 nibble bytes + 32 E4M3 scales = 288 B, vs 1024 B of
    bf16 and 512 B + scales of FP8 (about half, as the FP4 section says).
    Model-level accounting of 890 B/token: 3 encoder main-KV caches at r=2
    and one decoder cache at r=1 ("3 encoder + 1 decoder cache"), plus the
    same four index-K caches at 128 FP4 values + one 4-byte scale (68 B)."""
    assert fp4.ENTRY_BYTES == 288
    assert fp4.quantize_kv_fp4(np.zeros((3, 512), np.float32)).shape == (3, 288)
    assert 288 / (512 + 32) < 0.53
    main = 3 * 288 / 2 + 288
    index = 3 * 68 / 2 + 68
    assert main == 720 and index == 170 and main + index == 890
