"""Pins for the oracle's MXFP4 index-K entries (no GPU).

Pinned against hand-worked blocks (tests/golden/mxfp4_index_k_blocks.txt),
the ml_dtypes float4_e2m1fn conversion of x / 2^e and its float8_e8m0fnu
decoding of the scale bytes (independent library routines), the exponent
rule computed with frexp, and the 890 B/token accounting.
"""

import os

import ml_dtypes
import numpy as np
import pytest
import torch

from oracle import mxfp4

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "mxfp4_index_k_blocks.txt")


def _golden():
    out = []
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        name, xs, sc, codes, deq = [p.strip() for p in line.split("|")]
        out.append((name, np.array([float(v) for v in xs.split()], dtype=np.float32), int(sc),
                    np.array([int(c, 16) for c in codes.split()], dtype=np.uint8),
                    np.array([float(v) for v in deq.split()], dtype=np.float64)))
    return out


def _codes(packed):
    nib = packed[:, :64]
    c = np.empty((packed.shape[0], 128), dtype=np.uint8)
    c[:, 0::2] = nib & 0xF
    c[:, 1::2] = nib >> 4
    return c


@pytest.mark.parametrize("blk", _golden(), ids=lambda b: b[0])
def test_hand_worked_blocks(blk):
    name, xs, sc, codes, deq = blk
    for k in range(4):                                  # the block in each of the four positions
        x = np.zeros((1, 128), dtype=np.float32)
        x[0, 32 * k:32 * k + xs.shape[0]] = xs
        p = mxfp4.quantize_index_k_mxfp4(x)
        assert p.shape == (1, 68)
        assert int(p[0, 64 + k]) == sc, name
        others = [64 + j for j in range(4) if j != k]
        assert np.all(p[0, others] == 0)                # zero blocks: e = -127
        c = _codes(p)[0, 32 * k:32 * k + xs.shape[0]]
        np.testing.assert_array_equal(c, codes, err_msg=name)
        v = mxfp4.dequantize_index_k_mxfp4(p)[0, 32 * k:32 * k + xs.shape[0]]
        np.testing.assert_array_equal(v, deq)
        np.testing.assert_array_equal(np.signbit(v), np.signbit(deq))


def _random(seed, n=5000):
    rng = np.random.default_rng(seed)
    x = rng.normal(0, 1, (n, 4, 32)) * np.exp2(rng.uniform(-60, 60, (n, 4, 1)))
    x[::9, 1] = 0.0
    x = x.reshape(n, 128)
    return torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).to(torch.float32).numpy()


def test_exponent_rule_by_frexp():
    x = _random(1)
    p = mxfp4.quantize_index_k_mxfp4(x)
    amax = np.max(np.abs(x.reshape(-1, 4, 32)), axis=2)
    m, E = np.frexp(amax.astype(np.float64))            # amax = m 2^E, m in [0.5, 1)
    want = np.where(amax > 0, np.clip(E - 1 - 2, -127, 127), -127) + 127
    np.testing.assert_array_equal(p[:, 64:], want.astype(np.uint8))
    # the scale bytes decode through ml_dtypes' E8M0 to the same power of two
    s = p[:, 64:].copy().view(ml_dtypes.float8_e8m0fnu).astype(np.float64)
    np.testing.assert_array_equal(s, np.exp2(want.astype(np.float64) - 127))


def test_codes_match_the_library_e2m1_conversion():
    x = _random(2)
    p = mxfp4.quantize_index_k_mxfp4(x)
    e = p[:, 64:].astype(np.float64) - 127
    y = (x.reshape(-1, 4, 32) * np.exp2(-e)[..., None]).astype(np.float32).reshape(-1, 128)
    assert np.all(np.abs(y) < 8)
    ref = y.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    np.testing.assert_array_equal(_codes(p), ref)


def test_dequantised_values_are_exact_in_bf16_and_close():
    x = _random(3, n=400)
    v = mxfp4.dequantize_index_k_mxfp4(mxfp4.quantize_index_k_mxfp4(x))
    vb = torch.from_numpy(v).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(v, vb)
    # per block: |v - x| <= half the largest E2M1 step (1) times 2^e, or the
    # saturation of x/2^e < 8 down to 6
    e = mxfp4.block_exponent(np.max(np.abs(x.reshape(-1, 4, 32)), axis=2)).astype(np.float64)
    bound = np.repeat(2.0 * np.exp2(e), 32, axis=1)
    assert np.all(np.abs(v - x) <= bound)


def test_entry_bytes_close_the_890_accounting():
    """68 B per index-K entry: with 288 B main-KV entries and the pages'
    three encoder caches at r=2 plus one decoder cache, 720 + 170 = 890 B per
    token."""
    assert mxfp4.ENTRY_BYTES == 68
    main = 3 * 288 / 2 + 288
    index = 3 * mxfp4.ENTRY_BYTES / 2 + mxfp4.ENTRY_BYTES
    assert main + index == 890


def test_fake_quantize_is_idempotent_and_keeps_grid_values():
    """Index-Q goes through the same rule: values already on a block's grid
    (E2M1 x 2^e with the block maximum at 4 or 6 times 2^e) are fixed
    points, and quantising twice equals quantising once (the block maximum
    after quantisation is 4 or 6 times 2^e, so the exponent is kept)."""
    rng = np.random.default_rng(11)
    x = torch.from_numpy(rng.normal(0, 1, (300, 128)).astype(np.float32) *
                         np.exp2(rng.integers(-30, 30, (300, 1))).astype(np.float32)).to(torch.bfloat16).float().numpy()
    once = mxfp4.fake_quantize(x)
    twice = mxfp4.fake_quantize(once.astype(np.float32))
    np.testing.assert_array_equal(once, twice)
    # grid values: codes times 2^e, with the largest magnitude 6 * 2^e
    e = rng.integers(-20, 20, (50, 4, 1))
    codes = rng.integers(0, 16, (50, 4, 32)).astype(np.uint8)
    codes[:, :, 0] = 7
    grid = (mxfp4.e2m1_value(codes) * np.exp2(e)).reshape(50, 128)
    np.testing.assert_array_equal(mxfp4.fake_quantize(grid.astype(np.float32)), grid)
    # any leading shape: [B, Q, 32 heads, 128]
    q = x[:64].reshape(2, 1, 32, 128)
    np.testing.assert_array_equal(mxfp4.fake_quantize(q).reshape(64, 128), once[:64])
