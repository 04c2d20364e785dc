"""Pins for the oracle's compress -> RoPE -> FP4 step (no GPU): closed forms
that a wrong order, sign, pair layout or channel range would break."""

import numpy as np
import torch

from oracle import compress, fp4


def _bf16(a):
    return torch.from_numpy(np.asarray(a, dtype=np.float32)).to(torch.bfloat16).to(torch.float32).numpy()


def _x(n, seed):
    return _bf16(np.random.default_rng(seed).normal(0, 1, (n, 512)))


def test_r1_unit_weight_zero_angle_is_the_plain_quantiser():
    x = _x(64, 1)
    w = np.ones((1, 1, 512), np.float32)
    cos, sin = np.ones((64, 32), np.float32), np.zeros((64, 32), np.float32)
    np.testing.assert_array_equal(compress.compress_rope_quantize(x, w, 1, cos, sin), fp4.quantize_kv_fp4(x))


def test_one_hot_weights_pick_a_token():
    x = _x(40, 2)                                       # 20 entries of r = 2
    w = np.zeros((20, 2, 512), np.float32)
    w[::2, 1] = 1.0                                      # even entries take their second token
    w[1::2, 0] = 1.0                                     # odd entries their first
    e = compress.compress_entries(x, w, 2)
    np.testing.assert_array_equal(e[::2], x[1::4])
    np.testing.assert_array_equal(e[1::2], x[2::4])


def test_power_of_two_weights_are_exact_and_ordered():
    """0.5 x0 + 0.25 x1 has no rounding for these inputs; a shared weight
    row applies to every entry."""
    x = _x(8, 3)
    w = np.stack([np.full(512, 0.5, np.float32), np.full(512, 0.25, np.float32)])[None]
    e = compress.compress_entries(x, w, 2)
    np.testing.assert_array_equal(e, 0.5 * x[0::2].astype(np.float64) + 0.25 * x[1::2].astype(np.float64))


def test_quarter_turn_maps_pairs_to_minus_b_a_and_leaves_the_rest():
    x = _x(16, 4)
    cos, sin = np.zeros((16, 32), np.float32), np.ones((16, 32), np.float32)
    rot = compress.rope_rotate(x, cos, sin)
    np.testing.assert_array_equal(rot[:, :448], x[:, :448])
    np.testing.assert_array_equal(rot[:, 448::2], -x[:, 449::2])
    np.testing.assert_array_equal(rot[:, 449::2], x[:, 448::2])
    # so the fused step equals quantising the hand-rotated vectors
    w = np.ones((1, 1, 512), np.float32)
    man = x.copy()
    man[:, 448::2], man[:, 449::2] = -x[:, 449::2], x[:, 448::2]
    np.testing.assert_array_equal(compress.compress_rope_quantize(x, w, 1, cos, sin), fp4.quantize_kv_fp4(man))


def test_rotation_keeps_pair_norms_and_angles_add():
    rng = np.random.default_rng(5)
    x = _x(32, 5)
    th = rng.uniform(-np.pi, np.pi, (32, 32))
    cos, sin = np.cos(th).astype(np.float32), np.sin(th).astype(np.float32)
    rot = compress.rope_rotate(x, cos, sin).astype(np.float64)
    n0 = x[:, 448::2].astype(np.float64) ** 2 + x[:, 449::2].astype(np.float64) ** 2
    n1 = rot[:, 448::2] ** 2 + rot[:, 449::2] ** 2
    np.testing.assert_allclose(n1, n0, rtol=1e-5, atol=1e-6)
    # the rotated pair's angle is the original plus theta
    ang = np.arctan2(rot[:, 449::2], rot[:, 448::2]) - np.arctan2(x[:, 449::2], x[:, 448::2])
    d = np.angle(np.exp(1j * (ang - th)))
    assert np.max(np.abs(d[n0 > 1e-6])) < 1e-4
