"""Oracle: FP4 (E2M1 values, one E4M3 scale per 16 channels) main-KV entries.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

Source of the format: [eogee] §3.4 "FP4 主 KV 缓存" states the main-KV
cache stores E2M1 values with one E4M3 scale per 16 channels, like NVFP4
without its second-level global scale, quantised after RoPE and dequantised
before the attention math.  [ainewsway] section "KV 快取為何成為瓶頸" and
[nxbn] §2.3 repeat E2M1 + per-16-channel E4M3 scaling.  The pages give no
scale constant and no rounding mode; the readings used here are:

* scale  sf = fp32(amax / 6)  (6 = largest E2M1 magnitude), then
  s = E4M3(sf) rounded to nearest, ties to even code, saturating at 448;
* value  y  = fp32(x / s), then q = E2M1(y) rounded to nearest, ties to
  even code, saturating at 6; the sign bit is signbit(y), so -0 exists;
* if s == 0 every y of the block is a zero carrying the sign of x;
* packed entry (512 channels): 256 bytes of nibbles, channel 2i in the low
  nibble of byte i and channel 2i+1 in the high nibble, then 32 scale bytes
  (scale of block k at byte 256 + k)  ->  288 bytes per entry.

Both decisions are taken in IEEE float32 (numpy float32 division is
correctly rounded), the same precision the kernel uses.  The grids below are
enumerated from the bit-field definitions of the two formats, not from a
table shared with anything else.

Parity: pinned (tests/test_oracle_fp4.py) against hand-worked blocks, the
ml_dtypes and torch float8 conversions, and exhaustive code round-trips.
"""

import numpy as np

D_MAIN = 512          # main-KV entry width, [nxbn] §3.1 head_dim 512
BLOCK = 16            # channels per scale, [eogee] §3.4
N_BLOCKS = D_MAIN // BLOCK
ENTRY_BYTES = D_MAIN // 2 + N_BLOCKS   # 256 nibble bytes + 32 scale bytes


# ---------------------------------------------------------------------------
# Format definitions
# ---------------------------------------------------------------------------

def e4m3_value(code):
    """Decode E4M3 (FN variant: 4 exponent bits, bias 7, 3 mantissa bits,
    no infinities, S.1111.111 is NaN) to float64.  Works on arrays."""
    c = np.asarray(code, dtype=np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    normal = (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0)
    subnormal = (m / 8.0) * 2.0 ** -6
    mag = np.where(e == 0, subnormal, normal)
    mag = np.where((e == 15) & ((c & 7) == 7), np.nan, mag)
    return sign * mag


def e2m1_value(code):
    """Decode E2M1 (2 exponent bits, bias 1, 1 mantissa bit; subnormal when
    the exponent field is 0) to float64.  Works on arrays."""
    c = np.asarray(code, dtype=np.int64)
    sign = np.where(c & 0x8, -1.0, 1.0)
    e = (c >> 1) & 0x3
    m = (c & 0x1).astype(np.float64)
    mag = np.where(e == 0, m * 0.5, (1.0 + m / 2.0) * np.exp2(e.astype(np.float64) - 1.0))
    return sign * mag


# magnitudes of all non-negative finite codes, ascending in code order
_E4M3_MAGS = e4m3_value(np.arange(0x7F))        # codes 0x00..0x7E, max 448
_E2M1_MAGS = e2m1_value(np.arange(8))           # 0, .5, 1, 1.5, 2, 3, 4, 6


def _round_to_grid(a, mags):
    """Index of the grid magnitude nearest to a >= 0 (float64 array, values
    exactly representable), ties to the even index, saturating at the top.
    Grid values ascend with their code, so the code is the index."""
    a = np.asarray(a, dtype=np.float64)
    top = len(mags) - 1
    i = np.searchsorted(mags, a, side="right") - 1          # mags[i] <= a
    i = np.clip(i, 0, top)
    j = np.minimum(i + 1, top)
    d_lo = a - mags[i]
    d_hi = mags[j] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (i % 2 == 1))
    out = np.where(pick_hi & (j != i), j, i)
    return np.where(a >= mags[top], top, out).astype(np.int64)


def e4m3_encode(x):
    """float32 -> E4M3 code, round to nearest even, saturate to +-448."""
    x = np.asarray(x, dtype=np.float32)
    mag = _round_to_grid(np.abs(x).astype(np.float64), _E4M3_MAGS)
    return (np.where(np.signbit(x), 0x80, 0) | mag).astype(np.uint8)


def e2m1_encode(y):
    """float32 -> E2M1 code, round to nearest even, saturate to +-6; the sign
    bit is the sign bit of y (so -0 encodes as 0x8)."""
    y = np.asarray(y, dtype=np.float32)
    mag = _round_to_grid(np.abs(y).astype(np.float64), _E2M1_MAGS)
    return (np.where(np.signbit(y), 0x8, 0) | mag).astype(np.uint8)


# ---------------------------------------------------------------------------
# Entry quantisation
# ---------------------------------------------------------------------------

def quantize_block_codes(x):
    """Quantise blocks of 16 channels.

    x: float32 array [..., 16] of bf16-representable values (finite).
    Returns (value codes uint8 [..., 16], scale code uint8 [...]).
    """
    x = np.asarray(x, dtype=np.float32)
    assert x.shape[-1] == BLOCK
    amax = np.max(np.abs(x), axis=-1)
    sf = amax / np.float32(6.0)                     # fp32, correctly rounded
    s_code = e4m3_encode(sf)
    s = e4m3_value(s_code).astype(np.float32)       # exact in fp32
    s_b = s[..., None]
    with np.errstate(divide="ignore", invalid="ignore"):
        y = np.where(s_b != 0, x / np.where(s_b != 0, s_b, np.float32(1.0)),
                     np.copysign(np.float32(0.0), x))
    return e2m1_encode(y.astype(np.float32)), s_code


def quantize_kv_fp4(x):
    """Quantise main-KV entries.  x: [n, 512] float32 (bf16 values).
    Returns packed uint8 [n, 288]."""
    x = np.asarray(x, dtype=np.float32)
    n = x.shape[0]
    assert x.shape == (n, D_MAIN)
    codes, scales = quantize_block_codes(x.reshape(n, N_BLOCKS, BLOCK))
    codes = codes.reshape(n, D_MAIN)
    out = np.zeros((n, ENTRY_BYTES), dtype=np.uint8)
    out[:, :D_MAIN // 2] = codes[:, 0::2] | (codes[:, 1::2] << 4)
    out[:, D_MAIN // 2:] = scales
    return out


def unpack_codes(packed):
    """Packed [n, 288] -> (value codes [n, 512], scale codes [n, 32])."""
    packed = np.asarray(packed, dtype=np.uint8)
    n = packed.shape[0]
    nib = packed[:, :D_MAIN // 2]
    codes = np.empty((n, D_MAIN), dtype=np.uint8)
    codes[:, 0::2] = nib & 0xF
    codes[:, 1::2] = nib >> 4
    return codes, packed[:, D_MAIN // 2:]


def dequantize_kv_fp4(packed):
    """Packed [n, 288] -> float64 [n, 512]; v = E2M1(q) * E4M3(s), which is
    exact (at most 6 significant bits) in bf16, fp32 and fp64 ([eogee] §3.4:
    the cache is dequantised before the attention math)."""
    codes, scales = unpack_codes(packed)
    n = codes.shape[0]
    vals = e2m1_value(codes).reshape(n, N_BLOCKS, BLOCK)
    s = e4m3_value(scales)[..., None]
    return (vals * s).reshape(n, D_MAIN)
