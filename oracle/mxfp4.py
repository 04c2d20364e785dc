"""Oracle: FP4 index-K entries in the OCP MXFP4 format.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

Source: [eogee] §3.4 says V4 already trained the indexer's Q/K with FP4
quantisation and names the format family OCP MXFP4 (E2M1 values); the page
gives no layout for the index-K cache.  The byte accounting on
[ainewsway] "KV 快取為何成為瓶頸" (890 B per token = three encoder caches at
r=2 and one decoder cache, main KV 288 B per entry) leaves 170 B per token
for four index-K caches, i.e. 68 B per 128-channel index-K entry: 64 B of
E2M1 values and 4 B of scales.  OCP MXFP4 proper is exactly that: one
8-bit power-of-two scale (E8M0) per block of 32 elements.  Readings:

* block of 32 channels, shared scale X = 2^e with
  e = floor(log2(amax)) - 2 (2 = the largest E2M1 exponent, the OCP MX
  rule), clamped to the E8M0 range [-127, 127]; an all-zero block uses
  e = -127;
* q_i = E2M1(x_i / X), round to nearest, ties to the even code,
  saturating at 6 (x/X < 8 always); the sign bit is that of x_i;
* entry layout: byte i (0..63) holds channel 2i in its low nibble and
  channel 2i+1 in its high nibble, byte 64 + k holds e + 127 for
  channels 32k..32k+31 -> 68 bytes per entry;
* dequantised value E2M1(q) * 2^e, exact in bf16 and fp32.

x / X is a power-of-two scaling, exact in float32 for every bf16 input.

Index-Q: the same page says the indexer's Q and K are both FP4 (quantisation
aware training), so when index-K is MXFP4 the scores are those of index-Q
quantised by the same rule (per head row of 128 dims, blocks of 32) and
dequantised (``fake_quantize``); index-Q is never stored, so only its values
matter.

Parity: pinned (tests/test_oracle_mxfp4.py) against hand-worked blocks,
the ml_dtypes float4_e2m1fn conversion of x / X and its float8_e8m0fnu
decoding of the scale bytes, the exponent rule computed by frexp, and the
890 B accounting.
"""

import numpy as np

from .fp4 import e2m1_encode, e2m1_value

D_INDEX = 128         # index-K width, [nxbn] §3.3 index_head_dim
BLOCK = 32            # OCP MX block size
N_BLOCKS = D_INDEX // BLOCK
ENTRY_BYTES = D_INDEX // 2 + N_BLOCKS     # 64 + 4 = 68


def block_exponent(amax):
    """e = floor(log2(amax)) - 2, clamped to [-127, 127]; -127 for amax 0.
    Works on arrays of non-negative float32."""
    a = np.asarray(amax, dtype=np.float64)
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0))) - 2
    e = np.where(a > 0, e, -127)
    return np.clip(e, -127, 127).astype(np.int64)


def quantize_index_k_mxfp4(x):
    """x: float32 [n, 128] (bf16 values, finite) -> uint8 [n, 68]."""
    x = np.asarray(x, dtype=np.float32)
    n = x.shape[0]
    assert x.shape == (n, D_INDEX)
    xb = x.reshape(n, N_BLOCKS, BLOCK)
    e = block_exponent(np.max(np.abs(xb), axis=2))                  # [n, 4]
    y = (xb.astype(np.float64) * np.exp2(-e.astype(np.float64))[..., None]).astype(np.float32)
    codes = e2m1_encode(y).reshape(n, D_INDEX)
    out = np.zeros((n, ENTRY_BYTES), dtype=np.uint8)
    out[:, :D_INDEX // 2] = codes[:, 0::2] | (codes[:, 1::2] << 4)
    out[:, D_INDEX // 2:] = (e + 127).astype(np.uint8)
    return out


def dequantize_index_k_mxfp4(packed):
    """uint8 [n, 68] -> float64 [n, 128]."""
    packed = np.asarray(packed, dtype=np.uint8)
    n = packed.shape[0]
    nib = packed[:, :D_INDEX // 2]
    codes = np.empty((n, D_INDEX), dtype=np.uint8)
    codes[:, 0::2] = nib & 0xF
    codes[:, 1::2] = nib >> 4
    e = packed[:, D_INDEX // 2:].astype(np.float64) - 127.0
    vals = e2m1_value(codes).reshape(n, N_BLOCKS, BLOCK)
    return (vals * np.exp2(e)[..., None]).reshape(n, D_INDEX)


def fake_quantize(x):
    """Rows of 128 values (float32, bf16-representable; any leading shape)
    through the MXFP4 rule and back: float64 of the same shape.  Used for
    index-Q, whose scores with an MXFP4 index-K are defined on these values."""
    x = np.asarray(x, dtype=np.float32)
    shape = x.shape
    assert shape[-1] == D_INDEX
    rows = x.reshape(-1, D_INDEX)
    return dequantize_index_k_mxfp4(quantize_index_k_mxfp4(rows)).reshape(shape)
