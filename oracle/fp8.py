"""Oracle: FP8 sliding-window (SWA) KV rows.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

Source: [eogee] §3.4 "FP4 主 KV 缓存" keeps the quantisation-sensitive SWA KV
cache in FP8 while the main KV goes to FP4.  The pages name the precision
only.  The readings used here (the plainest per-row FP8 cache):

* element format E4M3 (the FN variant, max 448), the same FP8 format the
  pages use for the main KV's scales;
* one float32 scale per cached window row: s = fp32(amax / 448) with IEEE
  round-to-nearest-even division, so the largest element maps to 448;
* code_i = E4M3(fp32(x_i / s)), round to nearest, ties to the even code,
  saturating at 448 (s can round down, so |x/s| can exceed 448 by an ulp);
  the sign bit is signbit(x_i / s), so -0 exists;
* s == 0 (an all-zero row) makes every element a zero carrying its sign;
* dequantised value v_i = E4M3(code_i) * s (exact in float64).

The decision (the E4M3 code) is taken in IEEE float32, as the kernel takes
it.  The E4M3 grid and encoder are those of ``oracle.fp4`` (its scale
format), pinned there against two library conversions.

Parity: pinned (tests/test_oracle_fp8.py) against hand-worked rows
(tests/golden/fp8_window_rows.txt), the ml_dtypes float8_e4m3fn and torch
float8_e4m3fn conversions of x / s, and byte accounting.
"""

import numpy as np

from .fp4 import e4m3_encode, e4m3_value

D_ROW = 512           # window row width = attention head dim, [nxbn] §3.1
E4M3_MAX = 448.0


def quantize_window_fp8(x):
    """x: float32 [n, 512] (bf16 values, finite).  Returns (codes uint8
    [n, 512], scales float32 [n])."""
    x = np.asarray(x, dtype=np.float32)
    assert x.ndim == 2 and x.shape[1] == D_ROW
    amax = np.max(np.abs(x), axis=1)
    s = (amax / np.float32(E4M3_MAX)).astype(np.float32)        # fp32, correctly rounded
    s_b = s[:, None]
    with np.errstate(divide="ignore", invalid="ignore"):
        y = np.where(s_b != 0, x / np.where(s_b != 0, s_b, np.float32(1.0)),
                     np.copysign(np.float32(0.0), x)).astype(np.float32)
    return e4m3_encode(y), s


def dequantize_window_fp8(codes, scales):
    """codes uint8 [n, 512], scales float32 [n] -> float64 [n, 512]."""
    return e4m3_value(np.asarray(codes)) * np.asarray(scales, dtype=np.float64)[:, None]


def row_bytes():
    """Bytes of one cached window row: 512 E4M3 codes and a 4-byte scale."""
    return D_ROW + 4
