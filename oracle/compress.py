"""Oracle: new main-KV entries compressed, rotated and quantised to FP4.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

Sources: [eogee] §3.2: CSA2 compresses every r tokens into one main-KV entry
(r = 2 in the encoder, r = 1 in the decoder), without the overlap between
neighbouring entries and without absolute position encoding in the
compression; §3.4: the entry is quantised to FP4 after RoPE (quantising
before RoPE was measured to gain little accuracy and to cost decode time);
[nxbn] §3.1: a 64-dimensional RoPE slice of the 512-dimensional head.

The pages print neither the compressor's form nor the rotation's layout.
Readings used here:

* compression: entry e = sum over j < r of w[e][j] * x[e r + j], channel by
  channel, with the weights given by the caller (learned in the model);
  weights shared by every entry are the case w[e] = w[0];
* RoPE on channels 448..511 (the last 64), rotating adjacent pairs
  (448 + 2i, 449 + 2i) by the caller's angle for pair i of entry e, given
  as cos[e][i] and sin[e][i] (the frequencies, YaRN included, are the
  model's choice): (a, b) -> (a cos - b sin, a sin + b cos);
* every step in IEEE float32 with one rounding per operation, in the order
  written (products, then the sum over j in increasing j; a cos, b sin,
  then their difference); the rotated float32 entry goes to the FP4
  quantiser of ``oracle.fp4`` without an intermediate bf16 rounding.

Parity: pinned (tests/test_oracle_compress.py) against closed forms: r = 1
with unit weight and zero angle is the plain quantiser; one-hot weights pick
a token; a quarter turn maps (a, b) to (-b, a) exactly; channels below 448
are not rotated; pair norms are kept.
"""

import numpy as np

from .fp4 import D_MAIN, quantize_kv_fp4

ROPE_START = 448      # [nxbn] §3.1 qk_rope_head_dim 64 of head_dim 512: the last 64 channels
ROPE_PAIRS = 32


def compress_entries(x, w, r):
    """x float32 [n_entries * r, 512], w float32 [n_entries or 1, r, 512] ->
    float32 [n_entries, 512]."""
    x = np.asarray(x, dtype=np.float32)
    w = np.asarray(w, dtype=np.float32)
    n = x.shape[0] // r
    xs = x.reshape(n, r, D_MAIN)
    wb = np.broadcast_to(w, (n, r, D_MAIN)) if w.shape[0] == 1 else w
    acc = (wb[:, 0] * xs[:, 0]).astype(np.float32)
    for j in range(1, r):
        acc = (acc + (wb[:, j] * xs[:, j]).astype(np.float32)).astype(np.float32)
    return acc


def rope_rotate(e, cos, sin):
    """e float32 [n, 512]; cos, sin float32 [n, 32] -> rotated float32 copy."""
    e = np.array(e, dtype=np.float32, copy=True)
    cos = np.asarray(cos, dtype=np.float32)
    sin = np.asarray(sin, dtype=np.float32)
    a = e[:, ROPE_START::2].copy()
    b = e[:, ROPE_START + 1::2].copy()
    e[:, ROPE_START::2] = ((a * cos).astype(np.float32) - (b * sin).astype(np.float32)).astype(np.float32)
    e[:, ROPE_START + 1::2] = ((a * sin).astype(np.float32) + (b * cos).astype(np.float32)).astype(np.float32)
    return e


def compress_rope_quantize(x, w, r, cos, sin):
    """The fused step: packed FP4 entries uint8 [n_entries, 288]."""
    return quantize_kv_fp4(rope_rotate(compress_entries(x, w, r), cos, sin))
