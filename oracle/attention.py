"""Oracle: sparse MQA attention over selected FP4 entries plus the SWA window.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

Sources:
* [eogee] §3.2: each query attends only to its selected main-KV entries plus
  this layer's SWA KV; every layer keeps its own global Q and SWA KV; 64
  query heads, head dim 512, top-K 512, SWA window 128.
* [nxbn] §3.1 table: num_attention_heads 64, num_key_value_heads 1,
  head_dim 512, qk_rope_head_dim 64, sliding_window 128.
* [eogee] §3.4: the FP4 cache is dequantised before the attention math.

Readings (the pages are silent): one main-KV vector per entry serves as both
key and value (one KV head); the softmax is one joint softmax over the K
selected entries and the W window rows, with no de-duplication when a
selected entry and a window row describe the same token; scale 1/sqrt(512)
unless given; no attention sink; index -1 is skipped.  The 64-dim RoPE
slice is already rotated in the inputs, so it needs no separate treatment.

float64 throughout.  Parity: pinned (tests/test_oracle_attention.py) against
torch's scaled_dot_product_attention on the dense special case, softmax
normalisation, uniform-score and single-key closed forms.

Quantised Q ([eogee] §3.4 says the model deliberately does not rely on the
tensor cores' native FP4 matmul, which would need Q in FP4 as well): the
variant ``quantize_q`` puts every head row of Q through the main-KV rule
(E2M1 values, one E4M3 scale per 16 channels, s = E4M3(amax / 6)), and the
attention is then ``sparse_mqa`` on those values for every key, selected
entries and window rows alike.  Pinned by: grid-valued Q is unchanged (the
quantiser's idempotence) and the composition of pinned functions.
"""

import numpy as np

from . import fp4

H = 64        # [nxbn] §3.1 num_attention_heads
D = 512       # [nxbn] §3.1 head_dim
WIN = 128     # [nxbn] §3.1 sliding_window, [eogee] §3.2 win = 128


def sparse_mqa(q, kv_deq, idx, swa_rows, scale=None):
    """One query position.

    q        [64, 512]   query heads
    kv_deq   [N, 512]    dequantised main-KV entries (key = value)
    idx      [K]         selected entry positions, -1 = empty slot
    swa_rows [W, 512]    this layer's window rows visible to the query
    Returns (o [64, 512], lse [64]) with lse the natural-log sum of
    exp(scaled logits); no keys at all gives o = 0 and lse = -inf.
    """
    q = np.asarray(q, dtype=np.float64)
    idx = np.asarray(idx)
    sel = np.asarray(kv_deq, dtype=np.float64)[idx[idx >= 0]]
    keys = np.concatenate([sel, np.asarray(swa_rows, dtype=np.float64).reshape(-1, q.shape[1])], axis=0)
    if scale is None:
        scale = 1.0 / np.sqrt(q.shape[1])
    if keys.shape[0] == 0:
        return np.zeros_like(q), np.full(q.shape[0], -np.inf)
    logits = (q @ keys.T) * scale                 # [64, n_keys]
    m = logits.max(axis=1, keepdims=True)
    e = np.exp(logits - m)
    l = e.sum(axis=1, keepdims=True)
    p = e / l
    o = p @ keys
    lse = (m + np.log(l))[:, 0]
    return o, lse


def quantize_q(q):
    """[..., 512] query rows through the main-KV FP4 rule and back
    (float64, exact dequantised values)."""
    q = np.asarray(q, dtype=np.float32)
    rows = q.reshape(-1, q.shape[-1])
    return fp4.dequantize_kv_fp4(fp4.quantize_kv_fp4(rows)).reshape(q.shape)
