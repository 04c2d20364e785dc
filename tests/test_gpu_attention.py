"""GPU parity of csa2_sparse_attn against the float64 oracle on the same
index sets (1e-2 absolute + 1e-2 relative)."""

import numpy as np
import pytest
import torch

from fp4_kv_cache_mxfp4_b200 import csa2
from oracle import attention, fp4
from parity import check_attention, f32

pytestmark = pytest.mark.gpu


def _case(B, Q, N, K, W, swa_step, seed, q_std=512 ** -0.5, minus_one=0.0):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(B, N, 512, generator=g).to(torch.bfloat16)
    kv = np.stack([fp4.quantize_kv_fp4(f32(x[b])) for b in range(B)])       # oracle-made cache bytes
    q = (torch.randn(B, Q, 64, 512, generator=g) * q_std).to(torch.bfloat16)
    rows = W + (Q - 1) * swa_step if W else 1
    swa = torch.randn(B, rows, 512, generator=g).to(torch.bfloat16)
    rng = np.random.default_rng(seed)
    idx = np.stack([[rng.choice(N, K, replace=False) if K else np.zeros(0, int) for _ in range(Q)]
                    for _ in range(B)]).astype(np.int32).reshape(B, Q, K)
    if minus_one:
        idx[rng.random(idx.shape) < minus_one] = -1
    return kv, q, swa, idx


def _run(kv, q, swa, idx, W, swa_step, scale=0.0, want_lse=True):
    B, Q = q.shape[:2]
    d = "cuda"
    kv_d = torch.from_numpy(kv).to(d)
    q_d, swa_d = q.to(d), swa.to(d)
    idx_d = torch.from_numpy(idx).to(d)
    out = torch.full((B, Q, 64, 512), float("nan"), dtype=torch.bfloat16, device=d)
    lse = torch.full((B, Q, 64), float("nan"), device=d) if want_lse else None
    a = csa2.attn_args(q_d, kv_d, idx_d, swa_d, out, lse, W=W, swa_step=swa_step, scale=scale)
    ws = csa2.workspace(a, csa2.WS_ATTN)
    csa2.csa2_sparse_attn(a, ws)
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), (lse.cpu().numpy() if want_lse else None)


def _oracle(kv, q, swa, idx, W, swa_step, scale=None, quantised_q=False):
    B, Q = q.shape[:2]
    o = np.zeros((B, Q, 64, 512))
    lse = np.zeros((B, Q, 64))
    for b in range(B):
        deq = fp4.dequantize_kv_fp4(kv[b])
        for i in range(Q):
            rows = f32(swa[b])[i * swa_step: i * swa_step + W]
            qi = attention.quantize_q(f32(q[b, i])) if quantised_q else f32(q[b, i])
            o[b, i], lse[b, i] = attention.sparse_mqa(qi, deq, idx[b, i], rows, scale)
    return o, lse


@pytest.mark.parametrize("B,Q,N,K,W,step,seed,m1", [
    (1, 4, 2048, 512, 128, 0, 0, 0.0),
    (2, 3, 700, 512, 128, 0, 1, 0.1),      # some empty slots
    (1, 2, 300, 100, 37, 1, 2, 0.0),       # ragged slices, causal windows
    (3, 1, 64, 64, 0, 0, 3, 0.0),          # selected entries only
    (1, 1, 10, 0, 128, 0, 4, 0.0),         # window only
    (1, 130, 3000, 512, 128, 1, 7, 0.05),  # 130 queries: one CTA per query over all its slices
    (2, 70, 900, 200, 100, 1, 8, 0.0),     # per query, ragged slices
    (2, 1, 1500, 512, 256, 0, 10, 0.0),    # 6 slices merged in one cluster
    (1, 2, 1500, 896, 128, 0, 11, 0.02),   # 8 slices: the largest cluster
    (1, 2, 1500, 1024, 128, 0, 12, 0.0),   # 9 slices: partials and the merge kernel
    (3, 1, 500, 130, 0, 0, 13, 0.0),       # 2 slices, the second with 2 keys
])
def test_attention_parity(B, Q, N, K, W, step, seed, m1):
    kv, q, swa, idx = _case(B, Q, N, K, W, step, seed, minus_one=m1)
    out, lse = _run(kv, q, swa, idx, W, step)
    o_ref, lse_ref = _oracle(kv, q, swa, idx, W, step)
    check_attention(out, o_ref, what="out")
    np.testing.assert_allclose(lse, lse_ref, rtol=1e-3, atol=1e-3)


def test_peaked_softmax_and_explicit_scale():
    kv, q, swa, idx = _case(2, 1, 1000, 512, 128, 0, 5, q_std=1.0)
    out, lse = _run(kv, q, swa, idx, 128, 0, scale=0.125)
    o_ref, lse_ref = _oracle(kv, q, swa, idx, 128, 0, scale=0.125)
    check_attention(out, o_ref, what="peaked")
    np.testing.assert_allclose(lse, lse_ref, rtol=1e-3, atol=1e-2)


def test_per_query_reference_max_moves():
    """One CTA per query with a very peaked softmax (unit query scale and
    softmax scale 1): slice maxima differ by tens of log2 units, so later
    slices often move the running reference max and the accumulated output
    of the earlier slices is rescaled."""
    kv, q, swa, idx = _case(1, 128, 2000, 384, 128, 1, 9, q_std=1.0)
    out, lse = _run(kv, q, swa, idx, 128, 1, scale=1.0)
    o_ref, lse_ref = _oracle(kv, q, swa, idx, 128, 1, scale=1.0)
    check_attention(out, o_ref, what="rescaled")
    np.testing.assert_allclose(lse, lse_ref, rtol=1e-3, atol=1e-2)


def test_no_keys_at_all():
    for Q in (2, 128):                     # split slices and one CTA per query
        kv, q, swa, idx = _case(1, Q, 100, 64, 0, 0, 6)
        idx[:] = -1
        out, lse = _run(kv, q, swa, idx, 0, 0)
        assert np.all(out == 0)
        assert np.all(np.isneginf(lse))


def _q_rows_fp4(q):
    """Oracle-made FP4 rows of Q (the main-KV entry format per head)."""
    B, Q = q.shape[:2]
    return torch.from_numpy(fp4.quantize_kv_fp4(f32(q).reshape(-1, 512)).reshape(B, Q, 64, 288))


@pytest.mark.parametrize("B,Q,N,K,W,step,seed,m1", [
    (2, 1, 1500, 512, 128, 0, 20, 0.0),    # 5 slices in a cluster: FP4 slices on the FP4 tensor path
    (1, 2, 1500, 1024, 128, 0, 21, 0.05),  # 9 slices: partials and the merge kernel
    (3, 1, 500, 130, 0, 0, 22, 0.0),       # selected entries only, a 2-key slice
    (1, 1, 10, 0, 128, 0, 23, 0.0),        # window only (dequantised Q on the bf16 path)
    (1, 130, 3000, 512, 128, 1, 24, 0.05), # one CTA per query: dequantised Q for every slice
])
def test_quantised_q_parity(B, Q, N, K, W, step, seed, m1):
    """Quantised Q: Q given as FP4 rows; against the oracle's attention on
    the dequantised Q (the logits of every key use those values)."""
    kv, q, swa, idx = _case(B, Q, N, K, W, step, seed, minus_one=m1)
    out, lse = _run(kv, _q_rows_fp4(q), swa, idx, W, step)
    o_ref, lse_ref = _oracle(kv, q, swa, idx, W, step, quantised_q=True)
    check_attention(out, o_ref, what="quantised q")
    np.testing.assert_allclose(lse, lse_ref, rtol=1e-3, atol=1e-3)


def test_quantised_q_exact_on_grid_values():
    """Q already on the FP4 grid: the call on its FP4 rows equals the bf16
    call (the rows hold exactly these values and every product is exact)."""
    kv, q, swa, idx = _case(2, 1, 1500, 512, 128, 0, 25)
    codes = np.random.default_rng(25).integers(0, 16, (2, 1, 64, 32, 16)).astype(np.uint8)
    codes[..., 5] = 7
    qg = torch.from_numpy((fp4.e2m1_value(codes) * 2.0 ** -6).reshape(2, 1, 64, 512).astype(np.float32)).to(torch.bfloat16)
    a, la = _run(kv, qg, swa, idx, 128, 0)
    b, lb = _run(kv, _q_rows_fp4(qg), swa, idx, 128, 0)
    np.testing.assert_allclose(b, a, rtol=0, atol=2e-3 * np.abs(a).max())
    np.testing.assert_allclose(lb, la, rtol=1e-5, atol=1e-5)
