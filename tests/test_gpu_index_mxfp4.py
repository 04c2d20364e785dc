"""GPU parity of the MXFP4 index-K path ("DeepSeek V4.1-Flash 技术报告深度解析"
§3.4: FP4 indexer K in the OCP MXFP4 family; 68-byte entries):

* csa2_quantize_index_k_mxfp4: entries bit-exact against oracle.mxfp4;
* csa2_index_score_topk on those entries (oracle-made bytes): the top-K under
  the band rule of tests/parity.py against the oracle's scores on the
  dequantised index-K and the MXFP4-quantised index-Q (the page's FP4
  indexer Q and K), in Full scans (one to many queries, ragged tails, fewer
  visible entries than K), with the HSI pool, and pool re-scores.
"""

import numpy as np
import pytest
import torch

from fp4_kv_cache_mxfp4_b200 import csa2
from oracle import indexer, mxfp4
from parity import check_topk, f32

pytestmark = pytest.mark.gpu


def test_index_k_quantiser_bit_exact():
    g = torch.Generator().manual_seed(1)
    x = torch.randn(5000, 4, 32, generator=g) * torch.exp2(torch.randint(-60, 60, (5000, 4, 1), generator=g).float())
    x[::7, 2] = 0.0
    x[1::7, 1, ::3] = -0.0
    x = x.reshape(5000, 128).to(torch.bfloat16)
    # golden-like rows: ties and saturation at e = 0
    x[0, :6] = torch.tensor([6.0, -3.0, 1.25, 0.1, 5.0, 7.0]).to(torch.bfloat16)
    out = torch.full((5100, 68), 0xAA, dtype=torch.uint8, device="cuda")
    csa2.csa2_quantize_index_k_mxfp4(x.cuda(), out, row_offset=64)
    dst = torch.tensor([5099, 3, 5098], dtype=torch.int64, device="cuda")
    csa2.csa2_quantize_index_k_mxfp4(x[:3].cuda(), out, dst_rows=dst)
    torch.cuda.synchronize()
    want = mxfp4.quantize_index_k_mxfp4(f32(x))
    got = out.cpu().numpy()
    np.testing.assert_array_equal(got[64:5064], want)
    np.testing.assert_array_equal(got[[5099, 3, 5098]], want[:3])
    assert np.all(got[:3] == 0xAA) and np.all(got[4:64] == 0xAA)


def _case(B, Q, N, seed):
    g = torch.Generator().manual_seed(seed)
    qI = torch.randn(B, Q, 32, 128, generator=g).to(torch.bfloat16)
    w = torch.rand(B, Q, 32, generator=g)
    kI = torch.randn(B, N, 128, generator=g).to(torch.bfloat16)
    k4 = np.stack([mxfp4.quantize_index_k_mxfp4(f32(kI[b])) for b in range(B)])
    kdeq = np.stack([mxfp4.dequantize_index_k_mxfp4(k4[b]) for b in range(B)])
    return qI, w, k4, kdeq


def _run(mode, qI, w, k4, n_vis, K, hsi_blocks=0, pool_in=None):
    B, Q = qI.shape[:2]
    d = "cuda"
    nv = torch.as_tensor(n_vis, dtype=torch.int32).reshape(B, Q).to(d)
    idx = torch.full((B, Q, K), -7, dtype=torch.int32, device=d)
    sc = torch.empty((B, Q, K), device=d)
    pool_out = torch.full((B, Q, hsi_blocks), -7, dtype=torch.int32, device=d) if (hsi_blocks and mode == 0) else None
    pin = None if pool_in is None else torch.as_tensor(pool_in, dtype=torch.int32).to(d)
    a = csa2.index_args(mode, qI.to(d), w.to(d), torch.from_numpy(k4).to(d), nv, idx, sc, hsi_blocks=hsi_blocks,
                        hsi_block=8, pool_out=pool_out, pool_in=pin)
    csa2.csa2_index_score_topk(a, csa2.workspace(a, csa2.WS_INDEX))
    torch.cuda.synchronize()
    assert csa2.csa2_device_status() == (0, 0)
    return idx.cpu().numpy(), sc.cpu().numpy(), None if pool_out is None else pool_out.cpu().numpy()


@pytest.mark.parametrize("B,Q,N,seed,vis", [
    (4, 1, 20000, 1, "all"),        # decode, ragged last tile (20000 = 156 tiles + 32 rows)
    (2, 2, 6000, 2, "ragged"),      # two queries per MMA group, per-query visibility
    (1, 8, 3000, 3, "ragged"),      # eight queries per MMA group (sampled histogram)
    (1, 5, 1500, 4, "causal"),      # a verify block of 5 queries
    (2, 1, 400, 5, "few"),          # fewer visible entries than K
])
def test_scan_topk_against_dequantised_oracle(B, Q, N, seed, vis):
    qI, w, k4, kdeq = _case(B, Q, N, seed)
    rng = np.random.default_rng(seed)
    if vis == "all":
        n_vis = np.full((B, Q), N)
    elif vis == "ragged":
        n_vis = rng.integers(N // 2, N + 1, (B, Q))
    elif vis == "causal":
        n_vis = np.array([[N - Q + 1 + i for i in range(Q)]] * B)
    else:
        n_vis = np.array([[300], [0]])
    K = 512
    idx, sc, _ = _run(0, qI, w, k4, n_vis, K)
    for b in range(B):
        for q in range(Q):
            s = indexer.index_scores(mxfp4.fake_quantize(f32(qI[b, q])), f32(w[b, q]), kdeq[b], int(n_vis[b, q]))
            sel = check_topk(idx[b, q], s, K, what=f"b{b} q{q}")
            assert np.all(np.diff(sel) > 0)
            np.testing.assert_allclose(sc[b, q, :len(sel)], s[sel], rtol=2e-3, atol=2e-3)


def test_hsi_pool_and_pool_rescore():
    B, Q, N = 2, 1, 8 * 3000
    qI, w, k4, kdeq = _case(B, Q, N, 6)
    qI2 = torch.randn(B, Q, 32, 128, generator=torch.Generator().manual_seed(66)).to(torch.bfloat16)
    n_vis = np.array([[N], [N - 13]])
    idx, _, pool = _run(0, qI, w, k4, n_vis, 512, hsi_blocks=400)
    for b in range(B):
        s = indexer.index_scores(mxfp4.fake_quantize(f32(qI[b, 0])), f32(w[b, 0]), kdeq[b], int(n_vis[b, 0]))
        check_topk(idx[b, 0], s, 512, what=f"full b{b}")
        bs = indexer.block_scores(s, 8)
        v = pool[b, 0][pool[b, 0] >= 0]
        assert np.all(np.diff(v) > 0)
        check_topk(np.concatenate([v[np.argsort(-bs[v], kind="stable")], pool[b, 0][pool[b, 0] < 0]]), bs, 400,
                   what=f"pool b{b}")
    idx2, _, _ = _run(2, qI2, w, k4, n_vis, 300, hsi_blocks=400, pool_in=pool)
    for b in range(B):
        pos, ps = indexer.pool_scores(mxfp4.fake_quantize(f32(qI2[b, 0])), f32(w[b, 0]), kdeq[b], pool[b, 0],
                                      int(n_vis[b, 0]))
        check_topk(idx2[b, 0], ps, 300, positions=pos, what=f"pool rescore b{b}")


def test_n_not_a_multiple_of_four_is_refused():
    qI, w, k4, _ = _case(1, 1, 1000, 7)
    with pytest.raises(csa2.Csa2Error) as e:
        _run(0, qI, w, np.ascontiguousarray(k4[:, :999]), np.array([[999]]), 64)
    assert e.value.status == 2


def test_scores_exact_on_grid_values():
    """Index-Q and index-K already on their MXFP4 grids with small exponents:
    every product and partial sum is exact in f32, so the scores the kernel
    returns equal the oracle's float64 scores exactly, and the selection is
    compared index for index (ties to the lower position)."""
    B, Q, N, K = 1, 2, 4000, 256
    rng = np.random.default_rng(12)
    kc = rng.integers(0, 16, (N, 128)).astype(np.uint8)
    qc = rng.integers(0, 16, (B, Q, 32, 128)).astype(np.uint8)
    kx = mxfp4.e2m1_value(kc) * 0.5
    qx = mxfp4.e2m1_value(qc) * 0.25
    k4 = mxfp4.quantize_index_k_mxfp4(kx.astype(np.float32))[None]
    kdeq = mxfp4.dequantize_index_k_mxfp4(k4[0])
    qI = torch.from_numpy(qx.astype(np.float32)).to(torch.bfloat16)
    w = torch.from_numpy(rng.integers(0, 4, (B, Q, 32)).astype(np.float32))
    n_vis = np.array([[N, N - 777]])
    idx, sc, _ = _run(0, qI, w, k4, n_vis, K)
    for q in range(Q):
        s = indexer.index_scores(mxfp4.fake_quantize(f32(qI[0, q])), f32(w[0, q]), kdeq, int(n_vis[0, q]))
        want, _ = indexer.topk(s, K)
        np.testing.assert_array_equal(np.sort(idx[0, q]), np.sort(want))
        np.testing.assert_array_equal(sc[0, q][np.argsort(idx[0, q])], s[np.sort(want)])
