"""GPU parity of csa2_index_score_topk (Full, Reindex, HSI pool, pool
re-score) against the oracle, with the top-K band rule of tests/parity.py."""

import numpy as np
import pytest
import torch

from fp4_kv_cache_mxfp4_b200 import csa2
from oracle import indexer
from parity import check_topk, f32

pytestmark = pytest.mark.gpu


def _inputs(B, Q, N, seed, kind="normal"):
    g = torch.Generator().manual_seed(seed)
    if kind == "normal":
        qI = torch.randn(B, Q, 32, 128, generator=g)
        kI = torch.randn(B, N, 128, generator=g)
        w = torch.rand(B, Q, 32, generator=g)
    elif kind == "ints":        # small integers: every score exact in fp32, many ties
        qI = torch.randint(-1, 2, (B, Q, 32, 128), generator=g).float()
        kI = torch.randint(-1, 2, (B, N, 128), generator=g).float()
        w = torch.ones(B, Q, 32)
    elif kind == "zero":        # every score is 0
        qI = torch.zeros(B, Q, 32, 128)
        kI = torch.randn(B, N, 128, generator=g)
        w = torch.rand(B, Q, 32, generator=g)
    return qI.to(torch.bfloat16), w.float(), kI.to(torch.bfloat16)


def _run(mode, qI, w, kI, n_vis, K, hsi_blocks=0, pool_in=None, want_scores=True):
    B, Q = qI.shape[:2]
    d = "cuda"
    qI_d, w_d, kI_d = qI.to(d), w.to(d), kI.to(d)
    nv = torch.as_tensor(n_vis, dtype=torch.int32).reshape(B, Q).to(d)
    idx = torch.full((B, Q, K), -7, dtype=torch.int32, device=d)
    sc = torch.empty((B, Q, K), dtype=torch.float32, device=d) if want_scores else None
    pool_out = torch.full((B, Q, hsi_blocks), -7, dtype=torch.int32, device=d) if (hsi_blocks and mode == 0) else None
    pin = None if pool_in is None else torch.as_tensor(pool_in, dtype=torch.int32).to(d)
    a = csa2.index_args(mode, qI_d, w_d, kI_d, nv, idx, sc, hsi_blocks=hsi_blocks, hsi_block=8,
                        pool_out=pool_out, pool_in=pin)
    ws = csa2.workspace(a, csa2.WS_INDEX)
    csa2.csa2_index_score_topk(a, ws)
    torch.cuda.synchronize()
    assert csa2.csa2_device_status() == (0, 0)
    out = dict(idx=idx.cpu().numpy(), scores=None if sc is None else sc.cpu().numpy(),
               pool=None if pool_out is None else pool_out.cpu().numpy(), ws=ws)
    return out


def _oracle_scores(qI, w, kI, b, q, n_vis):
    return indexer.index_scores(f32(qI[b, q]), f32(w[b, q]), f32(kI[b]), n_vis)


@pytest.mark.parametrize("B,Q,N,seed", [(1, 4, 2048, 0), (3, 2, 1000, 1), (2, 1, 5000, 2), (1, 8, 777, 3),
                                         (1, 21, 3000, 4), (2, 13, 1500, 5)])
def test_full_scan_random(B, Q, N, seed):
    qI, w, kI = _inputs(B, Q, N, seed)
    rng = np.random.default_rng(seed)
    n_vis = rng.integers(0, N + 1, (B, Q))
    n_vis[0, 0] = N
    if B * Q > 2:
        n_vis.flat[1] = 0
        n_vis.flat[2] = 300                    # fewer than K visible: padded
    K = 512
    r = _run(0, qI, w, kI, n_vis, K)
    for b in range(B):
        for q in range(Q):
            s = _oracle_scores(qI, w, kI, b, q, int(n_vis[b, q]))
            sel = check_topk(r["idx"][b, q], s, K, what=f"b{b} q{q}")
            gs = r["scores"][b, q][:len(sel)]
            np.testing.assert_allclose(gs, s[sel], rtol=1e-4, atol=1e-3)
            assert np.all(np.isneginf(r["scores"][b, q][len(sel):]))
            assert np.all(np.diff(sel) > 0), "ascending position order"


def test_integer_scores_ties_exact():
    """Integer inputs make every fp32 score exact, so the tie-break to the
    lower position is compared index for index."""
    B, Q, N = 2, 3, 3000
    qI, w, kI = _inputs(B, Q, N, 11, kind="ints")
    n_vis = np.array([[3000, 2999, 1500], [129, 3000, 640]])
    for K in (1, 64, 512, 2048):
        r = _run(0, qI, w, kI, n_vis, K)
        for b in range(B):
            for q in range(Q):
                s = _oracle_scores(qI, w, kI, b, q, int(n_vis[b, q]))
                sel = check_topk(r["idx"][b, q], s, K, exact=True, what=f"K{K} b{b} q{q}")
                assert np.all(np.diff(sel) > 0)


def test_all_equal_scores_take_lowest_positions():
    # 40000 equal scores overflow the candidate list: the exact fallback runs
    B, Q, N = 1, 1, 40000
    qI, w, kI = _inputs(B, Q, N, 12, kind="zero")
    r = _run(0, qI, w, kI, [[N]], 512)
    np.testing.assert_array_equal(r["idx"][0, 0], np.arange(512))
    assert np.all(r["scores"][0, 0] == 0)


def test_many_ties_at_the_top():
    """2000 copies of one index-K row all tie for the top score: the tie
    break alone decides which 512 are taken (the lowest positions)."""
    B, Q, N = 1, 3, 9000
    qI, w, kI = _inputs(B, Q, N, 17)
    kI[0, 100:2100] = kI[0, 5000]
    qI[0, :, :, :] = kI[0, 5000].float().to(torch.bfloat16)      # the copied row scores highest
    r = _run(0, qI, w, kI, [[N, N, 2050]], 512)
    for q in range(Q):
        s = _oracle_scores(qI, w, kI, 0, q, [N, N, 2050][q])
        sel = check_topk(r["idx"][0, q], s, 512, exact=True, what=f"q{q}")
        assert np.all(np.diff(sel) > 0)
    np.testing.assert_array_equal(r["idx"][0, 0], np.arange(100, 612))


def test_reindex_equals_full_with_same_index_q():
    B, Q, N = 2, 1, 4096
    qI, w, kI = _inputs(B, Q, N, 13)
    r0 = _run(0, qI, w, kI, [[N], [N]], 512)
    r1 = _run(1, qI, w, kI, [[N], [N]], 512)
    np.testing.assert_array_equal(r0["idx"], r1["idx"])


def test_workspace_contents_do_not_matter():
    """The call clears what it needs: a reused workspace full of garbage
    gives the same answer."""
    B, Q, N = 2, 2, 3000
    qI, w, kI = _inputs(B, Q, N, 14)
    r = _run(0, qI, w, kI, [[N, N], [N, 17]], 256)
    ws = r["ws"]
    ws.fill_(0xAB)
    a_idx = torch.full((B, Q, 256), -7, dtype=torch.int32, device="cuda")
    a = csa2.index_args(0, qI.cuda(), w.cuda(), kI.cuda(),
                        torch.tensor([[N, N], [N, 17]], dtype=torch.int32, device="cuda"), a_idx)
    csa2.csa2_index_score_topk(a, ws)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(a_idx.cpu().numpy(), r["idx"])


def test_hsi_pool_and_pool_rescore():
    B, Q, N = 2, 1, 8 * 3000 + 5
    qI, w, kI = _inputs(B, Q, N, 15)
    n_vis = np.array([[N], [N - 1000]])
    nb = 2048
    r = _run(0, qI, w, kI, n_vis, 512, hsi_blocks=nb)
    pools = []
    for b in range(B):
        s = _oracle_scores(qI, w, kI, b, 0, int(n_vis[b, 0]))
        check_topk(r["idx"][b, 0], s, 512, what=f"pos b{b}")
        bs = indexer.block_scores(s, 8)
        pool = r["pool"][b, 0]
        valid = pool[pool >= 0]
        assert np.all(np.diff(valid) > 0), "pool must be ascending"
        # pool = top-2048 blocks under the band rule (ascending output order)
        best_first = valid[np.argsort(-bs[valid], kind="stable")]
        check_topk(np.concatenate([best_first, pool[pool < 0]]), bs, nb, what=f"blocks b{b}")
        pools.append(indexer.hsi_select_blocks(s, nb, 8)[0])     # oracle pool feeds the re-score
    # pool-restricted re-score with a fresh index-Q, fed the oracle's pool
    qI2, w2, _ = _inputs(B, Q, N, 16)
    pool_in = np.stack(pools)[:, None, :]
    r2 = _run(2, qI2, w2, kI, n_vis, 512, hsi_blocks=nb, pool_in=pool_in)
    for b in range(B):
        pos, ps = indexer.pool_scores(f32(qI2[b, 0]), f32(w2[b, 0]), f32(kI[b]), pool_in[b, 0], int(n_vis[b, 0]))
        check_topk(r2["idx"][b, 0], ps, 512, positions=pos, what=f"pool b{b}")


@pytest.mark.parametrize("Q", [2, 4, 5, 8])
def test_hsi_pool_with_query_blocks(Q):
    """Full scan with the HSI pool for several causal queries per MMA group
    (2, 4 and 8-query kernels; 5 is a verify block in the 8-query kernel):
    every query gets its own top-K and its own pool."""
    B, N = 2, 8 * 900 + 3
    qI, w, kI = _inputs(B, Q, N, 40 + Q)
    n_vis = np.array([[N - Q + 1 + i for i in range(Q)], [N - 700 + i for i in range(Q)]])
    nb = 300
    r = _run(0, qI, w, kI, n_vis, 512, hsi_blocks=nb)
    for b in range(B):
        for q in range(Q):
            s = _oracle_scores(qI, w, kI, b, q, int(n_vis[b, q]))
            check_topk(r["idx"][b, q], s, 512, what=f"pos b{b} q{q}")
            bs = indexer.block_scores(s, 8)
            pool = r["pool"][b, q]
            valid = pool[pool >= 0]
            assert len(valid) == nb and np.all(np.diff(valid) > 0), f"pool b{b} q{q}"
            check_topk(np.concatenate([valid[np.argsort(-bs[valid], kind="stable")], pool[pool < 0]]), bs, nb,
                       what=f"blocks b{b} q{q}")


def test_pool_with_padding_and_invisible_tail():
    B, Q, N = 1, 2, 4000
    qI, w, kI = _inputs(B, Q, N, 17)
    rng = np.random.default_rng(17)
    pool = np.full((1, 2, 100), -1, dtype=np.int32)
    pool[0, 0, :90] = np.sort(rng.choice(500, 90, replace=False))
    pool[0, 1, :100] = np.sort(rng.choice(500, 100, replace=False))
    n_vis = np.array([[4000, 2000]])
    r = _run(2, qI, w, kI, n_vis, 512, hsi_blocks=100, pool_in=pool)
    for q in range(2):
        pos, ps = indexer.pool_scores(f32(qI[0, q]), f32(w[0, q]), f32(kI[0]), pool[0, q], int(n_vis[0, q]))
        check_topk(r["idx"][0, q], ps, 512, positions=pos, what=f"q{q}")
