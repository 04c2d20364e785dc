"""Pins for the oracle's indexer, top-K and HSI pool (no GPU).

Pinned against closed forms of the score, brute-force subset search for
top-K (the unique set that beats every excluded element under the
(score, lower position) order), and the HSI identities stated on the pages
(a pool covering everything equals the full scan; the Full layer's own
top-K lies inside its pool).
"""

import itertools

import numpy as np
import pytest

from oracle import indexer


def _rng(s):
    return np.random.default_rng(s)


def test_score_closed_form_one_hot():
    """w = e_h and qI[h] = e_d give s_t = ReLU(kI[t, d]): no scale factor,
    ReLU applied, the right operand axes."""
    rng = _rng(0)
    kI = rng.normal(size=(50, 128))
    for h, d in [(0, 0), (5, 77), (31, 127)]:
        qI = np.zeros((32, 128)); qI[h, d] = 1.0
        w = np.zeros(32); w[h] = 1.0
        s = indexer.index_scores(qI, w, kI, 50)
        np.testing.assert_array_equal(s, np.maximum(kI[:, d], 0))


def test_score_relu_kills_negative_heads():
    rng = _rng(1)
    k = np.abs(rng.normal(size=(20, 128)))
    qI = -np.abs(rng.normal(size=(32, 128)))        # every q_h . k_t < 0
    w = rng.uniform(size=32)
    assert np.all(indexer.index_scores(qI, w, k, 20) == 0)


def test_score_linear_when_all_dots_positive():
    """With every q_h . k_t > 0 the ReLU is the identity, so
    s_t = (sum_h w_h q_h) . k_t."""
    rng = _rng(2)
    k = np.abs(rng.normal(size=(40, 128)))
    qI = np.abs(rng.normal(size=(32, 128)))
    w = rng.normal(size=32)                          # weights of either sign
    s = indexer.index_scores(qI, w, k, 40)
    np.testing.assert_allclose(s, k @ (w @ qI), rtol=1e-12)


def test_score_visibility():
    rng = _rng(3)
    k = rng.normal(size=(30, 128)); qI = rng.normal(size=(32, 128)); w = rng.uniform(size=32)
    s = indexer.index_scores(qI, w, k, 17)
    assert np.all(np.isfinite(s[:17])) and np.all(s[17:] == -np.inf)
    np.testing.assert_array_equal(s[:17], indexer.index_scores(qI, w, k[:17], 17))


def _brute_topk_set(s, K):
    """The unique K-subset S with: for i in S, j not in S, s_i > s_j or
    (s_i == s_j and i < j); found by trying every subset."""
    n = len(s)
    found = []
    for S in itertools.combinations(range(n), K):
        inS = set(S)
        ok = all((s[i] > s[j]) or (s[i] == s[j] and i < j)
                 for i in S for j in range(n) if j not in inS)
        if ok:
            found.append(S)
    assert len(found) == 1
    return set(found[0])


@pytest.mark.parametrize("seed", range(12))
def test_topk_against_brute_force_with_ties(seed):
    rng = _rng(100 + seed)
    n = int(rng.integers(5, 11))
    K = int(rng.integers(1, min(n, 5) + 1))
    s = rng.integers(0, 3, n).astype(np.float64)         # many ties
    pos, sc = indexer.topk(s, K)
    assert set(pos.tolist()) == _brute_topk_set(s, K)
    # best first: descending score, ascending position among equal scores
    keys = [(-s[p], p) for p in pos]
    assert keys == sorted(keys)
    np.testing.assert_array_equal(sc, s[pos])


def test_topk_pads_when_fewer_visible():
    s = np.array([3.0, -np.inf, 1.0, 2.0, -np.inf])
    pos, sc = indexer.topk(s, 5)
    assert pos.tolist() == [0, 3, 2, -1, -1]
    assert sc[3] == -np.inf and sc[4] == -np.inf


def test_topk_all_equal_takes_lowest_positions():
    pos, _ = indexer.topk(np.zeros(2048), 512)
    assert pos.tolist() == list(range(512))


def test_topk_with_explicit_positions():
    s = np.array([1.0, 5.0, 5.0, 2.0])
    pos, _ = indexer.topk(s, 2, positions=np.array([40, 90, 30, 10]))
    assert pos.tolist() == [30, 90]          # tie on 5.0 -> lower position 30 first


def test_topk_random_large_matches_sort():
    rng = _rng(7)
    s = rng.normal(size=2048)
    pos, _ = indexer.topk(s, 512)
    assert set(pos.tolist()) == set(np.argsort(-s, kind="stable")[:512].tolist())


def test_block_scores_planted():
    s = np.full(40, -np.inf)
    s[:34] = np.arange(34, dtype=np.float64) % 5      # 0 1 2 3 4 0 1 2 ...
    s[12] = 9.0
    bs = indexer.block_scores(s, 8)
    assert bs.tolist() == [4.0, 9.0, 4.0, 4.0, 3.0]   # block 4: only positions 32, 33 (2, 3) visible
    s2 = np.full(16, -np.inf); s2[:3] = 1.0
    assert indexer.block_scores(s2, 8).tolist() == [1.0, -np.inf]


def test_hsi_pool_covering_everything_equals_full_scan():
    """With blocks * 8 >= visible entries the pool is every block, so a pool
    re-score equals a full Reindex scan ([eogee] §3.3)."""
    rng = _rng(8)
    N, n_vis = 200, 187
    k = rng.normal(size=(N, 128)); qI = rng.normal(size=(32, 128)); w = rng.uniform(size=32)
    s = indexer.index_scores(qI, w, k, n_vis)
    blocks, _ = indexer.hsi_select_blocks(s, n_blocks=30, block=8)
    assert blocks[:24].tolist() == list(range(24)) and np.all(blocks[24:] == -1)
    pos, ps = indexer.pool_scores(qI, w, k, blocks, n_vis, 8)
    assert pos.tolist() == list(range(n_vis))
    np.testing.assert_allclose(ps, s[:n_vis], rtol=1e-13)
    p1, _ = indexer.topk(ps, 16, positions=pos)
    p2, _ = indexer.topk(s, 16)
    np.testing.assert_array_equal(p1, p2)


@pytest.mark.parametrize("seed", range(5))
def test_full_topk_lies_inside_its_pool(seed):
    """A block can outrank a block holding a top-K position only if it holds
    a top-K position itself, so the 2048-block pool contains the Full layer's
    top-512 whenever 512 <= 2048 (scores distinct)."""
    rng = _rng(20 + seed)
    N = 8 * 700
    k = rng.normal(size=(N, 128)); qI = rng.normal(size=(32, 128)); w = rng.uniform(size=32)
    s = indexer.index_scores(qI, w, k, N)
    top, _ = indexer.topk(s, 64)
    blocks, _ = indexer.hsi_select_blocks(s, n_blocks=256, block=8)
    pool = set(indexer.pool_positions(blocks, N, 8).tolist())
    assert set(top.tolist()) <= pool


def test_hsi_blocks_brute_force_tiny():
    rng = _rng(9)
    for _ in range(10):
        n = int(rng.integers(9, 40))
        s = rng.integers(0, 4, n).astype(np.float64)
        nb_keep = int(rng.integers(1, 4))
        blocks, bsc = indexer.hsi_select_blocks(s, n_blocks=nb_keep, block=4)
        nb = -(-n // 4)
        bmax = [max(s[4 * b: min(n, 4 * b + 4)]) for b in range(nb)]
        want = sorted(_brute_topk_set(np.array(bmax), min(nb_keep, nb)))
        assert blocks[blocks >= 0].tolist() == want
        assert bsc[:len(want)].tolist() == [bmax[b] for b in want]
