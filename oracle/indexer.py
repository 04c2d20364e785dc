"""Oracle: lightweight-indexer scoring, top-K selection, Hierarchical Sparse
Indexer (HSI) candidate pool.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

Sources:
* [eogee] §3.2: CSA2 keeps a lightweight indexer; index-Q and index-K score
  the main-KV entries, each query keeps its top-K entries (K = 512) and the
  indexer has 32 heads of dimension 128.  Full mode scores all visible
  entries; Reindex re-scores the shared index-K with the layer's own index-Q;
  Reuse consumes the earlier layer's top-K ([opskyn] "HBM 与 SSD，分别怎么省？",
  [titansim] "核心机制与研究方法" mode list).
* [eogee] §3.3 and [titansim] Figure 5: the first Full layer of the decoder
  also takes, for each block of 8 positions, the highest index score in the
  block, keeps the 2048 best blocks (a 16,384-position shared pool) and the
  later Reindex layers score only that pool.  [nxbn] §3.3 table:
  candidate_topk_blocks 2048, candidate_block_size 8, index_topk 512,
  index_n_heads 32, index_head_dim 128.

The pages print no score formula.  The definition implemented here is
    s[q, t] = sum_h w[q, h] * ReLU( sum_d qI[q, h, d] * kI[t, d] )
with per-query head weights w and no 1/sqrt(d) factor.  Ties in top-K go to
the lower position, ties between blocks to the lower block id; positions
t >= n_vis (not yet visible to the query) never score.  When fewer than K
positions are visible the result is padded with -1.

All scores are float64 (inputs are bf16 values held in float32/float64).
Parity: pinned (tests/test_oracle_indexer.py) against brute-force subset
search on tiny inputs, closed forms and mode identities.
"""

import numpy as np

H_I = 32          # indexer heads,     [nxbn] §3.3 index_n_heads
D_I = 128         # indexer head dim,  [nxbn] §3.3 index_head_dim
TOPK = 512        # [eogee] §3.2, [nxbn] §3.3 index_topk
HSI_BLOCK = 8     # [eogee] §3.3, [nxbn] §3.3 candidate_block_size
HSI_BLOCKS = 2048 # [eogee] §3.3, [nxbn] §3.3 candidate_topk_blocks


def index_scores(qI, w, kI, n_vis):
    """Scores of one query against the first n_vis index-K rows.

    qI [32, 128], w [32], kI [N, 128]; returns float64 [N] with -inf at
    t >= n_vis.
    """
    qI = np.asarray(qI, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    kI = np.asarray(kI, dtype=np.float64)
    N = kI.shape[0]
    n_vis = int(min(max(n_vis, 0), N))
    logits = kI[:n_vis] @ qI.T                      # [n_vis, 32]: q_h . k_t
    s = np.maximum(logits, 0.0) @ w                 # sum_h w_h ReLU(.)
    out = np.full(N, -np.inf)
    out[:n_vis] = s
    return out


def topk(scores, K, positions=None):
    """The K best entries of ``scores`` (1-D), best first.

    Order: larger score first, then lower position.  ``positions`` gives
    the position of each score (default: its index); only finite scores are
    eligible; the result is padded with -1 to length K.
    Returns (positions int64 [K], scores float64 [K] with -inf padding).
    """
    s = np.asarray(scores, dtype=np.float64)
    pos = np.arange(s.shape[0]) if positions is None else np.asarray(positions)
    ok = np.isfinite(s)
    s, pos = s[ok], pos[ok]
    order = np.lexsort((pos, -s))            # primary key -s, secondary pos
    take = order[:K]
    out_pos = np.full(K, -1, dtype=np.int64)
    out_s = np.full(K, -np.inf)
    out_pos[:take.shape[0]] = pos[take]
    out_s[:take.shape[0]] = s[take]
    return out_pos, out_s


def block_scores(scores, block=HSI_BLOCK):
    """HSI block score: max of the visible scores inside each block of
    ``block`` consecutive positions; a block with no visible position gets
    -inf (never selected)."""
    s = np.asarray(scores, dtype=np.float64)
    nb = -(-s.shape[0] // block)
    padded = np.full(nb * block, -np.inf)
    padded[:s.shape[0]] = s
    return padded.reshape(nb, block).max(axis=1)


def hsi_select_blocks(scores, n_blocks=HSI_BLOCKS, block=HSI_BLOCK):
    """Blocks kept for the shared candidate pool, as ascending block ids
    padded with -1 to ``n_blocks``; plus the kept blocks' scores in the
    same order."""
    bs = block_scores(scores, block)
    ids, _ = topk(bs, n_blocks)
    kept = np.sort(ids[ids >= 0])
    out = np.full(n_blocks, -1, dtype=np.int64)
    out[:kept.shape[0]] = kept
    sc = np.full(n_blocks, -np.inf)
    sc[:kept.shape[0]] = bs[kept]
    return out, sc


def pool_positions(block_ids, n_vis, block=HSI_BLOCK):
    """Visible positions covered by the pool blocks, in pool order."""
    b = np.asarray(block_ids)
    b = b[b >= 0]
    pos = (b[:, None] * block + np.arange(block)[None, :]).reshape(-1)
    return pos[pos < n_vis]


def pool_scores(qI, w, kI, block_ids, n_vis, block=HSI_BLOCK):
    """Reindex restricted to the pool: (positions, scores) of the visible
    pool positions, scored with this layer's own qI and w."""
    pos = pool_positions(block_ids, n_vis, block)
    qI = np.asarray(qI, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    k = np.asarray(kI, dtype=np.float64)[pos]
    s = np.maximum(k @ qI.T, 0.0) @ w
    return pos, s
