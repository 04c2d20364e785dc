"""Oracle: one CSA2 sharing group run layer by layer for one batch row.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

Sources: [eogee] §3.2 (Full / Reindex / Reuse static modes; layers of a
group share one main KV and one index-K; Reindex re-scores the shared keys
with its own index-Q; Reuse consumes the top-K of the previous indexing
layer and skips the indexer), [eogee] §3.3 (Reindex layers after the first
Full layer of the decoder score only the HSI pool), [eogee] §3.4 (new
entries are quantised after RoPE, before they join the cache).

Readings: Reuse takes the indices of the most recent indexing layer
([titansim] "核心机制与研究方法" describes Reuse as taking the previous
layer's already-selected indices);
REINDEX_POOL uses the pool built by the most recent Full layer, which may
sit in an earlier group: [eogee] §3.3 has the decoder's first Full layer
build the pool that every later Reindex layer re-scores, and the §3.2
configuration paragraph puts those Reindex layers at the head of decoder
groups 2..5 (each Reindex + 3 Reuse; group 1 is Full + 3 Reuse; the encoder
is 3 groups of Full + 5 Reuse at r=2).  The layers run strictly in order;
each layer's inputs are given.

Parity: pinned through the mode identities in tests/test_oracle_group.py,
including "a pool handed to a later group = the pool built in the same
group".
"""

import numpy as np

from . import fp4, indexer, attention

FULL, REINDEX, REINDEX_POOL, REUSE = 0, 1, 2, 3


def group_row(kv_fp4, kI, n_vis, layers, K=indexer.TOPK, W=attention.WIN,
              swa_step=0, hsi_blocks=0, hsi_block=indexer.HSI_BLOCK,
              kv_new=None, new_rows=None, scale=None, pool_in=None):
    """Run a group for one batch row.

    kv_fp4   uint8 [N, 288] packed cache (modified in place by kv_new)
    kI       [N, 128] index-K
    n_vis    [Q] visible entries per query position
    layers   list of dicts: mode, and qI [Q,32,128], w [Q,32] for indexing
             modes, q [Q,64,512], swa [rows,512] for every layer
    swa_step query position i sees window rows [i*swa_step, i*swa_step+W)
    hsi_blocks  0 = no pool; else a FULL layer also builds the pool
    kv_new   [n_new, 512] new entries quantised into rows new_rows first
    pool_in  [Q, hsi_blocks] pool built by an earlier group, used by
             REINDEX_POOL layers until a FULL layer here builds its own
    Returns a list of per-layer dicts: idx [Q,K], o [Q,64,512], lse [Q,64],
    and pool [Q,hsi_blocks] for a FULL layer that built one.
    """
    if kv_new is not None:
        kv_fp4[np.asarray(new_rows)] = fp4.quantize_kv_fp4(kv_new)
    n_vis = np.asarray(n_vis)
    Q = n_vis.shape[0]
    results = []
    last_idx = None
    last_pool = None if pool_in is None else np.asarray(pool_in)
    for L in layers:
        mode = L["mode"]
        res = {}
        if mode in (FULL, REINDEX):
            idx = np.full((Q, K), -1, dtype=np.int64)
            pool = np.full((Q, max(hsi_blocks, 1)), -1, dtype=np.int64)
            for i in range(Q):
                s = indexer.index_scores(L["qI"][i], L["w"][i], kI, n_vis[i])
                idx[i], _ = indexer.topk(s, K)
                if mode == FULL and hsi_blocks:
                    pool[i], _ = indexer.hsi_select_blocks(s, hsi_blocks, hsi_block)
            if mode == FULL and hsi_blocks:
                res["pool"] = pool
                last_pool = pool
            last_idx = idx
        elif mode == REINDEX_POOL:
            assert last_pool is not None, "REINDEX_POOL needs an earlier FULL layer with a pool"
            idx = np.full((Q, K), -1, dtype=np.int64)
            for i in range(Q):
                pos, s = indexer.pool_scores(L["qI"][i], L["w"][i], kI, last_pool[i], n_vis[i], hsi_block)
                idx[i], _ = indexer.topk(s, K, positions=pos)
            last_idx = idx
        elif mode == REUSE:
            assert last_idx is not None, "REUSE needs an earlier indexing layer"
            idx = last_idx
        else:
            raise ValueError(mode)
        o = np.zeros((Q, attention.H, attention.D))
        lse = np.zeros((Q, attention.H))
        swa = np.asarray(L["swa"], dtype=np.float64)
        for i in range(Q):
            rows = swa[i * swa_step: i * swa_step + W]
            # attention reads only the selected entries: dequantise those
            sel = idx[i][idx[i] >= 0]
            deq = fp4.dequantize_kv_fp4(kv_fp4[sel])
            o[i], lse[i] = attention.sparse_mqa(L["q"][i], deq, np.arange(sel.shape[0]), rows, scale)
        res.update(idx=idx, o=o, lse=lse)
        results.append(res)
    return results


def stack_row(groups, hsi_blocks=0, hsi_block=indexer.HSI_BLOCK, **kw):
    """Several groups of one batch row, run in order ([eogee] §3.2
    configuration paragraph).  ``groups`` is a list of dicts with the
    group_row arguments kv_fp4, kI, n_vis, layers (and optionally kv_new,
    new_rows): groups may share one cache (the decoder) or each hold their
    own (the encoder).  The most recent pool built by any group's Full
    layer is handed to the next groups (the decoder's first Full layer
    builds the pool every later Reindex layer re-scores, [eogee] §3.3).
    Returns the per-group lists of group_row."""
    out = []
    pool = None
    for G in groups:
        res = group_row(G["kv_fp4"], G["kI"], G["n_vis"], G["layers"], hsi_blocks=hsi_blocks,
                        hsi_block=hsi_block, kv_new=G.get("kv_new"), new_rows=G.get("new_rows"),
                        pool_in=pool, **kw)
        for r in res:
            if "pool" in r:
                pool = r["pool"]
        out.append(res)
    return out
