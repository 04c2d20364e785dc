"""Pins for the oracle's group schedule (no GPU): the mode identities the
pages imply ([eogee] §3.2/§3.3): Reindex with the Full layer's own index-Q
selects the same entries; Reuse then equals that Reindex layer; a pool that
covers every block makes a pool-restricted Reindex equal a full one; new
entries are quantised into the cache before scoring."""

import numpy as np

from oracle import fp4, group


def _setup(seed, N=640, Q=2):
    rng = np.random.default_rng(seed)
    kv = fp4.quantize_kv_fp4(rng.normal(size=(N, 512)).astype(np.float32))
    kI = rng.normal(size=(N, 128))
    n_vis = np.array([N - 3, N][:Q])

    def layer(mode, qI=None, w=None):
        return dict(mode=mode,
                    qI=rng.normal(size=(Q, 32, 128)) if qI is None else qI,
                    w=rng.uniform(size=(Q, 32)) if w is None else w,
                    q=rng.normal(size=(Q, 64, 512)) * 0.05,
                    swa=rng.normal(size=(128, 512)))
    return kv, kI, n_vis, layer


def test_reindex_with_shared_index_q_equals_full_and_reuse_equals_it():
    kv, kI, n_vis, layer = _setup(0)
    L0 = layer(group.FULL)
    L1 = layer(group.REINDEX, qI=L0["qI"], w=L0["w"])
    L2 = layer(group.REUSE)
    L2["q"], L2["swa"] = L1["q"], L1["swa"]
    res = group.group_row(kv, kI, n_vis, [L0, L1, L2], K=64, W=128)
    np.testing.assert_array_equal(res[0]["idx"], res[1]["idx"])
    np.testing.assert_array_equal(res[1]["idx"], res[2]["idx"])
    np.testing.assert_array_equal(res[1]["o"], res[2]["o"])
    np.testing.assert_array_equal(res[1]["lse"], res[2]["lse"])


def test_reuse_takes_the_most_recent_indexing_layer():
    kv, kI, n_vis, layer = _setup(1)
    res = group.group_row(kv, kI, n_vis, [layer(group.FULL), layer(group.REINDEX), layer(group.REUSE)], K=32)
    np.testing.assert_array_equal(res[2]["idx"], res[1]["idx"])
    assert not np.array_equal(res[0]["idx"], res[1]["idx"])


def test_pool_covering_all_blocks_equals_full_reindex():
    kv, kI, n_vis, layer = _setup(2)
    L0 = layer(group.FULL)
    L1 = layer(group.REINDEX_POOL)
    L1b = dict(L1, mode=group.REINDEX)
    r_pool = group.group_row(kv.copy(), kI, n_vis, [L0, L1], K=48, hsi_blocks=80, hsi_block=8)
    r_full = group.group_row(kv.copy(), kI, n_vis, [L0, L1b], K=48)
    np.testing.assert_array_equal(r_pool[1]["idx"], r_full[1]["idx"])
    np.testing.assert_allclose(r_pool[1]["o"], r_full[1]["o"], rtol=1e-12)
    assert r_pool[0]["pool"].shape == (2, 80)


def test_new_entries_are_quantised_before_scoring():
    kv, kI, n_vis, layer = _setup(3)
    rng = np.random.default_rng(33)
    new = rng.normal(size=(2, 512)).astype(np.float32) * 50       # large values: attention must see them
    kv2 = kv.copy()
    res = group.group_row(kv2, kI, n_vis, [layer(group.FULL)], K=16, kv_new=new, new_rows=[7, 9])
    np.testing.assert_array_equal(kv2[[7, 9]], fp4.quantize_kv_fp4(new))
    assert res[0]["o"].shape == (2, 64, 512)


def test_topk_indices_valid_and_visible():
    kv, kI, n_vis, layer = _setup(4, N=300, Q=2)
    res = group.group_row(kv, kI, n_vis, [layer(group.FULL)], K=512)
    for i in range(2):
        idx = res[0]["idx"][i]
        vis = idx[idx >= 0]
        assert len(vis) == n_vis[i] and len(set(vis.tolist())) == n_vis[i]
        assert np.all(idx[n_vis[i]:] == -1)
        assert vis.max() < n_vis[i]



def test_window_rows_follow_the_query_position():
    """Zero query and all-zero main-KV entries: every key gets the same
    weight, so channel 0 of the output is sum(window row ids) / (K + W).
    Query i must see window rows [i*step, i*step + W)."""
    N, Q, K, W, step = 64, 3, 8, 5, 2
    kv = fp4.quantize_kv_fp4(np.zeros((N, 512), np.float32))
    kI = np.random.default_rng(0).normal(size=(N, 128))
    swa = np.zeros((W + (Q - 1) * step, 512))
    swa[:, 0] = np.arange(swa.shape[0])
    L = dict(mode=group.FULL, qI=np.ones((Q, 32, 128)), w=np.ones((Q, 32)),
             q=np.zeros((Q, 64, 512)), swa=swa)
    res = group.group_row(kv, kI, np.array([N] * Q), [L], K=K, W=W, swa_step=step)
    for i in range(Q):
        want = sum(range(i * step, i * step + W)) / (K + W)
        np.testing.assert_allclose(res[0]["o"][i][:, 0], want, rtol=1e-12)


def test_prefill_visibility_follows_token_coverage():
    """Causal prefill inputs: entry j covers tokens [j*r, (j+1)*r) and a query
    at token p sees it once all its tokens are at or before p; the visible
    count per query, counted entry by entry, matches the workload's n_vis,
    and the window of query i starts at row i (one new window row per token)."""
    from fp4_kv_cache_mxfp4_b200 import workloads
    for r, n_prefix, n_new in [(2, 40, 12), (1, 17, 5), (4, 9, 6)]:
        N = n_prefix + n_new
        Q = n_new * r
        wl = workloads.Workload("t", 0, B=1, Q=Q, N=N, r=r, modes=[0], n_new=n_new, prefill=True, swa_step=1)
        p0 = n_prefix * r                             # first query's token
        for i in range(Q):
            p = p0 + i
            visible = sum(1 for j in range(N) if (j + 1) * r <= p + 1)
            assert wl.n_vis[i] == visible, (r, i)
        assert wl.n_vis[-1] == N                      # the last query sees every entry
        assert wl.swa_rows == wl.W + Q - 1


def test_pool_handed_to_a_later_group_equals_the_pool_built_in_the_group():
    """Decoder schedule: the pool of group 1's Full layer serves the Reindex
    layer heading group 2.  Running [Full, pool-Reindex, Reuse] as one group
    or as [Full] then [pool-Reindex, Reuse] with the pool handed over gives
    the same indices and outputs."""
    kv, kI, n_vis, layer = _setup(5)
    L0, L1, L2 = layer(group.FULL), layer(group.REINDEX_POOL), layer(group.REUSE)
    one = group.group_row(kv.copy(), kI, n_vis, [L0, L1, L2], K=40, hsi_blocks=24, hsi_block=8)
    first = group.group_row(kv.copy(), kI, n_vis, [L0], K=40, hsi_blocks=24, hsi_block=8)
    second = group.group_row(kv.copy(), kI, n_vis, [L1, L2], K=40, hsi_blocks=24, hsi_block=8,
                             pool_in=first[0]["pool"])
    np.testing.assert_array_equal(one[0]["pool"], first[0]["pool"])
    for a, b in ((one[1], second[0]), (one[2], second[1])):
        np.testing.assert_array_equal(a["idx"], b["idx"])
        np.testing.assert_array_equal(a["o"], b["o"])
    # the pool restricts the search: 24 blocks of 8 cannot hold every top-40
    # position of a fresh index-Q over 640 entries
    assert np.all(second[0]["idx"] >= 0)
    for i in range(2):
        blocks = set((second[0]["idx"][i] // 8).tolist())
        assert blocks <= set(first[0]["pool"][i].tolist())


def test_pool_reindex_without_any_pool_is_refused():
    kv, kI, n_vis, layer = _setup(6)
    try:
        group.group_row(kv, kI, n_vis, [layer(group.REINDEX_POOL)], K=8, hsi_blocks=4)
    except AssertionError:
        return
    raise AssertionError("a pool-restricted Reindex ran without a pool")


def test_stack_row_hands_the_decoder_pool_forward_and_keeps_encoder_caches_apart():
    """stack_row: decoder groups share one cache and the Full layer's pool
    reaches the later groups' Reindex layers; encoder groups each read their
    own cache (a group's attention sees only its own entries)."""
    kv, kI, n_vis, layer = _setup(7)
    g1 = dict(kv_fp4=kv, kI=kI, n_vis=n_vis, layers=[layer(group.FULL), layer(group.REUSE)])
    g2 = dict(kv_fp4=kv, kI=kI, n_vis=n_vis, layers=[layer(group.REINDEX_POOL), layer(group.REUSE)])
    g3 = dict(kv_fp4=kv, kI=kI, n_vis=n_vis, layers=[layer(group.REINDEX_POOL), layer(group.REUSE)])
    res = group.stack_row([g1, g2, g3], hsi_blocks=16, hsi_block=8, K=32)
    pool = res[0][0]["pool"]
    for gi in (1, 2):
        for i in range(2):
            assert set((res[gi][0]["idx"][i] // 8).tolist()) <= set(pool[i].tolist())
        np.testing.assert_array_equal(res[gi][1]["idx"], res[gi][0]["idx"])
    # encoder: two groups with their own caches; a zero cache gives outputs
    # that only the window explains
    kv_zero = fp4.quantize_kv_fp4(np.zeros((640, 512), np.float32))
    e1 = dict(kv_fp4=kv, kI=kI, n_vis=n_vis, layers=[layer(group.FULL), layer(group.REUSE)])
    L = layer(group.FULL)
    L["swa"] = np.zeros((128, 512))
    e2 = dict(kv_fp4=kv_zero, kI=kI, n_vis=n_vis, layers=[L])
    enc = group.stack_row([e1, e2], K=32)
    assert np.all(enc[1][0]["o"] == 0) and not np.all(enc[0][0]["o"] == 0)

