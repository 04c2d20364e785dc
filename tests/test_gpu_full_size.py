"""GPU parity at the full workload sizes, in the launch configuration the
bench times (one csa2_group_decode call over a workload staged by
fp4_kv_cache_mxfp4_b200.device_workload), checked on sampled outputs the
oracle computes one by one:

* FP4 bytes of every new entry and of sampled older entries: bit-exact;
* per indexing layer and sampled (row, query): the top-K under the band
  rule (and the HSI block pool, when the schedule has one);
* per layer and sampled (row, query): the attention output and its
  log-sum-exp against the float64 oracle on the GPU's (validated) indices.
"""

import numpy as np
import pytest
import torch

from fp4_kv_cache_mxfp4_b200 import csa2, workloads
from fp4_kv_cache_mxfp4_b200.device_workload import make_device_workload, run_step
from oracle import attention, fp4, fp8, indexer, mxfp4
from parity import check_attention, check_topk, f32

pytestmark = pytest.mark.gpu


def _samples(wl):
    """(b, q) pairs checked against the oracle."""
    if wl.Q == 1:
        return [(b, 0) for b in range(wl.B)]
    rng = np.random.default_rng(wl.seed)
    qs = sorted({q for q in (0, 1, 7, 8, wl.Q // 2 - 1, wl.Q - 2, wl.Q - 1, *rng.integers(0, wl.Q, 3).tolist())
                 if 0 <= q < wl.Q})
    return [(b, q) for b in range(wl.B) for q in qs]


def _attn_oracle(kv_host_b, sel, q, win):
    """Attention over the selected entries without dequantising the whole
    cache: the selected rows are dequantised into a compact array."""
    valid = sel[sel >= 0]
    deq = fp4.dequantize_kv_fp4(kv_host_b[valid])
    local = np.full(sel.shape, -1, dtype=np.int64)
    local[sel >= 0] = np.arange(valid.shape[0])
    return attention.sparse_mqa(q, deq, local, win)


def _index_k_for_oracle(wl, cw, b):
    """The index-K the scores are defined on: the bf16 draws, or their MXFP4
    entries dequantised (the pages' FP4 index-K)."""
    k = f32(workloads.index_k(cw, b))
    if wl.index_k_format == 2:
        return mxfp4.dequantize_index_k_mxfp4(mxfp4.quantize_index_k_mxfp4(k))
    return k


def _index_q_for_oracle(wl, qI):
    """A query's index-Q as the scores see it: bf16, or MXFP4-quantised when
    index-K is MXFP4 (the page's FP4 indexer Q and K)."""
    q = f32(qI)
    return mxfp4.fake_quantize(q) if wl.index_k_format == 2 else q


def _window_for_oracle(wl, swa_b):
    """A layer's window rows of one batch row as the attention sees them."""
    x = f32(swa_b)
    if wl.window_format == 1:
        return fp8.dequantize_window_fp8(*fp8.quantize_window_fp8(x))
    return x


@pytest.mark.parametrize("w", [1, 2, 3, 4, 6, 7, 8], ids=lambda w: workloads.WORKLOADS[w].name)
def test_full_size_sampled(w):
    """One step of a full-size workload (a stack of groups for 6 and 7)
    through the library call the bench times."""
    wl = workloads.WORKLOADS[w]
    csa2.load()
    T = make_device_workload(wl, csa2)
    run_step(T, csa2)
    torch.cuda.synchronize()
    assert csa2.csa2_device_status() == (0, 0)
    B, N = wl.B, wl.N
    rng = np.random.default_rng(100 + w)
    n_caches = len(T["caches"])

    # FP4 bytes of every cache: every new entry, and 64 sampled older ones per row
    for c in range(n_caches):
        cw = wl.cache_of_group(c)
        kv = T["caches"][c]["kv"]
        for b in range(B):
            new_host = kv[b, N - wl.n_new:].cpu().numpy()
            want = fp4.quantize_kv_fp4(f32(workloads.main_kv_rows(cw, b, N - wl.n_new, wl.n_new)))
            np.testing.assert_array_equal(new_host, want, err_msg=f"new entries of cache {c} row {b}")
            for r in rng.integers(0, N - wl.n_new, 64).tolist():
                got = kv[b, r].cpu().numpy()
                np.testing.assert_array_equal(got, fp4.quantize_kv_fp4(f32(workloads.main_kv_rows(cw, b, r, 1)))[0],
                                              err_msg=f"entry {r} of cache {c} row {b}")

    # MXFP4 index-K entries: 64 sampled rows per cache row, bit-exact
    if wl.index_k_format == 2:
        for c in range(n_caches):
            cw = wl.cache_of_group(c)
            for b in range(B):
                rows = rng.integers(0, N, 64)
                want = mxfp4.quantize_index_k_mxfp4(f32(workloads.index_k(cw, b))[rows])
                np.testing.assert_array_equal(T["caches"][c]["kI"][b][torch.as_tensor(rows, device="cuda")].cpu().numpy(), want)

    samples = _samples(wl)
    kv_host = {(c, b): T["caches"][c]["kv"][b].cpu().numpy() for c in range(n_caches) for b in range(B)}
    n_vis = np.asarray(wl.n_vis)
    pool = None
    last_idx = None
    for g in range(len(wl.groups)):
        c = g if wl.cache_per_group else 0
        cw = wl.cache_of_group(c)
        G = T["groups"][g]
        if G["pool"] is not None:
            pool = G["pool"].cpu().numpy()
        for l in wl.group_layers(g):
            mode = wl.modes[l]
            li = workloads.layer_inputs(wl, l)
            L = T["layers"][l]
            if mode != workloads.REUSE:
                last_idx = L["idx"].cpu().numpy()
            for b in range(B):
                kI = _index_k_for_oracle(wl, cw, b) if mode != workloads.REUSE else None
                win_b = _window_for_oracle(wl, li["swa"][b])
                for (bb, q) in samples:
                    if bb != b:
                        continue
                    what = f"{wl.name} group {g} layer {l} b{b} q{q}"
                    nv = int(n_vis[q])
                    if mode in (workloads.FULL, workloads.REINDEX):
                        s = indexer.index_scores(_index_q_for_oracle(wl, li["qI"][b, q]), f32(li["w"][b, q]), kI, nv)
                        check_topk(last_idx[b, q], s, wl.K, what=what)
                        if mode == workloads.FULL and wl.hsi_blocks:
                            bs = indexer.block_scores(s, 8)
                            gp = pool[b, q]
                            v = gp[gp >= 0]
                            assert np.all(np.diff(v) > 0), f"{what}: pool not ascending"
                            check_topk(np.concatenate([v[np.argsort(-bs[v], kind="stable")], gp[gp < 0]]), bs,
                                       wl.hsi_blocks, what=what + " pool")
                    elif mode == workloads.REINDEX_POOL:
                        pos, ps = indexer.pool_scores(_index_q_for_oracle(wl, li["qI"][b, q]), f32(li["w"][b, q]), kI, pool[b, q], nv)
                        check_topk(last_idx[b, q], ps, wl.K, positions=pos, what=what)
                    win = win_b[q * wl.swa_step: q * wl.swa_step + wl.W]
                    o, lse = _attn_oracle(kv_host[(c, b)], last_idx[b, q], f32(li["q"][b, q]), win)
                    check_attention(L["out"][b, q], o, what=what)
                    np.testing.assert_allclose(L["lse"][b, q].cpu().numpy(), lse, rtol=1e-3, atol=1e-3)
