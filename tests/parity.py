"""Shared parity checks between the CUDA path and the oracle.

Tolerances (the workload specification's parity bar):
* FP4 bytes and scales: bit-exact.
* top-K: exact index sets, except inside a band of +-1e-3 relative around
  the oracle's K-th score; indices scoring above the band must be selected,
  selected indices must score at least the band's floor, sizes equal.
* attention: |gpu - oracle| <= 1e-2 + 1e-2 |oracle| against the float64
  oracle evaluated on the same index set.
"""

import numpy as np
import torch

TOPK_BAND = 1e-3
ATTN_ATOL = 1e-2
ATTN_RTOL = 1e-2


def check_topk(gpu_idx, scores, K, positions=None, band=TOPK_BAND, exact=False, what=""):
    """Set comparison (the order of gpu_idx is not checked here).
    gpu_idx: int array [K] from the CUDA path.  scores: oracle scores of
    the candidate slots (float64, -inf = not visible).  positions: position
    of each slot (default: slot index).  Returns the GPU's valid indices."""
    gpu_idx = np.asarray(gpu_idx).astype(np.int64)
    s = np.asarray(scores, dtype=np.float64)
    pos = np.arange(s.shape[0]) if positions is None else np.asarray(positions)
    ok = np.isfinite(s)
    s_vis, p_vis = s[ok], pos[ok]
    kk = min(K, s_vis.shape[0])
    assert np.all(gpu_idx[kk:] == -1), f"{what}: padding"
    sel = gpu_idx[:kk]
    assert np.all(sel >= 0), f"{what}: -1 inside the first {kk}"
    assert len(set(sel.tolist())) == kk, f"{what}: duplicate indices"
    score_of = dict(zip(p_vis.tolist(), s_vis.tolist()))
    assert all(p in score_of for p in sel.tolist()), f"{what}: index not visible / not a candidate"
    if kk == 0:
        return sel
    order = np.lexsort((p_vis, -s_vis))
    oracle = p_vis[order[:kk]]
    if exact:
        np.testing.assert_array_equal(np.sort(sel), np.sort(oracle), err_msg=f"{what}: exact top-K")
        return sel
    sK = s_vis[order[kk - 1]]
    lo, hi = sK - band * abs(sK), sK + band * abs(sK)
    must = set(p_vis[s_vis > hi].tolist())
    got = set(sel.tolist())
    assert must <= got, f"{what}: {len(must - got)} indices above the band missing"
    floor = np.array([score_of[p] for p in sel.tolist()])
    assert np.all(floor >= lo), f"{what}: selected index below the band"
    return sel


def check_attention(out_gpu, o_oracle, what=""):
    o = np.asarray(o_oracle, dtype=np.float64)
    g = out_gpu.float().cpu().numpy().astype(np.float64) if torch.is_tensor(out_gpu) else np.asarray(out_gpu)
    err = np.abs(g - o)
    tol = ATTN_ATOL + ATTN_RTOL * np.abs(o)
    bad = err > tol
    assert not bad.any(), f"{what}: {bad.sum()} of {bad.size} outside tolerance, max err {err.max():.3e}"
    return float(err.max())


def f32(t):
    """CPU float32 numpy copy of a tensor (bf16 values are exact in fp32)."""
    return t.detach().float().cpu().numpy()
