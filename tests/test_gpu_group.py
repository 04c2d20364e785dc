"""GPU parity of csa2_group_decode (quantise the step's entries, then the
layers in order) against the oracle on small versions of each schedule."""

import numpy as np
import pytest
import torch

from fp4_kv_cache_mxfp4_b200 import csa2, workloads
from oracle import attention, fp4, indexer
from parity import check_attention, check_topk, f32

pytestmark = pytest.mark.gpu


def _make(wl):
    """Device inputs of a workload plus host copies for the oracle."""
    d = "cuda"
    B, N = wl.B, wl.N
    kv = torch.zeros(B, N, 288, dtype=torch.uint8, device=d)
    x_all = []
    for b in range(B):
        x = workloads.main_kv_rows(wl, b, 0, N)
        x_all.append(x)
        csa2.csa2_quantize_kv_fp4(x[: N - wl.n_new].to(d), kv[b])       # the cache before this step
    kI = torch.stack([workloads.index_k(wl, b) for b in range(B)])
    new = torch.cat([x[N - wl.n_new:] for x in x_all]).to(d)
    new_rows = torch.tensor([b * N + r for b in range(B) for r in wl.new_rows], dtype=torch.int64, device=d)
    layers = [workloads.layer_inputs(wl, l) for l in range(len(wl.modes))]
    return dict(kv=kv, kI=kI, kI_d=kI.to(d), x=x_all, new=new, new_rows=new_rows, layers=layers,
                n_vis=workloads.n_vis_tensor(wl))


def _run_group(wl, T):
    d = "cuda"
    B, Q, K = wl.B, wl.Q, wl.K
    Ls = []
    for l, mode in enumerate(wl.modes):
        li = T["layers"][l]
        Ls.append(dict(mode=mode, qI=li["qI"].to(d), w=li["w"].to(d), q=li["q"].to(d), swa=li["swa"].to(d),
                       out=torch.empty(B, Q, 64, 512, dtype=torch.bfloat16, device=d),
                       lse=torch.empty(B, Q, 64, device=d),
                       idx=torch.full((B, Q, K), -7, dtype=torch.int32, device=d) if mode != 3 else None))
    pool = torch.full((B, Q, wl.hsi_blocks), -7, dtype=torch.int32, device=d) if wl.hsi_blocks else None
    g = csa2.group_args(B, Q, K, wl.W, wl.N, T["n_vis"].to(d), T["kI_d"], T["kv"], Ls, kv_new=T["new"],
                        new_rows=T["new_rows"], swa_rows=wl.swa_rows, swa_step=wl.swa_step,
                        hsi_blocks=wl.hsi_blocks, hsi_block=wl.hsi_block, pool=pool)
    ws = csa2.workspace(g, csa2.WS_GROUP)
    csa2.csa2_group_decode(g, ws)
    torch.cuda.synchronize()
    assert csa2.csa2_device_status() == (0, 0)
    return Ls, pool


def _check(wl, T, Ls, pool):
    """Oracle, step by step: quantised bytes of the new rows, per layer the
    top-K under the band rule, attention on the GPU's (validated) indices."""
    B, Q, N = wl.B, wl.Q, wl.N
    kv_host = T["kv"].cpu().numpy()
    for b in range(B):
        want = fp4.quantize_kv_fp4(f32(T["x"][b][N - wl.n_new:]))
        np.testing.assert_array_equal(kv_host[b, N - wl.n_new:], want)
    n_vis = T["n_vis"].numpy()
    last_idx, last_pool = None, None
    for l, mode in enumerate(wl.modes):
        li = T["layers"][l]
        if mode in (0, 1):
            gidx = Ls[l]["idx"].cpu().numpy()
            for b in range(B):
                for q in range(Q):
                    s = indexer.index_scores(f32(li["qI"][b, q]), f32(li["w"][b, q]), f32(T["kI"][b]), int(n_vis[b, q]))
                    check_topk(gidx[b, q], s, wl.K, what=f"layer {l} b{b} q{q}")
                    if mode == 0 and wl.hsi_blocks:
                        bs = indexer.block_scores(s, 8)
                        gp = pool.cpu().numpy()[b, q]
                        v = gp[gp >= 0]
                        check_topk(np.concatenate([v[np.argsort(-bs[v], kind="stable")], gp[gp < 0]]), bs,
                                   wl.hsi_blocks, what=f"pool b{b}")
            if mode == 0 and wl.hsi_blocks:
                last_pool = pool.cpu().numpy()
            last_idx = gidx
        elif mode == 2:
            gidx = Ls[l]["idx"].cpu().numpy()
            for b in range(B):
                for q in range(Q):
                    pos, ps = indexer.pool_scores(f32(li["qI"][b, q]), f32(li["w"][b, q]), f32(T["kI"][b]),
                                                  last_pool[b, q], int(n_vis[b, q]))
                    check_topk(gidx[b, q], ps, wl.K, positions=pos, what=f"layer {l} pool b{b}")
            last_idx = gidx
        out = Ls[l]["out"].float().cpu().numpy()
        for b in range(B):
            for q in range(Q):
                sel = last_idx[b, q]
                rows_needed = sel[sel >= 0]
                deq = np.zeros((N, 512))
                deq[rows_needed] = fp4.dequantize_kv_fp4(kv_host[b, rows_needed])
                win = f32(li["swa"][b])[q * wl.swa_step: q * wl.swa_step + wl.W]
                o, lse = attention.sparse_mqa(f32(li["q"][b, q]), deq, sel, win)
                check_attention(out[b, q], o, what=f"layer {l} b{b} q{q}")
                np.testing.assert_allclose(Ls[l]["lse"].cpu().numpy()[b, q], lse, rtol=1e-3, atol=1e-3)


def _small(base, **kw):
    wl = workloads.WORKLOADS[base]
    args = dict(name=wl.name + "_small", seed=wl.seed, B=wl.B, Q=wl.Q, N=wl.N, r=wl.r, modes=list(wl.modes),
                K=wl.K, W=wl.W, hsi_blocks=wl.hsi_blocks, hsi_block=wl.hsi_block, n_new=wl.n_new,
                prefill=wl.prefill, swa_step=wl.swa_step)
    args.update(kw)
    return workloads.Workload(**args)


@pytest.mark.parametrize("wl", [
    workloads.WORKLOADS[0],
    _small(1, B=3, N=5000),
    _small(2, B=2, N=9000),
    _small(3, B=2, N=8 * 2500 + 3, hsi_blocks=512),
    _small(2, B=1, Q=3, N=3001, n_new=3),
    _small(4, Q=40, N=3000, n_new=20),                 # causal prefill: 5 query blocks of 8
    _small(4, B=2, Q=19, N=1333, n_new=10),            # two rows, a partial query block
], ids=lambda w: f"{w.name}_B{w.B}_Q{w.Q}_N{w.N}")
def test_group_small(wl):
    T = _make(wl)
    Ls, pool = _run_group(wl, T)
    _check(wl, T, Ls, pool)
