"""GPU parity of csa2_stack_decode (several sharing groups in one call)
against the oracle's stack_row, every layer and every query, on small
versions of the model's two schedules ("DeepSeek V4.1-Flash 技术报告深度解析"
§3.2 configuration paragraph, §3.3):

* decoder: groups over one shared cache; group 1 is Full (building the HSI
  pool) + Reuse layers, the later groups a pool-restricted Reindex + Reuse
  layers reading group 1's pool;
* encoder: groups of Full + Reuse layers at r=2, each with its own cache.

Both run several query positions per row with causal visibility (a draft
block being verified), and the stack's second call must repeat the first.
"""

import numpy as np
import pytest
import torch

from fp4_kv_cache_mxfp4_b200 import csa2, workloads
from fp4_kv_cache_mxfp4_b200.device_workload import make_device_workload, run_step
from oracle import fp4, group
from parity import check_attention, check_topk, f32
from oracle import indexer

pytestmark = pytest.mark.gpu

F, RI, RP, RU = workloads.FULL, workloads.REINDEX, workloads.REINDEX_POOL, workloads.REUSE

DECODER = workloads.Workload("decoder_stack_small", 61, B=2, Q=5, N=6001, r=1,
                             modes=[F, RU, RU] + [RP, RU, RU] * 2, groups=[3, 3, 3], hsi_blocks=200, n_new=5,
                             prefill=True, swa_step=1)
ENCODER = workloads.Workload("encoder_stack_small", 71, B=2, Q=5, N=3000, r=2,
                             modes=[F, RU, RU] * 3, groups=[3, 3, 3], cache_per_group=True, n_new=2,
                             prefill=True, swa_step=1)


def _oracle_row(wl, b):
    """stack_row inputs of batch row b, from the same seeded draws."""
    groups = []
    shared = None
    for g in range(len(wl.groups)):
        cw = wl.cache_of_group(g if wl.cache_per_group else 0)
        if wl.cache_per_group or shared is None:
            x = f32(workloads.main_kv_rows(cw, b, 0, wl.N))
            kv = fp4.quantize_kv_fp4(x[: wl.N - wl.n_new])
            kv = np.concatenate([kv, np.zeros((wl.n_new, 288), np.uint8)])
            cache = dict(kv_fp4=kv, kI=f32(workloads.index_k(cw, b)), kv_new=x[wl.N - wl.n_new:],
                         new_rows=wl.new_rows)
            shared = cache
        cache = shared
        layers = []
        for l in wl.group_layers(g):
            li = workloads.layer_inputs(wl, l)
            layers.append(dict(mode=wl.modes[l], qI=f32(li["qI"][b]), w=f32(li["w"][b]), q=f32(li["q"][b]),
                               swa=f32(li["swa"][b])))
        first = g == 0 or wl.cache_per_group
        groups.append(dict(kv_fp4=cache["kv_fp4"], kI=cache["kI"], n_vis=np.asarray(wl.n_vis), layers=layers,
                           kv_new=cache["kv_new"] if first else None, new_rows=cache["new_rows"] if first else None))
    return group.stack_row(groups, hsi_blocks=wl.hsi_blocks, hsi_block=wl.hsi_block, K=wl.K, W=wl.W,
                           swa_step=wl.swa_step), groups


@pytest.mark.parametrize("wl", [DECODER, ENCODER], ids=lambda w: w.name)
def test_stack_matches_oracle(wl):
    csa2.load()
    T = make_device_workload(wl, csa2)
    run_step(T, csa2)
    torch.cuda.synchronize()
    assert csa2.csa2_device_status() == (0, 0)
    first = [L["out"].clone() for L in T["layers"]]
    for b in range(wl.B):
        res, groups = _oracle_row(wl, b)
        pool = None
        for g in range(len(wl.groups)):
            c = g if wl.cache_per_group else 0
            np.testing.assert_array_equal(T["caches"][c]["kv"][b].cpu().numpy(), groups[g]["kv_fp4"],
                                          err_msg=f"cache {c} row {b}")
            G = T["groups"][g]
            if G["pool"] is not None:
                pool = G["pool"].cpu().numpy()[b]
            last = None
            for k, l in enumerate(wl.group_layers(g)):
                mode = wl.modes[l]
                L = T["layers"][l]
                li = groups[g]["layers"][k]
                if mode != RU:
                    last = L["idx"].cpu().numpy()[b]
                for q in range(wl.Q):
                    what = f"{wl.name} group {g} layer {l} b{b} q{q}"
                    nv = wl.n_vis[q]
                    if mode == F:
                        s = indexer.index_scores(li["qI"][q], li["w"][q], groups[g]["kI"], nv)
                        check_topk(last[q], s, wl.K, what=what)
                        if wl.hsi_blocks:
                            bs = indexer.block_scores(s, wl.hsi_block)
                            v = pool[q][pool[q] >= 0]
                            check_topk(np.concatenate([v[np.argsort(-bs[v], kind="stable")], pool[q][pool[q] < 0]]),
                                       bs, wl.hsi_blocks, what=what + " pool")
                    elif mode == RP:
                        pos, ps = indexer.pool_scores(li["qI"][q], li["w"][q], groups[g]["kI"], pool[q], nv)
                        check_topk(last[q], ps, wl.K, positions=pos, what=what)
                    # attention on the GPU's (validated) indices
                    sel = last[q]
                    deq = np.zeros((wl.N, 512))
                    rows = sel[sel >= 0]
                    deq[rows] = fp4.dequantize_kv_fp4(groups[g]["kv_fp4"][rows])
                    from oracle import attention
                    o, lse = attention.sparse_mqa(li["q"][q], deq, sel, li["swa"][q * wl.swa_step: q * wl.swa_step + wl.W])
                    check_attention(L["out"][b, q], o, what=what)
                    np.testing.assert_allclose(L["lse"][b, q].cpu().numpy(), lse, rtol=1e-3, atol=1e-3)
                if mode == RU:
                    np.testing.assert_array_equal(last.shape, (wl.Q, wl.K))
    # a second step on the same inputs gives the same outputs bit for bit
    run_step(T, csa2)
    torch.cuda.synchronize()
    for a, L in zip(first, T["layers"]):
        assert torch.equal(a, L["out"])
