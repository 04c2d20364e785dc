"""Stage a seeded workload on the GPU through the library's own calls.

The main-KV cache of every batch row (all entries but the step's new ones)
is quantised into FP4 with csa2_quantize_kv_fp4 in 65,536-row chunks; the
step's new entries, index-K and every layer's inputs are copied to the
device; the returned dict holds the csa2_group_args of one step and a
workspace of the size the library asks for.  The bench and the full-size
parity tests both build their step here, so both run the same launches.
"""

import torch

from . import workloads


def with_seed_shift(wl, shift):
    """The same workload drawn from another seed (one per replica)."""
    if not shift:
        return wl
    return workloads.Workload(**{**wl.__dict__, "seed": wl.seed + 7919 * shift, "n_vis": list(wl.n_vis)})


def make_device_workload(wl, csa2, seed_shift=0):
    d = "cuda"
    wl = with_seed_shift(wl, seed_shift)
    B, Q, N, K = wl.B, wl.Q, wl.N, wl.K
    kv = torch.empty(B, N, 288, dtype=torch.uint8, device=d)
    for b in range(B):
        for r0 in range(0, N - wl.n_new, workloads.KV_CHUNK):
            n = min(workloads.KV_CHUNK, N - wl.n_new - r0)
            x = workloads.main_kv_rows(wl, b, r0, n).to(d)
            csa2.csa2_quantize_kv_fp4(x, kv[b], row_offset=r0)
    kI = torch.stack([workloads.index_k(wl, b) for b in range(B)]).to(d)
    new = torch.cat([workloads.main_kv_rows(wl, b, N - wl.n_new, wl.n_new) for b in range(B)]).to(d)
    new_rows = torch.tensor([b * N + r for b in range(B) for r in wl.new_rows], dtype=torch.int64, device=d)
    layers = []
    for l, mode in enumerate(wl.modes):
        li = workloads.layer_inputs(wl, l)
        layers.append(dict(mode=mode, qI=li["qI"].to(d), w=li["w"].to(d), q=li["q"].to(d), swa=li["swa"].to(d),
                           out=torch.empty(B, Q, 64, 512, dtype=torch.bfloat16, device=d),
                           lse=torch.empty(B, Q, 64, device=d),
                           idx=torch.empty(B, Q, K, dtype=torch.int32, device=d) if mode != workloads.REUSE else None))
    pool = torch.empty(B, Q, wl.hsi_blocks, dtype=torch.int32, device=d) if wl.hsi_blocks else None
    n_vis = workloads.n_vis_tensor(wl).to(d)
    g = csa2.group_args(B, Q, K, wl.W, N, n_vis, kI, kv, layers, kv_new=new, new_rows=new_rows,
                        swa_rows=wl.swa_rows, swa_step=wl.swa_step, hsi_blocks=wl.hsi_blocks,
                        hsi_block=wl.hsi_block, pool=pool)
    ws = csa2.workspace(g, csa2.WS_GROUP)
    torch.cuda.synchronize()
    return dict(wl=wl, g=g, ws=ws, kv=kv, kI=kI, new=new, new_rows=new_rows, layers=layers, pool=pool, n_vis=n_vis)
