"""Stage a seeded workload on the GPU through the library's own calls.

The main-KV cache of every batch row (all entries but the step's new ones)
is quantised into FP4 with csa2_quantize_kv_fp4 in 65,536-row chunks; the
step's new entries, index-K and every layer's inputs are copied to the
device; the returned dict holds the csa2_group_args of each sharing group
(and, for a stack of groups, the csa2_stack_args) of one step, plus a
workspace of the size the library asks for.  The bench and the full-size
parity tests both build their step here, so both run the same launches.

A stack of groups either shares one cache (the decoder: the first group's
Full layer quantises the step's new entries and builds the HSI pool that
the later groups' pool-restricted Reindex layers read) or gives every group
its own cache (the encoder: each group quantises its own new entries).
"""

import torch

from . import workloads


def with_seed_shift(wl, shift):
    """The same workload drawn from another seed (one per replica)."""
    if not shift:
        return wl
    return workloads.Workload(**{**wl.__dict__, "seed": wl.seed + 7919 * shift, "n_vis": list(wl.n_vis),
                                 "groups": list(wl.groups)})


def _stage_cache(cw, csa2, d):
    """FP4 main KV of every row but the step's new entries, index-K (bf16,
    or quantised on the device to MXFP4 entries), the new entries and their
    absolute destination rows."""
    B, N = cw.B, cw.N
    kv = torch.empty(B, N, 288, dtype=torch.uint8, device=d)
    for b in range(B):
        for r0 in range(0, N - cw.n_new, workloads.KV_CHUNK):
            n = min(workloads.KV_CHUNK, N - cw.n_new - r0)
            x = workloads.main_kv_rows(cw, b, r0, n).to(d)
            csa2.csa2_quantize_kv_fp4(x, kv[b], row_offset=r0)
    if cw.index_k_format == csa2.FMT_MXFP4:
        kI = torch.empty(B, N, 68, dtype=torch.uint8, device=d)
        for b in range(B):
            csa2.csa2_quantize_index_k_mxfp4(workloads.index_k(cw, b).to(d), kI[b])
    else:
        kI = torch.stack([workloads.index_k(cw, b) for b in range(B)]).to(d)
    new = torch.cat([workloads.main_kv_rows(cw, b, N - cw.n_new, cw.n_new) for b in range(B)]).to(d)
    new_rows = torch.tensor([b * N + r for b in range(B) for r in cw.new_rows], dtype=torch.int64, device=d)
    return dict(kv=kv, kI=kI, new=new, new_rows=new_rows)


def _arena(tensors, d, copy=True):
    """One device buffer holding every tensor of `tensors` (each at a
    256-byte aligned offset): returns the buffer and the views, filled with
    the tensors' values when `copy`.  A step's inputs (or outputs) then
    move between host and device in one copy."""
    offs, off = [], 0
    for t in tensors:
        off = (off + 255) & ~255
        offs.append(off)
        off += t.numel() * t.element_size()
    buf = torch.empty(max(off, 1), dtype=torch.uint8, device=d)
    views = []
    for t, o in zip(tensors, offs):
        v = buf[o:o + t.numel() * t.element_size()].view(t.dtype).view(t.shape)
        if copy:
            v.copy_(t)
        views.append(v)
    return buf, views


def make_device_workload(wl, csa2, seed_shift=0):
    d = "cuda"
    wl = with_seed_shift(wl, seed_shift)
    B, Q, K = wl.B, wl.Q, wl.K
    n_groups = len(wl.groups)
    caches = [_stage_cache(wl.cache_of_group(g), csa2, d) for g in range(n_groups if wl.cache_per_group else 1)]
    layers = []
    for l, mode in enumerate(wl.modes):
        li = workloads.layer_inputs(wl, l)
        swa, swa_scale = li["swa"].to(d), None
        if wl.window_format == csa2.FMT_FP8:
            codes = torch.empty(B, wl.swa_rows, 512, dtype=torch.uint8, device=d)
            swa_scale = torch.empty(B, wl.swa_rows, device=d)
            for b in range(B):
                csa2.csa2_quantize_window_fp8(swa[b], codes[b], swa_scale[b])
            swa = codes
        q = li["q"].to(d)
        q4 = torch.empty(B, Q, 64, 288, dtype=torch.uint8, device=d)      # the same q as FP4 rows
        csa2.csa2_quantize_kv_fp4(q.reshape(-1, 512), q4.view(-1, 288))
        layers.append(dict(mode=mode, qI=li["qI"].to(d), w=li["w"].to(d), q=q, q4=q4, swa=swa,
                           swa_scale=swa_scale, out=torch.empty(B, Q, 64, 512, dtype=torch.bfloat16, device=d),
                           lse=torch.empty(B, Q, 64, device=d),
                           idx=torch.empty(B, Q, K, dtype=torch.int32, device=d) if mode != workloads.REUSE else None))
    # the step's inputs (new entries, every layer's qI, w and q) in one
    # device buffer and every layer's output in another
    ins = [C["new"] for C in caches] + [L[k] for L in layers for k in ("qI", "w", "q")]
    in_buf, in_views = _arena(ins, d)
    for C in caches:
        C["new"] = in_views.pop(0)
    for L in layers:
        for k in ("qI", "w", "q"):
            L[k] = in_views.pop(0)
    out_buf, out_views = _arena([L["out"] for L in layers], d, copy=False)
    for L, v in zip(layers, out_views):
        L["out"] = v
    n_vis = workloads.n_vis_tensor(wl).to(d)
    groups = []
    pool = None                      # the most recent pool built by a Full layer (handed to later groups)
    for g in range(n_groups):
        C = caches[g if wl.cache_per_group else 0]
        Ls = [layers[l] for l in wl.group_layers(g)]
        builds_pool = wl.hsi_blocks > 0 and any(L["mode"] == workloads.FULL for L in Ls)
        own_pool = torch.empty(B, Q, wl.hsi_blocks, dtype=torch.int32, device=d) if builds_pool else None
        quantise = g == 0 or wl.cache_per_group
        ga = csa2.group_args(B, Q, K, wl.W, wl.N, n_vis, C["kI"], C["kv"], Ls,
                             kv_new=C["new"] if quantise else None, new_rows=C["new_rows"] if quantise else None,
                             swa_rows=wl.swa_rows, swa_step=wl.swa_step, hsi_blocks=wl.hsi_blocks,
                             hsi_block=wl.hsi_block, pool=own_pool, pool_in=pool, swa_format=wl.window_format)
        groups.append(dict(g=ga, cache=C, layers=Ls, pool=own_pool, pool_in=pool))
        if own_pool is not None:
            pool = own_pool
    if n_groups == 1:
        stack = None
        ws = csa2.workspace(groups[0]["g"], csa2.WS_GROUP)
    else:
        stack = csa2.stack_args([G["g"] for G in groups])
        ws = csa2.workspace(stack, csa2.WS_STACK)
    torch.cuda.synchronize()
    C0 = caches[0]
    return dict(wl=wl, g=groups[0]["g"], groups=groups, stack=stack, ws=ws, caches=caches, kv=C0["kv"], kI=C0["kI"],
                new=C0["new"], new_rows=C0["new_rows"], layers=layers, pool=groups[0]["pool"], n_vis=n_vis,
                inputs=in_buf, outputs=out_buf)


def set_flags(T, flags):
    """Launch-order flags of every group call of a staged step."""
    if T["stack"] is None:
        T["g"].flags = flags
    else:
        for i in range(len(T["groups"])):
            T["stack"]._group_array[i].flags = flags


def set_q_format(T, q_format, csa2):
    """Attention Q of every layer of a staged step: bf16 rows (FMT_BF16) or
    their FP4 rows (FMT_NVFP4, quantised Q)."""
    for G in T["groups"]:
        for j, L in enumerate(G["layers"]):
            G["g"]._layer_array[j].q = (L["q4"] if q_format == csa2.FMT_NVFP4 else L["q"]).data_ptr()
    if T["stack"] is None:
        T["g"].q_format = q_format
    else:
        for i in range(len(T["groups"])):
            T["stack"]._group_array[i].q_format = q_format


def _span(views, base):
    """(offset, bytes) of the arena range that holds `views`."""
    lo = min(v.data_ptr() for v in views)
    hi = max(v.data_ptr() + v.numel() * v.element_size() for v in views)
    return lo - base, hi - lo


def io_copies(T, host_in, host_out, per_layer=False):
    """The host<->device copies of a staged step for the overlapped-copy
    calls, through host mirrors of its input and output buffers (same
    offsets): each cache's new entries before the first layer of the group
    that quantises them, each layer's qI, w and q (one range) before that
    layer, each layer's output after it.  Returns two lists of
    (dst, src, bytes, layer) in layer order.

    Every distinct layer named is a synchronisation point between the
    caller's stream and a copy stream.  per_layer=False names as few as the
    step allows: the inputs of layer 0 (and the new entries) before layer
    0, all other inputs before layer 1 (an earlier layer than they need);
    every output but the last layer's after the second-to-last layer (a
    later one than they need), the last layer's after it."""
    wl = T["wl"]
    n = len(T["layers"])

    def tag_in(l):
        return l if per_layer else min(l, 1)

    def tag_out(l):
        return l if per_layer else max(l, n - 2)

    din, dout = T["inputs"].data_ptr(), T["outputs"].data_ptr()
    hin, hout = host_in.data_ptr(), host_out.data_ptr()
    ins = []
    for g in range(len(wl.groups)):
        if g == 0 or wl.cache_per_group:
            off, nb = _span([T["caches"][g if wl.cache_per_group else 0]["new"]], din)
            ins.append((din + off, hin + off, nb, tag_in(wl.group_layers(g)[0])))
    for l, L in enumerate(T["layers"]):
        off, nb = _span([L["qI"], L["w"], L["q"]], din)
        ins.append((din + off, hin + off, nb, tag_in(l)))
    ins.sort(key=lambda c: c[3])
    outs = []
    for l, L in enumerate(T["layers"]):
        off, nb = _span([L["out"]], dout)
        outs.append((hout + off, dout + off, nb, tag_out(l)))
    return ins, outs


def run_step_io(T, csa2, io, stream=None):
    """One step with its copies overlapped: csa2_group_decode_io or
    csa2_stack_decode_io."""
    if T["stack"] is None:
        csa2.csa2_group_decode_io(T["g"], io, T["ws"], stream)
    else:
        csa2.csa2_stack_decode_io(T["stack"], io, T["ws"], stream)


def run_step(T, csa2, stream=None):
    """One step through the library's public call: csa2_group_decode for one
    group, csa2_stack_decode for a stack."""
    if T["stack"] is None:
        csa2.csa2_group_decode(T["g"], T["ws"], stream)
    else:
        csa2.csa2_stack_decode(T["stack"], T["ws"], stream)
