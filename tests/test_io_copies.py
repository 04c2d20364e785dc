"""The copy lists of the overlapped-copy calls (host logic, no GPU): every
input byte of a staged step moves in before the layer that first reads it,
every output byte moves out after the layer that writes it, ranges
disjoint, lists in layer order; per layer, or with the fewest
synchronisation points (two per direction)."""

import pytest
import torch

from fp4_kv_cache_mxfp4_b200 import device_workload as dw
from fp4_kv_cache_mxfp4_b200 import workloads


def _staged(wl):
    """A CPU stand-in for a staged step with the device workload's arena
    layout (small tensors of the real ones' kinds)."""
    n_caches = len(wl.groups) if wl.cache_per_group else 1
    news = [torch.zeros(3, 512, dtype=torch.bfloat16) for _ in range(n_caches)]
    per_layer = [(torch.zeros(2, 32, 128, dtype=torch.bfloat16), torch.zeros(2, 32),
                  torch.zeros(2, 64, 512, dtype=torch.bfloat16)) for _ in wl.modes]
    in_buf, views = dw._arena(news + [t for trio in per_layer for t in trio], "cpu")
    caches = [dict(new=views.pop(0)) for _ in range(n_caches)]
    layers = [dict(qI=views.pop(0), w=views.pop(0), q=views.pop(0)) for _ in wl.modes]
    out_buf, outs = dw._arena([torch.zeros(2, 64, 512, dtype=torch.bfloat16) for _ in wl.modes], "cpu", copy=False)
    for L, o in zip(layers, outs):
        L["out"] = o
    return dict(wl=wl, inputs=in_buf, outputs=out_buf, caches=caches, layers=layers)


def _nbytes(v):
    return v.numel() * v.element_size()


def _check(wl, per_layer):
    T = _staged(wl)
    host_in, host_out = torch.empty_like(T["inputs"]), torch.empty_like(T["outputs"])
    ins, outs = dw.io_copies(T, host_in, host_out, per_layer=per_layer)
    n = len(wl.modes)
    if per_layer:
        assert [c[3] for c in outs] == list(range(n))
    else:
        assert len({c[3] for c in ins}) <= 2 and len({c[3] for c in outs}) <= 2
    din, hin = T["inputs"].data_ptr(), host_in.data_ptr()
    dout, hout = T["outputs"].data_ptr(), host_out.data_ptr()
    assert [c[3] for c in ins] == sorted(c[3] for c in ins)
    assert [c[3] for c in outs] == sorted(c[3] for c in outs)
    assert all(0 <= c[3] < n for c in ins + outs)
    # the same offsets on both sides, ranges disjoint
    spans = sorted((dst - din, n) for dst, src, n, _ in ins)
    for dst, src, n, _ in ins:
        assert dst - din == src - hin
    for (a, n), (b, _) in zip(spans, spans[1:]):
        assert a + n <= b
    for dst, src, n, _ in outs:
        assert dst - hout == src - dout

    def covered(v, layer):
        o = v.data_ptr() - din
        return any(c[3] <= layer and c[0] - din <= o and o + _nbytes(v) <= c[0] - din + c[2] for c in ins)

    for l, L in enumerate(T["layers"]):
        for k in ("qI", "w", "q"):
            assert covered(L[k], l), (l, k)
        o = L["out"].data_ptr() - dout
        assert any(c[3] >= l and c[1] - dout <= o and o + _nbytes(L["out"]) <= c[1] - dout + c[2] for c in outs)
    for g in range(len(wl.groups)):
        if g == 0 or wl.cache_per_group:
            new = T["caches"][g if wl.cache_per_group else 0]["new"]
            first = wl.group_layers(g)[0]
            assert covered(new, first)
            assert any(c[3] <= first and c[0] == new.data_ptr() for c in ins)
    assert sum(c[2] for c in ins) <= T["inputs"].numel()


@pytest.mark.parametrize("per_layer", [True, False])
def test_group_copies(per_layer):
    _check(workloads.WORKLOADS[2], per_layer)
    _check(workloads.WORKLOADS[1], per_layer)                # one layer


@pytest.mark.parametrize("per_layer", [True, False])
def test_stack_copies_with_a_cache_per_group(per_layer):
    wl = workloads.WORKLOADS[7]
    assert wl.cache_per_group and len(wl.groups) > 1
    _check(wl, per_layer)


@pytest.mark.parametrize("per_layer", [True, False])
def test_stack_copies_with_one_cache(per_layer):
    wl = workloads.WORKLOADS[6]
    assert not wl.cache_per_group and len(wl.groups) > 1
    _check(wl, per_layer)
