"""C-ABI checks that need no GPU: the library loads, exports every function
include/csa2.h declares, the binding's struct layouts equal the C
compiler's, and host-side validation rejects bad arguments before any
device work.  Only argument combinations that fail validation (or touch no
device) are used here, so nothing can reach a kernel."""

import ctypes
import os
import re
import subprocess
import tempfile

import pytest

from fp4_kv_cache_mxfp4_b200 import build, csa2

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "csa2.h")
FAKE = 0x10000          # 16-byte aligned stand-in pointer, never dereferenced


@pytest.fixture(scope="module")
def L():
    build.build()
    return csa2.load()


def _declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\**\s+\**(csa2_\w+)\s*\(", text, re.M)))


def test_every_declared_function_is_exported(L):
    names = _declared_functions()
    assert {"csa2_quantize_kv_fp4", "csa2_index_score_topk", "csa2_sparse_attn", "csa2_group_decode",
            "csa2_workspace_size"} <= set(names)
    for n in names:
        assert hasattr(L, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", csa2.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (csa2_\w+)", out))
    assert set(names) <= exported


def test_version_and_status_strings(L):
    assert csa2.version() == 107
    assert csa2.status_string(0) == "ok"
    assert "workspace" in csa2.status_string(4)
    assert csa2.status_string(99) == "unknown status"


# Python field names that differ from the header's (`in` is a keyword)
_C_NAME = {"in_": "in"}


def _c_layout():
    fields = {
        "csa2_index_args": [f for f, _ in csa2.IndexArgs._fields_],
        "csa2_attn_args": [f for f, _ in csa2.AttnArgs._fields_],
        "csa2_layer": [f for f, _ in csa2.Layer._fields_],
        "csa2_group_args": [f for f, _ in csa2.GroupArgs._fields_],
        "csa2_stack_args": [f for f, _ in csa2.StackArgs._fields_],
        "csa2_compress_args": [f for f, _ in csa2.CompressArgs._fields_],
        "csa2_copy": [f for f, _ in csa2.Copy._fields_],
        "csa2_io": [_C_NAME.get(f, f) for f, _ in csa2.Io._fields_],
    }
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "csa2.h"', "int main(void) {"]
    for s, fs in fields.items():
        lines.append(f'printf("{s} %zu\\n", sizeof({s}));')
        for f in fs:
            lines.append(f'printf("{s}.{f} %zu\\n", offsetof({s}, {f}));')
    lines.append("return 0; }")
    with tempfile.TemporaryDirectory() as d:
        src, exe = os.path.join(d, "l.c"), os.path.join(d, "l")
        open(src, "w").write("\n".join(lines))
        subprocess.run(["gcc", "-I", os.path.dirname(HEADER), "-o", exe, src], check=True)
        out = subprocess.run([exe], capture_output=True, text=True, check=True).stdout
    return dict(line.split() for line in out.strip().splitlines())


def test_struct_layouts_match_the_header():
    c = _c_layout()
    for cname, py in [("csa2_index_args", csa2.IndexArgs), ("csa2_attn_args", csa2.AttnArgs),
                      ("csa2_layer", csa2.Layer), ("csa2_group_args", csa2.GroupArgs),
                      ("csa2_stack_args", csa2.StackArgs), ("csa2_compress_args", csa2.CompressArgs),
                      ("csa2_copy", csa2.Copy), ("csa2_io", csa2.Io)]:
        assert int(c[cname]) == ctypes.sizeof(py), cname
        for f, _ in py._fields_:
            assert int(c[f"{cname}.{_C_NAME.get(f, f)}"]) == getattr(py, f).offset, (cname, f)


def _index(**kw):
    a = csa2.IndexArgs(mode=0, B=1, Q=1, K=512, N=4096, qI=FAKE, w=FAKE, kI=FAKE, n_vis=FAKE, idx=FAKE,
                       scores=None, hsi_blocks=0, hsi_block=8, pool_out=None, pool_in=None)
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def _attn(**kw):
    a = csa2.AttnArgs(B=1, Q=1, K=512, W=128, N=4096, q=FAKE, kv_fp4=FAKE, idx=FAKE, swa=FAKE,
                      swa_rows=128, swa_step=0, scale=0.0, out=FAKE, lse=None)
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def _call_index(L, a, ws=FAKE, ws_bytes=0):
    return L.csa2_index_score_topk(ctypes.byref(a), ctypes.c_void_p(ws), ws_bytes, None)


def _call_attn(L, a, ws=FAKE, ws_bytes=0):
    return L.csa2_sparse_attn(ctypes.byref(a), ctypes.c_void_p(ws), ws_bytes, None)


@pytest.mark.parametrize("kw,status", [
    (dict(mode=3), 1), (dict(mode=7), 1), (dict(qI=None), 1), (dict(n_vis=None), 1), (dict(idx=None), 1),
    (dict(B=0), 2), (dict(Q=0), 2), (dict(B=2, Q=40000), 2), (dict(K=0), 2), (dict(K=2049), 2), (dict(N=0), 2),
    (dict(N=2 ** 31), 2), (dict(hsi_blocks=-1), 2), (dict(hsi_blocks=2048, hsi_block=16, pool_out=FAKE), 2),
    (dict(hsi_blocks=2048, pool_out=None), 1), (dict(mode=2, hsi_blocks=2048, pool_in=None), 1),
    (dict(qI=FAKE + 8), 3), (dict(kI=FAKE + 4), 3), (dict(scores=FAKE + 2), 3),
    # MXFP4 index-K: N a multiple of 4, and of 8 with an HSI pool (whole-block fetches)
    (dict(k_format=2, N=4098), 2), (dict(k_format=2, N=4100), 4),
    (dict(k_format=2, N=4100, hsi_blocks=512, pool_out=FAKE), 2),
    (dict(k_format=2, N=4100, mode=2, hsi_blocks=512, pool_in=FAKE), 2),
    (dict(k_format=2, N=4104, hsi_blocks=512, pool_out=FAKE), 4),
    (dict(k_format=2, N=4104, mode=2, hsi_blocks=512, pool_in=FAKE), 4),
    (dict(N=4100, hsi_blocks=512, pool_out=FAKE), 4),      # bf16 index-K: TMA bounds the blocks
    (dict(), 4),                       # valid arguments, zero-byte workspace
])
def test_index_validation(L, kw, status):
    assert _call_index(L, _index(**kw)) == status


def test_index_validation_null_struct(L):
    assert L.csa2_index_score_topk(None, None, 0, None) == 1


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), 1), (dict(out=None), 1), (dict(idx=None), 1), (dict(swa=None), 1),
    (dict(B=0), 2), (dict(B=3, Q=30000), 2), (dict(K=-1), 2), (dict(K=0, W=0), 2), (dict(W=1025), 2),
    (dict(swa_rows=100), 2), (dict(Q=2, swa_step=1, swa_rows=128), 2),
    (dict(out=FAKE + 8), 3), (dict(lse=FAKE + 4), 3), (dict(q_format=2), 1), (dict(q_format=4), 1),
    (dict(q_format=3), 4),             # quantised Q: valid, zero-byte workspace
    (dict(), 4),                       # valid arguments, zero-byte workspace
])
def test_attn_validation(L, kw, status):
    assert _call_attn(L, _attn(**kw)) == status


def test_quantize_validation(L):
    q = L.csa2_quantize_kv_fp4
    assert q(ctypes.c_void_p(FAKE), -1, 512, ctypes.c_void_p(FAKE), None, 0, None) == 2
    assert q(ctypes.c_void_p(FAKE), 4, 500, ctypes.c_void_p(FAKE), None, 0, None) == 2
    assert q(ctypes.c_void_p(FAKE), 4, 516, ctypes.c_void_p(FAKE), None, 0, None) == 2
    assert q(ctypes.c_void_p(FAKE), 4, 512, ctypes.c_void_p(FAKE), None, -3, None) == 2
    assert q(None, 4, 512, ctypes.c_void_p(FAKE), None, 0, None) == 1
    assert q(ctypes.c_void_p(FAKE + 2), 4, 512, ctypes.c_void_p(FAKE), None, 0, None) == 3
    assert q(ctypes.c_void_p(FAKE), 0, 512, None, None, 0, None) == 0      # nothing to do


def test_workspace_sizes(L):
    a = _index(B=4, Q=1, K=512, N=131072)
    n = L.csa2_workspace_size(ctypes.byref(a), csa2.WS_INDEX)
    # scores (4 B per entry per query) + one 4096-bin histogram and one
    # tile counter per query
    assert n >= 4 * 131072 * 4 + 4 * 4096 * 4
    assert n < 4 * 131072 * 4 + 4 * 4096 * 4 + 4096
    assert L.csa2_workspace_size(ctypes.byref(_index(Q=0)), csa2.WS_INDEX) == 0
    # 4 FP4 + 1 window slices of 128 keys merge inside a cluster: no partials
    assert 0 < L.csa2_workspace_size(ctypes.byref(_attn(B=4, Q=1, K=512, W=128)), csa2.WS_ATTN) <= 256
    # 16 + 1 slices: fp32 partials per slice and a merge kernel
    at = _attn(B=4, Q=1, K=2048, W=128)
    m = L.csa2_workspace_size(ctypes.byref(at), csa2.WS_ATTN)
    assert m >= 4 * 17 * 64 * 512 * 4
    assert L.csa2_workspace_size(ctypes.byref(at), 9) == 0
    # a workspace one byte short is refused
    assert _call_index(L, a, FAKE, n - 1) == 4
    assert _call_attn(L, at, FAKE, m - 1) == 4


def test_group_validation(L):
    layers = (csa2.Layer * 2)()
    layers[0] = csa2.Layer(mode=3, q=FAKE, swa=FAKE, out=FAKE)          # REUSE first: nothing to reuse
    layers[1] = csa2.Layer(mode=0, qI=FAKE, w=FAKE, q=FAKE, swa=FAKE, out=FAKE, idx=FAKE)
    g = csa2.GroupArgs(B=1, Q=1, K=512, W=128, N=4096, n_vis=FAKE, kI=FAKE, kv_fp4=FAKE, kv_new=None, n_new=0,
                       new_rows=None, swa_rows=128, swa_step=0, hsi_blocks=0, hsi_block=8, pool=None, scale=0.0,
                       n_layers=2, layers=ctypes.cast(layers, ctypes.POINTER(csa2.Layer)))
    assert L.csa2_group_decode(ctypes.byref(g), ctypes.c_void_p(FAKE), 0, None) == 1
    layers[0] = csa2.Layer(mode=0, qI=FAKE, w=FAKE, q=FAKE, swa=FAKE, out=FAKE, idx=FAKE)
    layers[1] = csa2.Layer(mode=2, qI=FAKE, w=FAKE, q=FAKE, swa=FAKE, out=FAKE, idx=FAKE)   # pool without HSI
    assert L.csa2_group_decode(ctypes.byref(g), ctypes.c_void_p(FAKE), 0, None) == 1
    layers[1] = csa2.Layer(mode=3, q=FAKE, swa=FAKE, out=FAKE)
    n = L.csa2_workspace_size(ctypes.byref(g), csa2.WS_GROUP)
    assert n > 0
    assert L.csa2_group_decode(ctypes.byref(g), ctypes.c_void_p(FAKE), n - 1, None) == 4
    g.flags = 4                                                           # unknown flag bit
    assert L.csa2_group_decode(ctypes.byref(g), ctypes.c_void_p(FAKE), n, None) == 1
    g.flags = csa2.GROUP_INPUTS_READY | csa2.GROUP_SERIAL
    assert L.csa2_workspace_size(ctypes.byref(g), csa2.WS_GROUP) == n


def _group(layers, **kw):
    g = csa2.GroupArgs(B=1, Q=1, K=512, W=128, N=4096, n_vis=FAKE, kI=FAKE, kv_fp4=FAKE, kv_new=None, n_new=0,
                       new_rows=None, swa_rows=128, swa_step=0, hsi_blocks=2048, hsi_block=8, pool=FAKE, scale=0.0,
                       n_layers=len(layers), layers=ctypes.cast(layers, ctypes.POINTER(csa2.Layer)), pool_in=None,
                       flags=0)
    for k, v in kw.items():
        setattr(g, k, v)
    return g


def test_group_pool_in_validation(L):
    """A group that starts with a pool-restricted Reindex layer needs the
    pool of an earlier call (pool_in); with it, it is valid."""
    layers = (csa2.Layer * 2)()
    layers[0] = csa2.Layer(mode=2, qI=FAKE, w=FAKE, q=FAKE, swa=FAKE, out=FAKE, idx=FAKE)
    layers[1] = csa2.Layer(mode=3, q=FAKE, swa=FAKE, out=FAKE)
    g = _group(layers)
    assert L.csa2_group_decode(ctypes.byref(g), ctypes.c_void_p(FAKE), 0, None) == 1
    assert L.csa2_workspace_size(ctypes.byref(g), csa2.WS_GROUP) == 0
    g.pool_in = FAKE + 4
    assert L.csa2_group_decode(ctypes.byref(g), ctypes.c_void_p(FAKE), 0, None) == 3
    g.pool_in = FAKE
    n = L.csa2_workspace_size(ctypes.byref(g), csa2.WS_GROUP)
    assert n > 0
    assert L.csa2_group_decode(ctypes.byref(g), ctypes.c_void_p(FAKE), n - 1, None) == 4


def test_stack_validation_and_workspace(L):
    """The stack call's workspace is the largest single group's; every
    group is validated before anything is enqueued."""
    first = (csa2.Layer * 2)()
    first[0] = csa2.Layer(mode=0, qI=FAKE, w=FAKE, q=FAKE, swa=FAKE, out=FAKE, idx=FAKE)
    first[1] = csa2.Layer(mode=3, q=FAKE, swa=FAKE, out=FAKE)
    later = (csa2.Layer * 2)()
    later[0] = csa2.Layer(mode=2, qI=FAKE, w=FAKE, q=FAKE, swa=FAKE, out=FAKE, idx=FAKE)
    later[1] = csa2.Layer(mode=3, q=FAKE, swa=FAKE, out=FAKE)
    g1, g2 = _group(first), _group(later, pool_in=FAKE)
    n1 = L.csa2_workspace_size(ctypes.byref(g1), csa2.WS_GROUP)
    n2 = L.csa2_workspace_size(ctypes.byref(g2), csa2.WS_GROUP)
    st = csa2.stack_args([g1, g2])
    assert L.csa2_workspace_size(ctypes.byref(st), csa2.WS_STACK) == max(n1, n2)
    assert L.csa2_stack_decode(ctypes.byref(st), ctypes.c_void_p(FAKE), max(n1, n2) - 1, None) == 4
    bad = csa2.stack_args([g1, _group(later)])                            # second group lacks its pool
    assert L.csa2_stack_decode(ctypes.byref(bad), ctypes.c_void_p(FAKE), 1 << 40, None) == 1
    assert L.csa2_workspace_size(ctypes.byref(bad), csa2.WS_STACK) == 0
    empty = csa2.StackArgs(n_groups=0, groups=None)
    assert L.csa2_stack_decode(ctypes.byref(empty), ctypes.c_void_p(FAKE), 0, None) == 1


def test_arg_structs_keep_their_tensors_alive():
    """The ctypes structs hold raw pointers: the binding must keep every
    tensor they point to alive, or a temporary's memory can be handed to the
    next allocation (a workspace) before the call runs."""
    import gc
    import weakref

    import torch
    n_vis = torch.zeros(1, 1, dtype=torch.int32)
    ref = weakref.ref(n_vis)
    a = csa2.index_args(0, torch.zeros(1, 1, 32, 128), torch.zeros(1, 1, 32), torch.zeros(1, 8, 128), n_vis,
                        torch.zeros(1, 1, 4, dtype=torch.int32))
    del n_vis
    gc.collect()
    assert ref() is not None
    q = torch.zeros(1, 1, 64, 512)
    ref_q = weakref.ref(q)
    at = csa2.attn_args(q, torch.zeros(1, 8, 288, dtype=torch.uint8), torch.zeros(1, 1, 4, dtype=torch.int32),
                        torch.zeros(1, 128, 512), torch.zeros(1, 1, 64, 512))
    del q
    gc.collect()
    assert ref_q() is not None
    nv = torch.zeros(1, 1, dtype=torch.int32)
    ref_nv = weakref.ref(nv)
    layer = dict(mode=0, qI=torch.zeros(1), w=torch.zeros(1), q=torch.zeros(1), swa=torch.zeros(1),
                 out=torch.zeros(1), lse=None, idx=torch.zeros(1, dtype=torch.int32))
    g = csa2.group_args(1, 1, 4, 128, 8, nv, torch.zeros(1), torch.zeros(1, dtype=torch.uint8), [layer])
    del nv, layer
    gc.collect()
    assert ref_nv() is not None
    assert a is not None and at is not None and g is not None


def test_workspace_sizes_for_prefill_shapes(L):
    """4096 causal queries over 133,120 entries: scores padded to a multiple
    of 4 slots per query, 2048-bin histograms for 8-query MMA groups, and
    attention with one CTA per query needs no partials."""
    a = _index(B=1, Q=4096, K=512, N=133121)
    n = L.csa2_workspace_size(ctypes.byref(a), csa2.WS_INDEX)
    ld = (133121 + 3) // 4 * 4
    assert n >= 4096 * ld * 4 + 4096 * 2048 * 4
    assert n < 4096 * ld * 4 + 4096 * 2048 * 4 + 4096
    at = _attn(B=1, Q=4096, K=512, W=128, swa_step=1, swa_rows=128 + 4095)
    assert 0 < L.csa2_workspace_size(ctypes.byref(at), csa2.WS_ATTN) <= 256
    small = _attn(B=1, Q=127, K=512, W=128, swa_step=1, swa_rows=128 + 126)
    assert 0 < L.csa2_workspace_size(ctypes.byref(small), csa2.WS_ATTN) <= 256
    many = _attn(B=1, Q=127, K=1024, W=128, swa_step=1, swa_rows=128 + 126)      # 9 slices
    assert L.csa2_workspace_size(ctypes.byref(many), csa2.WS_ATTN) >= 127 * 9 * 64 * 512 * 4


def test_compress_validation(L):
    def args(**kw):
        a = csa2.CompressArgs(x=FAKE, n_entries=4, ld_x=512, r=2, w=FAKE, w_stride=0, cos=FAKE, sin=FAKE,
                              kv_fp4=FAKE, dst_rows=None, row_offset=0)
        for k, v in kw.items():
            setattr(a, k, v)
        return L.csa2_compress_rope_quantize_kv_fp4(ctypes.byref(a), None)
    assert L.csa2_compress_rope_quantize_kv_fp4(None, None) == 1
    assert args(r=0) == 2 and args(r=17) == 2 and args(ld_x=500) == 2 and args(w_stride=7) == 2
    assert args(n_entries=-1) == 2 and args(row_offset=-1) == 2
    assert args(cos=None) == 1 and args(w=None) == 1 and args(kv_fp4=None) == 1
    assert args(x=FAKE + 8) == 3 and args(sin=FAKE + 2) == 3
    assert args(n_entries=0, x=None) == 0



def test_io_validation(L):
    """The overlapped-copy calls check their copy lists (layers inside the
    call, non-decreasing, no NULL pointer) before anything is enqueued; a
    valid list reaches the workspace check."""
    first = (csa2.Layer * 2)()
    first[0] = csa2.Layer(mode=0, qI=FAKE, w=FAKE, q=FAKE, swa=FAKE, out=FAKE, idx=FAKE)
    first[1] = csa2.Layer(mode=3, q=FAKE, swa=FAKE, out=FAKE)
    later = (csa2.Layer * 2)()
    later[0] = csa2.Layer(mode=2, qI=FAKE, w=FAKE, q=FAKE, swa=FAKE, out=FAKE, idx=FAKE)
    later[1] = csa2.Layer(mode=3, q=FAKE, swa=FAKE, out=FAKE)
    g1, g2 = _group(first), _group(later, pool_in=FAKE)
    st = csa2.stack_args([g1, g2])

    def group(io):
        return L.csa2_group_decode_io(ctypes.byref(g1), io and ctypes.byref(io), ctypes.c_void_p(FAKE), 0, None)

    def stack(io):
        return L.csa2_stack_decode_io(ctypes.byref(st), ctypes.byref(io), ctypes.c_void_p(FAKE), 0, None)

    ok_in = [(FAKE, FAKE, 64, 0), (FAKE, FAKE, 64, 0), (FAKE, FAKE, 0, 1)]
    ok_out = [(FAKE, FAKE, 64, 0), (FAKE, FAKE, 64, 1)]
    assert group(csa2.io_args(ok_in, ok_out)) == 4                          # valid: workspace next
    assert group(csa2.io_args([], [])) == 4
    assert group(None) == 1
    assert group(csa2.io_args([(FAKE, FAKE, 64, 2)], [])) == 1              # layer outside the group
    assert group(csa2.io_args([], [(FAKE, FAKE, 64, -1)])) == 1
    assert group(csa2.io_args([(FAKE, FAKE, 64, 1), (FAKE, FAKE, 64, 0)], [])) == 1   # out of order
    assert group(csa2.io_args([(None, FAKE, 64, 0)], [])) == 1
    assert group(csa2.io_args([], [(FAKE, None, 64, 0)])) == 1
    neg = csa2.io_args([], [])
    neg.n_in = -1
    assert group(neg) == 1
    missing = csa2.io_args([], [])
    missing.n_out, missing.out = 1, None
    assert group(missing) == 1
    # a stack counts its layers through the groups: 4 here
    assert stack(csa2.io_args([(FAKE, FAKE, 64, 0), (FAKE, FAKE, 64, 2)], [(FAKE, FAKE, 64, 3)])) == 4
    assert stack(csa2.io_args([(FAKE, FAKE, 64, 4)], [])) == 1
