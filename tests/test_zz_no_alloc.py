"""The no-allocation index entry point, csa2_index_score_topk_noalloc.

Some callers cannot allocate device memory: code that a host framework
hands only its input and output buffers, with no allocator of its own, or a
serving process that reserved its whole memory pool at start-up, where a
cudaMalloc would fail or stall the device.  For them the library offers the
index call with its scratch in a fixed device array inside the library.

The GPU test calls that entry point through the C ABI twice in a row, on
different inputs and modes, and checks each result against the ordinary
csa2_index_score_topk with a caller workspace: the selected positions must
be identical, the scores equal within the tolerance the other index tests
use.  The second call must not see anything left over from the first.  This
file is collected last so that a run stopping at the first failure has run
every other test already; it also passes alone in a fresh process.
"""

import ctypes

import numpy as np
import pytest
import torch

from fp4_kv_cache_mxfp4_b200 import build, csa2


def _inputs(B, Q, N, seed):
    g = torch.Generator().manual_seed(seed)
    qI = torch.randn(B, Q, 32, 128, generator=g).to(torch.bfloat16).cuda()
    w = torch.rand(B, Q, 32, generator=g).cuda()
    kI = torch.randn(B, N, 128, generator=g).to(torch.bfloat16).cuda()
    n_vis = torch.randint(N // 2, N + 1, (B, Q), generator=g, dtype=torch.int32).cuda()
    return qI, w, kI, n_vis


def _call(mode, qI, w, kI, n_vis, K, hsi_blocks, pool_in, noalloc):
    B, Q = qI.shape[:2]
    idx = torch.full((B, Q, K), -7, dtype=torch.int32, device="cuda")
    sc = torch.full((B, Q, K), 7.0, device="cuda")
    pool_out = torch.full((B, Q, hsi_blocks), -7, dtype=torch.int32, device="cuda") if mode == 0 and hsi_blocks else None
    a = csa2.index_args(mode, qI, w, kI, n_vis, idx, sc, hsi_blocks=hsi_blocks, hsi_block=8,
                        pool_out=pool_out, pool_in=pool_in)
    if noalloc:
        csa2.csa2_index_score_topk_noalloc(a)
    else:
        csa2.csa2_index_score_topk(a, csa2.workspace(a, csa2.WS_INDEX))
    torch.cuda.synchronize()
    return idx.cpu().numpy(), sc.cpu().numpy(), None if pool_out is None else pool_out


def _memory_state():
    """Free device memory as the driver sees it, and what torch's caching
    allocator holds."""
    torch.cuda.synchronize()
    return torch.cuda.mem_get_info()[0], torch.cuda.memory_reserved()


@pytest.mark.gpu
def test_noalloc_matches_workspace_call_twice():
    build.build()
    # call 1: Full scan with an HSI pool; call 2: pool-restricted Reindex
    # (different shapes, so the shared scratch is reused with a new layout)
    qI, w, kI, n_vis = _inputs(2, 2, 9000, 1)
    qI2, w2, _, _ = _inputs(2, 2, 9000, 2)
    ref_idx, ref_sc, ref_pool = _call(0, qI, w, kI, n_vis, 512, 256, None, noalloc=False)
    ref_idx2, ref_sc2, _ = _call(2, qI2, w2, kI, n_vis, 300, 256, ref_pool, noalloc=False)

    # the output buffers of the two calls, made before memory is measured
    outs = [(torch.full((2, 2, 512), -7, dtype=torch.int32, device="cuda"), torch.full((2, 2, 512), 7.0, device="cuda"),
             torch.full((2, 2, 256), -7, dtype=torch.int32, device="cuda")),
            (torch.full((2, 2, 300), -7, dtype=torch.int32, device="cuda"), torch.full((2, 2, 300), 7.0, device="cuda"),
             None)]
    args = [csa2.index_args(0, qI, w, kI, n_vis, outs[0][0], outs[0][1], hsi_blocks=256, hsi_block=8,
                            pool_out=outs[0][2]),
            csa2.index_args(2, qI2, w2, kI, n_vis, outs[1][0], outs[1][1], hsi_blocks=256, hsi_block=8,
                            pool_in=ref_pool)]
    # one call first, so that loading the library's module (which places
    # the scratch array) and the address lookup are behind us
    _call(0, qI2, w2, kI, n_vis, 64, 256, None, noalloc=True)
    before = _memory_state()
    for a in args:
        csa2.csa2_index_score_topk_noalloc(a)
    after = _memory_state()
    # the calls themselves take no device memory from the driver or torch
    assert after == before, (before, after)

    np.testing.assert_array_equal(outs[0][0].cpu().numpy(), ref_idx)
    np.testing.assert_allclose(outs[0][1].cpu().numpy(), ref_sc, rtol=1e-4, atol=1e-3)
    np.testing.assert_array_equal(outs[0][2].cpu().numpy(), ref_pool.cpu().numpy())
    np.testing.assert_array_equal(outs[1][0].cpu().numpy(), ref_idx2)
    np.testing.assert_allclose(outs[1][1].cpu().numpy(), ref_sc2, rtol=1e-4, atol=1e-3)
    assert csa2.csa2_device_status() == (0, 0)


def test_noalloc_refuses_requests_beyond_its_scratch():
    """Host-side check, no GPU needed: a request whose scratch exceeds the
    fixed array is refused with CSA2_ERR_WORKSPACE before any device work."""
    build.build()
    lib = csa2.load()
    fake = 0x10000
    big = csa2.IndexArgs(mode=0, B=8, Q=1, K=512, N=1 << 20, qI=fake, w=fake, kI=fake, n_vis=fake, idx=fake,
                         scores=None, hsi_blocks=0, hsi_block=8, pool_out=None, pool_in=None)
    assert lib.csa2_workspace_size(ctypes.byref(big), csa2.WS_INDEX) > csa2.noalloc_scratch_bytes()
    assert lib.csa2_index_score_topk_noalloc(ctypes.byref(big), None) == 4


def test_noalloc_scratch_size_matches_the_header():
    """The size compiled into the library is the header's
    CSA2_NOALLOC_SCRATCH_BYTES (no GPU needed)."""
    import os
    import re
    build.build()
    text = open(os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "csa2.h")).read()
    m = re.search(r"#define\s+CSA2_NOALLOC_SCRATCH_BYTES\s+\((\d+)u\s*\*\s*(\d+)u\s*\*\s*(\d+)u\)", text)
    assert m, "CSA2_NOALLOC_SCRATCH_BYTES not found in include/csa2.h"
    header = int(m.group(1)) * int(m.group(2)) * int(m.group(3))
    assert csa2.noalloc_scratch_bytes() == header == 16 * 1024 * 1024
