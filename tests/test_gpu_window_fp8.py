"""GPU parity of the FP8 window path ("DeepSeek V4.1-Flash 技术报告深度解析"
§3.4: the SWA KV cache stays FP8) against the oracle:

* csa2_quantize_window_fp8: codes and scales bit-exact against oracle.fp8;
* csa2_sparse_attn with FP8 window rows (oracle-made codes): outputs within
  1e-2 absolute + 1e-2 relative of the float64 oracle on the dequantised
  rows, in each attention mode (slices merged in a cluster, one CTA per
  query, window only);
* csa2_group_decode with the FP8 window on every layer.
"""

import numpy as np
import pytest
import torch

from fp4_kv_cache_mxfp4_b200 import csa2, workloads
from oracle import attention, fp4, fp8
from parity import check_attention, check_topk, f32
from oracle import indexer

pytestmark = pytest.mark.gpu


def _rows(n, seed):
    """bf16 rows with magnitudes from 2^-30 to 2^30 per row, zero rows,
    signed zeros and E4M3 ties (x/s on a midpoint of the grid)."""
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(n, 512, generator=g)
    x = x * torch.exp2(torch.randint(-30, 30, (n, 1), generator=g).float())
    x[0] = 0.0
    x[1, ::2] = -0.0
    x[2, 0] = 448.0
    x[2, 1:40] = torch.tensor([3.375, 3.125, -0.0009765625, 0.0029296875] * 9 + [1.0, 2.0, -2.0])
    return x.to(torch.bfloat16)


def test_window_quantiser_bit_exact():
    x = _rows(3000, 1)
    codes = torch.full((3100, 512), 0xAA, dtype=torch.uint8, device="cuda")
    scales = torch.full((3100,), 7.0, device="cuda")
    csa2.csa2_quantize_window_fp8(x.cuda(), codes, scales, row_offset=50)
    dst = torch.tensor([3099, 7, 3098], dtype=torch.int64, device="cuda")
    csa2.csa2_quantize_window_fp8(x[:3].cuda(), codes, scales, dst_rows=dst)
    torch.cuda.synchronize()
    want_c, want_s = fp8.quantize_window_fp8(f32(x))
    got_c, got_s = codes.cpu().numpy(), scales.cpu().numpy()
    np.testing.assert_array_equal(got_c[50:3050], want_c)
    np.testing.assert_array_equal(got_s[50:3050], want_s)
    np.testing.assert_array_equal(got_c[[3099, 7, 3098]], want_c[:3])
    np.testing.assert_array_equal(got_s[[3099, 7, 3098]], want_s[:3])
    assert np.all(got_c[:7] == 0xAA) and np.all(got_s[:7] == 7.0)


def _attn_case(B, Q, N, K, W, step, seed, q_std=512 ** -0.5):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(B, N, 512, generator=g).to(torch.bfloat16)
    kv = np.stack([fp4.quantize_kv_fp4(f32(x[b])) for b in range(B)])
    q = (torch.randn(B, Q, 64, 512, generator=g) * q_std).to(torch.bfloat16)
    rows = W + (Q - 1) * step
    # N(0, 1) rows (the workloads' distribution) scaled per row by 2^-3..1,
    # so that the row scales differ; bf16 softmax weights bound the error by
    # about 2^-9 max|row|, inside the tolerance for rows of this size
    win = (torch.randn(B, rows, 512, generator=g) * torch.exp2(torch.randint(-3, 1, (B, rows, 1), generator=g).float())
           ).to(torch.bfloat16)
    codes, scales = zip(*[fp8.quantize_window_fp8(f32(win[b])) for b in range(B)])
    rng = np.random.default_rng(seed)
    idx = np.stack([[rng.choice(N, K, replace=False) if K else np.zeros(0, int) for _ in range(Q)]
                    for _ in range(B)]).astype(np.int32).reshape(B, Q, K)
    return kv, q, np.stack(codes), np.stack(scales), idx


@pytest.mark.parametrize("B,Q,N,K,W,step,seed,qs", [
    (4, 1, 3000, 512, 128, 0, 1, 512 ** -0.5),     # slices merged in a cluster
    (1, 2, 800, 300, 100, 1, 2, 512 ** -0.5),      # ragged window, causal step
    (1, 1, 10, 0, 128, 0, 3, 1.0),                 # window only, peaked softmax
    (1, 130, 2000, 256, 128, 1, 4, 512 ** -0.5),   # one CTA per query
])
def test_attention_with_fp8_window(B, Q, N, K, W, step, seed, qs):
    kv, q, codes, scales, idx = _attn_case(B, Q, N, K, W, step, seed, qs)
    d = "cuda"
    out = torch.full((B, Q, 64, 512), float("nan"), dtype=torch.bfloat16, device=d)
    lse = torch.full((B, Q, 64), float("nan"), device=d)
    a = csa2.attn_args(q.to(d), torch.from_numpy(kv).to(d), torch.from_numpy(idx).to(d),
                       torch.from_numpy(codes).to(d), out, lse, W=W, swa_step=step,
                       swa_scale=torch.from_numpy(scales).to(d))
    csa2.csa2_sparse_attn(a, csa2.workspace(a, csa2.WS_ATTN))
    torch.cuda.synchronize()
    o_g, l_g = out.float().cpu().numpy(), lse.cpu().numpy()
    for b in range(B):
        deq = fp4.dequantize_kv_fp4(kv[b])
        wdeq = fp8.dequantize_window_fp8(codes[b], scales[b])
        for i in range(Q):
            o, l = attention.sparse_mqa(f32(q[b, i]), deq, idx[b, i], wdeq[i * step: i * step + W])
            check_attention(o_g[b, i], o, what=f"b{b} q{i}")
            np.testing.assert_allclose(l_g[b, i], l, rtol=1e-3, atol=1e-2)


def test_group_with_fp8_window():
    """Full, Reindex, Reuse over 4000 entries with FP8 windows quantised on
    the GPU (their bytes checked against the oracle first)."""
    wl = workloads.Workload("fp8win_small", 9, B=2, Q=1, N=4000, r=1, modes=[0, 1, 3], n_new=1)
    d = "cuda"
    B, N, K = wl.B, wl.N, wl.K
    kv = torch.empty(B, N, 288, dtype=torch.uint8, device=d)
    xs = [workloads.main_kv_rows(wl, b, 0, N) for b in range(B)]
    for b in range(B):
        csa2.csa2_quantize_kv_fp4(xs[b].to(d), kv[b])
    kI = torch.stack([workloads.index_k(wl, b) for b in range(B)])
    Ls, wins = [], []
    for l, mode in enumerate(wl.modes):
        li = workloads.layer_inputs(wl, l)
        codes = torch.empty(B, wl.swa_rows, 512, dtype=torch.uint8, device=d)
        scales = torch.empty(B, wl.swa_rows, device=d)
        for b in range(B):
            csa2.csa2_quantize_window_fp8(li["swa"][b].to(d), codes[b], scales[b])
        torch.cuda.synchronize()
        for b in range(B):
            wc, ws = fp8.quantize_window_fp8(f32(li["swa"][b]))
            np.testing.assert_array_equal(codes[b].cpu().numpy(), wc)
            np.testing.assert_array_equal(scales[b].cpu().numpy(), ws)
        wins.append([fp8.dequantize_window_fp8(codes[b].cpu().numpy(), scales[b].cpu().numpy()) for b in range(B)])
        Ls.append(dict(mode=mode, qI=li["qI"].to(d), w=li["w"].to(d), q=li["q"].to(d), swa=codes, swa_scale=scales,
                       out=torch.empty(B, 1, 64, 512, dtype=torch.bfloat16, device=d),
                       lse=torch.empty(B, 1, 64, device=d),
                       idx=torch.empty(B, 1, K, dtype=torch.int32, device=d) if mode != 3 else None))
    g = csa2.group_args(B, 1, K, wl.W, N, workloads.n_vis_tensor(wl).to(d), kI.to(d), kv, Ls,
                        swa_rows=wl.swa_rows, swa_format=csa2.FMT_FP8)
    csa2.csa2_group_decode(g, csa2.workspace(g, csa2.WS_GROUP))
    torch.cuda.synchronize()
    assert csa2.csa2_device_status() == (0, 0)
    kv_h = kv.cpu().numpy()
    last = None
    for l, mode in enumerate(wl.modes):
        li = workloads.layer_inputs(wl, l)
        if mode != 3:
            last = Ls[l]["idx"].cpu().numpy()
        for b in range(B):
            if mode != 3:
                s = indexer.index_scores(f32(li["qI"][b, 0]), f32(li["w"][b, 0]), f32(kI[b]), N)
                check_topk(last[b, 0], s, K, what=f"layer {l} b{b}")
            sel = last[b, 0]
            o, lse = attention.sparse_mqa(f32(li["q"][b, 0]), fp4.dequantize_kv_fp4(kv_h[b]), sel, wins[l][b][:wl.W])
            check_attention(Ls[l]["out"][b, 0], o, what=f"layer {l} b{b}")
