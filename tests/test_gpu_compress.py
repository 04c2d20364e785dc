"""GPU parity of csa2_compress_rope_quantize_kv_fp4 against the oracle:
packed FP4 entries bit-exact ("DeepSeek V4.1-Flash 技术报告深度解析" §3.2
compression of r tokens per entry, §3.4 quantisation after RoPE)."""

import numpy as np
import pytest
import torch

from fp4_kv_cache_mxfp4_b200 import csa2
from oracle import compress, fp4
from parity import f32

pytestmark = pytest.mark.gpu


def _inputs(n, r, seed, shared, spread=8):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(n * r, 512, generator=g)
    x = (x * torch.exp2(torch.randint(-spread, spread + 1, (n * r, 1), generator=g).float())).to(torch.bfloat16)
    x[0, :7] = -0.0
    if shared:
        w = torch.rand(1, r, 512, generator=g) * 2 - 0.5
    else:
        w = torch.softmax(torch.randn(n, r, 1, generator=g), dim=1).expand(n, r, 512).contiguous()
    w[..., 3] = 0.0                                    # zero weights: signed-zero products
    th = torch.rand(n, 32, generator=g, dtype=torch.float64) * 2 * np.pi - np.pi
    cos, sin = torch.cos(th).float(), torch.sin(th).float()
    return x, w.float(), cos, sin


@pytest.mark.parametrize("n,r,shared", [(3000, 2, False), (2500, 2, True), (700, 1, False), (333, 4, True)])
def test_fused_entries_bit_exact(n, r, shared):
    x, w, cos, sin = _inputs(n, r, n + r, shared)
    kv = torch.full((n + 40, 288), 0xAA, dtype=torch.uint8, device="cuda")
    csa2.csa2_compress_rope_quantize_kv_fp4(x.cuda(), r, w.cuda(), cos.cuda(), sin.cuda(), kv, row_offset=40)
    torch.cuda.synchronize()
    want = compress.compress_rope_quantize(f32(x), w.numpy(), r, cos.numpy(), sin.numpy())
    got = kv.cpu().numpy()
    np.testing.assert_array_equal(got[40:], want)
    assert np.all(got[:40] == 0xAA)


def test_identity_case_equals_the_plain_quantiser_on_the_gpu():
    """r = 1, unit weights, zero angles: the same bytes as csa2_quantize_kv_fp4."""
    x, _, _, _ = _inputs(1000, 1, 9, True)
    w = torch.ones(1, 1, 512)
    cos, sin = torch.ones(1000, 32), torch.zeros(1000, 32)
    a = torch.zeros(1000, 288, dtype=torch.uint8, device="cuda")
    b = torch.zeros(1000, 288, dtype=torch.uint8, device="cuda")
    csa2.csa2_compress_rope_quantize_kv_fp4(x.cuda(), 1, w.cuda(), cos.cuda(), sin.cuda(), a)
    csa2.csa2_quantize_kv_fp4(x.cuda(), b)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    np.testing.assert_array_equal(a.cpu().numpy(), fp4.quantize_kv_fp4(f32(x)))


def test_scattered_destinations():
    x, w, cos, sin = _inputs(64, 2, 11, False)
    rows = torch.randperm(500, generator=torch.Generator().manual_seed(3))[:64].to(torch.int64)
    kv = torch.zeros(500, 288, dtype=torch.uint8, device="cuda")
    csa2.csa2_compress_rope_quantize_kv_fp4(x.cuda(), 2, w.cuda(), cos.cuda(), sin.cuda(), kv, dst_rows=rows.cuda())
    torch.cuda.synchronize()
    want = compress.compress_rope_quantize(f32(x), w.numpy(), 2, cos.numpy(), sin.numpy())
    np.testing.assert_array_equal(kv.cpu().numpy()[rows.numpy()], want)
