"""GPU parity of csa2_quantize_kv_fp4 against the oracle: bit-exact bytes."""

import os

import numpy as np
import pytest
import torch

from fp4_kv_cache_mxfp4_b200 import csa2, workloads
from oracle import fp4
from parity import f32

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "fp4_blocks.txt")


def _gpu_quantize(x_bf16, dst_rows=None, row_offset=0, cap=None):
    x = x_bf16.cuda()
    n = x.shape[0]
    rows = cap if cap is not None else n + row_offset
    kv = torch.full((rows, 288), 0xAA, dtype=torch.uint8, device="cuda")
    dr = None if dst_rows is None else torch.as_tensor(dst_rows, dtype=torch.int64).cuda()
    csa2.csa2_quantize_kv_fp4(x, kv, dr, row_offset)
    torch.cuda.synchronize()
    return kv.cpu().numpy()


def test_random_entries_bit_exact():
    wl = workloads.WORKLOADS[0]
    x = workloads.main_kv_rows(wl, 0, 0, 2048)
    got = _gpu_quantize(x)
    want = fp4.quantize_kv_fp4(f32(x))
    np.testing.assert_array_equal(got, want)


def test_golden_blocks_bit_exact():
    blocks = []
    for line in open(GOLDEN):
        line = line.strip()
        if line and not line.startswith("#"):
            blocks.append([float(v) for v in line.split("|")[1].split()])
    x = np.zeros((len(blocks), 512), dtype=np.float32)
    for r, b in enumerate(blocks):
        x[r] = np.tile(b, 32)
    got = _gpu_quantize(torch.from_numpy(x).to(torch.bfloat16))
    np.testing.assert_array_equal(got, fp4.quantize_kv_fp4(x))


def _bf16_from_bits(bits):
    return torch.from_numpy(np.asarray(bits, dtype=np.uint16).view(np.int16)).view(torch.bfloat16)


def test_every_bf16_amax_and_ties():
    """Every positive finite bf16 value is the amax of one block; the other
    15 channels hold fractions of it that land on E2M1 ties and boundaries
    (bf16-rounded), with both signs."""
    amax_bits = np.arange(1, 0x7F80, dtype=np.uint32)          # positive finite, without 0
    n_blocks = -(-amax_bits.size // 32) * 32
    amax_bits = np.concatenate([amax_bits, np.full(n_blocks - amax_bits.size, 0x3F80, np.uint32)])
    amax = _bf16_from_bits(amax_bits).float().numpy()
    fr = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -0.75, -1.25, -1.75, -2.5, -3.5, -5.0, 0.0],
                  dtype=np.float32) / 6.0
    blk = np.concatenate([amax[:, None], amax[:, None] * fr[None, :]], axis=1)
    blk[1::2, 0] *= -1                                           # negative amax in every other block
    x = torch.from_numpy(blk.reshape(-1, 512).astype(np.float32)).to(torch.bfloat16)
    got = _gpu_quantize(x)
    np.testing.assert_array_equal(got, fp4.quantize_kv_fp4(f32(x)))


@pytest.mark.parametrize("seed", [1, 2])
def test_extreme_scales(seed):
    """Scales from E4M3 subnormals / zero to saturation."""
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(4096, 512, generator=g)
    e = torch.randint(-40, 20, (4096, 32, 1), generator=g).float()
    x = (x.view(4096, 32, 16) * torch.exp2(e)).view(4096, 512).to(torch.bfloat16)
    x[7, :17] = 0.0
    x[8, 3] = -0.0
    got = _gpu_quantize(x)
    np.testing.assert_array_equal(got, fp4.quantize_kv_fp4(f32(x)))


def test_scatter_rows_stride_and_ragged_count():
    g = torch.Generator().manual_seed(5)
    base = torch.randn(37, 640, generator=g).to(torch.bfloat16)     # row stride 640 elements
    x = base[:, :512]
    assert x.stride(0) == 640
    dst = np.random.default_rng(0).permutation(100)[:37]
    got = _gpu_quantize(x, dst_rows=dst, cap=100)
    want = fp4.quantize_kv_fp4(f32(x))
    np.testing.assert_array_equal(got[dst], want)
    untouched = np.setdiff1d(np.arange(100), dst)
    assert np.all(got[untouched] == 0xAA)
    got2 = _gpu_quantize(x.contiguous(), row_offset=11)
    np.testing.assert_array_equal(got2[11:], want)
    assert np.all(got2[:11] == 0xAA)


def test_zero_entries_is_a_no_op():
    kv = torch.full((4, 288), 7, dtype=torch.uint8, device="cuda")
    csa2.csa2_quantize_kv_fp4(torch.empty(0, 512, dtype=torch.bfloat16, device="cuda"), kv)
    torch.cuda.synchronize()
    assert torch.all(kv == 7)
