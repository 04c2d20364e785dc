"""Seeded synthetic workloads for CSA2 decode / prefill over an FP4 main KV.

This module only draws random inputs and describes shapes; it holds none of
the method's arithmetic (no quantisation, scoring, selection or attention),
so both the CUDA path and the CPU oracle can be fed from it.

Distributions (the pages' workloads are long-context agent traces; no data
set is involved): main-KV entries, index-K, index-Q and SWA rows ~ N(0, 1),
query heads ~ N(0, 1/512), per-head indexer weights ~ U(0, 1).  All tensors
are drawn on the CPU with torch's Philox-free CPU generator so that every
consumer sees identical bytes.

Streams: shared caches of workload c come from seed c (main KV in 65,536-row
chunks, each chunk from its own derived seed so any rows can be regenerated
alone); the inputs of layer l come from seed 1000*c + 100 + l.
"""

from dataclasses import dataclass, field
from typing import List

import torch

FULL, REINDEX, REINDEX_POOL, REUSE = 0, 1, 2, 3
MODE_NAMES = {FULL: "full", REINDEX: "reindex", REINDEX_POOL: "reindex_pool", REUSE: "reuse"}

D = 512        # main-KV / attention head dim
H = 64         # attention heads
H_I = 32       # indexer heads
D_I = 128      # indexer head dim
ENTRY_BYTES = 288
KV_CHUNK = 65536


@dataclass
class Workload:
    name: str
    seed: int
    B: int                 # batch rows (independent sequences)
    Q: int                 # query positions per row
    N: int                 # main-KV entries per row (visible to the last query)
    r: int                 # compression ratio (tokens per entry)
    modes: List[int]
    K: int = 512
    W: int = 128
    hsi_blocks: int = 0    # 0 = no HSI pool
    hsi_block: int = 8
    n_new: int = 1         # entries quantised into each row at the start of a step
    prefill: bool = False  # causal queries over the tail (n_vis per query)
    swa_step: int = 0      # window of query i starts at row i*swa_step
    desc: str = ""
    n_vis: List[int] = field(default_factory=list)   # per query, filled in __post_init__
    groups: List[int] = field(default_factory=list)  # layers per sharing group (default: one group)
    cache_per_group: bool = False  # each group has its own main KV and index-K (encoder), else one
                                   # cache for all groups (decoder)
    index_k_format: int = 0        # 0: bf16 index-K; 2: 68-byte MXFP4 entries
    window_format: int = 0         # 0: bf16 window rows; 1: E4M3 codes + one f32 scale per row

    def __post_init__(self):
        if not self.groups:
            self.groups = [len(self.modes)]
        assert sum(self.groups) == len(self.modes)
        if not self.n_vis:
            if self.prefill:
                # query i sits at token p0 + i, with p0 = (N - n_new) * r; entry e
                # (tokens [e*r, (e+1)*r)) is visible once all its tokens are
                p0 = (self.N - self.n_new) * self.r
                self.n_vis = [(p0 + i + 1) // self.r for i in range(self.Q)]
            else:
                self.n_vis = [self.N] * self.Q

    @property
    def swa_rows(self):
        return self.W + (self.Q - 1) * self.swa_step

    def group_layers(self, g):
        """Indices (into modes) of the layers of group g."""
        start = sum(self.groups[:g])
        return list(range(start, start + self.groups[g]))

    def cache_of_group(self, g):
        """The workload whose seed draws group g's shared caches: the same
        one for every group of a decoder stack, a derived seed per group of
        an encoder stack."""
        if not self.cache_per_group or g == 0:
            return self
        return Workload(**{**self.__dict__, "seed": self.seed + 97 * g, "n_vis": list(self.n_vis),
                           "groups": list(self.groups)})

    @property
    def new_rows(self):
        """Rows (within each batch row's cache) written at the start of a step."""
        return list(range(self.N - self.n_new, self.N))


WORKLOADS = {
    0: Workload("tiny_full_decode_ctx2k_b1_q4", 0, B=1, Q=4, N=2048, r=1, modes=[FULL], n_new=4,
                desc="Full-mode decode, batch 1, 4 query positions, 2048 entries"),
    1: Workload("full_decode_r2_ctx64k_b8", 1, B=8, Q=1, N=32768, r=2, modes=[FULL], n_new=1,
                desc="Full-mode decode, batch 8, 64K tokens at r=2 (32,768 entries)"),
    2: Workload("group4_decode_ctx128k_b4", 2, B=4, Q=1, N=131072, r=1,
                modes=[FULL, REINDEX, REINDEX, REUSE], n_new=1,
                desc="Decoder group Full, Reindex, Reindex, Reuse at 128K entries, batch 4"),
    3: Workload("hsi_decode_ctx1m_b2", 3, B=2, Q=1, N=1048576, r=1,
                modes=[FULL, REINDEX_POOL, REINDEX_POOL, REINDEX_POOL], hsi_blocks=2048, n_new=1,
                desc="Full + HSI pool (2048 x 8) then 3 pool-restricted Reindex layers at 1M entries, batch 2"),
    4: Workload("prefill_t4096_prefix256k_r2", 4, B=1, Q=4096, N=131072 + 2048, r=2, modes=[FULL],
                n_new=2048, prefill=True, swa_step=1,
                desc="Prefill chunk of 4096 tokens after a 256K-token prefix at r=2, causal"),
    6: Workload("decoder20_q5_ctx128k_b4", 6, B=4, Q=5, N=131072, r=1,
                modes=[FULL, REUSE, REUSE, REUSE] + [REINDEX_POOL, REUSE, REUSE, REUSE] * 4, groups=[4] * 5,
                hsi_blocks=2048, n_new=5, prefill=True, swa_step=1,
                desc="The decoder's 20 CSA2 layers as 5 groups over one 128K-entry cache (group 1: Full + HSI "
                     "pool + 3 Reuse; groups 2-5: pool Reindex + 3 Reuse), 5 query positions per row "
                     "(a verified draft block), batch 4"),
    7: Workload("encoder18_q5_ctx64k_r2_b4", 7, B=4, Q=5, N=32768, r=2,
                modes=([FULL] + [REUSE] * 5) * 3, groups=[6] * 3, cache_per_group=True, n_new=2,
                prefill=True, swa_step=1,
                desc="The encoder's 18 CSA2 layers as 3 groups (Full + 5 Reuse), each group with its own "
                     "cache of 32,768 entries (64K tokens at r=2), 5 query positions per row, batch 4"),
    8: Workload("group4_decode_ctx128k_b4_mxfp4ik_fp8win", 2, B=4, Q=1, N=131072, r=1,
                modes=[FULL, REINDEX, REINDEX, REUSE], n_new=1, index_k_format=2, window_format=1,
                desc="The decoder group of workload 2 (same draws) with the pages' other precisions: index-K "
                     "as 68-byte MXFP4 entries and FP8 window rows"),
    5: Workload("prefill_t1024_prefix64k_r2", 5, B=1, Q=1024, N=32768 + 512, r=2, modes=[FULL],
                n_new=512, prefill=True, swa_step=1,
                desc="Prefill chunk of 1024 tokens after a 64K-token prefix at r=2, causal: the prefill "
                     "kernels at a size small enough for full profiler captures"),
}


def _gen(seed):
    g = torch.Generator()
    g.manual_seed(int(seed))
    return g


def _kv_chunk_seed(wl, b, chunk):
    return (wl.seed * 1_000_003 + b * 7919 + chunk) * 2 + 1


def main_kv_rows(wl, b, start, count):
    """bf16 [count, 512] main-KV entries (already rotated) of batch row b,
    rows [start, start+count).  New-entry rows are drawn like any other."""
    out = torch.empty(count, D, dtype=torch.bfloat16)
    r = start
    while r < start + count:
        chunk = r // KV_CHUNK
        c0 = chunk * KV_CHUNK
        n_chunk = min(KV_CHUNK, wl.N - c0)
        x = torch.randn(n_chunk, D, generator=_gen(_kv_chunk_seed(wl, b, chunk))).to(torch.bfloat16)
        lo = r - c0
        hi = min(n_chunk, start + count - c0)
        out[r - start: r - start + hi - lo] = x[lo:hi]
        r = c0 + hi
    return out


def index_k(wl, b):
    """bf16 [N, 128] index-K of batch row b."""
    return torch.randn(wl.N, D_I, generator=_gen(wl.seed * 31 + 17 + b * 1_000_033)).to(torch.bfloat16)


def layer_inputs(wl, layer):
    """Per-layer inputs for all batch rows: qI bf16 [B,Q,32,128], w f32 [B,Q,32],
    q bf16 [B,Q,64,512], swa bf16 [B,swa_rows,512]."""
    g = _gen(1000 * wl.seed + 100 + layer)
    qI = torch.randn(wl.B, wl.Q, H_I, D_I, generator=g).to(torch.bfloat16)
    w = torch.rand(wl.B, wl.Q, H_I, generator=g, dtype=torch.float32)
    q = (torch.randn(wl.B, wl.Q, H, D, generator=g) / (D ** 0.5)).to(torch.bfloat16)
    swa = torch.randn(wl.B, wl.swa_rows, D, generator=g).to(torch.bfloat16)
    return {"qI": qI, "w": w, "q": q, "swa": swa}


def n_vis_tensor(wl):
    """int32 [B, Q] visible entries per query."""
    return torch.tensor([wl.n_vis] * wl.B, dtype=torch.int32)
