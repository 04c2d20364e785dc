// index_scan.cuh -- lightweight-indexer scoring on the 5th-generation tensor
// cores ("DeepSeek V4.1-Flash 技术报告深度解析" §3.2 indexer, §3.3 HSI).
//
//   s[q, t] = sum_h w[q, h] * ReLU(qI[q, h, :] . kI[t, :])
//
// The contraction is D[t, (q,h)] = kI_tile[t, :] . qI[(q,h), :]: a
// 128-entry tile of index-K (128 rows x 128 dims, bf16) is the A operand,
// the row's index-Q (32*Q heads x 128 dims) is the B operand, the fp32
// accumulator (128 lanes x 32*Q columns) lives in tensor memory.  Each
// epilogue thread then owns one entry: it reads its 32*Q head values from
// TMEM and reduces them to Q scores (ReLU, weight, sum).
//
// Warp roles (192 threads):
//   warp 0      TMA producer: streams index-K tiles into an S-stage ring
//   warp 1      TMEM allocator + single-thread MMA issuer
//   warps 2..5  epilogue: TMEM -> scores, fused score histogram (for the
//               top-K threshold) and, with HSI, the block max over 8
//               positions with its own histogram
// Pool mode (Reindex restricted to the HSI pool) gathers the tile as 16
// blocks of 8 contiguous index-K rows with one 1 KB TMA box per block half.
//
// HBM roofline: 256 B of index-K per entry per (row, layer) + 4 B of score
// write; index-Q, w and histograms are negligible.
#pragma once
#include "common.cuh"

namespace csa2 {

constexpr int kScanThreads = 192;
constexpr int kTileRows = 128;               // entries per MMA tile (M)
constexpr int kStageBytes = kTileRows * 128 * 2;   // 32 KB: two 128x64 swizzled boxes

struct ScanParams {
  int pool_mode;          // 0: scan [0, n_vis) of each row; 1: scan the pool of each (b,q)
  int B, Q;               // batch rows, queries per row
  int qg;                 // queries per MMA group: Q (scan) or 1 (pool)
  int64_t N;              // index-K rows per batch row
  int64_t n_elems;        // score slots per query: N (scan) or pool_blocks*8 (pool)
  const int32_t* n_vis;   // [B*Q]
  const float* w;         // [B*Q*32]
  const int32_t* pool;    // pool mode: [B*Q][pool_blocks]
  int pool_blocks;
  float* scores;          // [B*Q][n_elems]
  float* bscores;         // scan with HSI: [B*Q][nblk]
  int64_t nblk;
  uint32_t* hist;         // [B*Q][1 << hb]
  uint32_t* bhist;        // scan with HSI: [B*Q][1 << hb]
  int hb;                 // histogram bits
  int groups;             // B (scan) or B*Q (pool)
  int tiles_per_group;
  int ctas_per_group;
  int stages;
  int acc_bufs;
  uint32_t tmem_cols;
};

struct ScanSmem {
  // offsets inside the dynamic shared memory block
  uint32_t stage0, qi0, w0, hist0, bhist0, bar0, total;
};

__host__ __device__ inline ScanSmem scan_smem_layout(int stages, int qg, int hb, int hsi) {
  ScanSmem L;
  uint32_t off = 0;
  L.stage0 = off; off += stages * kStageBytes;
  L.qi0 = off;    off += 2 * (32 * qg) * 128;          // two 64-dim halves of [32*qg x 64] bf16
  L.w0 = off;     off += qg * 32 * 4;
  L.hist0 = off;  off += qg * (1u << hb) * 4;
  L.bhist0 = off; off += hsi ? qg * (1u << hb) * 4 : 0;
  off = (off + 15) & ~15u;
  L.bar0 = off;   off += (2 * stages + 2 * 4 + 2) * 8 + 16;
  L.total = off;
  return L;
}

__global__ void __launch_bounds__(kScanThreads, 1)
index_scan_kernel(const __grid_constant__ CUtensorMap tmap_k,
                  const __grid_constant__ CUtensorMap tmap_q,
                  ScanParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // the swizzle atoms need 1024-byte alignment of every operand tile
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int hsi = (p.bscores != nullptr);
  const ScanSmem L = scan_smem_layout(p.stages, p.qg, p.hb, hsi);
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + L.bar0);
  uint64_t* empty_bar = full_bar + p.stages;
  uint64_t* tfull_bar = empty_bar + p.stages;
  uint64_t* tempty_bar = tfull_bar + 4;
  uint64_t* q_bar = tempty_bar + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(q_bar + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* w_s = reinterpret_cast<float*>(smem + L.w0);
  uint32_t* hist_s = reinterpret_cast<uint32_t*>(smem + L.hist0);
  uint32_t* bhist_s = reinterpret_cast<uint32_t*>(smem + L.bhist0);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int group = blockIdx.x / p.ctas_per_group;
  const int cig = blockIdx.x % p.ctas_per_group;
  // batch row and first query of this MMA group
  const int b = p.pool_mode ? group / p.Q : group;
  const int q0 = p.pool_mode ? group % p.Q : 0;
  const int bq0 = b * p.Q + q0;              // first (b,q) of the group
  const int nbins = 1 << p.hb;

  // this CTA's tile range; in scan mode, tiles past every query's n_vis are skipped
  int tile_lo = static_cast<int>((static_cast<int64_t>(cig) * p.tiles_per_group) / p.ctas_per_group);
  int tile_hi = static_cast<int>((static_cast<int64_t>(cig + 1) * p.tiles_per_group) / p.ctas_per_group);
  if (!p.pool_mode) {
    int nmax = 0;
    for (int q = 0; q < p.qg; ++q) nmax = max(nmax, p.n_vis[bq0 + q]);
    tile_hi = min(tile_hi, (nmax + kTileRows - 1) / kTileRows);
  }
  const int ntiles = max(0, tile_hi - tile_lo);

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) { mbar_init(&full_bar[s], 1); mbar_init(&empty_bar[s], 1); }
    for (int a = 0; a < p.acc_bufs; ++a) { mbar_init(&tfull_bar[a], 1); mbar_init(&tempty_bar[a], 128); }
    mbar_init(q_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) { tma_prefetch_desc(&tmap_k); tma_prefetch_desc(&tmap_q); }
  if (warp == 1) { tmem_alloc(tmem_slot, p.tmem_cols); tmem_relinquish(); }
  for (int i = threadIdx.x; i < p.qg * nbins; i += blockDim.x) hist_s[i] = 0;
  if (hsi) for (int i = threadIdx.x; i < p.qg * nbins; i += blockDim.x) bhist_s[i] = 0;
  for (int i = threadIdx.x; i < p.qg * 32; i += blockDim.x) w_s[i] = p.w[bq0 * 32 + i];
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t n_mma = 32u * p.qg;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && ntiles > 0) {
      const uint64_t pol_stream = l2_policy_evict_first();
      const uint64_t pol_keep = l2_policy_evict_last();
      uint8_t* qi = smem + L.qi0;
      const uint32_t qbox = n_mma * 128;
      mbar_arrive_expect_tx(q_bar, 2 * qbox);
      tma_load_2d(qi, &tmap_q, q_bar, 0, bq0 * 32, pol_keep);
      tma_load_2d(qi + qbox, &tmap_q, q_bar, 64, bq0 * 32, pol_keep);
      for (int i = 0; i < ntiles; ++i) {
        const int s = i % p.stages;
        const uint32_t ph = (i / p.stages) & 1;
        if (!mbar_wait(&empty_bar[s], ph ^ 1, kErrWaitSmemEmpty, abort_flag)) break;
        uint8_t* st = smem + L.stage0 + s * kStageBytes;
        mbar_arrive_expect_tx(&full_bar[s], kStageBytes);
        const int tile = tile_lo + i;
        if (!p.pool_mode) {
          const int32_t y = static_cast<int32_t>(static_cast<int64_t>(b) * p.N + static_cast<int64_t>(tile) * kTileRows);
          tma_load_2d(st, &tmap_k, &full_bar[s], 0, y, pol_stream);
          tma_load_2d(st + kStageBytes / 2, &tmap_k, &full_bar[s], 64, y, pol_stream);
        } else {
          const int32_t* pool = p.pool + static_cast<int64_t>(bq0) * p.pool_blocks;
#pragma unroll 1
          for (int j = 0; j < kTileRows / 8; ++j) {
            const int slot = tile * (kTileRows / 8) + j;
            int blk = (slot < p.pool_blocks) ? pool[slot] : -1;
            if (blk < 0) blk = 0;                    // padding slot: load any block, scores masked
            const int32_t y = static_cast<int32_t>(static_cast<int64_t>(b) * p.N + static_cast<int64_t>(blk) * 8);
            tma_load_2d(st + j * 1024, &tmap_k, &full_bar[s], 0, y, pol_stream);
            tma_load_2d(st + kStageBytes / 2 + j * 1024, &tmap_k, &full_bar[s], 64, y, pol_stream);
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && ntiles > 0) {
      const uint32_t idesc = umma_idesc_bf16_f32(128, n_mma);
      const uint32_t qi_addr = smem_u32(smem + L.qi0);
      const uint32_t qbox = n_mma * 128;
      bool ok = mbar_wait(q_bar, 0, kErrWaitOperand, abort_flag);
      for (int i = 0; ok && i < ntiles; ++i) {
        const int s = i % p.stages;
        const int a = i % p.acc_bufs;
        if (!mbar_wait(&tempty_bar[a], ((i / p.acc_bufs) & 1) ^ 1, kErrWaitTmemEmpty, abort_flag)) break;
        if (!mbar_wait(&full_bar[s], (i / p.stages) & 1, kErrWaitTmaFull, abort_flag)) break;
        tc_fence_after();
        const uint32_t st_addr = smem_u32(smem + L.stage0 + s * kStageBytes);
        const uint32_t d_tmem = tmem_base + a * n_mma;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          // K step kk covers dims 16kk..16kk+15: half kk/4, 32-byte column (kk%4)
          const uint32_t koff = (kk >> 2) * (kStageBytes / 2) + (kk & 3) * 32;
          const uint32_t qoff = (kk >> 2) * qbox + (kk & 3) * 32;
          umma_bf16(d_tmem, umma_desc_sw128_kmajor(st_addr + koff),
                    umma_desc_sw128_kmajor(qi_addr + qoff), idesc, kk > 0 ? 1u : 0u);
        }
        umma_commit(&empty_bar[s]);
        umma_commit(&tfull_bar[a]);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;                 // TMEM lanes this warp may read
    const int row = quarter * 32 + lane;          // entry within the tile
    int nv[8];
    for (int q = 0; q < p.qg; ++q) nv[q] = p.n_vis[bq0 + q];
    const int32_t* pool = p.pool_mode ? p.pool + static_cast<int64_t>(bq0) * p.pool_blocks : nullptr;
    for (int i = 0; i < ntiles; ++i) {
      const int a = i % p.acc_bufs;
      // tcgen05.ld is warp-collective: leave the loop as a whole warp
      const bool ok = mbar_wait(&tfull_bar[a], (i / p.acc_bufs) & 1, kErrWaitTmemFull, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const int tile = tile_lo + i;
      const int64_t e = static_cast<int64_t>(tile) * kTileRows + row;   // score slot
      for (int q = 0; q < p.qg; ++q) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + a * n_mma + 32 * q, r);
        tmem_ld_wait();
        float s = 0.0f;
        const float* wq = w_s + 32 * q;
#pragma unroll
        for (int h = 0; h < 32; ++h) s = fmaf(wq[h], fmaxf(__uint_as_float(r[h]), 0.0f), s);
        bool valid;
        if (!p.pool_mode) {
          valid = e < nv[q];
        } else {
          const int64_t slot = e >> 3;
          const int blk = (slot < p.pool_blocks) ? pool[slot] : -1;
          valid = blk >= 0 && (static_cast<int64_t>(blk) * 8 + (e & 7)) < nv[q];
        }
        if (!valid) s = -INFINITY;
        if (e < p.n_elems) {
          p.scores[static_cast<int64_t>(bq0 + q) * p.n_elems + e] = s;
          if (valid) atomicAdd(&hist_s[q * nbins + (okey(s) >> (32 - p.hb))], 1u);
        }
        if (hsi) {
          float m = s;
          m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
          m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
          m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
          const int64_t jb = e >> 3;
          if ((lane & 7) == 0 && jb < p.nblk) {
            p.bscores[static_cast<int64_t>(bq0 + q) * p.nblk + jb] = m;
            if (m != -INFINITY) atomicAdd(&bhist_s[q * nbins + (okey(m) >> (32 - p.hb))], 1u);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty_bar[a]);
    }
    // flush the CTA's histograms into the global ones
    named_bar_sync(1, 128);
    const int et = threadIdx.x - 64;
    for (int i = et; i < p.qg * nbins; i += 128) {
      const uint32_t v = hist_s[i];
      if (v) atomicAdd(&p.hist[static_cast<int64_t>(bq0 + i / nbins) * nbins + (i % nbins)], v);
      if (hsi) {
        const uint32_t bv = bhist_s[i];
        if (bv) atomicAdd(&p.bhist[static_cast<int64_t>(bq0 + i / nbins) * nbins + (i % nbins)], bv);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, p.tmem_cols);
  }
}

}  // namespace csa2
