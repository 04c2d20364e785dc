// index_scan.cuh -- lightweight-indexer scoring on the 5th-generation tensor
// cores ("DeepSeek V4.1-Flash 技术报告深度解析" §3.2 indexer, §3.3 HSI).
//
//   s[q, t] = sum_h w[q, h] * ReLU(qI[q, h, :] . kI[t, :])
//
// The contraction is D[t, (q,h)] = kI_tile[t, :] . qI[(q,h), :]: a
// 128-entry tile of index-K (128 rows x 128 dims, bf16) is the A operand,
// the row's index-Q (32*QG heads x 128 dims) is the B operand, the fp32
// accumulator (128 lanes x 32*QG columns) lives in tensor memory.  Each
// epilogue thread then owns one entry: it reads its 32*QG head values from
// TMEM and reduces them to QG scores (ReLU, weight, sum).
//
// This kernel serves rows with two or more queries (query blocks, prefill).
// One query per group (decode rows, HSI pool re-scores) runs the transposed
// kernel of index_scan_t.cuh, which shares these parameters and constants.
//
// Warp roles (320 threads; 448 with MXFP4 index-K):
//   warp 0      TMA producer: streams index-K tiles into an S-stage ring
//   warp 1      TMEM allocator + single-thread MMA issuer
//   warps 2..9  epilogue, two sets of four warps taking alternate tiles
//               (each set covers the 128 TMEM lanes): TMEM -> scores, the
//               score histogram used for the top-K threshold and, with HSI,
//               the block max over 8 positions with its own histogram
//   warps 10..13  MXFP4 index-K only: quantise the index-Q tile, then
//               repack each raw tile into the stage the MMA reads, one
//               entry per thread
// After the last tile every CTA adds its histograms to the global ones.
// Pool mode (Reindex restricted to the HSI pool) gathers the tile as 16
// blocks of 8 contiguous index-K rows with one 1 KB TMA box per block half.
//
// MXFP4 index-K (68-byte entries: 64 bytes of E2M1 nibbles, 4 E8M0 block
// scales; "DeepSeek V4.1-Flash 技术报告深度解析" §3.4, where the indexer's
// Q and K are both FP4): the contraction runs on the block-scaled FP4 tensor
// path (tcgen05.mma kind::mxf4, E2M1 x E2M1 with one UE8M0 scale per 32
// values, f32 accumulation), so no value is widened.
//   - index-Q is quantised to the same MXFP4 rule once per CTA by the four
//     extra warps: E2M1 codes in a 64-byte-swizzled tile (the B operand)
//     and its scales in the block-scale chunk layout, copied once into
//     tensor memory;
//   - the producer streams raw tiles (128 entries, 8.5 KB, one bulk copy;
//     pool mode one 544-byte copy per block of 8) into a ring of its own;
//   - the extra warps repack each raw tile: the 64 nibble bytes of entry c
//     become row c of a 64-byte-swizzled 128 x 128 E2M1 tile (the A
//     operand) and its 4 scale bytes go to the tile's scale chunk, which
//     the MMA issuer copies into tensor memory (tcgen05.cp) before the two
//     K = 64 MMAs of the tile.
// E2M1 x E2M1 x 2^(ea + eb) products are exact and the sum is f32, as in
// the bf16 path: the score is that of the dequantised Q and K.
//
// HBM roofline: 256 B (bf16) or 68 B (MXFP4) of index-K per entry per
// (row, layer) + 4 B of score write; index-Q, w and histograms are
// negligible.
#pragma once
#include "common.cuh"

namespace csa2 {

constexpr int kScanEpiWarps = 8;
constexpr int kScanEpiThreads = kScanEpiWarps * 32;
constexpr int kScanThreads = 64 + kScanEpiThreads;
constexpr int kScanCvtWarps = 4;                   // MXFP4 index-K: warps expanding raw tiles, one row per thread
constexpr int kScanThreadsF4 = kScanThreads + kScanCvtWarps * 32;
constexpr int kTileRows = 128;                     // entries per MMA tile (M)
constexpr int kStageBytes = kTileRows * 128 * 2;   // 32 KB: two 128x64 swizzled boxes
constexpr int kAccBufs = 4;                        // TMEM accumulator slots (barriers)
constexpr int kRawStageBytes = kTileRows * 68;     // MXFP4 index-K: one raw tile of 68-byte entries
constexpr int kF4NibBytes = kTileRows * 64;        // MXFP4: repacked E2M1 tile, 128 rows x 64 B
constexpr int kF4StageBytes = kF4NibBytes + 1024;  // + its 512-byte scale chunk, padded to the swizzle alignment
constexpr int kF4MaxQG = 4;                        // MXFP4: queries per MMA group (TMEM room for scales)
constexpr int kF4RawStages = 8;                    // MXFP4: raw tiles in flight per CTA (12-20 measured no faster)

// accumulators in flight: as many as fit the 512 TMEM columns (less the
// block-scale columns of the MXFP4 path), at most 4
__host__ __device__ constexpr int scan_acc_bufs(int QG, bool kf4 = false) {
  return 32 * QG * 4 + (kf4 ? 64 : 0) <= 512 ? 4 : 2;
}
// MXFP4: 512-byte scale chunks (128 rows each) of the index-Q tile
__host__ __device__ constexpr int scan_q_chunks(int QG) { return (32 * QG + 127) / 128; }
// tensor-memory columns: accumulators, then (MXFP4) 4 scale columns per
// stage and per index-Q chunk; a power of two >= 32
__host__ __device__ inline uint32_t scan_tmem_cols(int QG, bool kf4, int stages) {
  uint32_t need = static_cast<uint32_t>(scan_acc_bufs(QG, kf4) * 32 * QG + (kf4 ? 4 * (stages + scan_q_chunks(QG)) : 0));
  uint32_t cols = 32;
  while (cols < need) cols <<= 1;
  return cols;
}

struct ScanParams {
  int pool_mode;          // 0: scan [0, n_vis) of each row; 1: scan the pool of each (b,q)
  int B, Q;               // batch rows, queries per row
  int qg;                 // queries per MMA group: min(Q, QG) (scan) or 1 (pool)
  int qblocks;            // scan: query blocks per batch row, ceil(Q / qg)
  int64_t N;              // index-K rows per batch row
  int64_t n_elems;        // score slots per query: N (scan) or pool_blocks*8 (pool)
  int64_t ld, bld;        // row strides of scores and bscores (multiples of 4)
  const int32_t* n_vis;   // [B*Q]
  const float* w;         // [B*Q*32]
  const int32_t* pool;    // pool mode: [B*Q][pool_blocks]
  int pool_blocks;
  float* scores;          // [B*Q][ld]
  float* bscores;         // scan with HSI: [B*Q][bld]
  int64_t nblk;
  uint32_t* hist;         // [B*Q][1 << hb]       (zero at launch)
  uint32_t* bhist;        // scan with HSI: [B*Q][1 << hb]
  int hb;                 // histogram bits
  int hist_every;         // the score histogram counts tiles with tile % hist_every == 0
  int groups;             // B*qblocks (scan) or B*Q (pool)
  int tiles_per_group;
  int ctas_per_group;
  int stages;
  uint32_t tmem_cols;
  int early_q;            // 1: index-Q and w are complete at launch (load them before waiting on
                          // the predecessor); 0: they may be the predecessor's results
  const uint8_t* k4;      // MXFP4 index-K: [B*N][68] entries (N a multiple of 4)
  int raw_stages;         // MXFP4 index-K: raw tiles in flight
  int* tile_ctr;          // one query per group: [groups] tiles claimed past the first
                          // ctas_per_group (zero at launch)
};

struct ScanSmem {
  // offsets inside the dynamic shared memory block
  uint32_t stage0, raw0, qi0, q40, sfb0, w0, hist0, bhist0, bar0, total;
};

// raw_stages: MXFP4 index-K raw tiles (0 for bf16 index-K, which also
// selects the bf16 stage size)
__host__ __device__ inline ScanSmem scan_smem_layout(int stages, int QG, int hb, int hsi, int raw_stages = 0) {
  ScanSmem L;
  const bool kf4 = raw_stages > 0;
  uint32_t off = 0;
  L.stage0 = off; off += stages * (kf4 ? kF4StageBytes : kStageBytes);
  L.raw0 = off;   off += raw_stages * kRawStageBytes;
  off = (off + 1023) & ~1023u;                          // swizzled operand tiles start on 1 KB
  L.qi0 = off;    off += 2 * (32 * QG) * 128;          // two 64-dim halves of [32*QG x 64] bf16
  L.q40 = off;    off += kf4 ? (32 * QG) * 64 : 0;     // MXFP4 index-Q, [32*QG x 64 B] swizzled
  L.sfb0 = off;   off += kf4 ? scan_q_chunks(QG) * 512 : 0;
  L.w0 = off;     off += QG * 32 * 4;
  L.hist0 = off;  off += QG * (1u << hb) * 4;
  L.bhist0 = off; off += hsi ? QG * (1u << hb) * 4 : 0;
  off = (off + 15) & ~15u;
  L.bar0 = off;   off += (2 * stages + 2 * kAccBufs + 2 * raw_stages + 2) * 8 + 16 + 64;   // barriers, TMEM slot, flags
  L.total = off;
  return L;
}

template <int QG, bool HSI, bool KF4>
__global__ void __launch_bounds__(KF4 ? kScanThreadsF4 : kScanThreads, 1)
index_scan_kernel(const __grid_constant__ CUtensorMap tmap_k,
                  const __grid_constant__ CUtensorMap tmap_q,
                  ScanParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // the swizzle atoms need 1024-byte alignment of every operand tile
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int R = KF4 ? p.raw_stages : 0;
  const ScanSmem L = scan_smem_layout(p.stages, QG, p.hb, HSI, R);
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + L.bar0);
  uint64_t* empty_bar = full_bar + p.stages;
  uint64_t* tfull_bar = empty_bar + p.stages;
  uint64_t* tempty_bar = tfull_bar + kAccBufs;
  uint64_t* rfull_bar = tempty_bar + kAccBufs;     // MXFP4: raw tile landed
  uint64_t* rempty_bar = rfull_bar + R;            // MXFP4: raw tile expanded
  uint64_t* q_bar = rempty_bar + R;
  uint64_t* q4_bar = q_bar + 1;                    // MXFP4: index-Q quantised
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(q_bar + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* w_s = reinterpret_cast<float*>(smem + L.w0);
  uint32_t* hist_s = reinterpret_cast<uint32_t*>(smem + L.hist0);
  uint32_t* bhist_s = reinterpret_cast<uint32_t*>(smem + L.bhist0);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int group = blockIdx.x / p.ctas_per_group;
  const int cig = blockIdx.x % p.ctas_per_group;
  // batch row and first query of this MMA group
  const int b = p.pool_mode ? group / p.Q : group / p.qblocks;
  const int q0 = p.pool_mode ? group % p.Q : (group % p.qblocks) * p.qg;
  const int bq0 = b * p.Q + q0;              // first (b,q) of the group
  const int qn = p.pool_mode ? 1 : min(p.qg, p.Q - q0);   // queries of this group
  const int nbins = 1 << p.hb;

  if (threadIdx.x == 0) {
    // with MXFP4 index-K a stage is full once every repacking warp has
    // written its part of the tile; arrivals from several warps come one
    // per warp (lane 0, after a warp barrier), not one per thread
    for (int s = 0; s < p.stages; ++s) { mbar_init(&full_bar[s], KF4 ? kScanCvtWarps : 1); mbar_init(&empty_bar[s], 1); }
    for (int r = 0; r < R; ++r) { mbar_init(&rfull_bar[r], 1); mbar_init(&rempty_bar[r], kScanCvtWarps); }
    for (int a = 0; a < scan_acc_bufs(QG, KF4); ++a) { mbar_init(&tfull_bar[a], 1); mbar_init(&tempty_bar[a], 4); }
    mbar_init(q_bar, 1);
    mbar_init(q4_bar, kScanCvtWarps);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) { if (!KF4) tma_prefetch_desc(&tmap_k); tma_prefetch_desc(&tmap_q); }
  if (warp == 1) { tmem_alloc(tmem_slot, p.tmem_cols); tmem_relinquish(); }
  for (int i = threadIdx.x; i < QG * nbins; i += blockDim.x) hist_s[i] = 0;
  if (HSI) for (int i = threadIdx.x; i < QG * nbins; i += blockDim.x) bhist_s[i] = 0;

  // Index-K and n_vis are the caller's cache and step metadata: complete
  // before this kernel can start (its predecessor is the call's memset node
  // or a kernel of this library that waited for everything before it), so
  // the first index-K tiles are requested at once.  What waits for the
  // predecessor: index-Q and w unless early_q (in a model they come from
  // the previous layer's output), the HSI pool (a previous top-K wrote it)
  // and every global store (the score buffer is shared with the previous
  // layer's top-K).
  pdl_launch_dependents();

  // this CTA's tile range; in scan mode, tiles past every query's n_vis are skipped
  int tile_lo = static_cast<int>((static_cast<int64_t>(cig) * p.tiles_per_group) / p.ctas_per_group);
  int tile_hi = static_cast<int>((static_cast<int64_t>(cig + 1) * p.tiles_per_group) / p.ctas_per_group);
  int nv[QG];
#pragma unroll
  for (int q = 0; q < QG; ++q) nv[q] = (q < qn) ? p.n_vis[bq0 + q] : 0;
  if (!p.pool_mode) {
    int nmax = 0;
#pragma unroll
    for (int q = 0; q < QG; ++q) nmax = max(nmax, nv[q]);
    tile_hi = min(tile_hi, (nmax + kTileRows - 1) / kTileRows);
  }
  const int ntiles = max(0, tile_hi - tile_lo);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  constexpr uint32_t n_mma = 32u * QG;
  constexpr int ACC = scan_acc_bufs(QG, KF4);
  static_assert(!KF4 || QG <= kF4MaxQG, "MXFP4 index-K: at most 4 queries per MMA group");

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && ntiles > 0) {
      if (p.pool_mode) pdl_wait();
      const uint64_t pol_stream = l2_policy_evict_first();
      const uint64_t pol_keep = l2_policy_evict_last();
      uint8_t* qi = smem + L.qi0;
      constexpr uint32_t qbox = n_mma * 128;
      auto load_q = [&]() {
        mbar_arrive_expect_tx(q_bar, 2 * qbox);
        tma_load_2d(qi, &tmap_q, q_bar, 0, bq0 * 32, pol_keep);
        tma_load_2d(qi + qbox, &tmap_q, q_bar, 64, bq0 * 32, pol_keep);
      };
      // index-Q before the tiles when it is complete; otherwise after the
      // first ring of index-K tiles is in flight and the predecessor is done
      const bool q_late = !p.early_q && !p.pool_mode;
      if (!q_late) load_q();
      if constexpr (KF4) {
        // raw MXFP4 tiles: one bulk copy per tile (its valid rows), or one
        // per pool block of 8 entries
        for (int i = 0; i < ntiles; ++i) {
          const int r = i % R;
          if (q_late && i == min(R, ntiles)) { pdl_wait(); load_q(); }
          if (!mbar_wait(&rempty_bar[r], ((i / R) & 1) ^ 1, kErrWaitSmemEmpty, abort_flag)) break;
          uint8_t* dst = smem + L.raw0 + r * kRawStageBytes;
          const int tile = tile_lo + i;
          if (!p.pool_mode) {
            const int64_t row0 = static_cast<int64_t>(tile) * kTileRows;
            const uint32_t rows = static_cast<uint32_t>(min(static_cast<int64_t>(kTileRows), p.N - row0));
            mbar_arrive_expect_tx(&rfull_bar[r], rows * 68u);
            bulk_load(dst, p.k4 + (static_cast<int64_t>(b) * p.N + row0) * 68, rows * 68u, &rfull_bar[r]);
          } else {
            const int32_t* pool = p.pool + static_cast<int64_t>(bq0) * p.pool_blocks;
            mbar_arrive_expect_tx(&rfull_bar[r], (kTileRows / 8) * 544u);
#pragma unroll 1
            for (int j = 0; j < kTileRows / 8; ++j) {
              const int slot = tile * (kTileRows / 8) + j;
              int blk = (slot < p.pool_blocks) ? pool[slot] : -1;
              if (blk < 0) blk = 0;                  // padding slot: load any block, scores masked
              bulk_load(dst + j * 544, p.k4 + (static_cast<int64_t>(b) * p.N + static_cast<int64_t>(blk) * 8) * 68,
                        544u, &rfull_bar[r]);
            }
          }
        }
        if (q_late && ntiles <= R) { pdl_wait(); load_q(); }
      }
      for (int i = 0; !KF4 && i < ntiles; ++i) {
        const int s = i % p.stages;
        const uint32_t ph = (i / p.stages) & 1;
        if (q_late && i == min(p.stages, ntiles)) { pdl_wait(); load_q(); }
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
      if (!KF4 && q_late && ntiles <= p.stages) { pdl_wait(); load_q(); }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (KF4 && lane == 0 && ntiles > 0) {
      // block-scaled FP4: per tile, its scale chunk into this stage's 4
      // scale columns, then two K = 64 MMAs (scale bytes 0-1, then 2-3)
      const uint32_t sfa_col = tmem_base + ACC * n_mma;
      const uint32_t sfb_col = sfa_col + 4 * p.stages;
      const uint32_t q4_addr = smem_u32(smem + L.q40);
      bool ok = mbar_wait(q4_bar, 0, kErrWaitOperand, abort_flag);
      if (ok) {
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < scan_q_chunks(QG); ++c)
          tmem_cp_sf_chunk(sfb_col + 4 * c, umma_desc_sf_chunk(smem_u32(smem + L.sfb0 + 512 * c)));
      }
      for (int i = 0; ok && i < ntiles; ++i) {
        const int s = i % p.stages;
        const int a = i % ACC;
        if (!mbar_wait(&tempty_bar[a], ((i / ACC) & 1) ^ 1, kErrWaitTmemEmpty, abort_flag)) break;
        if (!mbar_wait(&full_bar[s], (i / p.stages) & 1, kErrWaitTmaFull, abort_flag)) break;
        tc_fence_after();
        const uint32_t st_addr = smem_u32(smem + L.stage0 + s * kF4StageBytes);
        const uint32_t d_tmem = tmem_base + a * n_mma;
        tmem_cp_sf_chunk(sfa_col + 4 * s, umma_desc_sf_chunk(st_addr + kF4NibBytes));
#pragma unroll
        for (int ks = 0; ks < 2; ++ks)
          umma_mxf4(d_tmem, umma_desc_sw64_kmajor(st_addr + 32 * ks), umma_desc_sw64_kmajor(q4_addr + 32 * ks),
                    umma_idesc_mxf4(128, n_mma, 2u * ks), sfa_col + 4 * s, sfb_col, ks > 0 ? 1u : 0u);
        umma_commit(&empty_bar[s]);
        umma_commit(&tfull_bar[a]);
      }
    }
    if (!KF4 && lane == 0 && ntiles > 0) {
      constexpr uint32_t idesc = umma_idesc_bf16_f32(128, n_mma);
      const uint32_t qi_addr = smem_u32(smem + L.qi0);
      constexpr uint32_t qbox = n_mma * 128;
      bool ok = mbar_wait(q_bar, 0, kErrWaitOperand, abort_flag);
      for (int i = 0; ok && i < ntiles; ++i) {
        const int s = i % p.stages;
        const int a = i % ACC;
        if (!mbar_wait(&tempty_bar[a], ((i / ACC) & 1) ^ 1, kErrWaitTmemEmpty, abort_flag)) break;
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
  } else if (KF4 && warp >= 2 + kScanEpiWarps) {
    // ------------------------------------------------------------ MXFP4 repacking
    const int crow = threadIdx.x - 64 - kScanEpiThreads;      // 0..127
    const int Rc = R > 0 ? R : 1;                  // R >= 2 here (this role exists with MXFP4 index-K only)
    // index-Q to MXFP4 (the index-K rule: e = floor(log2 amax) - 2 per 32
    // values, q = E2M1(x / 2^e)), one (head row, 32-value block) per thread
    auto quantize_q = [&]() {
      if (mbar_wait(q_bar, 0, kErrWaitOperand, abort_flag)) {
        constexpr uint32_t qbox = n_mma * 128;
        const uint8_t* qi = smem + L.qi0;
        uint8_t* q4 = smem + L.q40;
        uint8_t* sfb = smem + L.sfb0;
        for (int item = crow; item < static_cast<int>(n_mma) * 4; item += kScanCvtWarps * 32) {
          const int rr = item >> 2, k = item & 3;
          const uint8_t* box = qi + (k >> 1) * qbox;
          float v[32];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint4 u = *reinterpret_cast<const uint4*>(box + sw128_off(rr, 4 * (k & 1) + c));
            const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&uw[j]));
              v[8 * c + 2 * j] = f.x;
              v[8 * c + 2 * j + 1] = f.y;
            }
          }
          float amax = 0.0f;
#pragma unroll
          for (int j = 0; j < 32; ++j) amax = fmaxf(amax, fabsf(v[j]));
          // floor(log2 amax) from the bits (a bf16 value: normal, subnormal or 0)
          const uint32_t ab = __float_as_uint(amax);
          const int fl = ab >= 0x00800000u ? static_cast<int>(ab >> 23) - 127 : (31 - __clz(ab)) - 149;
          const int e = ab ? max(-127, min(127, fl - 2)) : -127;
          // 2^-e is a normal float (e <= 125 for bf16 inputs); x * 2^-e is
          // exact unless it underflows, where E2M1 gives 0 either way
          const float inv = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);
          uint32_t packed[4] = {0u, 0u, 0u, 0u};
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float a = v[2 * j] * inv, b = v[2 * j + 1] * inv;
            uint32_t byte = e2m1x2_rn_sat(fabsf(a), fabsf(b));
            byte |= (__float_as_uint(a) >> 31) << 3;
            byte |= (__float_as_uint(b) >> 31) << 7;
            packed[j >> 2] |= byte << (8 * (j & 3));
          }
          *reinterpret_cast<uint4*>(q4 + sw64_off(rr, k)) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
          sfb[(rr >> 7) * 512 + sf_chunk_off(rr & 127, k)] = static_cast<uint8_t>(e + 127);
        }
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) mbar_arrive(q4_bar);
    };
    // index-Q first when it is there from the start; otherwise (it may
    // arrive only once the previous kernel has finished) the first ring of
    // stages is repacked before it is needed
    bool q_done = false;
    if (ntiles > 0 && (p.early_q || p.pool_mode)) { quantize_q(); q_done = true; }
    for (int t = 0; t < ntiles; ++t) {
      if (!q_done && t == min(p.stages, ntiles)) { quantize_q(); q_done = true; }
      const int r = t % Rc, st = t % p.stages;
      bool okc = mbar_wait(&rfull_bar[r], (t / Rc) & 1, kErrWaitTmaFull, abort_flag);
      okc = okc && mbar_wait(&empty_bar[st], ((t / p.stages) & 1) ^ 1, kErrWaitSmemEmpty, abort_flag);
      if (!__all_sync(0xffffffffu, okc)) break;
      const uint32_t* src = reinterpret_cast<const uint32_t*>(smem + L.raw0 + r * kRawStageBytes + crow * 68);
      uint32_t wv[17];
#pragma unroll
      for (int k = 0; k < 17; ++k) wv[k] = src[k];
      uint8_t* stage = smem + L.stage0 + st * kF4StageBytes;
#pragma unroll
      for (int c = 0; c < 4; ++c)
        *reinterpret_cast<uint4*>(stage + sw64_off(crow, c)) = make_uint4(wv[4 * c], wv[4 * c + 1], wv[4 * c + 2], wv[4 * c + 3]);
      // the entry's scale bytes are its 4 K blocks in order: one word
      *reinterpret_cast<uint32_t*>(stage + kF4NibBytes + sf_chunk_off(crow, 0)) = wv[16];
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&full_bar[st]);
        mbar_arrive(&rempty_bar[r]);
      }
    }
    if (!q_done && ntiles > 0) quantize_q();       // with no tiles nothing loads index-Q
  } else {
    // ------------------------------------------------------------ epilogue
    pdl_wait();                                   // before w and the first score store
    {
      const int et = threadIdx.x - 64;
      for (int i = et; i < QG * 32; i += kScanEpiThreads) w_s[i] = (i < qn * 32) ? p.w[bq0 * 32 + i] : 0.0f;
      named_bar_sync(1, kScanEpiThreads);
    }
    const int quarter = warp & 3;                 // TMEM lanes this warp may read
    const int set = (warp - 2) >> 2;              // tiles set, set+2, set+4, ...
    const int row = quarter * 32 + lane;          // entry within the tile
    const int32_t* pool = p.pool_mode ? p.pool + static_cast<int64_t>(bq0) * p.pool_blocks : nullptr;
    // the weights of one or two queries stay in registers
    constexpr int WREG = (QG <= 2) ? QG * 32 : 1;
    float wr[WREG];
#pragma unroll
    for (int h = 0; h < WREG; ++h) wr[h] = (QG <= 2) ? w_s[h] : 0.0f;
    // one tile's accumulator -> scores, histograms (false: a wait gave up)
    auto epi_tile = [&](int i) -> bool {
      const int a = i % ACC;
      // tcgen05.ld is warp-collective: leave the loop as a whole warp
      const bool ok = mbar_wait(&tfull_bar[a], (i / ACC) & 1, kErrWaitTmemFull, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) return false;
      tc_fence_after();
      const int tile = tile_lo + i;
      const int64_t e = static_cast<int64_t>(tile) * kTileRows + row;   // score slot
      bool pool_valid = true;
      int64_t pos = e;
      if (p.pool_mode) {
        const int64_t slot = e >> 3;
        const int blk = (slot < p.pool_blocks) ? pool[slot] : -1;
        pool_valid = blk >= 0;
        pos = static_cast<int64_t>(blk) * 8 + (e & 7);
      }
      // QB queries' head values per TMEM round trip: the loads of a batch
      // are in flight together and one wait covers them
      constexpr int QB = (QG >= 4) ? (HSI ? 2 : 4) : QG;
#pragma unroll
      for (int qb = 0; qb < QG; qb += QB) {
        uint32_t r[QB][32];
#pragma unroll
        for (int j = 0; j < QB; ++j)
          tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + a * n_mma + 32 * (qb + j), r[j]);
        tmem_ld_wait();
        if (qb + QB >= QG) {
          // every head value of the tile is in registers: hand the
          // accumulator back to the MMA issuer before the reductions
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty_bar[a]);
        }
#pragma unroll
        for (int j = 0; j < QB; ++j) {
          const int q = qb + j;
          float acc[4] = {0.f, 0.f, 0.f, 0.f};
          if (QG <= 2) {
#pragma unroll
            for (int h = 0; h < 32; ++h)
              acc[h & 3] = fmaf(wr[(QG <= 2 ? q : 0) * 32 + h], fmaxf(__uint_as_float(r[j][h]), 0.0f), acc[h & 3]);
          } else {
            const float4* w4 = reinterpret_cast<const float4*>(w_s + q * 32);
#pragma unroll
            for (int h4 = 0; h4 < 8; ++h4) {
              const float4 wv = w4[h4];
              acc[0] = fmaf(wv.x, fmaxf(__uint_as_float(r[j][4 * h4 + 0]), 0.0f), acc[0]);
              acc[1] = fmaf(wv.y, fmaxf(__uint_as_float(r[j][4 * h4 + 1]), 0.0f), acc[1]);
              acc[2] = fmaf(wv.z, fmaxf(__uint_as_float(r[j][4 * h4 + 2]), 0.0f), acc[2]);
              acc[3] = fmaf(wv.w, fmaxf(__uint_as_float(r[j][4 * h4 + 3]), 0.0f), acc[3]);
            }
          }
          float s = (acc[0] + acc[1]) + (acc[2] + acc[3]);
          const bool valid = pool_valid && pos < nv[q] && q < qn;
          if (!valid) s = -INFINITY;
          const bool in_range = e < p.n_elems && q < qn;
          if (in_range) p.scores[static_cast<int64_t>(bq0 + q) * p.ld + e] = s;
          if (tile % p.hist_every == 0) {               // uniform over the warp
            // decode scores rarely share a bin: one shared atomic per
            // score; with query blocks (prefill, many near-equal scores)
            // the warp's increments of a bin are combined first
            const uint32_t bin = okey(s) >> (32 - p.hb);
            if (QG <= 2) {
              if (in_range && valid) atomicAdd(&hist_s[q * nbins + bin], 1u);
            } else {
              warp_hist_add(hist_s + q * nbins, bin, in_range && valid);
            }
          }
          if (HSI) {
            float m = s;
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
            const int64_t jb = e >> 3;
            const bool writer = (lane & 7) == 0 && jb < p.nblk && q < qn;
            if (writer) p.bscores[static_cast<int64_t>(bq0 + q) * p.bld + jb] = m;
            warp_hist_add(bhist_s + q * nbins, okey(m) >> (32 - p.hb), writer && m != -INFINITY);
          }
        }
      }
      return true;
    };
    for (int i = set; i < ntiles; i += 2)
      if (!epi_tile(i)) break;
    // flush the CTA's histograms into the global ones
    named_bar_sync(1, kScanEpiThreads);
    const int et = threadIdx.x - 64;
    for (int i = et; i < qn * nbins; i += kScanEpiThreads) {
      const uint32_t v = hist_s[i];
      if (v) atomicAdd(&p.hist[static_cast<int64_t>(bq0 + i / nbins) * nbins + (i % nbins)], v);
      if (HSI) {
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
