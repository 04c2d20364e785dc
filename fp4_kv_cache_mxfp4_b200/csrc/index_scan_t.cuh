// index_scan_t.cuh -- the decode index scan with the entries on the MMA's N
// side ("DeepSeek V4.1-Flash 技术报告深度解析" §3.2 indexer, §3.3 HSI, §3.4
// FP4 indexer Q/K).
//
//   s[t] = sum_h w[h] * ReLU(qI[h, :] . kI[t, :])      (one query per CTA group)
//
// A tcgen05.mma instruction costs about the same issue time whatever its N,
// and a decode query has only 32 heads.  With index-K as the M = 128
// operand (index_scan.cuh) a 128-entry tile takes N = 32; here the
// contraction is transposed, D[(replica, h), t] = qI[h, :] . kI_tile[t, :]:
//   A (M = 128): the query's 32 head rows, repeated in each of the four
//                TMEM lane quarters (rows 32 r + h);
//   B (N = 256): a tile of 256 index-K entries;
// so one instruction covers 256 entries and every lane quarter holds the
// full 32 x 256 head-by-entry block.  Epilogue warp w (lane quarter w % 4)
// takes the entries 64 (w % 4) .. + 63 of the tile: its lane h reads head h's
// values of those entries from TMEM, forms w[h] * ReLU(.), and a butterfly
// over the 32 lanes (31 shuffles per 32 entries) leaves in lane l the sum
// over heads for entry l; scores, histogram and the HSI block max then
// follow as in the other kernel.
//
//   bf16 index-K   stages of 256 x 128 bf16 (64 KB, two 128-byte-swizzled
//                  boxes), 8 x K16 MMAs per tile, two accumulators of 256
//                  columns (the whole TMEM);
//   MXFP4 index-K  raw 192-entry tiles (12.75 KB bulk copies) repacked by
//                  four extra warps into 64-byte-swizzled E2M1 tiles and
//                  two scale chunks; index-Q quantised by the same rule
//                  into the replicated A tile; 2 x K64 block-scaled MMAs
//                  (kind::mxf4) per tile, two accumulators of 192 columns
//                  beside the scale columns (N = 192 leaves tensor memory
//                  for the scales while the MMA of one tile overlaps the
//                  epilogue of the other).
//
// Tiles are claimed, not assigned: CTA c of a query's group starts with
// tile c and then takes the next unclaimed one from the query's counter
// (one atomic per tile, claimed a tile ahead).  Under programmatic
// dependent launch the CTAs whose SMs are still held by the previous
// kernel start tens of microseconds late; with a fixed share of the tiles
// they, not the bandwidth, set the end of the scan.  The producer passes
// each tile's id beside its stage (a negative id ends the stream), the
// MMA thread beside its accumulator.
//
// Warp roles as in index_scan.cuh.  HBM roofline: the same bytes per entry.
#pragma once
#include "index_scan.cuh"

namespace csa2 {

// entries per tile (the MMA's N, and the columns of one accumulator)
__host__ __device__ constexpr int scan_t_tile(bool kf4) { return kf4 ? 192 : 256; }
// bf16: two 128-byte-swizzled boxes of 64 dims; MXFP4: E2M1 rows + two scale chunks
__host__ __device__ constexpr int scan_t_stage_bytes(bool kf4) { return kf4 ? 192 * 64 + 1024 : 256 * 128 * 2; }
constexpr int kTRawBytes = 192 * 68;                 // MXFP4: one raw tile of 68-byte entries

// tensor memory: two accumulators (bf16: all 512 columns; MXFP4: 384, then
// 4 scale columns for index-Q and 8 per stage for the entries)
__host__ __device__ inline uint32_t scan_t_tmem_cols(bool, int) { return 512u; }

struct ScanTSmem {
  uint32_t stage0, raw0, qa0, qi0, sfa0, w0, hist0, bhist0, bar0, tid0, total;
};

// stages / raw_stages: repacked (or bf16) stages and MXFP4 raw tiles
__host__ __device__ inline ScanTSmem scan_t_smem_layout(int stages, int hb, int hsi, bool kf4, int raw_stages) {
  ScanTSmem L;
  uint32_t off = 0;
  L.stage0 = off; off += stages * scan_t_stage_bytes(kf4);
  L.raw0 = off;   off += kf4 ? raw_stages * kTRawBytes : 0;
  off = (off + 1023) & ~1023u;
  L.qa0 = off;    off += kf4 ? 128 * 64 : 128 * 256;       // A: 128 replicated head rows
  L.qi0 = off;    off += kf4 ? 32 * 256 : 0;               // MXFP4: the bf16 head rows (two 32 x 64 boxes)
  L.sfa0 = off;   off += kf4 ? 512 : 0;
  L.w0 = off;     off += 32 * 4;
  L.hist0 = off;  off += (1u << hb) * 4;
  L.bhist0 = off; off += hsi ? (1u << hb) * 4 : 0;
  off = (off + 15) & ~15u;
  L.bar0 = off;   off += (2 * stages + 2 * 2 + 2 * raw_stages + 2) * 8 + 16 + 64;
  L.tid0 = off;   off += (stages + raw_stages + 2) * 4;   // tile ids of the stages, raw tiles, accumulators
  L.total = off;
  return L;
}

template <bool HSI, bool KF4>
__global__ void __launch_bounds__(KF4 ? kScanThreadsF4 : kScanThreads, 1)
index_scan_t_kernel(const __grid_constant__ CUtensorMap tmap_k,
                    const __grid_constant__ CUtensorMap tmap_q,
                    ScanParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr int TILE = scan_t_tile(KF4);
  constexpr int STAGE = scan_t_stage_bytes(KF4);
  constexpr int CPQ = TILE / 4;                    // entries per lane quarter: 64 (bf16) or 48 (MXFP4)
  const int R = KF4 ? p.raw_stages : 0;
  const ScanTSmem L = scan_t_smem_layout(p.stages, p.hb, HSI, KF4, R);
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + L.bar0);
  uint64_t* empty_bar = full_bar + p.stages;
  uint64_t* tfull_bar = empty_bar + p.stages;
  uint64_t* tempty_bar = tfull_bar + 2;
  uint64_t* rfull_bar = tempty_bar + 2;            // MXFP4: raw tile landed
  uint64_t* rempty_bar = rfull_bar + R;            // MXFP4: raw tile repacked
  uint64_t* q_bar = rempty_bar + R;                // index-Q landed
  uint64_t* q4_bar = q_bar + 1;                    // MXFP4: index-Q quantised
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(q_bar + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* w_s = reinterpret_cast<float*>(smem + L.w0);
  uint32_t* hist_s = reinterpret_cast<uint32_t*>(smem + L.hist0);
  uint32_t* bhist_s = reinterpret_cast<uint32_t*>(smem + L.bhist0);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bq0 = blockIdx.x / p.ctas_per_group;     // one query per group: (b, q) = bq0
  const int cig = blockIdx.x % p.ctas_per_group;
  const int b = bq0 / p.Q;
  const int nbins = 1 << p.hb;
  volatile int* stile = reinterpret_cast<volatile int*>(smem + L.tid0);   // tile of each stage
  volatile int* rtile = stile + p.stages;                                 // MXFP4: tile of each raw slot
  volatile int* acc_tile = rtile + R;                                     // tile of each accumulator

  // tiles of this query: [0, tlim); CTA cig takes tile cig first and then
  // claims tiles ctas_per_group, ctas_per_group + 1, ... from the query's
  // counter, so that CTAs that start late (their SM still busy with the
  // previous kernel) take fewer tiles
  const int nv = p.n_vis[bq0];
  const int tlim = p.pool_mode ? p.tiles_per_group : min(p.tiles_per_group, (nv + TILE - 1) / TILE);
  const int first_tile = cig < tlim ? cig : -1;

  uint64_t pol_stream = 0;
  // producer step i: wait for the slot, record the tile (or the end marker,
  // tile < 0), request its index-K
  auto issue = [&](int i, int tile) -> bool {
    if constexpr (KF4) {
      const int r = i % R;
      if (!mbar_wait(&rempty_bar[r], ((i / R) & 1) ^ 1, kErrWaitSmemEmpty, abort_flag)) return false;
      rtile[r] = tile;
      if (tile < 0) { mbar_arrive(&rfull_bar[r]); return true; }
      uint8_t* dst = smem + L.raw0 + r * kTRawBytes;
      if (!p.pool_mode) {
        const int64_t row0 = static_cast<int64_t>(tile) * TILE;
        const uint32_t rows = static_cast<uint32_t>(min(static_cast<int64_t>(TILE), p.N - row0));
        mbar_arrive_expect_tx(&rfull_bar[r], rows * 68u);
        bulk_load(dst, p.k4 + (static_cast<int64_t>(b) * p.N + row0) * 68, rows * 68u, &rfull_bar[r]);
      } else {
        const int32_t* pool = p.pool + static_cast<int64_t>(bq0) * p.pool_blocks;
        mbar_arrive_expect_tx(&rfull_bar[r], (TILE / 8) * 544u);
#pragma unroll 1
        for (int j = 0; j < TILE / 8; ++j) {
          const int slot = tile * (TILE / 8) + j;
          int blk = (slot < p.pool_blocks) ? pool[slot] : -1;
          if (blk < 0) blk = 0;                      // padding slot: load any block, scores masked
          bulk_load(dst + j * 544, p.k4 + (static_cast<int64_t>(b) * p.N + static_cast<int64_t>(blk) * 8) * 68,
                    544u, &rfull_bar[r]);
        }
      }
    } else {
      const int s = i % p.stages;
      if (!mbar_wait(&empty_bar[s], ((i / p.stages) & 1) ^ 1, kErrWaitSmemEmpty, abort_flag)) return false;
      stile[s] = tile;
      if (tile < 0) { mbar_arrive(&full_bar[s]); return true; }
      uint8_t* st = smem + L.stage0 + s * STAGE;
      mbar_arrive_expect_tx(&full_bar[s], STAGE);
      if (!p.pool_mode) {
        const int32_t y = static_cast<int32_t>(static_cast<int64_t>(b) * p.N + static_cast<int64_t>(tile) * TILE);
        tma_load_2d(st, &tmap_k, &full_bar[s], 0, y, pol_stream);
        tma_load_2d(st + STAGE / 2, &tmap_k, &full_bar[s], 64, y, pol_stream);
      } else {
        const int32_t* pool = p.pool + static_cast<int64_t>(bq0) * p.pool_blocks;
#pragma unroll 1
        for (int j = 0; j < TILE / 8; ++j) {
          const int slot = tile * (TILE / 8) + j;
          int blk = (slot < p.pool_blocks) ? pool[slot] : -1;
          if (blk < 0) blk = 0;
          const int32_t y = static_cast<int32_t>(static_cast<int64_t>(b) * p.N + static_cast<int64_t>(blk) * 8);
          tma_load_2d(st + j * 1024, &tmap_k, &full_bar[s], 0, y, pol_stream);
          tma_load_2d(st + STAGE / 2 + j * 1024, &tmap_k, &full_bar[s], 64, y, pol_stream);
        }
      }
    }
    return true;
  };

  // the first tile of a full scan is requested before the block-wide set-up
  // (it needs only the barriers); a pool re-score waits for its pool first
  const bool early_first = !p.pool_mode && first_tile >= 0;
  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) { mbar_init(&full_bar[s], KF4 ? kScanCvtWarps : 1); mbar_init(&empty_bar[s], 1); }
    for (int r = 0; r < R; ++r) { mbar_init(&rfull_bar[r], 1); mbar_init(&rempty_bar[r], kScanCvtWarps); }
    // tfull: the MMA commit and the MMA thread's arrival after it records
    // the accumulator's tile; tempty: the four warps of the epilogue set
    for (int a = 0; a < 2; ++a) { mbar_init(&tfull_bar[a], 2); mbar_init(&tempty_bar[a], 4); }
    mbar_init(q_bar, 1);
    mbar_init(q4_bar, kScanCvtWarps);
    *abort_flag = 0;
    fence_barrier_init();
    if (!KF4) tma_prefetch_desc(&tmap_k);
    tma_prefetch_desc(&tmap_q);
    pol_stream = l2_policy_evict_first();
    if (early_first) issue(0, first_tile);
  }
  if (warp == 1) { tmem_alloc(tmem_slot, p.tmem_cols); tmem_relinquish(); }
  for (int i = threadIdx.x; i < nbins; i += blockDim.x) hist_s[i] = 0;
  if (HSI) for (int i = threadIdx.x; i < nbins; i += blockDim.x) bhist_s[i] = 0;
  // what may start before the predecessor finishes: as in index_scan.cuh
  pdl_launch_dependents();

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && first_tile >= 0) {
      if (p.pool_mode) pdl_wait();
      const uint64_t pol_keep = l2_policy_evict_last();
      // bf16: the 32 head rows straight into the four replicas of each of
      // the A tile's two 128-byte-wide boxes; MXFP4: once, for quantising
      auto load_q = [&]() {
        if constexpr (KF4) {
          uint8_t* qi = smem + L.qi0;
          mbar_arrive_expect_tx(q_bar, 2 * 32 * 128);
          tma_load_2d(qi, &tmap_q, q_bar, 0, bq0 * 32, pol_keep);
          tma_load_2d(qi + 32 * 128, &tmap_q, q_bar, 64, bq0 * 32, pol_keep);
        } else {
          uint8_t* qa = smem + L.qa0;
          mbar_arrive_expect_tx(q_bar, 128 * 256);
#pragma unroll
          for (int c = 0; c < 2; ++c)
#pragma unroll
            for (int rep = 0; rep < 4; ++rep)
              tma_load_2d(qa + c * 16384 + rep * 4096, &tmap_q, q_bar, 64 * c, bq0 * 32, pol_keep);
        }
      };
      bool q_loaded = false;
      if (p.early_q || p.pool_mode) { load_q(); q_loaded = true; }
      // the slots a late index-Q may trail: the consumers free none before it lands
      const int ring = KF4 ? R : p.stages;
      auto claim = [&]() { return p.ctas_per_group + atomicAdd(p.tile_ctr + bq0, 1); };
      int i = 0;
      // producer step with the tile a claim returned: claim again in its
      // place, issue; false once the stream has ended
      auto step = [&](int& c) -> bool {
        const int tile = c < tlim ? c : -1;
        if (tile >= 0) c = claim();
        if (!q_loaded && i == ring) { pdl_wait(); load_q(); q_loaded = true; }
        const bool go = issue(i, tile) && tile >= 0;
        ++i;
        return go;
      };
      bool go = true;
      if (early_first) {
        i = 1;
      } else {
        if (!q_loaded && i == ring) { pdl_wait(); load_q(); q_loaded = true; }
        go = issue(0, first_tile);
        i = 1;
      }
      if constexpr (KF4) {
        // four claims in flight (separate registers, oldest first), so that
        // filling the six-tile raw ring does not wait on one atomic per tile
        int c0 = claim(), c1 = claim(), c2 = claim(), c3 = claim();
        while (go && step(c0) && step(c1) && step(c2) && step(c3)) {}
      } else {
        int c0 = claim();                           // one claim ahead
        while (go && step(c0)) {}
      }
      if (!q_loaded) { pdl_wait(); load_q(); }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && first_tile >= 0) {
      const uint32_t qa_addr = smem_u32(smem + L.qa0);
      const uint32_t sfa_col = tmem_base + 2 * TILE;      // MXFP4 scale columns
      const uint32_t sfb_col = sfa_col + 4;
      // local tile i is the end marker: it closes both epilogue sets
      auto close_sets = [&](int i) {
#pragma unroll 1
        for (int k = 0; k < 2; ++k) {
          const int ii = i + k, a = ii & 1;
          if (k > 0 && !mbar_wait(&tempty_bar[a], ((ii >> 1) & 1) ^ 1, kErrWaitTmemEmpty, abort_flag)) return;
          acc_tile[a] = -1;
          mbar_arrive(&tfull_bar[a]);
          mbar_arrive(&tfull_bar[a]);
        }
      };
      bool have_q = false;
      for (int i = 0;; ++i) {
        const int s = i % p.stages;
        const int a = i & 1;
        if (!mbar_wait(&full_bar[s], (i / p.stages) & 1, kErrWaitTmaFull, abort_flag)) break;
        const int tile = stile[s];
        if (!mbar_wait(&tempty_bar[a], ((i >> 1) & 1) ^ 1, kErrWaitTmemEmpty, abort_flag)) break;
        if (tile < 0) { close_sets(i); break; }
        if (!have_q) {
          if (!mbar_wait(KF4 ? q4_bar : q_bar, 0, kErrWaitOperand, abort_flag)) break;
          have_q = true;
          if constexpr (KF4) {
            tc_fence_after();
            tmem_cp_sf_chunk(sfa_col, umma_desc_sf_chunk(smem_u32(smem + L.sfa0)));
          }
        }
        tc_fence_after();
        const uint32_t st_addr = smem_u32(smem + L.stage0 + s * STAGE);
        if constexpr (KF4) {
          tmem_cp_sf_chunk(sfb_col + 8 * s, umma_desc_sf_chunk(st_addr + TILE * 64));
          tmem_cp_sf_chunk(sfb_col + 8 * s + 4, umma_desc_sf_chunk(st_addr + TILE * 64 + 512));
#pragma unroll
          for (int ks = 0; ks < 2; ++ks)
            umma_mxf4(tmem_base + a * TILE, umma_desc_sw64_kmajor(qa_addr + 32 * ks),
                      umma_desc_sw64_kmajor(st_addr + 32 * ks), umma_idesc_mxf4(128, TILE, 2u * ks), sfa_col,
                      sfb_col + 8 * s, ks > 0 ? 1u : 0u);
        } else {
          constexpr uint32_t idesc = umma_idesc_bf16_f32(128, TILE);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            // K step kk covers dims 16kk..16kk+15: box kk/4, 32-byte column (kk%4)
            umma_bf16(tmem_base + a * TILE, umma_desc_sw128_kmajor(qa_addr + (kk >> 2) * 16384 + (kk & 3) * 32),
                      umma_desc_sw128_kmajor(st_addr + (kk >> 2) * (STAGE / 2) + (kk & 3) * 32), idesc,
                      kk > 0 ? 1u : 0u);
          }
        }
        umma_commit(&empty_bar[s]);
        acc_tile[a] = tile;
        umma_commit(&tfull_bar[a]);
        mbar_arrive(&tfull_bar[a]);
      }
    }
  } else if (KF4 && warp >= 2 + kScanEpiWarps) {
    // ------------------------------------------------------------ MXFP4 repacking
    const int crow = threadIdx.x - 64 - kScanEpiThreads;      // 0..127
    const int Rc = R > 0 ? R : 1;
    // index-Q to MXFP4 (the index-K rule), one (head, 32-value block) per
    // thread, written to the four replica rows of the A tile
    auto quantize_q = [&]() {
      if (mbar_wait(q_bar, 0, kErrWaitOperand, abort_flag)) {
        const int h = crow >> 2, k = crow & 3;
        const uint8_t* box = smem + L.qi0 + (k >> 1) * (32 * 128);
        float v[32];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint4 u = *reinterpret_cast<const uint4*>(box + sw128_off(h, 4 * (k & 1) + c));
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
        const uint32_t ab = __float_as_uint(amax);
        const int fl = ab >= 0x00800000u ? static_cast<int>(ab >> 23) - 127 : (31 - __clz(ab)) - 149;
        const int e = ab ? max(-127, min(127, fl - 2)) : -127;
        const float inv = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);
        uint32_t packed[4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float a = v[2 * j] * inv, c2 = v[2 * j + 1] * inv;
          uint32_t byte = e2m1x2_rn_sat(fabsf(a), fabsf(c2));
          byte |= (__float_as_uint(a) >> 31) << 3;
          byte |= (__float_as_uint(c2) >> 31) << 7;
          packed[j >> 2] |= byte << (8 * (j & 3));
        }
        uint8_t* qa = smem + L.qa0;
        uint8_t* sfa = smem + L.sfa0;
#pragma unroll
        for (int rep = 0; rep < 4; ++rep) {
          const int row = 32 * rep + h;
          *reinterpret_cast<uint4*>(qa + sw64_off(row, k)) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
          sfa[sf_chunk_off(row, k)] = static_cast<uint8_t>(e + 127);
        }
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) mbar_arrive(q4_bar);
    };
    bool q_done = false;
    int t = 0;
    for (; first_tile >= 0; ++t) {
      // a late index-Q: once every stage holds a tile, the MMA needs it to go on
      if (!q_done && t == p.stages) { quantize_q(); q_done = true; }
      const int r = t % Rc, st = t % p.stages;
      bool okc = mbar_wait(&rfull_bar[r], (t / Rc) & 1, kErrWaitTmaFull, abort_flag);
      const int tile = okc ? rtile[r] : -1;
      if (!__all_sync(0xffffffffu, okc)) break;
      if (!q_done && t == 0 && tile >= 0 && (p.early_q || p.pool_mode)) { quantize_q(); q_done = true; }
      okc = mbar_wait(&empty_bar[st], ((t / p.stages) & 1) ^ 1, kErrWaitSmemEmpty, abort_flag);
      if (!__all_sync(0xffffffffu, okc)) break;
      if (tile < 0) {                             // end marker: pass it on to the MMA
        if (crow == 0) stile[st] = -1;
        __syncwarp();
        if (lane == 0) mbar_arrive(&full_bar[st]);
        break;
      }
      uint8_t* stage = smem + L.stage0 + st * STAGE;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int row = crow + 128 * half;          // rows 128.. exist for the first 64 threads
        if (row < TILE) {
          const uint32_t* src = reinterpret_cast<const uint32_t*>(smem + L.raw0 + r * kTRawBytes + row * 68);
          uint32_t wv[17];
#pragma unroll
          for (int k = 0; k < 17; ++k) wv[k] = src[k];
#pragma unroll
          for (int c = 0; c < 4; ++c)
            *reinterpret_cast<uint4*>(stage + sw64_off(row, c)) = make_uint4(wv[4 * c], wv[4 * c + 1], wv[4 * c + 2], wv[4 * c + 3]);
          *reinterpret_cast<uint32_t*>(stage + TILE * 64 + half * 512 + sf_chunk_off(crow, 0)) = wv[16];
        }
      }
      if (crow == 0) stile[st] = tile;
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&full_bar[st]);
        mbar_arrive(&rempty_bar[r]);
      }
    }
    if (!q_done && t > 0) quantize_q();
  } else {
    // ------------------------------------------------------------ epilogue
    pdl_wait();                                   // before w and the first score store
    {
      const int et = threadIdx.x - 64;
      if (et < 32) w_s[et] = p.w[bq0 * 32 + et];
      named_bar_sync(1, kScanEpiThreads);
    }
    const int quarter = warp & 3;                 // TMEM lanes this warp may read: one replica of the heads
    const int set = (warp - 2) >> 2;              // tiles set, set+2, set+4, ...
    const float wr = w_s[lane];                   // lane = head
    const int32_t* pool = p.pool_mode ? p.pool + static_cast<int64_t>(bq0) * p.pool_blocks : nullptr;
    // one group of 32 (or, second group of MXFP4, 16) entries of this
    // warp: lane h's values of head h -> lane l's sum over heads of entry l
    auto score_group = [&](float (&x)[32], int ng, int64_t e0, int tile) {
      if (ng == 32) {
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) {
          const bool upper = (lane & off) != 0;
#pragma unroll
          for (int j = 0; j < off; ++j) {
            const float send = upper ? x[j] : x[j + off];
            const float keep = upper ? x[j + off] : x[j];
            x[j] = keep + __shfl_xor_sync(0xffffffffu, send, off);
          }
        }
      } else {
        // 16 entries: fold lane pairs (l, l ^ 16), then halve over the
        // 16-lane halves; lanes l and l ^ 16 end with entry l & 15
#pragma unroll
        for (int j = 0; j < 16; ++j) x[j] += __shfl_xor_sync(0xffffffffu, x[j], 16);
#pragma unroll
        for (int off = 8; off >= 1; off >>= 1) {
          const bool upper = (lane & off) != 0;
#pragma unroll
          for (int j = 0; j < off; ++j) {
            const float send = upper ? x[j] : x[j + off];
            const float keep = upper ? x[j + off] : x[j];
            x[j] = keep + __shfl_xor_sync(0xffffffffu, send, off);
          }
        }
      }
      const bool owner = ng == 32 || lane < 16;     // the lane that reports its entry
      float s = x[0];
      const int64_t e = e0 + (lane & (ng - 1));     // score slot
      bool pool_valid = true;
      int64_t pos = e;
      if (p.pool_mode) {
        const int64_t slot = e >> 3;
        const int blk = (slot < p.pool_blocks) ? pool[slot] : -1;
        pool_valid = blk >= 0;
        pos = static_cast<int64_t>(blk) * 8 + (e & 7);
      }
      const bool valid = pool_valid && pos < nv;
      if (!valid) s = -INFINITY;
      const bool in_range = e < p.n_elems && owner;
      if (in_range) p.scores[static_cast<int64_t>(bq0) * p.ld + e] = s;
      if (in_range && valid) atomicAdd(&hist_s[okey(s) >> (32 - p.hb)], 1u);
      if (HSI) {
        float m = s;
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
        const int64_t jb = e >> 3;
        const bool writer = owner && (lane & 7) == 0 && jb < p.nblk;
        if (writer) p.bscores[static_cast<int64_t>(bq0) * p.bld + jb] = m;
        warp_hist_add(bhist_s, okey(m) >> (32 - p.hb), writer && m != -INFINITY);
      }
    };
    // local tile i: false at the end marker or a failed wait
    auto epi_tile = [&](int i) -> bool {
      const int a = i & 1;                          // accumulator (and its barriers)
      const bool ok = mbar_wait(&tfull_bar[a], (i >> 1) & 1, kErrWaitTmemFull, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) return false;
      const int tile = acc_tile[a];
      if (tile < 0) return false;
      tc_fence_after();
      // this warp's entries: columns CPQ quarter .. + CPQ - 1 of the accumulator
      const uint32_t col = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + a * TILE + CPQ * quarter;
      uint32_t r0[32], r1[32];
      tmem_ld_32x32b_x32(col, r0);
      if constexpr (CPQ == 64) {
        tmem_ld_32x32b_x32(col + 32, r1);
      } else {
        uint32_t r16[16];
        tmem_ld_32x32b_x16(col + 32, r16);
#pragma unroll
        for (int k = 0; k < 16; ++k) { r1[k] = r16[k]; r1[k + 16] = 0u; }
      }
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty_bar[a]);
      const int64_t e0 = static_cast<int64_t>(tile) * TILE + CPQ * quarter;
      float x[32];
#pragma unroll
      for (int k = 0; k < 32; ++k) x[k] = wr * fmaxf(__uint_as_float(r0[k]), 0.0f);
      score_group(x, 32, e0, tile);
#pragma unroll
      for (int k = 0; k < 32; ++k) x[k] = wr * fmaxf(__uint_as_float(r1[k]), 0.0f);
      score_group(x, CPQ - 32, e0 + 32, tile);
      return true;
    };
    for (int i = set; first_tile >= 0; i += 2)
      if (!epi_tile(i)) break;
    named_bar_sync(1, kScanEpiThreads);
    const int et = threadIdx.x - 64;
    for (int i = et; i < nbins; i += kScanEpiThreads) {
      const uint32_t v = hist_s[i];
      if (v) atomicAdd(&p.hist[static_cast<int64_t>(bq0) * nbins + i], v);
      if (HSI) {
        const uint32_t bv = bhist_s[i];
        if (bv) atomicAdd(&p.bhist[static_cast<int64_t>(bq0) * nbins + i], bv);
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
