// topk.cuh -- exact top-K selection with ties to the lower position
// ("DeepSeek V4.1-Flash 技术报告深度解析" §3.2 top-512, §3.3 top-2048 blocks).
//
// Keys: key64 = okey(score) << 32 | ~position.  okey orders floats, the low
// word inverts the position, so every key is distinct and "larger key" means
// "higher score, then lower position": the top-K set is the K largest keys.
//
// One thread-block cluster of C CTAs per selection problem (grid (C,
// queries), 512 threads per CTA); CTA r of the cluster owns the r-th of C
// contiguous slices of the query's slots, and warp w of a CTA the w-th of
// 16 contiguous ranges of its slice.
//  0. every CTA reads the query's score histogram (built by the scan
//     epilogue, coalesced) and finds the threshold bin tb, the highest bin
//     whose suffix count reaches need = min(K, visible): every top-K key has
//     its top bits >= tb;
//  1. every warp streams its range in 2 KB bulk copies through its own
//     three-stage ring (issued before the histogram is read) and compacts
//     the keys whose bin is >= tb into its own region, in position order
//     (four ballots per vector, no block-wide barrier); the warp lists are
//     then joined into the CTA's list;
//  2. the CTAs exchange their counts over distributed shared memory and push
//     their lists into the cluster's first CTA (in slice order, so the list
//     stays in position order), which radix-selects the need-th largest key
//     (8-bit digits) and writes the keys at or above it by an ordered
//     compaction: the result comes out in ascending position order,
//     deterministically, without a sort.
// If the candidates do not fit (massive ties) or an estimated threshold
// fails, step 2 runs over the scores themselves with the same filter
// (slower, exact).
// HBM roofline: 4 B per score read (normally still resident in L2).
#pragma once
#include <cooperative_groups.h>
#include "common.cuh"

namespace csa2 {

namespace cg = cooperative_groups;

constexpr int kTopkThreads = 512;
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr int kTopkVec = 4;                                  // float4 per lane per chunk
constexpr int kTopkWarpSlots = 32 * 4 * kTopkVec;            // 512 slots (2 KB) per warp chunk
constexpr int kTopkStages = 3;                               // chunks in flight per warp (bulk copies)
constexpr int kTopkWarpCap = 768;                            // candidates a warp may hold (kTopkCap / 16)
constexpr int kTopkCap = 12288;                             // candidate keys a CTA holds (the cluster's total)
constexpr int kTopkMaxCluster = 16;                         // 16 needs the non-portable cluster attribute

struct TopkParams {
  const float* scores;      // [BQ][ld]
  int64_t ld;               // row stride of scores, a multiple of 4
  int64_t n_elems;          // score slots per query
  const int32_t* n_vis;     // optional [BQ]: valid slots = ceil(n_vis / vis_div)
  int vis_div;
  const int32_t* pool;      // pool mode: position of slot e = pool[e/8]*8 + e%8
  int pool_blocks;
  const uint32_t* hist;     // [BQ][1 << hb] score histogram from the scan
  int hb;
  int hist_sample;          // 1: exact histogram; s > 1: it counts one tile in s, so the threshold
                            // is an estimate (with a margin on the count), checked against the
                            // exact candidate count before it is used
  int K;
  int32_t* out_idx;         // [BQ][K]
  float* out_scores;        // optional [BQ][K]
  const uint8_t* prefetch_kv;  // optional [B][prefetch_N][288]: FP4 rows the attention reads next,
  int64_t prefetch_N;          // pulled into L2 as their indices are written
  int Q;                       // queries per batch row (bq / Q = batch row)
};

struct TopkShared {
  uint32_t h256[256];
  uint32_t warp_tot[kTopkWarps];
  uint32_t cnt[kTopkMaxCluster];   // candidates found by each CTA of the cluster
  int d, gt, eq, total, tb, above;  // above: visible slots in bins higher than tb
  int abort_flag;
  uint32_t wcnt[kTopkWarps];                 // candidates found by each warp
  alignas(8) uint64_t wbar[kTopkWarps][kTopkStages];
};

__device__ __forceinline__ int64_t topk_valid_slots(const TopkParams& p, int bq) {
  if (!p.n_vis) return p.n_elems;
  const int64_t v = (static_cast<int64_t>(max(p.n_vis[bq], 0)) + p.vis_div - 1) / p.vis_div;
  return min(v, p.n_elems);
}

__device__ __forceinline__ uint32_t topk_position(const TopkParams& p, int bq, int64_t e) {
  if (!p.pool) return static_cast<uint32_t>(e);
  const int blk = p.pool[static_cast<int64_t>(bq) * p.pool_blocks + (e >> 3)];
  return static_cast<uint32_t>(blk * 8 + static_cast<int>(e & 7));
}

// is score s a candidate: visible (not -inf) and in bin tb or above
__device__ __forceinline__ bool topk_is_cand(float s, int tb, int hb) {
  return s != -INFINITY && static_cast<int>(okey(s) >> (32 - hb)) >= tb;
}

__device__ __forceinline__ uint64_t topk_make_key(const TopkParams& p, int bq, int64_t e, float s) {
  return (static_cast<uint64_t>(okey(s)) << 32) | static_cast<uint32_t>(~topk_position(p, bq, e));
}

// key of slot e, or 0 when the slot holds no visible score or sits below tb
__device__ __forceinline__ uint64_t topk_slot_key(const TopkParams& p, int bq, int64_t e, int tb) {
  const float s = p.scores[static_cast<int64_t>(bq) * p.ld + e];
  return topk_is_cand(s, tb, p.hb) ? topk_make_key(p, bq, e, s) : 0;
}

// Exclusive prefix sum over the block; *total gets the sum.  Ends with a
// barrier so the scratch can be reused.
__device__ __forceinline__ uint32_t topk_block_scan(uint32_t v, TopkShared& S, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) S.warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const uint32_t x = (lane < kTopkWarps) ? S.warp_tot[lane] : 0;
    uint32_t xi = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_up_sync(0xffffffffu, xi, o);
      if (lane >= o) xi += t;
    }
    if (lane < kTopkWarps) S.warp_tot[lane] = xi - x;   // exclusive per warp
    if (lane == 31) S.total = static_cast<int>(xi);
  }
  __syncthreads();
  const uint32_t r = S.warp_tot[warp] + incl - v;
  *total = static_cast<uint32_t>(S.total);
  __syncthreads();
  return r;
}

// Highest digit d of the 256-bin histogram with suffix(d) >= remaining, run
// by warp 0; lane l owns bins 255-8l .. 248-8l.
__device__ __forceinline__ void topk_pick_digit(TopkShared& S, int remaining) {
  const int lane = threadIdx.x & 31;
  uint32_t c[8], local = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) { c[i] = S.h256[255 - 8 * lane - i]; local += c[i]; }
  uint32_t incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  const uint32_t excl = incl - local;
  if (excl < static_cast<uint32_t>(remaining) && incl >= static_cast<uint32_t>(remaining)) {
    uint32_t acc = excl;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (acc + c[i] >= static_cast<uint32_t>(remaining)) {
        S.d = 255 - 8 * lane - i; S.gt = acc; S.eq = c[i];
        break;
      }
      acc += c[i];
    }
  }
}

// Radix select over a key source: returns P such that the keys >= P are
// exactly the `need` largest (keys are distinct; key 0 means "absent").
// The caller knows the top `bits0` bits of the need-th key (its histogram
// bin), `prefix0` holding them, and that `above` keys lie strictly above
// that bin: the passes only look at keys sharing the prefix.
// AGG: aggregate equal digits per warp before the shared atomic (for key
// sources that may hold long runs of equal keys, as the fallback does).
template <bool AGG, class KeyAt>
__device__ uint64_t topk_radix_select(TopkShared& S, int64_t n, int need, int bits0, uint64_t prefix0, int above,
                                      KeyAt key_at) {
  uint64_t prefix = prefix0;
  int bits = bits0, remaining = need - above;
  while (true) {
    const int width = min(8, 64 - bits);
    const int shift = 64 - bits - width;
    for (int i = threadIdx.x; i < 256; i += blockDim.x) S.h256[i] = 0;
    if (threadIdx.x == 0) S.d = -1;
    __syncthreads();
    for (int64_t i0 = 0; i0 < n; i0 += blockDim.x) {
      const int64_t i = i0 + threadIdx.x;
      const uint64_t k = (i < n) ? key_at(i) : 0;
      const bool act = k != 0 && (bits == 0 || (k >> (64 - bits)) == (prefix >> (64 - bits)));
      const uint32_t digit = static_cast<uint32_t>((k >> shift) & ((1u << width) - 1));
      if (AGG) warp_hist_add(S.h256, digit, act);
      else if (act) atomicAdd(&S.h256[digit], 1u);       // digits below the threshold bin spread out
    }
    __syncthreads();
    if (threadIdx.x < 32) topk_pick_digit(S, remaining);
    __syncthreads();
    if (S.d < 0) { if (threadIdx.x == 0) record_error(kErrSelectCount); return prefix; }
    prefix |= static_cast<uint64_t>(S.d) << shift;
    bits += width;
    remaining -= S.gt;
    const bool done = (S.eq == remaining) || bits == 64;
    __syncthreads();
    if (done) return prefix;
  }
}

__device__ __forceinline__ void prefetch_l2(const void* ptr) {
  asm volatile("prefetch.global.L2 [%0];" :: "l"(ptr));
}

__device__ __forceinline__ void topk_emit(const TopkParams& p, int bq, int32_t* out_idx, float* out_sc, uint32_t slot,
                                          uint64_t k) {
  if (slot >= static_cast<uint32_t>(p.K)) return;
  const int32_t pos = static_cast<int32_t>(~static_cast<uint32_t>(k));
  out_idx[slot] = pos;
  if (out_sc) out_sc[slot] = okey_to_float(static_cast<uint32_t>(k >> 32));
  if (p.prefetch_kv && pos >= 0 && pos < p.prefetch_N) {
    // the 288-byte row spans three or four 128-byte lines
    const uint8_t* row = p.prefetch_kv + (static_cast<int64_t>(bq / p.Q) * p.prefetch_N + pos) * 288;
    prefetch_l2(row);
    prefetch_l2(row + 128);
    prefetch_l2(row + 256);
    prefetch_l2(row + 287);
  }
}

__device__ __forceinline__ void fence_async_smem_generic() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__global__ void __launch_bounds__(kTopkThreads, 1)
topk_select_kernel(TopkParams p) {
  extern __shared__ __align__(1024) uint8_t topk_smem_raw[];
  TopkShared& S = *reinterpret_cast<TopkShared*>(topk_smem_raw);
  uint64_t* keys_s = reinterpret_cast<uint64_t*>(topk_smem_raw + ((sizeof(TopkShared) + 15) & ~size_t(15)));
  cg::cluster_group cluster = cg::this_cluster();
  const int C = static_cast<int>(cluster.num_blocks());
  const int rank = static_cast<int>(cluster.block_rank());

  // every CTA of the cluster must have started before another one writes
  // its shared memory: arrive now, wait just before the first remote store
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");

  const int bq = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_launch_dependents();
  pdl_wait();
  const float* row = p.scores + static_cast<int64_t>(bq) * p.ld;
  // stage ring [warp][stage][512 floats]; after streaming the same bytes hold
  // the CTA's contiguous candidate list (kTopkCap keys)
  float* ring_s = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(keys_s) + static_cast<size_t>(kTopkCap) * 8);
  uint64_t* cand_s = reinterpret_cast<uint64_t*>(ring_s);

  // this CTA's slice of the slots, cut into 16 contiguous warp ranges; each
  // warp streams its range in 512-slot chunks through its own ring of bulk
  // copies and compacts its candidates into its own region of keys_s, in
  // position order, without block-wide barriers.  Slices split all n_elems
  // slots, so the first copies go out before the visible count arrives;
  // slots at or past it are masked afterwards.
  const int64_t span = (((p.n_elems + C - 1) / C) + 3) & ~static_cast<int64_t>(3);
  const int64_t lo = min(p.n_elems, static_cast<int64_t>(rank) * span);
  const int64_t hi_copy = min(p.n_elems, lo + span);   // copies stay inside the slice's padded row
  const int64_t wspan = (((hi_copy - lo + kTopkWarps - 1) / kTopkWarps) + 3) & ~static_cast<int64_t>(3);
  const int64_t wlo = min(hi_copy, lo + warp * wspan);
  const int64_t whi_copy = min(hi_copy, wlo + wspan);
  float* wring = ring_s + warp * kTopkStages * kTopkWarpSlots;
  uint64_t* wbar = S.wbar[warp];
  auto issue_chunk = [&](int64_t c0, int k) {          // lane 0: chunk at slot c0 into stage k % kTopkStages
    if (c0 >= whi_copy) return;
    const int st = k % kTopkStages;
    const uint32_t n4 = static_cast<uint32_t>(min(static_cast<int64_t>(kTopkWarpSlots), whi_copy - c0) + 3) & ~3u;
    mbar_arrive_expect_tx(&wbar[st], n4 * 4);
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        :: "r"(smem_u32(wring + st * kTopkWarpSlots)), "l"(row + c0), "r"(n4 * 4), "r"(smem_u32(&wbar[st]))
        : "memory");
  };
  if (lane == 0) {
    for (int k = 0; k < kTopkStages; ++k) mbar_init(&wbar[k], 1);
    fence_barrier_init();
    for (int k = 0; k < kTopkStages; ++k) issue_chunk(wlo + static_cast<int64_t>(k) * kTopkWarpSlots, k);
  }
  if (tid == 0) S.abort_flag = 0;
  const int64_t nvalid = topk_valid_slots(p, bq);
  const int64_t whi = min(whi_copy, nvalid);

  // -- 0. threshold bin: thread t owns the `per` bins just below bin
  //       nbins - per*t (descending ranges), read with coalesced loads
  int need;
  {
    const int nbins = 1 << p.hb;
    const int per = nbins / kTopkThreads;             // 8 (12-bit), 4 (11-bit) or 2 (10-bit)
    const uint32_t* hq = p.hist + static_cast<int64_t>(bq) * nbins;
    const int lo_bin = nbins - per * (tid + 1);
    uint32_t c[8];
    if (per == 8) {
      const uint4 v0 = __ldcg(reinterpret_cast<const uint4*>(hq + lo_bin));
      const uint4 v1 = __ldcg(reinterpret_cast<const uint4*>(hq + lo_bin) + 1);
      c[0] = v0.x; c[1] = v0.y; c[2] = v0.z; c[3] = v0.w; c[4] = v1.x; c[5] = v1.y; c[6] = v1.z; c[7] = v1.w;
    } else if (per == 4) {
      const uint4 v0 = __ldcg(reinterpret_cast<const uint4*>(hq + lo_bin));
      c[0] = v0.x; c[1] = v0.y; c[2] = v0.z; c[3] = v0.w;
#pragma unroll
      for (int j = 4; j < 8; ++j) c[j] = 0;
    } else {
      const uint2 v0 = __ldcg(reinterpret_cast<const uint2*>(hq + lo_bin));
      c[0] = v0.x; c[1] = v0.y;
#pragma unroll
      for (int j = 2; j < 8; ++j) c[j] = 0;
    }
    uint32_t local = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) local += c[j];
    uint32_t total;
    uint32_t above = topk_block_scan(local, S, &total);   // bins above this thread's range
    // target: the suffix count the threshold bin must reach
    uint32_t target;
    if (p.hist_sample == 1) {
      need = static_cast<int>(total < static_cast<uint32_t>(p.K) ? total : static_cast<uint32_t>(p.K));
      target = static_cast<uint32_t>(need);
    } else {
      // a quarter more than the expected sampled count, plus 8 (about three
      // standard deviations of the sample at K = 512, s = 8)
      need = static_cast<int>(min(static_cast<int64_t>(p.K), nvalid));
      target = static_cast<uint32_t>((5 * need + 4 * p.hist_sample - 1) / (4 * p.hist_sample)) + 8;
    }
    if (tid == 0) { S.tb = (p.hist_sample == 1) ? nbins : 0; S.above = 0; }
    __syncthreads();
    if (need > 0 && above < target && above + local >= target) {
      bool found = false;
#pragma unroll
      for (int j = 7; j >= 0; --j) {
        if (j < per && !found) {
          if (above + c[j] >= target) {
            S.tb = lo_bin + j;
            S.above = static_cast<int>(above);
            found = true;
          }
          above += c[j];
        }
      }
    }
    __syncthreads();
  }
  const int tb = S.tb;

  // -- 1. this warp's range: candidates into its region, in position order
  uint32_t n = 0;                                     // the CTA's candidates (after the gather below)
  {
    const uint32_t lt = (1u << lane) - 1u;             // lanes below this one
    uint64_t* wkeys = keys_s + warp * kTopkWarpCap;
    uint32_t wn = 0;                                   // this warp's candidates so far (uniform in the warp)
    int k = 0;
    for (int64_t c0 = wlo; c0 < whi; c0 += kTopkWarpSlots, ++k) {
      const int st = k % kTopkStages;
      const bool ok = mbar_wait(&wbar[st], (k / kTopkStages) & 1, kErrWaitOperand, &S.abort_flag);
      float4 cur[kTopkVec];
      const int64_t left = whi - c0 - 4 * lane;        // visible slots from this lane's first on
      const float4* src = reinterpret_cast<const float4*>(wring + st * kTopkWarpSlots) + lane;
#pragma unroll
      for (int j = 0; j < kTopkVec; ++j) {
        cur[j] = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
        const int64_t rem = left - 128 * j;
        if (ok && need > 0 && rem > 0) {
          cur[j] = src[32 * j];
          if (rem < 4) {
            cur[j].w = -INFINITY;
            if (rem < 3) cur[j].z = -INFINITY;
            if (rem < 2) cur[j].y = -INFINITY;
          }
        }
      }
      __syncwarp();
      if (lane == 0) {                                 // every lane holds its values: refill the stage
        fence_async_smem_generic();
        issue_chunk(c0 + static_cast<int64_t>(kTopkStages) * kTopkWarpSlots, k + kTopkStages);
      }
      // position order inside the chunk is (j, lane, component): four
      // ballots per j give each lane its offset without a serial scan
#pragma unroll
      for (int j = 0; j < kTopkVec; ++j) {
        const bool f0 = topk_is_cand(cur[j].x, tb, p.hb), f1 = topk_is_cand(cur[j].y, tb, p.hb);
        const bool f2 = topk_is_cand(cur[j].z, tb, p.hb), f3 = topk_is_cand(cur[j].w, tb, p.hb);
        const uint32_t b0 = __ballot_sync(0xffffffffu, f0), b1 = __ballot_sync(0xffffffffu, f1);
        const uint32_t b2 = __ballot_sync(0xffffffffu, f2), b3 = __ballot_sync(0xffffffffu, f3);
        const uint32_t tot = __popc(b0) + __popc(b1) + __popc(b2) + __popc(b3);
        if (tot != 0) {
          uint32_t o = wn + __popc(b0 & lt) + __popc(b1 & lt) + __popc(b2 & lt) + __popc(b3 & lt);
          const int64_t s0 = c0 + 128 * j + 4 * lane;
          const float v[4] = {cur[j].x, cur[j].y, cur[j].z, cur[j].w};
          const bool f[4] = {f0, f1, f2, f3};
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            if (f[c]) {
              if (o < static_cast<uint32_t>(kTopkWarpCap)) wkeys[o] = topk_make_key(p, bq, s0 + c, v[c]);
              ++o;
            }
          }
        }
        wn += tot;
      }
    }
    // copies issued past the visible end (speculatively) land before the
    // ring is reused
    if (lane == 0) {
      const int64_t kcopy = (whi_copy - wlo + kTopkWarpSlots - 1) / kTopkWarpSlots;   // chunks in the range
      const int64_t kissued = min(kcopy, static_cast<int64_t>(k) + kTopkStages);
      volatile int keep_waiting = 0;                   // bounded even after an earlier wait gave up
      for (int64_t kk = k; kk < kissued; ++kk)
        mbar_wait(&wbar[kk % kTopkStages], static_cast<uint32_t>((kk / kTopkStages) & 1), kErrWaitOperand,
                  &keep_waiting);
      S.wcnt[warp] = wn;
    }
    __syncthreads();
    // the warp lists, in warp order, into one contiguous list over the ring
    bool wfit = true;
    uint32_t off = 0;
    for (int w = 0; w < kTopkWarps; ++w) {
      const uint32_t c = S.wcnt[w];
      wfit = wfit && c <= static_cast<uint32_t>(kTopkWarpCap);
      if (w < warp) off += min(c, static_cast<uint32_t>(kTopkWarpCap));
      n += c;
    }
    for (uint32_t i = lane; i < min(wn, static_cast<uint32_t>(kTopkWarpCap)); i += 32) cand_s[off + i] = wkeys[i];
    if (!wfit) n = kTopkCap + 1;                       // a warp overflowed: take the exact path
    __syncthreads();
  }

  // -- 2. counts to every CTA; the others push their lists into the first
  //       CTA's shared memory behind its own, in slice (= position) order
  asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
  if (tid < C) *cluster.map_shared_rank(&S.cnt[rank], tid) = n;
  cluster.sync();                                     // counts visible cluster-wide
  bool fits = true;
  uint32_t n_all = 0, my_off = 0;
  for (int r = 0; r < C; ++r) {
    const uint32_t c = S.cnt[r];
    fits = fits && c <= static_cast<uint32_t>(kTopkCap);
    if (r < rank) my_off += c;
    n_all += c;
  }
  fits = fits && n_all <= static_cast<uint32_t>(kTopkCap);
  if (fits && need > 0 && rank > 0) {
    uint64_t* dst = cluster.map_shared_rank(cand_s, 0) + my_off;
    for (uint32_t i = tid; i < n; i += kTopkThreads) dst[i] = cand_s[i];
  }
  cluster.sync();                                     // the first CTA holds every list; the rest may exit
  if (rank != 0) return;

  int32_t* out_idx = p.out_idx + static_cast<int64_t>(bq) * p.K;
  float* out_sc = p.out_scores ? p.out_scores + static_cast<int64_t>(bq) * p.K : nullptr;
  uint32_t written = 0;
  // an estimated threshold holds when at least `need` keys sit at or above it
  if (p.hist_sample != 1 && n_all < static_cast<uint32_t>(need)) fits = false;
  if (need > 0) {
    if (fits) {
      uint64_t P;
      if (p.hist_sample == 1)
        P = topk_radix_select<false>(S, n_all, need, p.hb, static_cast<uint64_t>(tb) << (64 - p.hb), S.above,
                                     [&](int64_t i) { return cand_s[i]; });
      else    // the K-th key's bin is unknown: full-width passes, equal digits aggregated
        P = topk_radix_select<true>(S, n_all, need, 0, 0, 0, [&](int64_t i) { return cand_s[i]; });
      // ordered compaction of the keys >= P (4 consecutive keys per thread)
      for (uint32_t i0 = 0; i0 < n_all; i0 += 4 * kTopkThreads) {
        uint64_t k[4];
        uint32_t m = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t j = i0 + 4 * tid + i;
          k[i] = (j < n_all) ? cand_s[j] : 0;
          if (k[i] < P) k[i] = 0;
          m += (k[i] != 0);
        }
        uint32_t tot;
        uint32_t o = written + topk_block_scan(m, S, &tot);
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (k[i] != 0) topk_emit(p, bq, out_idx, out_sc, o++, k[i]);
        written += tot;
      }
    } else {
      // candidates do not fit (or an estimated threshold failed): select
      // and compact over the scores themselves.  With an estimate, every
      // visible finite score takes part and `need` is counted exactly.
      const int tbf = (p.hist_sample == 1) ? tb : 0;
      uint64_t P;
      if (p.hist_sample == 1) {
        P = topk_radix_select<true>(S, nvalid, need, p.hb, static_cast<uint64_t>(tb) << (64 - p.hb), S.above,
                                    [&](int64_t e) { return topk_slot_key(p, bq, e, tbf); });
      } else {
        uint32_t cnt = 0;
        for (int64_t e = tid; e < nvalid; e += kTopkThreads) cnt += (row[e] != -INFINITY);
        uint32_t tot;
        topk_block_scan(cnt, S, &tot);
        need = static_cast<int>(min(tot, static_cast<uint32_t>(p.K)));
        P = need > 0 ? topk_radix_select<true>(S, nvalid, need, 0, 0, 0, [&](int64_t e) { return topk_slot_key(p, bq, e, 0); })
                     : ~0ull;
      }
      for (int64_t e0 = 0; need > 0 && e0 < nvalid; e0 += 4 * kTopkThreads) {
        uint64_t k[4];
        uint32_t m = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int64_t e = e0 + 4 * tid + i;
          k[i] = (e < nvalid) ? topk_slot_key(p, bq, e, tbf) : 0;
          if (k[i] < P) k[i] = 0;
          m += (k[i] != 0);
        }
        uint32_t tot;
        uint32_t o = written + topk_block_scan(m, S, &tot);
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (k[i] != 0) topk_emit(p, bq, out_idx, out_sc, o++, k[i]);
        written += tot;
      }
    }
    if (written != static_cast<uint32_t>(need) && tid == 0) record_error(kErrSelectCount);
  }
  for (int i = static_cast<int>(min(written, static_cast<uint32_t>(p.K))) + tid; i < p.K; i += kTopkThreads) {
    out_idx[i] = -1;
    if (out_sc) out_sc[i] = -INFINITY;
  }
}

inline size_t topk_smem_bytes() {
  // warp regions of candidates, then the stage rings (which later hold the
  // contiguous candidate list: both are kTopkCap keys)
  return ((sizeof(TopkShared) + 15) & ~size_t(15)) + static_cast<size_t>(kTopkCap) * 8 +
         static_cast<size_t>(kTopkWarps) * kTopkStages * kTopkWarpSlots * 4;
}

// CTAs per selection problem: enough to spread a long score row over SMs
// (one CTA per 8K slots, at most max_cluster), fewer once the problems
// alone fill the GPU twice over.
inline int topk_cluster_size(int64_t n_elems, int problems, int sms, int max_cluster) {
  int c = 1;
  while (c < max_cluster && static_cast<int64_t>(c) * 8192 < n_elems) c <<= 1;
  while (c > 1 && static_cast<int64_t>(problems) * c > 2 * static_cast<int64_t>(sms)) c >>= 1;
  return c;
}

}  // namespace csa2
