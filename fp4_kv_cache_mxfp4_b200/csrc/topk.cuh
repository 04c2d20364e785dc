// topk.cuh -- exact top-K selection with ties to the lower position
// ("DeepSeek V4.1-Flash 技术报告深度解析" §3.2 top-512, §3.3 top-2048 blocks).
//
// Keys: key64 = okey(score) << 32 | ~position.  okey orders floats, the low
// word inverts the position, so every key is distinct and "larger key" means
// "higher score, then lower position": the top-K set is the K largest keys.
//
// One launch per selection problem, grid (chunks, queries):
//  1. every CTA reads the query's score histogram (built by the scan
//     epilogue) and finds the threshold bin tb: the highest bin whose
//     suffix count reaches K;
//  2. every CTA appends the keys of its chunk whose bin is >= tb to the
//     query's candidate list (warp-aggregated atomics);
//  3. the last CTA to finish (ticket counter) radix-selects the K-th key
//     among the candidates (8-bit digits, from the top), gathers the K keys
//     at or above it, sorts them (bitonic, descending) and writes positions
//     and scores.  If the candidate list overflowed, step 3 runs over the scores
//     themselves (same filter), which is slower but exact.
// HBM roofline: 4 B per score read (the scores are usually still in L2).
#pragma once
#include "common.cuh"

namespace csa2 {

constexpr int kTopkThreads = 1024;
constexpr int kTopkSmemKeys = 4096;      // candidates cached in shared memory
constexpr int kTopkMaxK = 2048;

struct TopkParams {
  const float* scores;
  int64_t n_elems;          // score slots per query (row stride)
  const int32_t* n_vis;     // optional [BQ]: valid slots = ceil(n_vis / vis_div)
  int vis_div;
  const int32_t* pool;      // pool mode: position of slot e = pool[e/8]*8 + e%8
  int pool_blocks;
  uint32_t* hist;           // [BQ][1 << hb]
  int hb;
  uint64_t* cand;           // [BQ][cap]
  int cap;
  uint32_t* ctr;            // [BQ][4]: candidate count, finished CTAs (zero at launch)
  int K;
  int chunk;                // slots per CTA
  int32_t* out_idx;         // [BQ][K]
  float* out_scores;        // optional [BQ][K]
  int out_by_pos;           // 1: ascending positions (pool output), 0: best first
};

struct TopkShared {
  uint32_t h256[256];
  int tb, need, last, d, gt, eq, cnt, total;
  uint32_t warp_sum[32];
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

// key of slot e, or 0 when the slot holds no visible score or sits below tb
__device__ __forceinline__ uint64_t topk_slot_key(const TopkParams& p, int bq, int64_t e, int tb) {
  const float s = p.scores[static_cast<int64_t>(bq) * p.n_elems + e];
  if (s == -INFINITY) return 0;
  const uint32_t k = okey(s);
  if (static_cast<int>(k >> (32 - p.hb)) < tb) return 0;
  return (static_cast<uint64_t>(k) << 32) | static_cast<uint32_t>(~topk_position(p, bq, e));
}

// Highest digit d of a 256-bin histogram with suffix(d) >= remaining, run by
// warp 0; lane l owns bins 255-8l .. 248-8l.
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
template <class KeyAt>
__device__ uint64_t topk_radix_select(TopkShared& S, int64_t n, int need, KeyAt key_at) {
  uint64_t prefix = 0;
  int bits = 0, remaining = need;
  while (true) {
    const int shift = 56 - bits;
    for (int i = threadIdx.x; i < 256; i += blockDim.x) S.h256[i] = 0;
    if (threadIdx.x == 0) S.d = -1;
    __syncthreads();
    for (int64_t i = threadIdx.x; i < n; i += blockDim.x) {
      const uint64_t k = key_at(i);
      if (k == 0) continue;
      if (bits > 0 && (k >> (64 - bits)) != (prefix >> (64 - bits))) continue;
      atomicAdd(&S.h256[(k >> shift) & 255], 1u);
    }
    __syncthreads();
    if (threadIdx.x < 32) topk_pick_digit(S, remaining);
    __syncthreads();
    if (S.d < 0) { if (threadIdx.x == 0) record_error(kErrSelectCount); return prefix; }
    prefix |= static_cast<uint64_t>(S.d) << shift;
    bits += 8;
    remaining -= S.gt;
    const bool done = (S.eq == remaining) || bits == 64;
    __syncthreads();
    if (done) return prefix;
  }
}

__global__ void __launch_bounds__(kTopkThreads)
topk_select_kernel(TopkParams p) {
  extern __shared__ __align__(1024) uint8_t topk_smem_raw[];
  TopkShared& S = *reinterpret_cast<TopkShared*>(topk_smem_raw);
  uint32_t* hist_s = reinterpret_cast<uint32_t*>(topk_smem_raw + sizeof(TopkShared));
  const int nbins = 1 << p.hb;
  uint64_t* keys_s = reinterpret_cast<uint64_t*>(hist_s + nbins);        // kTopkSmemKeys
  uint64_t* sort_s = keys_s + kTopkSmemKeys;                              // kTopkMaxK

  const int bq = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t* hist = p.hist + static_cast<int64_t>(bq) * nbins;
  uint32_t* ctr = p.ctr + bq * 4;
  const int64_t nvalid = topk_valid_slots(p, bq);

  // -- 1. threshold bin from the histogram --------------------------------
  for (int i = tid; i < nbins; i += blockDim.x) hist_s[i] = __ldcg(hist + i);
  __syncthreads();
  const int per = (nbins + blockDim.x - 1) / blockDim.x;      // bins per thread, from the top
  const int hi_bin = nbins - 1 - tid * per;                   // this thread: [hi_bin-per+1, hi_bin]
  uint32_t local = 0;
  for (int j = 0; j < per; ++j) if (hi_bin - j >= 0) local += hist_s[hi_bin - j];
  uint32_t incl = local;
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) S.warp_sum[warp] = incl;
  if (tid == 0) S.tb = nbins;
  __syncthreads();
  uint32_t wbase = 0, total = 0;
  for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) {
    if (w < warp) wbase += S.warp_sum[w];
    total += S.warp_sum[w];
  }
  const int need = static_cast<int>(total < static_cast<uint32_t>(p.K) ? total : static_cast<uint32_t>(p.K));
  uint32_t above = wbase + incl - local;                      // count in bins above this thread's range
  if (need > 0 && above < static_cast<uint32_t>(need) && above + local >= static_cast<uint32_t>(need)) {
    for (int j = 0; j < per; ++j) {
      const int bin = hi_bin - j;
      if (bin < 0) break;
      above += hist_s[bin];
      if (above >= static_cast<uint32_t>(need)) { S.tb = bin; break; }
    }
  }
  if (tid == 0) { S.need = need; S.total = static_cast<int>(total); }
  __syncthreads();
  const int tb = S.tb;

  // -- 2. candidates of this chunk -----------------------------------------
  if (need > 0) {
    const int64_t lo = static_cast<int64_t>(blockIdx.x) * p.chunk;
    const int64_t hi = min(lo + p.chunk, nvalid);
    uint64_t* cand = p.cand + static_cast<int64_t>(bq) * p.cap;
    for (int64_t base = lo + warp * 32; base < hi; base += blockDim.x) {
      const int64_t e = base + lane;
      const uint64_t k = (e < hi) ? topk_slot_key(p, bq, e, tb) : 0;
      const uint32_t m = __ballot_sync(0xffffffffu, k != 0);
      if (m == 0) continue;
      uint32_t off = 0;
      if (lane == 0) off = atomicAdd(&ctr[0], __popc(m));
      off = __shfl_sync(0xffffffffu, off, 0);
      if (k != 0) {
        const uint32_t slot = off + __popc(m & ((1u << lane) - 1));
        if (slot < static_cast<uint32_t>(p.cap)) cand[slot] = k;
      }
    }
  }

  // -- 3. the last CTA of this query selects --------------------------------
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    const uint32_t t = atomicAdd(&ctr[1], 1u);
    S.last = (t == gridDim.x - 1);
  }
  __syncthreads();
  if (!S.last) return;
  __threadfence();

  int32_t* out_idx = p.out_idx + static_cast<int64_t>(bq) * p.K;
  float* out_sc = p.out_scores ? p.out_scores + static_cast<int64_t>(bq) * p.K : nullptr;
  int cnt = 0;
  if (need > 0) {
    const uint32_t C = __ldcg(&ctr[0]);
    uint64_t P;
    if (C <= static_cast<uint32_t>(p.cap)) {
      const uint64_t* cand = p.cand + static_cast<int64_t>(bq) * p.cap;
      if (C <= static_cast<uint32_t>(kTopkSmemKeys)) {
        for (uint32_t i = tid; i < C; i += blockDim.x) keys_s[i] = __ldcg(cand + i);
        __syncthreads();
        P = topk_radix_select(S, C, need, [&](int64_t i) { return keys_s[i]; });
        if (tid == 0) S.cnt = 0;
        __syncthreads();
        for (uint32_t i = tid; i < C; i += blockDim.x) {
          const uint64_t k = keys_s[i];
          if (k >= P) { const int s = atomicAdd(&S.cnt, 1); if (s < kTopkMaxK) sort_s[s] = k; }
        }
      } else {
        P = topk_radix_select(S, C, need, [&](int64_t i) { return __ldcg(cand + i); });
        if (tid == 0) S.cnt = 0;
        __syncthreads();
        for (uint32_t i = tid; i < C; i += blockDim.x) {
          const uint64_t k = __ldcg(cand + i);
          if (k >= P) { const int s = atomicAdd(&S.cnt, 1); if (s < kTopkMaxK) sort_s[s] = k; }
        }
      }
    } else {
      // candidate list overflowed: select over the scores themselves
      P = topk_radix_select(S, nvalid, need, [&](int64_t e) { return topk_slot_key(p, bq, e, tb); });
      if (tid == 0) S.cnt = 0;
      __syncthreads();
      for (int64_t e = tid; e < nvalid; e += blockDim.x) {
        const uint64_t k = topk_slot_key(p, bq, e, tb);
        if (k != 0 && k >= P) { const int s = atomicAdd(&S.cnt, 1); if (s < kTopkMaxK) sort_s[s] = k; }
      }
    }
    __syncthreads();
    cnt = S.cnt;
    if (cnt != need && tid == 0) record_error(kErrSelectCount);
    cnt = min(cnt, need);
    // re-key for ascending-position output
    if (p.out_by_pos) {
      for (int i = tid; i < cnt; i += blockDim.x) {
        const uint64_t k = sort_s[i];
        const uint32_t pos = ~static_cast<uint32_t>(k);
        sort_s[i] = (static_cast<uint64_t>(0xFFFFFFFFu - pos) << 32) | (k >> 32);
      }
    }
    int M = 1;
    while (M < cnt) M <<= 1;
    for (int i = cnt + tid; i < M; i += blockDim.x) sort_s[i] = 0;
    __syncthreads();
    for (int k = 2; k <= M; k <<= 1) {
      for (int j = k >> 1; j > 0; j >>= 1) {
        for (int i = tid; i < M; i += blockDim.x) {
          const int ixj = i ^ j;
          if (ixj > i) {
            const uint64_t a = sort_s[i], c = sort_s[ixj];
            const bool desc = (i & k) == 0;
            if (desc ? (a < c) : (a > c)) { sort_s[i] = c; sort_s[ixj] = a; }
          }
        }
        __syncthreads();
      }
    }
  }
  for (int i = tid; i < p.K; i += blockDim.x) {
    int32_t pos = -1;
    float sc = -INFINITY;
    if (i < cnt) {
      const uint64_t k = sort_s[i];
      if (p.out_by_pos) {
        pos = static_cast<int32_t>(0xFFFFFFFFu - static_cast<uint32_t>(k >> 32));
        sc = okey_to_float(static_cast<uint32_t>(k));
      } else {
        pos = static_cast<int32_t>(~static_cast<uint32_t>(k));
        sc = okey_to_float(static_cast<uint32_t>(k >> 32));
      }
    }
    out_idx[i] = pos;
    if (out_sc) out_sc[i] = sc;
  }
}

inline size_t topk_smem_bytes(int hb) {
  return sizeof(TopkShared) + (static_cast<size_t>(1) << hb) * 4 + (kTopkSmemKeys + kTopkMaxK) * 8;
}

}  // namespace csa2
