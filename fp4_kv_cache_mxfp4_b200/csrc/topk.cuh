// topk.cuh -- exact top-K selection with ties to the lower position
// ("DeepSeek V4.1-Flash 技术报告深度解析" §3.2 top-512, §3.3 top-2048 blocks).
//
// Keys: key64 = okey(score) << 32 | ~position.  okey orders floats, the low
// word inverts the position, so every key is distinct and "larger key" means
// "higher score, then lower position": the top-K set is the K largest keys.
//
// One launch per selection problem, grid (chunks, queries), 256 threads:
//  0. every CTA reads the query's score histogram (built by the scan
//     epilogue, coalesced) and finds the threshold bin tb, the highest bin
//     whose suffix count reaches need = min(K, visible): every top-K key has
//     its top bits >= tb;
//  1. every CTA compacts the keys of its 4096-slot chunk whose bin is >= tb
//     into the chunk's own segment, in position order (block prefix scan),
//     and records the segment's length;
//  2. the last CTA of the query (ticket counter) gathers the segments in
//     chunk order into shared memory, radix-selects the need-th largest key
//     (8-bit digits from the top) and writes the keys at or above it by an
//     ordered compaction: the result comes out in ascending position order,
//     deterministically, without a sort.
// If the candidates do not fit in shared memory, step 2 runs over the
// scores themselves with the same filter (slower, exact).
// HBM roofline: 4 B per score read (normally still resident in L2).
#pragma once
#include "common.cuh"

namespace csa2 {

constexpr int kTopkThreads = 256;
constexpr int kTopkPer = 16;              // slots per thread
constexpr int kTopkChunk = kTopkThreads * kTopkPer;   // 4096 slots per CTA
constexpr int kTopkSegCap = 1024;         // candidates kept per chunk (more: exact fallback)
constexpr int kTopkSmemKeys = 6144;       // candidates cached in shared memory
constexpr int kTopkMaxChunks = 2048;      // chunk offsets kept in shared memory

struct TopkParams {
  const float* scores;
  int64_t n_elems;          // score slots per query (row stride)
  const int32_t* n_vis;     // optional [BQ]: valid slots = ceil(n_vis / vis_div)
  int vis_div;
  const int32_t* pool;      // pool mode: position of slot e = pool[e/8]*8 + e%8
  int pool_blocks;
  const uint32_t* hist;     // [BQ][1 << hb] score histogram from the scan
  int hb;
  uint64_t* seg;            // [BQ][nchunks][kTopkSegCap]: chunk c's candidates
  uint32_t* seg_cnt;        // [BQ][nchunks]
  int nchunks;
  uint32_t* ctr;            // [BQ][8], zero at the scan's launch
  int ticket_slot;          // ctr[ticket_slot]: finished CTAs of the query
  int ovf_slot;             // ctr[ovf_slot] != 0: a chunk had more than kTopkSegCap candidates
  int K;
  int32_t* out_idx;         // [BQ][K]
  float* out_scores;        // optional [BQ][K]
};

struct TopkShared {
  uint32_t h256[256];
  uint32_t warp_tot[32];
  uint32_t chunk_off[kTopkMaxChunks + 1];
  int last, d, gt, eq, total, tb;
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

// key of score s at slot e, or 0 when the slot holds no visible score or
// sits below tb
__device__ __forceinline__ uint64_t topk_key_of(const TopkParams& p, int bq, int64_t e, float s, int tb) {
  if (s == -INFINITY) return 0;
  const uint32_t k = okey(s);
  if (static_cast<int>(k >> (32 - p.hb)) < tb) return 0;
  return (static_cast<uint64_t>(k) << 32) | static_cast<uint32_t>(~topk_position(p, bq, e));
}

// key of slot e, or 0 when the slot holds no visible score or sits below tb
__device__ __forceinline__ uint64_t topk_slot_key(const TopkParams& p, int bq, int64_t e, int tb) {
  const float s = p.scores[static_cast<int64_t>(bq) * p.n_elems + e];
  if (s == -INFINITY) return 0;
  const uint32_t k = okey(s);
  if (static_cast<int>(k >> (32 - p.hb)) < tb) return 0;
  return (static_cast<uint64_t>(k) << 32) | static_cast<uint32_t>(~topk_position(p, bq, e));
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
    const uint32_t x = (lane < kTopkThreads / 32) ? S.warp_tot[lane] : 0;
    uint32_t xi = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_up_sync(0xffffffffu, xi, o);
      if (lane >= o) xi += t;
    }
    S.warp_tot[lane] = xi - x;                      // exclusive per warp
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
template <class KeyAt>
__device__ uint64_t topk_radix_select(TopkShared& S, int64_t n, int need, KeyAt key_at) {
  uint64_t prefix = 0;
  int bits = 0, remaining = need;
  while (true) {
    const int shift = 56 - bits;
    for (int i = threadIdx.x; i < 256; i += blockDim.x) S.h256[i] = 0;
    if (threadIdx.x == 0) S.d = -1;
    __syncthreads();
    for (int64_t i0 = 0; i0 < n; i0 += blockDim.x) {
      const int64_t i = i0 + threadIdx.x;
      const uint64_t k = (i < n) ? key_at(i) : 0;
      const bool act = k != 0 && (bits == 0 || (k >> (64 - bits)) == (prefix >> (64 - bits)));
      warp_hist_add(S.h256, static_cast<uint32_t>((k >> shift) & 255), act);
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

__device__ __forceinline__ void topk_emit(const TopkParams& p, int32_t* out_idx, float* out_sc, uint32_t slot,
                                          uint64_t k) {
  if (slot >= static_cast<uint32_t>(p.K)) return;
  out_idx[slot] = static_cast<int32_t>(~static_cast<uint32_t>(k));
  if (out_sc) out_sc[slot] = okey_to_float(static_cast<uint32_t>(k >> 32));
}

__global__ void __launch_bounds__(kTopkThreads)
topk_select_kernel(TopkParams p) {
  extern __shared__ __align__(1024) uint8_t topk_smem_raw[];
  TopkShared& S = *reinterpret_cast<TopkShared*>(topk_smem_raw);
  uint64_t* keys_s = reinterpret_cast<uint64_t*>(topk_smem_raw + ((sizeof(TopkShared) + 15) & ~size_t(15)));

  const int bq = blockIdx.y;
  const int tid = threadIdx.x;
  uint32_t* ctr = p.ctr + static_cast<int64_t>(bq) * 8;
  const int64_t nvalid = topk_valid_slots(p, bq);

  // this thread's 16 slots of the chunk, loaded before the histogram so the
  // two reads overlap
  const int64_t slot0 = static_cast<int64_t>(blockIdx.x) * kTopkChunk + kTopkPer * tid;
  float sv[kTopkPer];
#pragma unroll
  for (int i = 0; i < kTopkPer; ++i)
    sv[i] = (slot0 + i < nvalid) ? p.scores[static_cast<int64_t>(bq) * p.n_elems + slot0 + i] : -INFINITY;

  // -- 0. threshold bin: thread t owns the `per` bins just below bin
  //       nbins - per*t (descending ranges), read with coalesced loads
  int need;
  {
    const int nbins = 1 << p.hb;
    const int per = nbins / kTopkThreads;             // 16 (12-bit) or 4 (10-bit)
    const uint32_t* hq = p.hist + static_cast<int64_t>(bq) * nbins;
    const int lo_bin = nbins - per * (tid + 1);
    uint32_t c[16];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint4 v = make_uint4(0, 0, 0, 0);
      if (4 * j < per) v = __ldcg(reinterpret_cast<const uint4*>(hq + lo_bin) + j);
      c[4 * j] = v.x; c[4 * j + 1] = v.y; c[4 * j + 2] = v.z; c[4 * j + 3] = v.w;
    }
    uint32_t local = 0;
#pragma unroll
    for (int j = 0; j < 16; ++j) local += c[j];
    uint32_t total;
    uint32_t above = topk_block_scan(local, S, &total);   // bins above this thread's range
    need = static_cast<int>(total < static_cast<uint32_t>(p.K) ? total : static_cast<uint32_t>(p.K));
    if (tid == 0) S.tb = nbins;
    __syncthreads();
    if (need > 0 && above < static_cast<uint32_t>(need) && above + local >= static_cast<uint32_t>(need)) {
      bool found = false;
#pragma unroll
      for (int j = 15; j >= 0; --j) {
        if (j < per && !found) {
          above += c[j];
          if (above >= static_cast<uint32_t>(need)) { S.tb = lo_bin + j; found = true; }
        }
      }
    }
    __syncthreads();
  }
  const int tb = S.tb;
  uint64_t* seg_q = p.seg + static_cast<int64_t>(bq) * p.nchunks * kTopkSegCap;
  uint32_t* cnt_q = p.seg_cnt + static_cast<int64_t>(bq) * p.nchunks;

  // -- 1. this chunk's candidates, in position order ------------------------
  {
    uint64_t k[kTopkPer];
    uint32_t n = 0;
#pragma unroll
    for (int i = 0; i < kTopkPer; ++i) {
      k[i] = (need > 0) ? topk_key_of(p, bq, slot0 + i, sv[i], tb) : 0;
      n += (k[i] != 0);
    }
    uint32_t total;
    uint32_t off = topk_block_scan(n, S, &total);
    uint64_t* seg = seg_q + static_cast<int64_t>(blockIdx.x) * kTopkSegCap;
#pragma unroll
    for (int i = 0; i < kTopkPer; ++i) {
      if (k[i] != 0 && off < static_cast<uint32_t>(kTopkSegCap)) seg[off] = k[i];
      off += (k[i] != 0);
    }
    if (tid == 0) {
      cnt_q[blockIdx.x] = min(total, static_cast<uint32_t>(kTopkSegCap));
      if (total > static_cast<uint32_t>(kTopkSegCap)) atomicOr(ctr + p.ovf_slot, 1u);
    }
    __threadfence();                                      // publish this thread's writes before the ticket
  }

  // -- 2. the last CTA of this query selects ---------------------------------
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    S.last = (atomicAdd(ctr + p.ticket_slot, 1u) == gridDim.x - 1);
  }
  __syncthreads();
  if (!S.last) return;
  __threadfence();

  int32_t* out_idx = p.out_idx + static_cast<int64_t>(bq) * p.K;
  float* out_sc = p.out_scores ? p.out_scores + static_cast<int64_t>(bq) * p.K : nullptr;
  uint32_t written = 0;
  if (need > 0) {
    // chunk offsets (exclusive scan of the segment lengths)
    uint32_t C = 0;
    bool fits = p.nchunks <= kTopkMaxChunks && __ldcg(ctr + p.ovf_slot) == 0;
    if (fits) {
      for (int c0 = 0; c0 < p.nchunks; c0 += kTopkThreads) {
        const int c = c0 + tid;
        const uint32_t v = (c < p.nchunks) ? __ldcg(cnt_q + c) : 0;
        uint32_t tot;
        const uint32_t o = topk_block_scan(v, S, &tot);
        if (c < p.nchunks) S.chunk_off[c] = C + o;
        C += tot;
      }
      if (tid == 0) S.chunk_off[p.nchunks] = C;
      __syncthreads();
      fits = C <= static_cast<uint32_t>(kTopkSmemKeys);
    }
    if (fits) {
      // gather the segments in chunk order: one warp per chunk
      const int lane = tid & 31, warp = tid >> 5;
      for (int c = warp; c < p.nchunks; c += kTopkThreads / 32) {
        const uint32_t o = S.chunk_off[c], n = S.chunk_off[c + 1] - o;
        const uint64_t* seg = seg_q + static_cast<int64_t>(c) * kTopkSegCap;
        for (uint32_t i = lane; i < n; i += 32) keys_s[o + i] = __ldcg(seg + i);
      }
      __syncthreads();
      const uint64_t P = topk_radix_select(S, C, need, [&](int64_t i) { return keys_s[i]; });
      // ordered compaction of the keys >= P (4 consecutive keys per thread)
      for (uint32_t i0 = 0; i0 < C; i0 += 4 * kTopkThreads) {
        uint64_t k[4];
        uint32_t n = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t j = i0 + 4 * tid + i;
          k[i] = (j < C) ? keys_s[j] : 0;
          if (k[i] < P) k[i] = 0;
          n += (k[i] != 0);
        }
        uint32_t tot;
        uint32_t o = written + topk_block_scan(n, S, &tot);
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (k[i] != 0) topk_emit(p, out_idx, out_sc, o++, k[i]);
        written += tot;
      }
    } else {
      // candidates do not fit: select and compact over the scores themselves
      const uint64_t P = topk_radix_select(S, nvalid, need, [&](int64_t e) { return topk_slot_key(p, bq, e, tb); });
      for (int64_t e0 = 0; e0 < nvalid; e0 += 4 * kTopkThreads) {
        uint64_t k[4];
        uint32_t n = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int64_t e = e0 + 4 * tid + i;
          k[i] = (e < nvalid) ? topk_slot_key(p, bq, e, tb) : 0;
          if (k[i] < P) k[i] = 0;
          n += (k[i] != 0);
        }
        uint32_t tot;
        uint32_t o = written + topk_block_scan(n, S, &tot);
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (k[i] != 0) topk_emit(p, out_idx, out_sc, o++, k[i]);
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
  return ((sizeof(TopkShared) + 15) & ~size_t(15)) + static_cast<size_t>(kTopkSmemKeys) * 8;
}

}  // namespace csa2
