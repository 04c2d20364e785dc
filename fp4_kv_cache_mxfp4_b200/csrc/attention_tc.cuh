// attention_tc.cuh -- sparse MQA on the 5th-generation tensor cores
// ("DeepSeek V4.1-Flash 技术报告深度解析" §3.2 attention, §3.4 dequantise
// before the attention math).
//
// A query's keys are cut into 128-key slices: ceil(K/128) slices of selected
// FP4 entries, then ceil(W/128) slices of window rows.  A CTA (512 threads)
// takes one slice (split mode: many CTAs per query, for few queries) or all
// slices of its query in turn (one CTA per query, for many queries).  Per
// slice the keys (FP4 entries, loaded straight into registers by the CTA's
// threads, 16 nibble bytes and two scales per thread and item, and
// dequantised there, or window rows brought by TMA) form a 128 x 512 bf16
// tile K in shared memory, stored K-major with the 128-byte swizzle; the
// query's 64 heads form Q (64 x 512, TMA, loaded once).  Then:
//   MMA 1   S^T[key, head] = K . Q^T            M = 128 keys, N = 64, K = 512
//   softmax per head over the slice's keys in registers (fp32; shuffles and
//           a 2 KB exchange between key quarters) against a running
//           reference max that only moves when a slice's max exceeds it by
//           more than 2^8 (the accumulator is then rescaled in TMEM);
//           P^T[key, head] = exp2(S^T - ref) rounded to bf16, stored
//           [key][head] as an MN-major operand
//   MMA 2   O^T[dim, head] += V^T . P^T         the same key tile read
//           MN-major (M = 128 dims per MMA, 4 tiles), N = 64, K = 128 keys
//   epilogue, by mode:
//     cluster merge (split mode with at most 8 slices): the query's slice
//                  CTAs form one thread-block cluster.  Each CTA sends its
//                  per-head (max, sum) to all the others through distributed
//                  shared memory; every CTA then knows the joint max M and
//                  sum L, scales its own O^T by exp2(m - M) / L while reading
//                  it from TMEM and sends each 32-dim chunk, rounded to bf16
//                  (the output's precision; the sum is taken in fp32), to
//                  the CTA that owns it (chunk c belongs to rank c mod C);
//                  the owner adds the chunks and writes bf16.  No partial
//                  leaves the SMs.
//     split mode, more slices: coalesced 16-byte stores of the unnormalised
//                  partial and the slice's (max, sum) per head;
//                  sparse_attn_combine_kernel merges the slices;
//     one CTA per query: normalised by the running sum, written as bf16 with
//                  the log-sum-exp.
// Quantised Q (q_fp4): Q arrives as FP4 rows in the main-KV entry format
// (E2M1 values, one E4M3 scale per 16 channels, 288 bytes per head; one
// bulk copy).  A split-mode CTA of an FP4 slice repacks Q's codes and
// scales and its gathered entries' codes and scales for the block-scaled
// FP4 tensor path and runs MMA 1 as 8 instructions (tcgen05 kind::mxf4nvf4,
// K = 64, a UE4M3 scale per 16 values: exactly the cache's format) while
// its threads expand the entries to bf16 for MMA 2; every other CTA expands
// Q to bf16 (exact) and runs MMA 1 on that.
// Accumulators: S^T in TMEM columns [0, 64), O^T tile t in [64 + 64t, 128 + 64t),
// block scales of the FP4 MMA 1 in [320, 384).
#pragma once
#include "common.cuh"
#include "quantize.cuh"
#include "attention.cuh"

namespace csa2 {

constexpr int kTcAttnThreads = 512;
constexpr int kTcAttnKeys = 128;                       // keys per slice (MMA M)
constexpr uint32_t kTcKeyTileBytes = 128 * 512 * 2;    // 128 KB: 8 chunks of [128 rows x 64 dims]
constexpr uint32_t kTcQTileBytes = 64 * 512 * 2;       // 64 KB: 8 chunks of [64 rows x 64 dims]
constexpr uint32_t kTcPTileBytes = 128 * 64 * 2;       // 16 KB: P^T [128 keys][64 heads]
constexpr uint32_t kTcMiscBytes = 8192;                // barriers, flags, softmax scratch, cluster statistics
constexpr int kTcMaxClusterSlices = 8;                 // cluster merge: at most this many slices per query
constexpr uint32_t kTcStatOff = 4096;                  // misc offset of the cluster statistics [8 ranks][64][2]
constexpr uint32_t kTcAttnSmem = kTcKeyTileBytes + kTcQTileBytes + kTcPTileBytes + kTcMiscBytes + 1024;
constexpr float kTcRefSlack = 8.0f;                    // log2 units a slice max may exceed the reference

struct TcAttnParams {
  int B, Q, K, W;
  int64_t N;
  const uint8_t* kv;
  const int32_t* idx;
  int swa_rows, swa_step;
  int kv_slices;             // ceil(K / 128): slices 0..kv_slices-1 hold FP4 entries, the rest window rows
  int slices;
  float scale_log2;
  int per_query;             // 1: one CTA per query over all slices, final output; 0: one slice per CTA
  int cluster_merge;         // split mode in clusters of `slices` CTAs: merge over distributed shared
                             // memory and write the final output (no partials)
  int early_inputs;          // 1: q and the window rows are complete at launch (the predecessor is a
                             // kernel of this library): load them before waiting on it
  int swa_fp8;               // 1: window rows are E4M3 codes [B][swa_rows][512] with one fp32 scale per row
  const uint8_t* swa8;
  const float* swa_scale;    // [B][swa_rows]
  float* opart;              // split: [BQ][slices][64][512]
  float* ml;                 // split: [BQ][slices][64][2]
  __nv_bfloat16* out;        // per query: [BQ][64][512]
  float* lse;                // per query, optional: [BQ][64]
  int q_fp4;                 // 1: Q given as FP4 rows (the main-KV entry format, 288 B per head);
                             // in split mode the FP4 slices run MMA 1 on the block-scaled FP4 path
  const uint8_t* q4;         // q_fp4: [BQ][64][288]
};

// Shared-memory descriptor of an MN-major operand in the 128-byte-swizzle
// canonical layout: 64-element (128 B) rows along M, 8-row swizzle atoms
// along K 1024 B apart (stride byte offset), the next 64 M-elements `lbo`
// bytes away (leading byte offset).
__device__ __forceinline__ uint64_t umma_desc_sw128_mnmajor(uint32_t smem_addr, uint32_t lbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFF);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFF) << 16;
  d |= static_cast<uint64_t>(1024 >> 4) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(2) << 61;
  return d;
}

// Four E4M3 codes (bytes of w) to four bf16 values, exactly.  Placing the
// code's exponent and mantissa bits at the bottom of a bf16 exponent field
// gives E4M3(c) * 2^-120 for normal and subnormal codes alike (both formats
// have a hidden bit and gradual underflow); one multiply by 2^120 restores
// the value.  lo = codes 0, 1; hi = codes 2, 3.
__device__ __forceinline__ void e4m3x4_to_bf16(uint32_t w, uint32_t& lo, uint32_t& hi) {
  const uint32_t a = __byte_perm(w, 0u, 0x4140);     // bytes 0, 1 -> bits 0-7, 16-23
  const uint32_t c = __byte_perm(w, 0u, 0x4342);     // bytes 2, 3
  const uint32_t ma = ((a & 0x007F007Fu) << 4) | ((a & 0x00800080u) << 8);
  const uint32_t mc = ((c & 0x007F007Fu) << 4) | ((c & 0x00800080u) << 8);
  const __nv_bfloat162 k = __floats2bfloat162_rn(1.329227995784916e36f, 1.329227995784916e36f);   // 2^120
  __nv_bfloat162 x = __hmul2(*reinterpret_cast<const __nv_bfloat162*>(&ma), k);
  __nv_bfloat162 y = __hmul2(*reinterpret_cast<const __nv_bfloat162*>(&mc), k);
  lo = *reinterpret_cast<uint32_t*>(&x);
  hi = *reinterpret_cast<uint32_t*>(&y);
}

__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Distributed shared memory: the address of the same shared-memory location
// in CTA `rank` of the cluster, and a store there.
__device__ __forceinline__ uint32_t dsmem_map(uint32_t local_addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local_addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void dsmem_st_f32x2(uint32_t addr, float a, float b) {
  asm volatile("st.shared::cluster.v2.f32 [%0], {%1, %2};" :: "r"(addr), "f"(a), "f"(b) : "memory");
}
__device__ __forceinline__ void dsmem_st_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared::cluster.v4.b32 [%0], {%1, %2, %3, %4};" :: "r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
               : "memory");
}
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_arrive_release() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_size() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
      :: "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
         "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
         "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]),
         "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Reduce 16 per-lane values (16 heads) over the 32 lanes of a warp with 16
// shuffles: each halving step trades half of the values with the partner
// lane, so afterwards lane l holds the reduction of head l >> 1.
template <bool MAX>
__device__ __forceinline__ float warp_reduce_heads16(const float (&v)[16], int lane) {
  float a[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {                        // lane bit 4 keeps heads 8..15, else 0..7
    const bool hi = lane & 16;
    const float keep = hi ? v[j + 8] : v[j], give = hi ? v[j] : v[j + 8];
    const float got = __shfl_xor_sync(0xffffffffu, give, 16);
    a[j] = MAX ? fmaxf(keep, got) : keep + got;
  }
  float b[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const bool hi = lane & 8;
    const float keep = hi ? a[j + 4] : a[j], give = hi ? a[j] : a[j + 4];
    const float got = __shfl_xor_sync(0xffffffffu, give, 8);
    b[j] = MAX ? fmaxf(keep, got) : keep + got;
  }
  float c[2];
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const bool hi = lane & 4;
    const float keep = hi ? b[j + 2] : b[j], give = hi ? b[j] : b[j + 2];
    const float got = __shfl_xor_sync(0xffffffffu, give, 4);
    c[j] = MAX ? fmaxf(keep, got) : keep + got;
  }
  const bool hi = lane & 2;
  const float keep = hi ? c[1] : c[0], give = hi ? c[0] : c[1];
  const float got = __shfl_xor_sync(0xffffffffu, give, 2);
  float d = MAX ? fmaxf(keep, got) : keep + got;
  const float e = __shfl_xor_sync(0xffffffffu, d, 1);
  return MAX ? fmaxf(d, e) : d + e;
}

__global__ void __launch_bounds__(kTcAttnThreads, 1)
sparse_attn_tc_kernel(const __grid_constant__ CUtensorMap tmap_q,
                      const __grid_constant__ CUtensorMap tmap_swa,
                      TcAttnParams p) {
  extern __shared__ __align__(1024) uint8_t tc_attn_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(tc_attn_smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* kt = smem;                                   // key tile (K-major), later read MN-major as V^T
  uint8_t* qt = smem + kTcKeyTileBytes;                 // Q (K-major), kept for every slice
  uint8_t* pt = qt + kTcQTileBytes;                     // P^T [128 keys][64 heads] bf16, swizzled (MN-major)
  uint8_t* misc = pt + kTcPTileBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(misc);   // [0] Q TMA, [1] MMA 1 done, [2] MMA 2 done,
                                                        // [3] FP4 row gather, [4] window rows TMA
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc + 48);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 52);
  int* rescale_flag = reinterpret_cast<int*>(misc + 56);
  int* valid_s = reinterpret_cast<int*>(misc + 64);                  // [128]
  float* red_s = reinterpret_cast<float*>(misc + 576);               // [2][4 quarters][64 heads]: max, sum
  float* ref_s = reinterpret_cast<float*>(misc + 2624);              // [64] running reference max (log2 units)
  float* sum_s = reinterpret_cast<float*>(misc + 2880);              // [64] running sum of P
  float* fac_s = reinterpret_cast<float*>(misc + 3136);              // [64] rescale factor of this slice
  float* wsc_s = reinterpret_cast<float*>(misc + 3392);              // [128] FP8 window: row scale per key

  const int bq = blockIdx.y;
  const int b = bq / p.Q, qi = bq % p.Q;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int first_slice = p.per_query ? 0 : static_cast<int>(blockIdx.x);
  const int n_iter = p.per_query ? p.slices : 1;

  if (tid == 0) {
    for (int i = 0; i < 5; ++i) mbar_init(&bars[i], 1);
    *abort_flag = 0;
    *rescale_flag = 0;
    fence_barrier_init();
  }
  if (tid < 64) { ref_s[tid] = -INFINITY; sum_s[tid] = 0.0f; }
  // cluster merge: every CTA of the cluster has started before another one
  // writes its shared memory (arrive now, wait before the first remote store)
  if (p.cluster_merge) cluster_arrive_relaxed();
  if (warp == 1) { tmem_alloc(tmem_slot, 512); tmem_relinquish(); }
  if (tid == 0) { tma_prefetch_desc(&tmap_q); tma_prefetch_desc(&tmap_swa); }
  pdl_launch_dependents();
  // idx comes from the previous kernel, and the partial outputs overwrite a
  // buffer the previous layer's merge reads: those wait for the predecessor
  if (!p.early_inputs) pdl_wait();
  uint8_t* qstage = kt + 65536;                         // q_fp4: [64][288] FP4 rows (past the gather's staging)
  if (tid == 0) {                                       // this thread initialised the barrier
    if (p.q_fp4) {
      mbar_arrive_expect_tx(&bars[0], 64 * 288);
      bulk_load(qstage, p.q4 + static_cast<int64_t>(bq) * 64 * 288, 64 * 288, &bars[0]);
    } else {
      mbar_arrive_expect_tx(&bars[0], kTcQTileBytes);
      const uint64_t pol = l2_policy_evict_last();
      for (int c = 0; c < 8; ++c) tma_load_2d(qt + c * 8192, &tmap_q, &bars[0], 64 * c, bq * 64, pol);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // ---- quantised Q.  The FP4 path's operands live in the Q region: codes
  //      [64 heads][256 B] (two 128-byte-swizzled boxes), then 8 scale
  //      chunks (one per MMA step of 64 dims), then the slice's entries
  //      repacked the same way ([128 keys][256 B] and 8 scale chunks).
  const bool fp4_mma = p.q_fp4 && !p.per_query && first_slice < p.kv_slices;
  uint8_t* q4 = qt;
  uint8_t* sfq = qt + 16384;
  uint8_t* k4 = qt + 20480;
  uint8_t* sfk = qt + 53248;
  // FP4 Q rows -> the FP4 MMA's operands (to_fp4: codes in two
  // 128-byte-swizzled boxes, scales in 8 chunks, one per MMA step), or the
  // values expanded to bf16 (exact) into the bf16 Q tile.  Thread t: head
  // t / 8, dims 64 (t % 8).. (32 code bytes, 4 scales).  Every thread of
  // the CTA calls it at the same point (it ends with a CTA barrier).
  auto unpack_q = [&](bool to_fp4) {
    const bool okq = mbar_wait(&bars[0], 0, kErrWaitOperand, abort_flag);
    const int h = tid >> 3, part = tid & 7;
    const uint8_t* row = qstage + h * 288;
    const uint4 c0 = okq ? *reinterpret_cast<const uint4*>(row + 32 * part) : make_uint4(0, 0, 0, 0);
    const uint4 c1 = okq ? *reinterpret_cast<const uint4*>(row + 32 * part + 16) : make_uint4(0, 0, 0, 0);
    const uint32_t scw = okq ? *reinterpret_cast<const uint32_t*>(row + 256 + 4 * part) : 0u;
    if (to_fp4) {
      // dims 64 part.. = box part/4, bytes 32 (part % 4).. of the row: chunks 2 (part % 4), +1
      uint8_t* box = q4 + (part >> 2) * 8192 + (h >> 3) * 1024 + (h & 7) * 128;
      const int ch = 2 * (part & 3);
      *reinterpret_cast<uint4*>(box + ((ch ^ (h & 7)) << 4)) = c0;
      *reinterpret_cast<uint4*>(box + (((ch + 1) ^ (h & 7)) << 4)) = c1;
      *reinterpret_cast<uint32_t*>(sfq + part * 512 + sf_chunk_off(h, 0)) = scw;
    } else {
      // dims 64 part.. = bf16 box part, 16-byte units 0..7 of row h
      uint8_t* box = qt + part * 8192;
      const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
      for (int wd = 0; wd < 8; ++wd) {
        const float sv = e4m3_code_to_float((scw >> (8 * (wd >> 1))) & 0xFF);   // 16 values per scale
        uint32_t o[4];
        e2m1x8_to_bf16(words[wd], __floats2bfloat162_rn(sv, sv), o);
        *reinterpret_cast<uint4*>(box + sw128_off(h, wd)) = make_uint4(o[0], o[1], o[2], o[3]);
      }
    }
    fence_async_smem();
    __syncthreads();
  };
  // CTAs of the FP4 MMA unpack Q while their entry rows are on the way
  if (p.q_fp4 && !fp4_mma) unpack_q(false);

  for (int it = 0; it < n_iter; ++it) {
    const int slice = first_slice + it;
    const bool window = slice >= p.kv_slices;
    const int key0 = window ? (slice - p.kv_slices) * kTcAttnKeys : slice * kTcAttnKeys;   // first key of the slice
    const int nkeys = window ? min(kTcAttnKeys, p.W - key0) : min(kTcAttnKeys, p.K - key0);
    const uint32_t ph = static_cast<uint32_t>(it & 1);                 // MMA barriers complete once per slice
    // the window barrier completes once per window slice (KV slices come
    // first); in split mode it is used at most once
    const uint32_t ph_win = p.per_query ? static_cast<uint32_t>((slice - p.kv_slices) & 1) : 0u;

    // the key tile and P^T are free once the previous slice's MMA 2 is done
    if (it > 0) {
      mbar_wait(&bars[2], ph ^ 1, kErrWaitTmemFull, abort_flag);
      tc_fence_after();
    }
    if (p.early_inputs && !window && it == 0) pdl_wait();
    int v = 0;
    if (tid < kTcAttnKeys) {
      if (tid < nkeys) {
        if (window) {
          v = 1;
        } else {
          const int32_t e = p.idx[static_cast<int64_t>(bq) * p.K + key0 + tid];
          v = (e >= 0 && e < p.N) ? e + 1 : 0;            // entry + 1, 0 = empty slot
        }
      }
      valid_s[tid] = v;
    }
    __syncthreads();

    // ---- operands: window rows by TMA; FP4 rows loaded by the threads
    //      (read-only path, 16 nibble bytes + 2 scales per item) and
    //      dequantised in registers
    if (tid == 0 && window && !p.swa_fp8) {
      const uint64_t pol = l2_policy_evict_last();
      mbar_arrive_expect_tx(&bars[4], kTcKeyTileBytes);
      const int32_t y = b * p.swa_rows + qi * p.swa_step + key0;
      for (int c = 0; c < 8; ++c) tma_load_2d(kt + c * 16384, &tmap_swa, &bars[4], 64 * c, y, pol);
    }
    if (window && p.swa_fp8) {
      // FP8 window rows: warp w loads rows 8w..8w+7 (512 codes, 16 per lane,
      // one coalesced load per row), expands E4M3 to bf16 exactly and
      // stores the key tile; the row scale multiplies the row's logits and
      // its softmax weights later (wsc_s)
      const int64_t row0 = static_cast<int64_t>(b) * p.swa_rows + qi * p.swa_step + key0;
      if (tid < kTcAttnKeys) wsc_s[tid] = (tid < nkeys) ? p.swa_scale[row0 + tid] : 0.0f;
      uint4 raw[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int r = 8 * warp + j;
        raw[j] = (r < nkeys) ? __ldg(reinterpret_cast<const uint4*>(p.swa8 + (row0 + r) * 512) + lane)
                             : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int r = 8 * warp + j;
        uint32_t o[8];
        e4m3x4_to_bf16(raw[j].x, o[0], o[1]);
        e4m3x4_to_bf16(raw[j].y, o[2], o[3]);
        e4m3x4_to_bf16(raw[j].z, o[4], o[5]);
        e4m3x4_to_bf16(raw[j].w, o[6], o[7]);
        // channels 16 lane .. 16 lane + 15 = chunk lane/4, units 2(lane%4), +1
        uint8_t* chunk = kt + (lane >> 2) * 16384;
        *reinterpret_cast<uint4*>(chunk + sw128_off(r, 2 * (lane & 3))) = make_uint4(o[0], o[1], o[2], o[3]);
        *reinterpret_cast<uint4*>(chunk + sw128_off(r, 2 * (lane & 3) + 1)) = make_uint4(o[4], o[5], o[6], o[7]);
      }
      fence_async_smem();
    }
    if (!window) {
      // Gather: warp w loads keys 8w..8w+7, one 288-byte row per load (lane
      // l < 18 loads bytes 16l..16l+15), all eight loads in flight at once,
      // into a staging area at the start of the key tile.  Then every thread
      // takes four items (key r, 32-channel chunk c: 16 nibble bytes and two
      // scales) from the staging area into registers, and after a barrier
      // expands them into the tile, which overwrites the staging area.  A
      // warp's items are 32 consecutive keys of one chunk, so its swizzled
      // 16-byte stores hit 32 different bank groups.
      uint8_t* stage = kt;                                // [128 keys][288 B]
      uint4 raw[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int vr = valid_s[8 * warp + j];
        raw[j] = make_uint4(0, 0, 0, 0);
        if (vr != 0 && lane < 18)
          raw[j] = __ldg(reinterpret_cast<const uint4*>(p.kv + (static_cast<int64_t>(b) * p.N + (vr - 1)) * 288) + lane);
      }
      if (fp4_mma && it == 0) unpack_q(true);            // the row loads are in flight meanwhile
      if (lane < 18) {
#pragma unroll
        for (int j = 0; j < 8; ++j) *reinterpret_cast<uint4*>(stage + (8 * warp + j) * 288 + 16 * lane) = raw[j];
      }
      __syncthreads();
      constexpr int kItems = kTcAttnKeys * 16 / kTcAttnThreads;
      uint4 nib[kItems];
      uint32_t sc[kItems];
#pragma unroll
      for (int k = 0; k < kItems; ++k) {
        const int i = tid + k * kTcAttnThreads;
        const int r = i & (kTcAttnKeys - 1), c = i >> 7;
        nib[k] = *reinterpret_cast<const uint4*>(stage + r * 288 + c * 16);
        sc[k] = *reinterpret_cast<const uint16_t*>(stage + r * 288 + 256 + 2 * c);
      }
      if (fp4_mma) {
        // repack for the FP4 MMA 1: thread (key r, quarter qq) moves dims
        // 128 qq..128 qq+127 (64 nibble bytes: box qq/2, chunks 4(qq%2)..)
        // and their 8 scales (MMA steps 2qq, 2qq+1: one word each)
        const int r = tid & (kTcAttnKeys - 1), qq = tid >> 7;
        const uint8_t* src = stage + r * 288;
        uint8_t* box = k4 + (qq >> 1) * 16384 + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int ch = 4 * (qq & 1) + u;
          *reinterpret_cast<uint4*>(box + ((ch ^ (r & 7)) << 4)) = *reinterpret_cast<const uint4*>(src + 64 * qq + 16 * u);
        }
        const uint2 scw = *reinterpret_cast<const uint2*>(src + 256 + 8 * qq);
        *reinterpret_cast<uint32_t*>(sfk + (2 * qq) * 512 + sf_chunk_off(r, 0)) = scw.x;
        *reinterpret_cast<uint32_t*>(sfk + (2 * qq + 1) * 512 + sf_chunk_off(r, 0)) = scw.y;
        fence_async_smem();
      }
      __syncthreads();
      if (fp4_mma && warp == 1 && lane == 0) {
        // MMA 1 on the FP4 tensor path, while the threads expand the
        // entries for MMA 2: scale chunks into tensor memory, then 8 steps
        tc_fence_after();
        const uint32_t sfq_col = tmem + 320, sfk_col = tmem + 352;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          tmem_cp_sf_chunk(sfq_col + 4 * j, umma_desc_sf_chunk(smem_u32(sfq + 512 * j)));
          tmem_cp_sf_chunk(sfk_col + 4 * j, umma_desc_sf_chunk(smem_u32(sfk + 512 * j)));
        }
        constexpr uint32_t idesc = umma_idesc_nvf4(128, 64);
        const uint32_t ka = smem_u32(k4), qa = smem_u32(q4);
#pragma unroll
        for (int j = 0; j < 8; ++j)
          umma_nvf4(tmem, umma_desc_sw128_kmajor(ka + (j >> 2) * 16384 + (j & 3) * 32),
                    umma_desc_sw128_kmajor(qa + (j >> 2) * 8192 + (j & 3) * 32), idesc, sfk_col + 4 * j,
                    sfq_col + 4 * j, j > 0 ? 1u : 0u);
        umma_commit(&bars[1]);
      }
#pragma unroll
      for (int k = 0; k < kItems; ++k) {
        const int i = tid + k * kTcAttnThreads;
        const int r = i & (kTcAttnKeys - 1), c = i >> 7;
        const float s0 = e4m3_code_to_float(sc[k] & 0xFF), s1 = e4m3_code_to_float(sc[k] >> 8);
        const __nv_bfloat162 S0 = __floats2bfloat162_rn(s0, s0), S1 = __floats2bfloat162_rn(s1, s1);
        uint32_t o[4][4];
        e2m1x8_to_bf16(nib[k].x, S0, o[0]);          // channels 32c .. 32c+7
        e2m1x8_to_bf16(nib[k].y, S0, o[1]);          //          .. 32c+15 (first scale block)
        e2m1x8_to_bf16(nib[k].z, S1, o[2]);
        e2m1x8_to_bf16(nib[k].w, S1, o[3]);          // empty slot: zero nibbles and scale -> zero key
        // channels 32c..32c+31 = chunk c/2 of the tile, units 4(c&1)..4(c&1)+3
        uint8_t* chunk = kt + (c >> 1) * 16384;
#pragma unroll
        for (int t = 0; t < 4; ++t)
          *reinterpret_cast<uint4*>(chunk + sw128_off(r, 4 * (c & 1) + t)) = make_uint4(o[t][0], o[t][1], o[t][2], o[t][3]);
      }
      fence_async_smem();
    }
    __syncthreads();

    // ---- MMA 1: S^T = K . Q^T  (M = 128 keys, N = 64 heads, K = 512 dims);
    //      already issued on the FP4 path for quantised Q
    if (warp == 1 && lane == 0 && !(fp4_mma && !window)) {
      bool ok = mbar_wait(&bars[0], 0, kErrWaitOperand, abort_flag);
      if (ok && window && !p.swa_fp8) ok = mbar_wait(&bars[4], ph_win, kErrWaitOperand, abort_flag);
      if (ok) {
        tc_fence_after();
        constexpr uint32_t idesc = umma_idesc_bf16_f32(128, 64);
        const uint32_t ka = smem_u32(kt), qa = smem_u32(qt);
#pragma unroll
        for (int kk = 0; kk < 32; ++kk) {
          const uint32_t koff = (kk >> 2) * 16384 + (kk & 3) * 32;
          const uint32_t qoff = (kk >> 2) * 8192 + (kk & 3) * 32;
          umma_bf16(tmem, umma_desc_sw128_kmajor(ka + koff), umma_desc_sw128_kmajor(qa + qoff), idesc, kk > 0);
        }
      }
      umma_commit(&bars[1]);
    }

    // ---- softmax in registers.  Warp w reads TMEM lanes 32(w%4).. (its 32
    //      keys) for heads 16(w/4)..16(w/4)+15; per-head max and sum reduce
    //      over the lanes by shuffles and over the four key quarters through
    //      shared memory.
    {
      const int quarter = warp & 3, hg = warp >> 2;
      const int key = quarter * 32 + lane;
      float sv[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) sv[j] = -INFINITY;
      const bool ok = mbar_wait(&bars[1], ph, kErrWaitTmemFull, abort_flag);
      if (__all_sync(0xffffffffu, ok)) {
        tc_fence_after();
        const bool kv_ok = valid_s[key] != 0;
        // an FP8 window key's logits carry its row scale
        const float ls = p.scale_log2 * ((window && p.swa_fp8) ? wsc_s[key] : 1.0f);
        uint32_t r[16];
        tmem_ld_32x32b_x16(tmem + (static_cast<uint32_t>(quarter * 32) << 16) + 16 * hg, r);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j) sv[j] = kv_ok ? __uint_as_float(r[j]) * ls : -INFINITY;
      }
      {
        const float m = warp_reduce_heads16<true>(sv, lane);
        if ((lane & 1) == 0) red_s[quarter * 64 + 16 * hg + (lane >> 1)] = m;
      }
      __syncthreads();
      // reference max per head: the running one unless this slice's max
      // exceeds it by more than kTcRefSlack
      float lj[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int h = 16 * hg + j;
        const float mt = fmaxf(fmaxf(red_s[h], red_s[64 + h]), fmaxf(red_s[128 + h], red_s[192 + h]));
        const float ref = ref_s[h];
        const float nref = (mt > ref + kTcRefSlack) ? mt : ref;
        lj[j] = exp2f(sv[j] - ((nref == -INFINITY) ? 0.0f : nref));
      }
      uint32_t pk[8];
      if (window && p.swa_fp8) {
        // MMA 2 multiplies the weight by the key's unscaled codes: fold the
        // row scale into the weight it sees, and sum the weights that this
        // rounded product stands for (weight = bf16(P s) / s), so that the
        // output stays a normalised combination of the rows
        const float rs = wsc_s[key];
        const float inv = (rs != 0.0f) ? 1.0f / rs : 0.0f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const __nv_bfloat162 v2 = __floats2bfloat162_rn(lj[2 * j] * rs, lj[2 * j + 1] * rs);
          pk[j] = *reinterpret_cast<const uint32_t*>(&v2);
          if (rs != 0.0f) {
            const float2 f = __bfloat1622float2(v2);
            lj[2 * j] = f.x * inv;
            lj[2 * j + 1] = f.y * inv;
          }
        }
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const __nv_bfloat162 v2 = __floats2bfloat162_rn(lj[2 * j], lj[2 * j + 1]);
          pk[j] = *reinterpret_cast<const uint32_t*>(&v2);
          const float2 f = __bfloat1622float2(v2);      // the sum uses the rounded weights MMA 2 sees
          lj[2 * j] = f.x;
          lj[2 * j + 1] = f.y;
        }
      }
      *reinterpret_cast<uint4*>(pt + sw128_off(key, 2 * hg)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      *reinterpret_cast<uint4*>(pt + sw128_off(key, 2 * hg + 1)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
      {
        const float l = warp_reduce_heads16<false>(lj, lane);
        if ((lane & 1) == 0) red_s[256 + quarter * 64 + 16 * hg + (lane >> 1)] = l;
      }
      fence_async_smem();
      __syncthreads();
      if (tid < 64) {
        const int h = tid;
        const float mt = fmaxf(fmaxf(red_s[h], red_s[64 + h]), fmaxf(red_s[128 + h], red_s[192 + h]));
        const float l = (red_s[256 + h] + red_s[320 + h]) + (red_s[384 + h] + red_s[448 + h]);
        const float ref = ref_s[h];
        const float nref = (mt > ref + kTcRefSlack) ? mt : ref;
        const float f = (nref == ref || ref == -INFINITY) ? 1.0f : exp2f(ref - nref);
        fac_s[h] = f;
        if (f != 1.0f && it > 0) *rescale_flag = 1;       // the accumulator holds earlier slices
        ref_s[h] = nref;
        sum_s[h] = sum_s[h] * f + l;
        if (!p.per_query && !p.cluster_merge) {
          if (p.early_inputs && window) pdl_wait();
          float* ml = p.ml + ((static_cast<int64_t>(bq) * p.slices + slice) * 64 + h) * 2;
          ml[0] = nref;
          ml[1] = l;
        }
      }
      // one slice per CTA: nothing below reads the running state, and P^T is
      // already published to the MMA issuer by the barrier above
      if (p.per_query) {
        tc_fence_before();
        __syncthreads();
      }
    }

    // ---- rescale the accumulator (rare: a slice max far above the reference)
    if (p.per_query && *rescale_flag) {
      const int quarter = warp & 3, t = warp >> 2;
#pragma unroll 1
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t r[32];
        const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + 64 + 64 * t + 32 * hh;
        tc_fence_after();
        tmem_ld_32x32b_x32(taddr, r);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(__uint_as_float(r[j]) * fac_s[32 * hh + j]);
        tmem_st_32x32b_x32(taddr, r);
        tmem_st_wait();
      }
      tc_fence_before();
      __syncthreads();
      if (tid == 0) *rescale_flag = 0;
    }

    // ---- MMA 2: O^T += V^T . P^T  (M = 128 dims per tile, N = 64 heads, K = 128 keys)
    if (warp == 1 && lane == 0) {
      tc_fence_after();
      if (!*abort_flag) {
        // A (V^T) and B (P^T) both MN-major
        constexpr uint32_t idesc = umma_idesc_bf16_f32(128, 64) | (1u << 15) | (1u << 16);
        const uint32_t ka = smem_u32(kt), pa = smem_u32(pt);
#pragma unroll
        for (int t = 0; t < 4; ++t) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t adesc = umma_desc_sw128_mnmajor(ka + (2 * t) * 16384 + kk * 2048, 16384);
            const uint64_t bdesc = umma_desc_sw128_mnmajor(pa + kk * 2048, 16384);
            umma_bf16(tmem + 64 + 64 * t, adesc, bdesc, idesc, (it > 0 || kk > 0) ? 1u : 0u);
          }
        }
      }
      umma_commit(&bars[2]);
    }
  }

  if (p.cluster_merge) {
    // ---- cluster merge.  Every CTA reaches both cluster barriers whatever
    //      happened before (all earlier waits are bounded), so no CTA of the
    //      cluster can be left waiting.
    const uint32_t C = cluster_size(), rank = cluster_rank();
    const uint32_t jmax = (16 + C - 1) / C;              // 32-dim chunks per owner
    float* stat = reinterpret_cast<float*>(misc + kTcStatOff);    // [rank][64 heads][max, sum]
    // recv[source rank][chunk j][head group 0..7][dim 0..31][8 heads bf16]:
    // one warp store puts 32 consecutive 16-byte pieces (512 contiguous
    // bytes) into the owner, the fewest and largest remote packets
    uint8_t* recv = kt;
    const bool ok = mbar_wait(&bars[2], 0, kErrWaitTmemFull, abort_flag);   // MMA 2 done
    cluster_wait_acquire();                              // pairs with the arrive at the start
    if (tid < 64) {
      const uint32_t la = smem_u32(stat + (rank * 64 + tid) * 2);
      for (uint32_t r = 0; r < C; ++r) dsmem_st_f32x2(dsmem_map(la, r), ref_s[tid], sum_s[tid]);
    }
    tc_fence_before();
    cluster_arrive_release();
    cluster_wait_acquire();                              // statistics everywhere; every CTA's MMA 2 done
    tc_fence_after();
    float* mj_s = red_s;                                 // [64] joint max, [64] joint sum (scratch reuse)
    if (tid < 64) {
      float M = -INFINITY;
      for (uint32_t r = 0; r < C; ++r) M = fmaxf(M, stat[(r * 64 + tid) * 2]);
      float L = 0.0f;
      if (M != -INFINITY)
        for (uint32_t r = 0; r < C; ++r) {
          const float m = stat[(r * 64 + tid) * 2];
          if (m != -INFINITY) L += exp2f(m - M) * stat[(r * 64 + tid) * 2 + 1];
        }
      const float m = ref_s[tid];
      fac_s[tid] = (L > 0.0f && m != -INFINITY) ? exp2f(m - M) / L : 0.0f;
      mj_s[tid] = M;
      mj_s[64 + tid] = L;
    }
    __syncthreads();
    {
      // warp w holds dims 32w..32w+31 (TMEM lanes 32(w%4).., tile w/4) for
      // all 64 heads; chunk w goes, scaled and rounded to bf16 (the final
      // output's precision), to rank w mod C: 8 vector stores of 8 heads
      const int quarter = warp & 3, t = warp >> 2;
      const uint32_t owner = static_cast<uint32_t>(warp) % C, j = static_cast<uint32_t>(warp) / C;
      const uint32_t base = smem_u32(recv + ((rank * jmax + j) * 8) * 512 + 16 * lane);
      const uint32_t rbase = dsmem_map(base, owner);
      const bool all_ok = __all_sync(0xffffffffu, ok);
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t r[32];
        if (all_ok) {
          tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(quarter * 32) << 16) + 64 + 64 * t + 32 * hh, r);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) r[jj] = 0u;
        }
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          uint32_t pk[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int h = 32 * hh + 8 * g + 2 * e;
            pk[e] = pack_bf16x2(__uint_as_float(r[8 * g + 2 * e]) * fac_s[h],
                                __uint_as_float(r[8 * g + 2 * e + 1]) * fac_s[h + 1]);
          }
          dsmem_st_v4(rbase + (4 * hh + g) * 512, pk[0], pk[1], pk[2], pk[3]);
        }
      }
    }
    tc_fence_before();
    cluster_arrive_release();
    cluster_wait_acquire();                              // every chunk delivered to its owner
    if (p.early_inputs) pdl_wait();                      // stores wait for the predecessor
    if (!*abort_flag) {
      // this CTA's chunks c = rank + C j: item (j, head group of 8, dim d) sums
      // the C sources in fp32; lanes run over d, so each of the 8 bf16 stores
      // of an item writes 64 contiguous bytes per warp
      const uint32_t nown = (16 - rank + C - 1) / C;
      for (uint32_t it = warp; it < nown * 8; it += kTcAttnThreads / 32) {
        const uint32_t j = it >> 3, hg = it & 7, d = lane;
        float a[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (uint32_t r = 0; r < C; ++r) {
          const uint4 v = *reinterpret_cast<const uint4*>(recv + ((r * jmax + j) * 8 + hg) * 512 + 16 * d);
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  #pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[e]));
            a[2 * e] += f.x;
            a[2 * e + 1] += f.y;
          }
        }
        const uint32_t c = rank + C * j;
        __nv_bfloat16* o = p.out + (static_cast<int64_t>(bq) * 64 + 8 * hg) * 512 + 32 * c + d;
  #pragma unroll
        for (int e = 0; e < 8; ++e) o[e * 512] = __float2bfloat16_rn(a[e]);
      }
      if (rank == 0 && p.lse && tid < 64) {
        const float L = mj_s[64 + tid];
        p.lse[static_cast<int64_t>(bq) * 64 + tid] = (L > 0.0f) ? (mj_s[tid] + log2f(L)) * 0.69314718055994531f : -INFINITY;
      }
    }
    if (warp == 1) {                                     // TMEM was last read before the second barrier
      tc_fence_after();
      tmem_dealloc(tmem, 512);
    }
    return;
  }

  // ---- epilogue: O^T tile (warp / 4), dims 32(warp % 4).. -> shared
  //      [head][dim] (the key tile is free now)
  float* obuf = reinterpret_cast<float*>(kt);
  {
    const bool ok = mbar_wait(&bars[2], static_cast<uint32_t>((n_iter - 1) & 1), kErrWaitTmemFull, abort_flag);
    if (__all_sync(0xffffffffu, ok)) {
      tc_fence_after();
      const int quarter = warp & 3, t = warp >> 2;
      const int d = 128 * t + 32 * quarter + lane;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(quarter * 32) << 16) + 64 + 64 * t + 32 * hh, r);
        tmem_ld_wait();
        if (p.per_query) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float l = sum_s[32 * hh + j];
            obuf[(32 * hh + j) * 512 + d] = (l > 0.0f) ? __uint_as_float(r[j]) / l : 0.0f;
          }
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) obuf[(32 * hh + j) * 512 + d] = __uint_as_float(r[j]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {                                      // TMEM is no longer read: free it early
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (p.early_inputs) pdl_wait();                       // window-only CTAs have not waited yet
  if (*abort_flag) return;
  if (!p.per_query) {
    float4* op = reinterpret_cast<float4*>(p.opart + (static_cast<int64_t>(bq) * p.slices + first_slice) * 64 * 512);
    const float4* src = reinterpret_cast<const float4*>(obuf);
#pragma unroll 4
    for (int j = tid; j < 64 * 512 / 4; j += kTcAttnThreads) op[j] = src[j];
  } else {
    // bf16 output, 8 dims (16 bytes) per store
    uint4* op = reinterpret_cast<uint4*>(p.out + static_cast<int64_t>(bq) * 64 * 512);
#pragma unroll 4
    for (int j = tid; j < 64 * 512 / 8; j += kTcAttnThreads) {
      const float4 a = reinterpret_cast<const float4*>(obuf)[2 * j];
      const float4 c = reinterpret_cast<const float4*>(obuf)[2 * j + 1];
      op[j] = make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(c.x, c.y), pack_bf16x2(c.z, c.w));
    }
    if (p.lse && tid < 64) {
      const float l = sum_s[tid];
      p.lse[static_cast<int64_t>(bq) * 64 + tid] =
          (l > 0.0f) ? (ref_s[tid] + log2f(l)) * 0.69314718055994531f : -INFINITY;
    }
  }
}

}  // namespace csa2
