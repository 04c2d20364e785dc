// attention_tc.cuh -- sparse MQA slice kernel on the 5th-generation tensor
// cores ("DeepSeek V4.1-Flash 技术报告深度解析" §3.2 attention, §3.4
// dequantise before the attention math).
//
// One CTA (512 threads) per (128-key slice, query).  The slice's keys (FP4
// entries, each 288-byte row fetched by one bulk copy and dequantised by the
// CTA's threads, or window rows brought by TMA) form a 128 x 512 bf16 tile
// K in shared memory, stored K-major with the 128-byte swizzle.  The
// query's 64 heads form Q (64 x 512, TMA).  Then:
//   MMA 1   S^T[key, head] = K . Q^T            M = 128 keys, N = 64, K = 512
//   softmax per head over the slice's keys (fp32, from TMEM via shared
//           memory), P^T[head, key] = exp2(S^T - max) rounded to bf16 and
//           stored as a K-major operand
//   MMA 2   O^T[dim, head] = V^T . P^T          the same key tile read
//           MN-major (M = 128 dims per MMA, 4 tiles), N = 64, K = 128 keys
//   epilogue: O^T from TMEM to shared memory as [head][dim] fp32, then
//           coalesced 16-byte stores to the slice's partial output; with the
//           slice's (max, sum) per head, sparse_attn_combine_kernel merges the
//           slices.
// Accumulators: S^T in TMEM columns [0, 64), O^T tile t in [64 + 64t, 128 + 64t).
#pragma once
#include "common.cuh"
#include "attention.cuh"

namespace csa2 {

constexpr int kTcAttnThreads = 512;
constexpr int kTcAttnWarps = kTcAttnThreads / 32;
constexpr int kTcAttnKeys = 128;                       // keys per slice (MMA M)
constexpr uint32_t kTcKeyTileBytes = 128 * 512 * 2;    // 128 KB: 8 chunks of [128 rows x 64 dims]
constexpr uint32_t kTcQTileBytes = 64 * 512 * 2;       // 64 KB: 8 chunks of [64 rows x 64 dims]
constexpr int kTcSPitch = kTcAttnKeys + 4;             // fp32 row pitch of the transposed scores
constexpr uint32_t kTcMiscBytes = 2048;
constexpr uint32_t kTcAttnSmem = kTcKeyTileBytes + kTcQTileBytes + kTcMiscBytes + 1024;

struct TcAttnParams {
  int B, Q, K, W;
  int64_t N;
  const uint8_t* kv;
  const int32_t* idx;
  int swa_rows, swa_step;
  int kv_slices;             // ceil(K / 128): slices 0..kv_slices-1 hold FP4 entries, the rest window rows
  int slices;
  float scale_log2;
  float* opart;              // [BQ][slices][64][512]
  float* ml;                 // [BQ][slices][64][2]
};

// byte offset of the 16-byte unit u (0..7) of row r in a K-major operand
// chunk of 128-byte rows with the 128-byte swizzle
__device__ __forceinline__ uint32_t sw128_off(int r, int u) {
  return static_cast<uint32_t>((r >> 3) * 1024 + (r & 7) * 128 + ((u ^ (r & 7)) << 4));
}

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

// Eight E2M1 codes (one 32-bit word of nibbles, code k in bits 4k..4k+3)
// to eight bf16 values (out[j] = codes 2j, 2j+1), times a bf16 scale.
// The magnitude (3 bits) selects the high and the low byte of the bf16
// pattern from two 8-byte tables held in registers (byte_perm); the sign
// bit is placed separately.  Products E2M1 x E4M3 are exact in bf16.
//   magnitude code:  0    1     2     3     4     5     6     7
//   value:           0    0.5   1     1.5   2     3     4     6
//   bf16:            0000 3F00  3F80  3FC0  4000  4040  4080  40C0
__device__ __forceinline__ void e2m1x8_to_bf16(uint32_t w, __nv_bfloat162 scale, uint32_t (&out)[4]) {
  const uint32_t m = w & 0x77777777u;
  const uint32_t lo_a = __byte_perm(0xC0800000u, 0xC0804000u, m);
  const uint32_t hi_a = __byte_perm(0x3F3F3F00u, 0x40404040u, m);
  const uint32_t lo_b = __byte_perm(0xC0800000u, 0xC0804000u, m >> 16);
  const uint32_t hi_b = __byte_perm(0x3F3F3F00u, 0x40404040u, m >> 16);
  uint32_t o[4];
  o[0] = __byte_perm(lo_a, hi_a, 0x5140) | ((w << 12) & 0x8000u) | ((w << 24) & 0x80000000u);
  o[1] = __byte_perm(lo_a, hi_a, 0x7362) | ((w << 4) & 0x8000u) | ((w << 16) & 0x80000000u);
  o[2] = __byte_perm(lo_b, hi_b, 0x5140) | ((w >> 4) & 0x8000u) | ((w << 8) & 0x80000000u);
  o[3] = __byte_perm(lo_b, hi_b, 0x7362) | ((w >> 12) & 0x8000u) | (w & 0x80000000u);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    __nv_bfloat162 x = *reinterpret_cast<__nv_bfloat162*>(&o[j]);
    x = __hmul2(x, scale);
    out[j] = *reinterpret_cast<uint32_t*>(&x);
  }
}

__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__global__ void __launch_bounds__(kTcAttnThreads, 1)
sparse_attn_tc_kernel(const __grid_constant__ CUtensorMap tmap_q,
                      const __grid_constant__ CUtensorMap tmap_swa,
                      TcAttnParams p) {
  extern __shared__ __align__(1024) uint8_t tc_attn_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(tc_attn_smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* kt = smem;                                   // key tile (K-major), later read MN-major as V^T
  uint8_t* qt = smem + kTcKeyTileBytes;                 // Q (K-major); after MMA 1: scores and P^T
  float* st = reinterpret_cast<float*>(qt);             // [64 heads][kTcSPitch] scaled scores
  uint8_t* pt = qt + 64 * kTcSPitch * 4;                // P^T: 2 chunks of [64 rows x 64 keys] (1024-aligned)
  uint8_t* misc = qt + kTcQTileBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(misc);   // [0] q/window TMA, [1] MMA 1 done, [2] MMA 2 done,
                                                        // [3] FP4 row gather
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* valid_s = reinterpret_cast<int*>(misc + 64);                  // [128]

  const int slice = blockIdx.x, bq = blockIdx.y;
  const int b = bq / p.Q, qi = bq % p.Q;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool window = slice >= p.kv_slices;
  const int key0 = window ? (slice - p.kv_slices) * kTcAttnKeys : slice * kTcAttnKeys;   // first key of the slice
  const int nkeys = window ? min(kTcAttnKeys, p.W - key0) : min(kTcAttnKeys, p.K - key0);

  if (tid == 0) {
    mbar_init(&bars[0], 1); mbar_init(&bars[1], 1); mbar_init(&bars[2], 1); mbar_init(&bars[3], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) { tmem_alloc(tmem_slot, 512); tmem_relinquish(); }
  if (tid == 0) { tma_prefetch_desc(&tmap_q); tma_prefetch_desc(&tmap_swa); }
  pdl_wait();                                           // idx, q and the FP4 rows come from earlier kernels
  pdl_launch_dependents();
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
  tc_fence_before();
  const int n_rows = __syncthreads_count(!window && v != 0);   // FP4 rows to gather
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // ---- operands: Q (and window rows) by TMA; FP4 rows by one bulk copy
  //      each into a staging area inside the key tile, then dequantised
  uint8_t* stage = kt;                                  // [128][288] raw rows (overwritten below)
  if (tid == 0) {
    const uint64_t pol = l2_policy_evict_last();
    if (n_rows) mbar_arrive_expect_tx(&bars[3], static_cast<uint32_t>(n_rows) * 288u);
    else mbar_arrive(&bars[3]);
    mbar_arrive_expect_tx(&bars[0], kTcQTileBytes + (window ? kTcKeyTileBytes : 0));
    for (int c = 0; c < 8; ++c) tma_load_2d(qt + c * 8192, &tmap_q, &bars[0], 64 * c, bq * 64, pol);
    if (window) {
      const int32_t y = b * p.swa_rows + qi * p.swa_step + key0;
      for (int c = 0; c < 8; ++c) tma_load_2d(kt + c * 16384, &tmap_swa, &bars[0], 64 * c, y, pol);
    }
  }
  if (!window) {
    __syncthreads();                                    // expect_tx is posted before any copy lands
    if (tid < kTcAttnKeys && v != 0) {
      const uint8_t* row = p.kv + (static_cast<int64_t>(b) * p.N + (v - 1)) * 288;
      asm volatile(
          "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], 288, [%2];"
          :: "r"(smem_u32(stage + tid * 288)), "l"(row), "r"(smem_u32(&bars[3])) : "memory");
    }
    // item = (key r, 32-channel chunk c): 16 nibble bytes + 2 scales -> four
    // 16-byte units of the key tile.  A warp takes 32 consecutive keys of one
    // chunk (conflict-free swizzled stores).  All raw items go to registers
    // before anything is written, since the tile overwrites the staging area.
    constexpr int kItems = kTcAttnKeys * 16 / kTcAttnThreads;
    const bool ok = mbar_wait(&bars[3], 0, kErrWaitOperand, abort_flag);
    uint4 nib[kItems];
    uint32_t sc[kItems];
#pragma unroll
    for (int k = 0; k < kItems; ++k) {
      const int i = tid + k * kTcAttnThreads;
      const int r = i & (kTcAttnKeys - 1), c = i >> 7;
      nib[k] = make_uint4(0, 0, 0, 0);
      sc[k] = 0;
      if (ok && valid_s[r]) {
        nib[k] = *reinterpret_cast<const uint4*>(stage + r * 288 + c * 16);
        sc[k] = *reinterpret_cast<const uint16_t*>(stage + r * 288 + 256 + 2 * c);
      }
    }
    __syncthreads();
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

  // ---- MMA 1: S^T = K . Q^T  (M = 128 keys, N = 64 heads, K = 512 dims)
  if (warp == 1 && lane == 0) {
    if (mbar_wait(&bars[0], 0, kErrWaitOperand, abort_flag)) {
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

  // ---- scores: TMEM -> scaled, masked, transposed into shared memory.
  //      Warp w reads TMEM lanes 32(w%4).. (its keys) and heads 16(w/4)..
  {
    const bool ok = mbar_wait(&bars[1], 0, kErrWaitTmemFull, abort_flag);
    if (__all_sync(0xffffffffu, ok)) {
      tc_fence_after();
      const int quarter = warp & 3, hg = warp >> 2;
      const int key = quarter * 32 + lane;
      const bool kv_ok = valid_s[key] != 0;
      uint32_t r[16];
      tmem_ld_32x32b_x16(tmem + (static_cast<uint32_t>(quarter * 32) << 16) + 16 * hg, r);
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 16; ++j)
        st[(16 * hg + j) * kTcSPitch + key] = kv_ok ? __uint_as_float(r[j]) * p.scale_log2 : -INFINITY;
    }
  }
  tc_fence_before();
  __syncthreads();

  // ---- softmax statistics per head; P^T in bf16 as the K-major B operand
  {
    const int h = tid >> 3, part = tid & 7;               // 8 threads per head, 16 keys each
    const float* srow = st + h * kTcSPitch + part * 16;
    float m = -INFINITY;
#pragma unroll
    for (int j = 0; j < 16; ++j) m = fmaxf(m, srow[j]);
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
    const float mu = (m == -INFINITY) ? 0.0f : m;
    float l = 0.0f;
    uint32_t pk[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const __nv_bfloat162 v = __floats2bfloat162_rn(exp2f(srow[2 * j] - mu), exp2f(srow[2 * j + 1] - mu));
      const float2 f = __bfloat1622float2(v);
      l += f.x + f.y;
      pk[j] = *reinterpret_cast<const uint32_t*>(&v);
    }
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    l += __shfl_xor_sync(0xffffffffu, l, 4);
    __syncthreads();                                      // every thread has read the scores it needs
    // keys 16part .. 16part+15 = chunk part/4, units 2(part&3), 2(part&3)+1 of row h
    uint8_t* chunk = pt + (part >> 2) * 8192;
#pragma unroll
    for (int t = 0; t < 2; ++t)
      *reinterpret_cast<uint4*>(chunk + sw128_off(h, 2 * (part & 3) + t)) =
          make_uint4(pk[4 * t], pk[4 * t + 1], pk[4 * t + 2], pk[4 * t + 3]);
    if (part == 0) {
      float* ml = p.ml + ((static_cast<int64_t>(bq) * p.slices + slice) * 64 + h) * 2;
      ml[0] = m;
      ml[1] = l;
    }
    fence_async_smem();
  }
  tc_fence_before();
  __syncthreads();

  // ---- MMA 2: O^T = V^T . P^T  (M = 128 dims per tile, N = 64 heads, K = 128 keys)
  if (warp == 1 && lane == 0) {
    tc_fence_after();
    if (!*abort_flag) {
      constexpr uint32_t idesc = umma_idesc_bf16_f32(128, 64) | (1u << 15);   // A MN-major
      const uint32_t ka = smem_u32(kt), pa = smem_u32(pt);
#pragma unroll
      for (int t = 0; t < 4; ++t) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t adesc = umma_desc_sw128_mnmajor(ka + (2 * t) * 16384 + kk * 2048, 16384);
          const uint64_t bdesc = umma_desc_sw128_kmajor(pa + (kk >> 2) * 8192 + (kk & 3) * 32);
          umma_bf16(tmem + 64 + 64 * t, adesc, bdesc, idesc, kk > 0);
        }
      }
    }
    umma_commit(&bars[2]);
  }

  // ---- epilogue: O^T tile (warp / 4), dims 32(warp % 4).. -> shared
  //      [head][dim] (the key tile is free now)
  float* obuf = reinterpret_cast<float*>(kt);
  {
    const bool ok = mbar_wait(&bars[2], 0, kErrWaitTmemFull, abort_flag);
    if (__all_sync(0xffffffffu, ok)) {
      tc_fence_after();
      const int quarter = warp & 3, t = warp >> 2;
      const int d = 128 * t + 32 * quarter + lane;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(quarter * 32) << 16) + 64 + 64 * t + 32 * hh, r);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 32; ++j) obuf[(32 * hh + j) * 512 + d] = __uint_as_float(r[j]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {                                      // TMEM is no longer read: free it early
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }

  if (!*abort_flag) {
    float4* op = reinterpret_cast<float4*>(p.opart + (static_cast<int64_t>(bq) * p.slices + slice) * 64 * 512);
    const float4* src = reinterpret_cast<const float4*>(obuf);
#pragma unroll 4
    for (int j = tid; j < 64 * 512 / 4; j += kTcAttnThreads) op[j] = src[j];
  }
}

}  // namespace csa2
