// attention.cuh -- sparse MQA over selected FP4 entries plus the SWA window
// ("DeepSeek V4.1-Flash 技术报告深度解析" §3.2 attention, §3.4 dequantise
// before the attention math).
//
// Keys of query (b,q): slot j < K is entry idx[j] of the FP4 cache (-1 =
// empty), slot K + r is window row q*swa_step + r.  Every key is also its
// value.  The key slots are split into 64-key slices; one CTA per
// (slice, query):
//   - stages the query's 64 heads x 512 dims and the slice's 64 keys in
//     shared memory as bf16 (FP4 entries are dequantised on the way in:
//     a 256-entry table turns each nibble byte into two E2M1 values and one
//     bf16x2 multiply applies the E4M3 scale, exactly);
//   - S = Q K^T (64 x 64) with m16n8k16 bf16 tensor-core MMAs, fp32
//     accumulate, softmax statistics (max, sum) per head in fp32;
//   - O_slice = P V (64 x 512) with P rounded to bf16, written unnormalised
//     in fp32 with its (max, sum) to the workspace.
// A second kernel merges the slices with a log-sum-exp combine and writes
// bf16 outputs and the natural-log LSE.
// HBM roofline per query: 288 B per selected entry + 1 KB per window row +
// 64 KB of queries + 64 KB of output (slice partials stay in L2).
#pragma once
#include "common.cuh"

namespace csa2 {

constexpr int kAttnThreads = 128;
constexpr int kAttnMaxK = 2048;      // largest K (CSA2_MAX_K)
constexpr int kAttnMaxW = 1024;      // largest window (CSA2_MAX_W)
constexpr int kAttnKeys = 64;        // key slots per slice
constexpr int kAttnSmem = 64 * 1024 * 2 + 1024 + 256 + 1024;   // q, keys, nibble table, flags, align

struct AttnParams {
  int B, Q, K, W;
  int64_t N;
  const __nv_bfloat16* q;
  const uint8_t* kv;
  const int32_t* idx;
  const __nv_bfloat16* swa;
  int swa_rows, swa_step;
  float scale_log2;          // logit scale * log2(e)
  float* opart;              // [BQ][slices][64][512]
  float* ml;                 // [BQ][slices][64][2]: running max (log2 units), sum
  int slices;
  __nv_bfloat16* out;        // [BQ][64][512]
  float* lse;                // optional [BQ][64]
};

// byte offset of 16-byte chunk c (0..63) of row r in a [rows][512] bf16 tile,
// XOR-swizzled so that ldmatrix rows fall in distinct banks
__device__ __forceinline__ uint32_t attn_swz(int r, int c) {
  return static_cast<uint32_t>(r) * 1024u + static_cast<uint32_t>((c ^ (r & 7)) << 4);
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" :: "r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// E2M1 magnitude of code c (0..7), from the bit fields: exponent e = c>>1
// (bias 1), mantissa m = c&1; subnormal when e == 0.
__device__ __forceinline__ float e2m1_code_value(int c) {
  const int e = (c >> 1) & 3, m = c & 1;
  const float mag = e ? ldexpf(1.0f + 0.5f * m, e - 1) : 0.5f * m;
  return (c & 8) ? -mag : mag;
}

__global__ void __launch_bounds__(kAttnThreads)
sparse_attn_slice_kernel(AttnParams p) {
  extern __shared__ __align__(1024) uint8_t attn_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(attn_smem_raw) + 127) & ~uintptr_t(127));
  uint8_t* q_s = smem;                                   // [64][512] bf16, swizzled
  uint8_t* k_s = smem + 65536;                           // [64][512] bf16, swizzled
  uint32_t* lut = reinterpret_cast<uint32_t*>(smem + 131072);   // 256 x bf16x2
  int* valid_s = reinterpret_cast<int*>(lut + 256);             // [64]

  const int slice = blockIdx.x, bq = blockIdx.y;
  const int b = bq / p.Q, qi = bq % p.Q;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t q_base = smem_u32(q_s), k_base = smem_u32(k_s);

  // query heads -> shared (async)
  const __nv_bfloat16* qg = p.q + static_cast<int64_t>(bq) * 64 * 512;
  for (int i = tid; i < 64 * 64; i += kAttnThreads) {
    const int r = i >> 6, c = i & 63;
    cp_async16(q_base + attn_swz(r, c), qg + r * 512 + c * 8);
  }
  // nibble-byte table: low nibble -> low half, high nibble -> high half
  for (int i = tid; i < 256; i += kAttnThreads)
    lut[i] = pack_bf16x2(e2m1_code_value(i & 15), e2m1_code_value(i >> 4));
  // which key slots of this slice hold a key
  if (tid < kAttnKeys) {
    const int j = slice * kAttnKeys + tid;
    int v = 0;
    if (j < p.K) {
      const int32_t e = p.idx[static_cast<int64_t>(bq) * p.K + j];
      v = e >= 0 && e < p.N;                 // anything outside the cache is an empty slot
    }
    else if (j < p.K + p.W) v = 1;
    valid_s[tid] = v;
  }
  __syncthreads();

  // window rows -> shared (async); FP4 entries -> dequantised bf16
  for (int i = tid; i < kAttnKeys * 64; i += kAttnThreads) {
    const int r = i >> 6, c = i & 63;
    const int j = slice * kAttnKeys + r;
    if (j >= p.K && j < p.K + p.W) {
      const __nv_bfloat16* src = p.swa + (static_cast<int64_t>(b) * p.swa_rows + qi * p.swa_step + (j - p.K)) * 512 + c * 8;
      cp_async16(k_base + attn_swz(r, c), src);
    } else if (!valid_s[r]) {
      *reinterpret_cast<uint4*>(k_s + attn_swz(r, c)) = make_uint4(0, 0, 0, 0);
    }
  }
  for (int i = tid; i < kAttnKeys * 16; i += kAttnThreads) {
    const int r = i >> 4, c = i & 15;                    // row r, 32-channel chunk c
    const int j = slice * kAttnKeys + r;
    if (j >= p.K || !valid_s[r]) continue;
    const int32_t e = p.idx[static_cast<int64_t>(bq) * p.K + j];
    const uint8_t* row = p.kv + (static_cast<int64_t>(b) * p.N + e) * 288;
    const uint4 nib = __ldg(reinterpret_cast<const uint4*>(row) + c);
    const uint16_t sc = __ldg(reinterpret_cast<const uint16_t*>(row + 256) + c);
    const float s0 = e4m3_code_to_float(sc & 0xFF), s1 = e4m3_code_to_float(sc >> 8);
    const __nv_bfloat162 S0 = __floats2bfloat162_rn(s0, s0), S1 = __floats2bfloat162_rn(s1, s1);
    const uint32_t w[4] = {nib.x, nib.y, nib.z, nib.w};
    uint32_t o[16];
#pragma unroll
    for (int t = 0; t < 16; ++t) {
      const uint32_t byte = (w[t >> 2] >> (8 * (t & 3))) & 0xFF;
      uint32_t v = lut[byte];
      __nv_bfloat162 x = *reinterpret_cast<__nv_bfloat162*>(&v);
      x = __hmul2(x, t < 8 ? S0 : S1);
      o[t] = *reinterpret_cast<uint32_t*>(&x);
    }
#pragma unroll
    for (int t = 0; t < 4; ++t)
      *reinterpret_cast<uint4*>(k_s + attn_swz(r, 4 * c + t)) = make_uint4(o[4 * t], o[4 * t + 1], o[4 * t + 2], o[4 * t + 3]);
  }
  cp_async_wait_all();
  __syncthreads();

  // ---------------- S = Q K^T for heads 16*warp .. 16*warp+15
  float sacc[8][4];
#pragma unroll
  for (int j = 0; j < 8; ++j) sacc[j][0] = sacc[j][1] = sacc[j][2] = sacc[j][3] = 0.0f;
#pragma unroll 4
  for (int kk = 0; kk < 32; ++kk) {
    uint32_t a[4];
    {
      const int r = 16 * warp + (lane & 7) + 8 * ((lane >> 3) & 1);
      const int c = 2 * kk + (lane >> 4);
      ldsm_x4(q_base + attn_swz(r, c), a[0], a[1], a[2], a[3]);
    }
#pragma unroll
    for (int jp = 0; jp < 4; ++jp) {
      uint32_t b0, b1, b2, b3;
      const int r = 16 * jp + (lane & 7) + 8 * (lane >> 4);
      const int c = 2 * kk + ((lane >> 3) & 1);
      ldsm_x4(k_base + attn_swz(r, c), b0, b1, b2, b3);
      mma_bf16_16816(sacc[2 * jp], a, b0, b1);
      mma_bf16_16816(sacc[2 * jp + 1], a, b2, b3);
    }
  }

  // ---------------- softmax statistics per head (rows g and g+8 of the warp)
  float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int n = 8 * j + 2 * (lane & 3);
    const bool v0 = valid_s[n], v1 = valid_s[n + 1];
    sacc[j][0] = v0 ? sacc[j][0] * p.scale_log2 : -INFINITY;
    sacc[j][1] = v1 ? sacc[j][1] * p.scale_log2 : -INFINITY;
    sacc[j][2] = v0 ? sacc[j][2] * p.scale_log2 : -INFINITY;
    sacc[j][3] = v1 ? sacc[j][3] * p.scale_log2 : -INFINITY;
    m0 = fmaxf(m0, fmaxf(sacc[j][0], sacc[j][1]));
    m1 = fmaxf(m1, fmaxf(sacc[j][2], sacc[j][3]));
  }
  m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, 1));
  m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, 2));
  m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, 1));
  m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, 2));
  const float mu0 = (m0 == -INFINITY) ? 0.0f : m0, mu1 = (m1 == -INFINITY) ? 0.0f : m1;
  float l0 = 0.0f, l1 = 0.0f;
  uint32_t pa[4][4];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const __nv_bfloat162 lo = __floats2bfloat162_rn(exp2f(sacc[j][0] - mu0), exp2f(sacc[j][1] - mu0));
    const __nv_bfloat162 hi = __floats2bfloat162_rn(exp2f(sacc[j][2] - mu1), exp2f(sacc[j][3] - mu1));
    const float2 flo = __bfloat1622float2(lo), fhi = __bfloat1622float2(hi);
    l0 += flo.x + flo.y;
    l1 += fhi.x + fhi.y;
    pa[j >> 1][(j & 1) * 2 + 0] = *reinterpret_cast<const uint32_t*>(&lo);
    pa[j >> 1][(j & 1) * 2 + 1] = *reinterpret_cast<const uint32_t*>(&hi);
  }
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);

  const int h0 = 16 * warp + (lane >> 2);
  float* ml = p.ml + (static_cast<int64_t>(bq) * p.slices + slice) * 64 * 2;
  if ((lane & 3) == 0) {
    ml[h0 * 2 + 0] = m0; ml[h0 * 2 + 1] = l0;
    ml[(h0 + 8) * 2 + 0] = m1; ml[(h0 + 8) * 2 + 1] = l1;
  }

  // ---------------- O = P V, 128 dims at a time
  float* op = p.opart + (static_cast<int64_t>(bq) * p.slices + slice) * 64 * 512;
#pragma unroll 1
  for (int dc = 0; dc < 4; ++dc) {
    float oacc[16][4];
#pragma unroll
    for (int j = 0; j < 16; ++j) oacc[j][0] = oacc[j][1] = oacc[j][2] = oacc[j][3] = 0.0f;
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      // A fragment of P for keys 16kk..16kk+15: n-tiles 2kk and 2kk+1
      const uint32_t a[4] = {pa[kk][0], pa[kk][1], pa[kk][2], pa[kk][3]};
#pragma unroll
      for (int jp = 0; jp < 8; ++jp) {
        uint32_t b0, b1, b2, b3;
        const int r = 16 * kk + (lane & 7) + 8 * ((lane >> 3) & 1);
        const int c = 16 * dc + 2 * jp + (lane >> 4);
        ldsm_x4_t(k_base + attn_swz(r, c), b0, b1, b2, b3);
        mma_bf16_16816(oacc[2 * jp], a, b0, b1);
        mma_bf16_16816(oacc[2 * jp + 1], a, b2, b3);
      }
    }
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int d = dc * 128 + 8 * j + 2 * (lane & 3);
      *reinterpret_cast<float2*>(op + h0 * 512 + d) = make_float2(oacc[j][0], oacc[j][1]);
      *reinterpret_cast<float2*>(op + (h0 + 8) * 512 + d) = make_float2(oacc[j][2], oacc[j][3]);
    }
  }
}

// Merge the slices of one (query, head): 128 threads x 4 dims.  The slice
// statistics are loaded once into shared memory; the partial outputs are
// fetched eight slices at a time so their L2 latencies overlap.
constexpr int kAttnMaxSlices = (kAttnMaxK + kAttnMaxW + kAttnKeys - 1) / kAttnKeys;

__global__ void __launch_bounds__(128)
sparse_attn_combine_kernel(AttnParams p) {
  __shared__ float m_s[kAttnMaxSlices], l_s[kAttnMaxSlices];
  const int bq = blockIdx.x >> 6, h = blockIdx.x & 63;
  const int t = threadIdx.x;
  const float* ml = p.ml + static_cast<int64_t>(bq) * p.slices * 128;
  if (t < p.slices) { m_s[t] = ml[t * 128 + h * 2]; l_s[t] = ml[t * 128 + h * 2 + 1]; }
  __syncthreads();
  float M = -INFINITY;
  for (int s = 0; s < p.slices; ++s) M = fmaxf(M, m_s[s]);
  float L = 0.0f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (M != -INFINITY) {
    const float4* op = reinterpret_cast<const float4*>(p.opart + (static_cast<int64_t>(bq) * p.slices * 64 + h) * 512) + t;
    const int64_t stride = 64 * 512 / 4;             // float4s between consecutive slices
    for (int s0 = 0; s0 < p.slices; s0 += 8) {
      float4 o[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (s0 + j < p.slices) o[j] = __ldcg(op + (s0 + j) * stride);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (s0 + j >= p.slices || m_s[s0 + j] == -INFINITY) continue;
        const float f = exp2f(m_s[s0 + j] - M);
        L += f * l_s[s0 + j];
        acc.x += f * o[j].x; acc.y += f * o[j].y; acc.z += f * o[j].z; acc.w += f * o[j].w;
      }
    }
  }
  const float inv = (L > 0.0f) ? 1.0f / L : 0.0f;
  uint2 packed;
  packed.x = pack_bf16x2(acc.x * inv, acc.y * inv);
  packed.y = pack_bf16x2(acc.z * inv, acc.w * inv);
  *reinterpret_cast<uint2*>(p.out + (static_cast<int64_t>(bq) * 64 + h) * 512 + 4 * t) = packed;
  if (p.lse && t == 0)
    p.lse[static_cast<int64_t>(bq) * 64 + h] = (L > 0.0f) ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
}

}  // namespace csa2
