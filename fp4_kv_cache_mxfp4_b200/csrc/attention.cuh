// attention.cuh -- merge of the per-slice partial results of the sparse MQA
// ("DeepSeek V4.1-Flash 技术报告深度解析" §3.2): each slice of a query's keys
// (attention_tc.cuh) leaves an unnormalised fp32 output and its per-head
// (max, sum) in log2 units; the combine rescales them to the common max,
// sums, normalises and writes bf16 outputs and the natural-log LSE.
// L2 traffic per query: slices x 128 KB of partials, read once.
#pragma once
#include "common.cuh"

namespace csa2 {

constexpr int kAttnMaxK = 2048;      // largest K (CSA2_MAX_K)
constexpr int kAttnMaxW = 1024;      // largest window (CSA2_MAX_W)
constexpr int kAttnSliceKeys = 128;  // keys per slice

struct AttnParams {
  float* opart;              // [BQ][slices][64][512] unnormalised partial outputs
  float* ml;                 // [BQ][slices][64][2]: max (log2 units), sum
  int slices;
  __nv_bfloat16* out;        // [BQ][64][512]
  float* lse;                // optional [BQ][64]
};

// Merge the slices of one (query, head): 128 threads x 4 dims.  The slice
// statistics are loaded once into shared memory; the partial outputs are
// fetched eight slices at a time so their L2 latencies overlap.
constexpr int kAttnMaxSlices = (kAttnMaxK + kAttnSliceKeys - 1) / kAttnSliceKeys + (kAttnMaxW + kAttnSliceKeys - 1) / kAttnSliceKeys;

__global__ void __launch_bounds__(128)
sparse_attn_combine_kernel(AttnParams p) {
  __shared__ float m_s[kAttnMaxSlices], l_s[kAttnMaxSlices];
  const int bq = blockIdx.x >> 6, h = blockIdx.x & 63;
  const int t = threadIdx.x;
  pdl_launch_dependents();
  pdl_wait();
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
