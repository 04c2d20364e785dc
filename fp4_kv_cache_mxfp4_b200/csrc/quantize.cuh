// quantize.cuh -- FP4 main-KV entry quantisation (E2M1 values, one E4M3
// scale per 16 channels), "DeepSeek V4.1-Flash 技术报告深度解析" §3.4.
//
// One warp per 512-channel entry, one lane per 16-channel scale block: the
// lane reads its 32 input bytes (two 16-byte loads, the warp covers the
// 1 KB row), decides its scale and 16 codes in fp32 with correctly rounded
// division, and writes 8 bytes of nibbles (the warp writes the 256-byte
// nibble area in one coalesced store) plus one scale byte.
// HBM roofline: 1024 B read + 288 B written per entry.
#pragma once
#include "common.cuh"

namespace csa2 {

// E4M3 code -> exact fp32 value (codes come from a satfinite conversion, so
// the NaN encoding never occurs).
__device__ __forceinline__ float e4m3_code_to_float(uint32_t c) {
  const uint32_t e = (c >> 3) & 0xF, m = c & 7;
  const float mag = e ? __uint_as_float(((e + 120u) << 23) | (m << 20))   // (1+m/8)*2^(e-7)
                      : static_cast<float>(m) * 0.001953125f;            // m * 2^-9
  return (c & 0x80) ? -mag : mag;
}

// Round to nearest even on the E4M3 grid, saturating at 448; returns the
// code of `v` in the low byte.
__device__ __forceinline__ uint32_t e4m3_rn_sat(float v) {
  uint16_t out;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(out) : "f"(0.0f), "f"(v));
  return out & 0xFF;
}

// Two magnitudes to E2M1 (round to nearest even, saturate at 6): `lo` lands
// in bits 0-3, `hi` in bits 4-7.
__device__ __forceinline__ uint32_t e2m1x2_rn_sat(float lo, float hi) {
  uint32_t out;
  asm("{\n\t.reg .b8 b;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b, %1, %2;\n\t"
      "cvt.u32.u8 %0, b;\n\t}"
      : "=r"(out) : "f"(hi), "f"(lo));
  return out & 0xFF;
}

__global__ void __launch_bounds__(256)
quantize_kv_fp4_kernel(const __nv_bfloat16* __restrict__ x, int64_t n, int64_t ld_x,
                       uint8_t* __restrict__ kv, const int64_t* __restrict__ dst_rows,
                       int64_t row_offset) {
  const int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  pdl_wait();
  pdl_launch_dependents();
  if (row >= n) return;

  const uint4* src = reinterpret_cast<const uint4*>(x + row * ld_x + lane * 16);
  uint4 raw[2];
  raw[0] = __ldg(src);
  raw[1] = __ldg(src + 1);
  const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(raw);
  float v[16];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float2 f = __bfloat1622float2(h2[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));

  const float sf = __fdiv_rn(amax, 6.0f);
  const uint32_t s_code = e4m3_rn_sat(sf);
  const float s = e4m3_code_to_float(s_code);

  uint32_t packed[2] = {0u, 0u};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float a = v[2 * i], b = v[2 * i + 1];
    const float ya = (s != 0.0f) ? __fdiv_rn(a, s) : 0.0f;
    const float yb = (s != 0.0f) ? __fdiv_rn(b, s) : 0.0f;
    uint32_t byte = e2m1x2_rn_sat(fabsf(ya), fabsf(yb));
    // sign bits come from the inputs (x and x/s share their sign, and a
    // zero scale keeps the sign of x)
    byte |= (__float_as_uint(a) >> 31) << 3;
    byte |= (__float_as_uint(b) >> 31) << 7;
    packed[i >> 2] |= byte << (8 * (i & 3));
  }

  const int64_t dst = dst_rows ? dst_rows[row] : row_offset + row;
  uint8_t* out = kv + dst * 288;
  *reinterpret_cast<uint2*>(out + lane * 8) = make_uint2(packed[0], packed[1]);
  out[256 + lane] = static_cast<uint8_t>(s_code);
}

inline cudaError_t launch_quantize(const void* x, int64_t n, int64_t ld_x, void* kv,
                                   const int64_t* dst_rows, int64_t row_offset, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  const int warps = 8;
  const int64_t blocks = (n + warps - 1) / warps;
  trace_pre(kKQuantize, st);
  const cudaError_t e = launch_ex(quantize_kv_fp4_kernel, dim3(static_cast<unsigned>(blocks)), dim3(warps * 32), 0, st,
                                  0, static_cast<const __nv_bfloat16*>(x), n, ld_x, static_cast<uint8_t*>(kv),
                                  dst_rows, row_offset);
  trace_post(st);
  return e;
}

}  // namespace csa2
