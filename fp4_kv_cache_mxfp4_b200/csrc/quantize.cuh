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

// The same block quantiser for bf16-valued inputs with one division per
// block: q = E2M1(x / s) by comparing |x| with the grid's midpoints times s.
// Both are exact in fp32 (a midpoint has at most 3 significant bits, s at
// most 4), and for x with 8 significant bits x / s is either exactly a
// midpoint or at least 2^-8 (relative) away from one, so fp32(x / s) rounds
// to the same code; ties go to the even code as in round-to-nearest-even.
__device__ __forceinline__ void fp4_block16_bf16(const float (&v)[16], uint2& nib, uint32_t& s_code) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
  s_code = e4m3_rn_sat(__fdiv_rn(amax, 6.0f));
  const float s = e4m3_code_to_float(s_code);
  // code >= 1 iff |x| > 0.25 s (tie to 0), >= 2 iff |x| >= 0.75 s (tie to 2), ...
  const float t1 = 0.25f * s, t2 = 0.75f * s, t3 = 1.25f * s, t4 = 1.75f * s, t5 = 2.5f * s, t6 = 3.5f * s, t7 = 5.0f * s;
  uint32_t packed[2] = {0u, 0u};
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float a = fabsf(v[i]);
    uint32_t c = (a > t1) + (a >= t2) + (a > t3) + (a >= t4) + (a > t5) + (a >= t6) + (a > t7);
    if (s == 0.0f) c = 0;
    c |= (__float_as_uint(v[i]) >> 31) << 3;
    packed[i >> 3] |= c << (4 * (i & 7));
  }
  nib = make_uint2(packed[0], packed[1]);
}

// One block of 16 channels (fp32 values) to its 8 nibble bytes and E4M3
// scale code: sf = amax / 6, s = E4M3(sf), q = E2M1(x / s), sign kept.
__device__ __forceinline__ void fp4_block16(const float (&v)[16], uint2& nib, uint32_t& s_code) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const float sf = __fdiv_rn(amax, 6.0f);
  s_code = e4m3_rn_sat(sf);
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
  nib = make_uint2(packed[0], packed[1]);
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
  uint2 nib;
  uint32_t s_code;
  fp4_block16_bf16(v, nib, s_code);                   // bf16 inputs: one division per block
  const int64_t dst = dst_rows ? dst_rows[row] : row_offset + row;
  uint8_t* out = kv + dst * 288;
  *reinterpret_cast<uint2*>(out + lane * 8) = nib;
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

// ---------------------------------------------------------------------------
// FP8 window rows ("DeepSeek V4.1-Flash 技术报告深度解析" §3.4: the SWA KV cache
// stays FP8): one E4M3 code per channel and one fp32 scale per 512-channel
// row, s = amax / 448, code = E4M3(x / s) (round to nearest even,
// saturating; a zero row gives signed zeros).  One warp per row, 16
// channels per lane; the warp reduces amax, then writes its 512 codes with
// one coalesced 16-byte store per lane.
// HBM roofline: 1024 B read + 516 B written per row.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
quantize_window_fp8_kernel(const __nv_bfloat16* __restrict__ x, int64_t n, int64_t ld_x,
                           uint8_t* __restrict__ codes, float* __restrict__ scales,
                           const int64_t* __restrict__ dst_rows, int64_t row_offset) {
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
    const float2 f = __bfloat1622float2(h2[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float s = __fdiv_rn(amax, 448.0f);
  uint32_t w[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    uint32_t word = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float a = v[4 * k + j];
      // a zero scale keeps the sign of x: cvt of a signed zero keeps it
      const float y = (s != 0.0f) ? __fdiv_rn(a, s) : copysignf(0.0f, a);
      word |= e4m3_rn_sat(y) << (8 * j);
    }
    w[k] = word;
  }
  const int64_t dst = dst_rows ? dst_rows[row] : row_offset + row;
  *reinterpret_cast<uint4*>(codes + dst * 512 + lane * 16) = make_uint4(w[0], w[1], w[2], w[3]);
  if (lane == 0) scales[dst] = s;
}

inline cudaError_t launch_quantize_window(const void* x, int64_t n, int64_t ld_x, void* codes, float* scales,
                                          const int64_t* dst_rows, int64_t row_offset, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  const int warps = 8;
  const int64_t blocks = (n + warps - 1) / warps;
  trace_pre(kKQuantizeWindow, st);
  const cudaError_t e = launch_ex(quantize_window_fp8_kernel, dim3(static_cast<unsigned>(blocks)), dim3(warps * 32), 0,
                                  st, 0, static_cast<const __nv_bfloat16*>(x), n, ld_x, static_cast<uint8_t*>(codes),
                                  scales, dst_rows, row_offset);
  trace_post(st);
  return e;
}

// ---------------------------------------------------------------------------
// MXFP4 index-K entries ("DeepSeek V4.1-Flash 技术报告深度解析" §3.4: FP4
// indexer Q/K in the OCP MXFP4 format): per block of 32 channels a shared
// scale 2^e, e = floor(log2(amax)) - 2 clamped to [-127, 127] (-127 for an
// all-zero block), codes E2M1(x / 2^e) (round to nearest even, saturate at
// 6, sign kept); entry = 64 nibble bytes (channel 2i low nibble of byte i)
// + 4 scale bytes e + 127 = 68 B.  One warp per entry, 4 channels per lane,
// 8 lanes per block.
// HBM roofline: 256 B read + 68 B written per entry.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
quantize_index_k_mxfp4_kernel(const __nv_bfloat16* __restrict__ x, int64_t n, int64_t ld_x,
                              uint8_t* __restrict__ out, const int64_t* __restrict__ dst_rows,
                              int64_t row_offset) {
  const int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  pdl_wait();
  pdl_launch_dependents();
  if (row >= n) return;
  const uint2 raw = __ldg(reinterpret_cast<const uint2*>(x + row * ld_x + lane * 4));
  const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.x));
  const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.y));
  const float v[4] = {f0.x, f0.y, f1.x, f1.y};
  float amax = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  int e = -127;
  if (amax > 0.0f) {
    int E;
    frexpf(amax, &E);                                  // amax = m 2^E, m in [0.5, 1)
    e = max(-127, min(127, E - 1 - 2));
  }
  uint32_t nib = 0;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float a = ldexpf(v[2 * i], -e), b = ldexpf(v[2 * i + 1], -e);   // exact: powers of two
    uint32_t byte = e2m1x2_rn_sat(fabsf(a), fabsf(b));
    byte |= (__float_as_uint(a) >> 31) << 3;
    byte |= (__float_as_uint(b) >> 31) << 7;
    nib |= byte << (8 * i);
  }
  const int64_t dst = dst_rows ? dst_rows[row] : row_offset + row;
  uint8_t* entry = out + dst * 68;
  *reinterpret_cast<uint16_t*>(entry + 2 * lane) = static_cast<uint16_t>(nib);
  if ((lane & 7) == 0) entry[64 + (lane >> 3)] = static_cast<uint8_t>(e + 127);
}

inline cudaError_t launch_quantize_index_k(const void* x, int64_t n, int64_t ld_x, void* out, const int64_t* dst_rows,
                                           int64_t row_offset, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  const int warps = 8;
  const int64_t blocks = (n + warps - 1) / warps;
  trace_pre(kKQuantizeIndexK, st);
  const cudaError_t e = launch_ex(quantize_index_k_mxfp4_kernel, dim3(static_cast<unsigned>(blocks)), dim3(warps * 32),
                                  0, st, 0, static_cast<const __nv_bfloat16*>(x), n, ld_x, static_cast<uint8_t*>(out),
                                  dst_rows, row_offset);
  trace_post(st);
  return e;
}

// ---------------------------------------------------------------------------
// New main-KV entries compressed, rotated and quantised in one pass
// ("DeepSeek V4.1-Flash 技术报告深度解析" §3.2 compression of r tokens per
// entry without overlap, §3.4 quantisation after RoPE): entry e =
// sum_j w[e][j] * x[e r + j] channel by channel (float32, one rounding per
// operation, j ascending), then channels 448..511 rotated in adjacent pairs
// by the caller's cos/sin (a cos - b sin, a sin + b cos), then the FP4 block
// quantiser on the float32 result.  One warp per entry, 16 channels (one
// scale block) per lane.
// HBM roofline: r * 1024 B of tokens + 288 B written per entry (+ weights
// and angles, shared or 256 B per entry).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
compress_rope_quantize_kernel(const __nv_bfloat16* __restrict__ x, int64_t n, int64_t ld_x, int r,
                              const float* __restrict__ w, int64_t w_stride, const float* __restrict__ cosv,
                              const float* __restrict__ sinv, uint8_t* __restrict__ kv,
                              const int64_t* __restrict__ dst_rows, int64_t row_offset) {
  const int64_t e = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  pdl_wait();
  pdl_launch_dependents();
  if (e >= n) return;
  float v[16] = {};                                   // every element is set at j = 0
  const float* we = w + e * w_stride;
#pragma unroll 1
  for (int j = 0; j < r; ++j) {
    const uint4* src = reinterpret_cast<const uint4*>(x + (e * r + j) * ld_x + lane * 16);
    const uint4 raw0 = __ldg(src), raw1 = __ldg(src + 1);
    const uint32_t rw[8] = {raw0.x, raw0.y, raw0.z, raw0.w, raw1.x, raw1.y, raw1.z, raw1.w};
    const float4* wj = reinterpret_cast<const float4*>(we + j * 512 + lane * 16);
    float wv[16];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float4 t = __ldg(wj + k);
      wv[4 * k] = t.x; wv[4 * k + 1] = t.y; wv[4 * k + 2] = t.z; wv[4 * k + 3] = t.w;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&rw[i]));
      const float p0 = __fmul_rn(wv[2 * i], f.x), p1 = __fmul_rn(wv[2 * i + 1], f.y);
      v[2 * i] = (j == 0) ? p0 : __fadd_rn(v[2 * i], p0);
      v[2 * i + 1] = (j == 0) ? p1 : __fadd_rn(v[2 * i + 1], p1);
    }
  }
  if (lane >= 28) {                                   // channels 448..511: pairs 8 (lane - 28) ..
    const int p0 = 8 * (lane - 28);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float c = __ldg(cosv + e * 32 + p0 + k), sn = __ldg(sinv + e * 32 + p0 + k);
      const float a = v[2 * k], b = v[2 * k + 1];
      v[2 * k] = __fsub_rn(__fmul_rn(a, c), __fmul_rn(b, sn));
      v[2 * k + 1] = __fadd_rn(__fmul_rn(a, sn), __fmul_rn(b, c));
    }
  }
  uint2 nib;
  uint32_t s_code;
  fp4_block16(v, nib, s_code);
  const int64_t dst = dst_rows ? dst_rows[e] : row_offset + e;
  uint8_t* out = kv + dst * 288;
  *reinterpret_cast<uint2*>(out + lane * 8) = nib;
  out[256 + lane] = static_cast<uint8_t>(s_code);
}

inline cudaError_t launch_compress_rope_quantize(const void* x, int64_t n, int64_t ld_x, int r, const float* w,
                                                 int64_t w_stride, const float* cosv, const float* sinv, void* kv,
                                                 const int64_t* dst_rows, int64_t row_offset, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  const int warps = 8;
  const int64_t blocks = (n + warps - 1) / warps;
  trace_pre(kKCompressRope, st);
  const cudaError_t e = launch_ex(compress_rope_quantize_kernel, dim3(static_cast<unsigned>(blocks)),
                                  dim3(warps * 32), 0, st, 0, static_cast<const __nv_bfloat16*>(x), n, ld_x, r, w,
                                  w_stride, cosv, sinv, static_cast<uint8_t*>(kv), dst_rows, row_offset);
  trace_post(st);
  return e;
}

}  // namespace csa2
