// common.cuh -- sm_100a building blocks shared by the libcsa2 kernels:
// mbarriers with bounded waits, TMA tile loads, tcgen05 (TMEM allocation,
// UMMA descriptors, MMA issue, TMEM loads), order-preserving float keys.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda.h>
#include <stdint.h>
#include <string.h>

namespace csa2 {

// ---------------------------------------------------------------------------
// Host-side launch tracing: when on, every kernel launch is bracketed by two
// pre-created CUDA events recorded on the launch stream.
// ---------------------------------------------------------------------------
enum KernelId : int { kKQuantize = 0, kKIndexScan = 1, kKTopk = 2, kKAttnSlice = 3, kKAttnCombine = 4,
                      kKQuantizeWindow = 5, kKQuantizeIndexK = 6, kKCompressRope = 7, kKCount = 8 };

struct LaunchTrace {
  bool on = false;
  int max = 0, n = 0;
  cudaEvent_t* ev = nullptr;   // 2 * max events
  int* kid = nullptr;          // max kernel ids
};
static LaunchTrace g_trace;

// Launch with programmatic stream serialisation: the kernel's CTAs may be
// scheduled while the previous kernel in the stream is finishing, run their
// set-up (barriers, tensor memory, descriptor prefetch) and then wait in
// pdl_wait() until that kernel has completed and its writes are visible.
// cluster_x > 0 adds a (cluster_x, 1, 1) thread-block cluster shape.
// Tracing records events between launches, which serialises them as usual.
static bool g_pdl = true;
// set for the duration of a call whose kernels must run in plain stream
// order (CSA2_GROUP_SERIAL); launches happen on the calling host thread
static thread_local bool g_serial_launch = false;
// last CUDA failure seen by a launch on this host thread (csa2_cuda_error_string)
static thread_local cudaError_t g_last_cuda_error = cudaSuccess;
template <typename... KArgs, typename... Args>
inline cudaError_t launch_ex(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                             unsigned cluster_x, Args... args) {
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  if (g_pdl && !g_serial_launch) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  if (cluster_x > 0) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, args...);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) g_last_cuda_error = e;
  return e;
}

// External records: under stream capture they become event-record nodes of
// the graph (so a replayed graph times its kernels), not capture edges.
inline void trace_pre(int kid, cudaStream_t st) {
  if (g_trace.on && g_trace.n < g_trace.max) {
    g_trace.kid[g_trace.n] = kid;
    cudaEventRecordWithFlags(g_trace.ev[2 * g_trace.n], st, cudaEventRecordExternal);
  }
}
inline void trace_post(cudaStream_t st) {
  if (g_trace.on && g_trace.n < g_trace.max) {
    cudaEventRecordWithFlags(g_trace.ev[2 * g_trace.n + 1], st, cudaEventRecordExternal);
    ++g_trace.n;
  }
}

// ---------------------------------------------------------------------------
// Device-side failure word (read and cleared by csa2_device_status).
// ---------------------------------------------------------------------------
enum DeviceError : int {
  kErrNone = 0,
  kErrWaitTmaFull = 1,      // scan: MMA issuer gave up waiting for a TMA stage
  kErrWaitSmemEmpty = 2,    // scan: producer gave up waiting for a free stage
  kErrWaitTmemFull = 3,     // scan: epilogue gave up waiting for an accumulator
  kErrWaitTmemEmpty = 4,    // scan: MMA issuer gave up waiting for a free accumulator
  kErrWaitOperand = 5,      // scan: index-Q operand never arrived
  kErrSelectCount = 6,      // top-K: selected count differs from the request
};

__device__ int g_device_error;

// Programmatic dependent launch: block until the previous kernel in the
// stream has completed (returns at once when launched without the
// attribute), and let the next kernel's CTAs be scheduled.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ void record_error(int code) {
  atomicCAS(&g_device_error, 0, code);
}

// Bound for every spin on an mbarrier: about two seconds of wall time.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
               :: "r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0;
}

// Waits until the phase with the given parity has completed.  Gives up after
// kWaitLimitNs (or at once when *abort is set by another role), records
// `err` and returns false.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int err,
                                          volatile int* abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (global_ns() - t0 > kWaitLimitNs) {
      record_error(err);
      *abort = 1;
      return false;
    }
  }
}

// ---------------------------------------------------------------------------
// TMA (bulk tensor copies global -> shared, completion on an mbarrier)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" :: "l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// 2-D tile load; x is the inner (contiguous) coordinate in elements.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t x, int32_t y, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;"
      :: "r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y),
         "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// Untiled bulk copy global -> shared (both 16-byte aligned, size a multiple
// of 16), completion on an mbarrier, streamed past L2 (evict first).
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;"
      :: "r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(l2_policy_evict_first())
      : "memory");
}

// ---------------------------------------------------------------------------
// tcgen05: tensor memory and the 5th-generation MMA
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
               :: "r"(smem_u32(dst_smem)), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor for a K-major operand stored in the
// 128-byte-swizzle canonical layout: rows of 128 B (64 bf16), groups of 8
// rows 1024 B apart.  Fields: start address >> 4 (bits 0-13), leading byte
// offset >> 4 (16-29, unused for swizzled K-major, set to 1), stride byte
// offset >> 4 (32-45), version 1 (46-47), base offset 0, layout 2 = 128B
// swizzle (61-63).
__device__ __forceinline__ uint64_t umma_desc_sw128_kmajor(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFF);
  d |= static_cast<uint64_t>(1) << 16;
  d |= static_cast<uint64_t>(1024 >> 4) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(2) << 61;
  return d;
}

// Instruction descriptor, kind::f16 with bf16 A/B, f32 accumulator, both
// operands K-major, shape M x N.
__host__ __device__ constexpr uint32_t umma_idesc_bf16_f32(int M, int N) {
  return (1u << 4)                                   // D format: f32
       | (1u << 7)                                   // A format: bf16
       | (1u << 10)                                  // B format: bf16
       | (static_cast<uint32_t>(N >> 3) << 17)       // N / 8
       | (static_cast<uint32_t>(M >> 4) << 24);      // M / 16
}

// D[tmem] (+)= A[smem] * B[smem]^T, issued by a single thread.
__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      :: "r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate) : "memory");
}

// Arrive on an mbarrier once every MMA issued so far by this thread is done.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               :: "r"(smem_u32(bar)) : "memory");
}

// 32 lanes x 32 columns of 32-bit values: thread i of the warp gets lane
// (warp's quarter base + i), registers = consecutive columns.
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Named barrier over a subset of warps.
__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" :: "r"(id), "r"(nthreads) : "memory");
}

// ---------------------------------------------------------------------------
// Order-preserving keys: okey(a) < okey(b) iff a < b for non-NaN floats;
// -0 is folded onto +0 so equal scores always tie.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t okey(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u << 1) == 0) u = 0;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float okey_to_float(uint32_t k) {
  uint32_t u = (k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k;
  return __uint_as_float(u);
}

// Shared-memory histogram increment aggregated over the lanes of a warp
// that hit the same bin (one atomic per distinct bin instead of one per
// lane); `active` says whether this lane counts.  Warp-collective.
__device__ __forceinline__ void warp_hist_add(uint32_t* hist, uint32_t bin, bool active) {
  const uint32_t live = __ballot_sync(0xffffffffu, active);
  if (!active) return;
  const uint32_t peers = __match_any_sync(live, bin);
  if ((threadIdx.x & 31) == static_cast<uint32_t>(__ffs(peers) - 1)) atomicAdd(&hist[bin], __popc(peers));
}

// byte offset of the 16-byte unit u (0..7) of row r in a K-major operand
// chunk of 128-byte rows with the 128-byte swizzle
__device__ __forceinline__ uint32_t sw128_off(int r, int u) {
  return static_cast<uint32_t>((r >> 3) * 1024 + (r & 7) * 128 + ((u ^ (r & 7)) << 4));
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

// ---------------------------------------------------------------- block-scaled FP4 MMA
// Shared-memory descriptor for a K-major operand in the 64-byte-swizzle
// canonical layout: rows of 64 B (128 packed E2M1 values), groups of 8 rows
// 512 B apart, the 16-byte chunk c of row r stored at chunk c ^ ((r >> 1) & 3).
// Layout type 4 = 64-byte swizzle; the other fields as for 128-byte swizzle.
__device__ __forceinline__ uint64_t umma_desc_sw64_kmajor(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFF);
  d |= static_cast<uint64_t>(1) << 16;
  d |= static_cast<uint64_t>(512 >> 4) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(4) << 61;
  return d;
}
// byte offset of 16-byte chunk c of row r in a 64-byte-swizzled tile
__host__ __device__ __forceinline__ uint32_t sw64_off(int r, int c) {
  return static_cast<uint32_t>(r) * 64u + static_cast<uint32_t>((c ^ ((r >> 1) & 3)) * 16);
}

// Descriptor of a 32-row x 16-byte block-scale chunk (no swizzle, rows
// contiguous, 8-row core matrices 128 B apart) for tcgen05.cp.
__device__ __forceinline__ uint64_t umma_desc_sf_chunk(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFF);
  d |= static_cast<uint64_t>(1) << 16;
  d |= static_cast<uint64_t>(128 >> 4) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  return d;
}

// Block-scale chunk of 128 operand rows x 4 scale bytes (512 B), the
// arrangement the MMA reads from tensor memory after one
// tcgen05.cp.32x128b.warpx4: 16-byte line m0 holds rows m0, m0+32, m0+64,
// m0+96 (4 bytes each: the scales of K blocks 0..3).  Byte offset of the
// scale of row r (0..127), K block k.
__host__ __device__ __forceinline__ uint32_t sf_chunk_off(int r, int k) {
  return static_cast<uint32_t>(16 * (r & 31) + 4 * (r >> 5) + k);
}

// Copy one 512-byte scale chunk into 4 tensor-memory columns at taddr; the
// 32 lines land in lanes 0..31 and are repeated in every lane quarter.
__device__ __forceinline__ void tmem_cp_sf_chunk(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" :: "r"(taddr), "l"(sdesc) : "memory");
}

// Instruction descriptor, kind::mxf4 (E2M1 A and B, UE8M0 scales per 32
// values, f32 accumulator, both K-major, K = 64 per instruction), shape
// M x N; sf_id selects the scale byte of each 32-bit scale column (the
// instruction uses bytes sf_id and sf_id + 1).
__host__ __device__ constexpr uint32_t umma_idesc_mxf4(int M, int N, uint32_t sf_id) {
  return (sf_id << 4)                                // B scale byte
       | (1u << 7)                                   // A format: E2M1
       | (1u << 10)                                  // B format: E2M1
       | (static_cast<uint32_t>(N >> 3) << 17)       // N / 8
       | (1u << 23)                                  // scale format: UE8M0
       | (static_cast<uint32_t>(M >> 4) << 24)       // M / 16
       | (sf_id << 29);                              // A scale byte
}

// D[tmem] (+)= (A * SFA)[smem] * (B * SFB)[smem]^T, block-scaled E2M1,
// issued by a single thread; tsfa / tsfb: tensor-memory scale columns.
__device__ __forceinline__ void umma_mxf4(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t tsfa, uint32_t tsfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
      :: "r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(tsfa), "r"(tsfb) : "memory");
}

// Instruction descriptor, kind::mxf4nvf4 with 16-value blocks (E2M1 A and
// B, one UE4M3 scale per 16 values, f32 accumulator, both K-major, K = 64
// per instruction: 4 scale bytes per row and instruction), shape M x N.
__host__ __device__ constexpr uint32_t umma_idesc_nvf4(int M, int N) {
  return (1u << 7)                                   // A format: E2M1
       | (1u << 10)                                  // B format: E2M1
       | (static_cast<uint32_t>(N >> 3) << 17)       // N / 8
       | (static_cast<uint32_t>(M >> 4) << 24);      // M / 16; scale format 0 = UE4M3
}

__device__ __forceinline__ void umma_nvf4(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t tsfa, uint32_t tsfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
      :: "r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(tsfa), "r"(tsfb) : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

}  // namespace csa2
