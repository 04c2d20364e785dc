// csa2_api.cu -- the C ABI of libcsa2 (declared in include/csa2.h): host-side
// validation, workspace layout, TMA descriptor set-up and kernel launches.
// The library is built as this single translation unit.
#include "../../include/csa2.h"

#include <cudaTypedefs.h>
#include <math.h>
#include <algorithm>
#include <mutex>
#include <vector>
#include <string.h>

#include "common.cuh"
#include "quantize.cuh"
#include "index_scan.cuh"
#include "index_scan_t.cuh"
#include "topk.cuh"
#include "attention.cuh"
#include "attention_tc.cuh"

namespace csa2 {
namespace {

constexpr int kMaxDevices = 64;
constexpr int kMaxDynSmem = 227 * 1024;
constexpr int kScanStages = 3;

struct DeviceInfo {
  bool init = false;
  bool ok = false;
  int sms = 0;
  bool attrs_set = false;
  int topk_max_cluster = 8;   // 16 where the GPU can place clusters of 16 top-K CTAs
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_mu;
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

// index_scan_kernel instances: queries per MMA group (1, 2, 4, 8) x HSI
// Every kernel asks for the full shared-memory carveout, so consecutive
// kernels of a step never make an SM reconfigure its L1/shared split.
template <class F>
cudaError_t set_smem_attrs(F* f, int dyn_bytes) {
  cudaError_t e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn_bytes);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(f, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
}

template <int QG, bool HSI, bool KF4>
cudaError_t set_scan_attr_one() {
  return set_smem_attrs(index_scan_kernel<QG, HSI, KF4>, kMaxDynSmem);
}
template <bool KF4>
cudaError_t set_scan_attrs_k() {
  cudaError_t e = cudaSuccess;
  cudaError_t r[8] = {set_scan_attr_one<1, false, KF4>(), set_scan_attr_one<1, true, KF4>(),
                      set_scan_attr_one<2, false, KF4>(), set_scan_attr_one<2, true, KF4>(),
                      set_scan_attr_one<4, false, KF4>(), set_scan_attr_one<4, true, KF4>(),
                      cudaSuccess, cudaSuccess};
  if constexpr (!KF4) {                      // MXFP4 index-K groups at most 4 queries
    r[6] = set_scan_attr_one<8, false, KF4>();
    r[7] = set_scan_attr_one<8, true, KF4>();
  }
  for (cudaError_t x : r) if (x != cudaSuccess) e = x;
  return e;
}
cudaError_t set_scan_attrs() {
  const cudaError_t a = set_scan_attrs_k<false>(), b = set_scan_attrs_k<true>();
  const cudaError_t t[4] = {set_smem_attrs(index_scan_t_kernel<false, false>, kMaxDynSmem),
                            set_smem_attrs(index_scan_t_kernel<true, false>, kMaxDynSmem),
                            set_smem_attrs(index_scan_t_kernel<false, true>, kMaxDynSmem),
                            set_smem_attrs(index_scan_t_kernel<true, true>, kMaxDynSmem)};
  for (cudaError_t x : t) if (x != cudaSuccess) return x;
  return a != cudaSuccess ? a : b;
}
cudaError_t launch_scan_t1(bool hsi, bool kf4, unsigned grid, size_t smem, cudaStream_t st, const CUtensorMap& tk,
                           const CUtensorMap& tq, const ScanParams& sp) {
  const dim3 block(kf4 ? kScanThreadsF4 : kScanThreads);
  if (kf4) return hsi ? launch_ex(index_scan_t_kernel<true, true>, dim3(grid), block, smem, st, 0, tk, tq, sp)
                      : launch_ex(index_scan_t_kernel<false, true>, dim3(grid), block, smem, st, 0, tk, tq, sp);
  return hsi ? launch_ex(index_scan_t_kernel<true, false>, dim3(grid), block, smem, st, 0, tk, tq, sp)
             : launch_ex(index_scan_t_kernel<false, false>, dim3(grid), block, smem, st, 0, tk, tq, sp);
}
inline int scan_qg(int qg) { return qg <= 1 ? 1 : qg <= 2 ? 2 : qg <= 4 ? 4 : 8; }

template <int QG, bool HSI, bool KF4>
cudaError_t launch_scan_t(unsigned grid, size_t smem, cudaStream_t st, const CUtensorMap& tk, const CUtensorMap& tq,
                          const ScanParams& sp) {
  return launch_ex(index_scan_kernel<QG, HSI, KF4>, dim3(grid), dim3(KF4 ? kScanThreadsF4 : kScanThreads), smem, st, 0,
                   tk, tq, sp);
}
template <bool KF4>
cudaError_t launch_scan_k(int QG, bool hsi, unsigned grid, size_t smem, cudaStream_t st, const CUtensorMap& tk,
                          const CUtensorMap& tq, const ScanParams& sp) {
  switch (QG * 2 + (hsi ? 1 : 0)) {
    case 2: return launch_scan_t<1, false, KF4>(grid, smem, st, tk, tq, sp);
    case 3: return launch_scan_t<1, true, KF4>(grid, smem, st, tk, tq, sp);
    case 4: return launch_scan_t<2, false, KF4>(grid, smem, st, tk, tq, sp);
    case 5: return launch_scan_t<2, true, KF4>(grid, smem, st, tk, tq, sp);
    case 8: return launch_scan_t<4, false, KF4>(grid, smem, st, tk, tq, sp);
    case 9: return launch_scan_t<4, true, KF4>(grid, smem, st, tk, tq, sp);
    default:
      if constexpr (KF4) return cudaErrorInvalidValue;   // plan_index caps MXFP4 groups at 4 queries
      else return hsi ? launch_scan_t<8, true, KF4>(grid, smem, st, tk, tq, sp)
                      : launch_scan_t<8, false, KF4>(grid, smem, st, tk, tq, sp);
  }
}
cudaError_t launch_scan(int QG, bool hsi, bool kf4, unsigned grid, size_t smem, cudaStream_t st, const CUtensorMap& tk,
                        const CUtensorMap& tq, const ScanParams& sp) {
  return kf4 ? launch_scan_k<true>(QG, hsi, grid, smem, st, tk, tq, sp)
             : launch_scan_k<false>(QG, hsi, grid, smem, st, tk, tq, sp);
}

// Largest top-K cluster this GPU can place: 16 (non-portable) when at least
// one such cluster fits, else the portable 8.
int topk_cluster_limit() {
  if (cudaFuncSetAttribute(topk_select_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
    cudaGetLastError();
    return 8;
  }
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(16, 1, 1);
  cfg.blockDim = dim3(kTopkThreads, 1, 1);
  cfg.dynamicSmemBytes = topk_smem_bytes();
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = 16;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, topk_select_kernel, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 8;
  }
  return n >= 1 ? 16 : 8;
}

csa2_status device_info(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return CSA2_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.init) {
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return CSA2_ERR_CUDA;
    // CSA2_PDL=0 launches every kernel with plain stream order
    const char* pdl = getenv("CSA2_PDL");
    if (pdl && pdl[0] == '0') g_pdl = false;
    d.ok = (prop.major == 10);
    d.sms = prop.multiProcessorCount;
    d.init = true;
  }
  if (!d.ok) return CSA2_ERR_ARCH;
  if (!d.attrs_set) {
    if (set_scan_attrs() != cudaSuccess ||
        set_smem_attrs(topk_select_kernel, static_cast<int>(topk_smem_bytes())) != cudaSuccess ||
        set_smem_attrs(sparse_attn_tc_kernel, static_cast<int>(kTcAttnSmem)) != cudaSuccess ||
        set_smem_attrs(sparse_attn_combine_kernel, 0) != cudaSuccess ||
        set_smem_attrs(quantize_kv_fp4_kernel, 0) != cudaSuccess ||
        set_smem_attrs(quantize_window_fp8_kernel, 0) != cudaSuccess ||
        set_smem_attrs(quantize_index_k_mxfp4_kernel, 0) != cudaSuccess ||
        set_smem_attrs(compress_rope_quantize_kernel, 0) != cudaSuccess)
      return CSA2_ERR_CUDA;
    d.topk_max_cluster = topk_cluster_limit();
    if (!g_encode) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
          q != cudaDriverEntryPointSuccess || !fn)
        return CSA2_ERR_CUDA;
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    d.attrs_set = true;
  }
  *out = &d;
  return CSA2_OK;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }
inline size_t up256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// bf16 [rows][128] matrix as a 2-D TMA map with 128-byte swizzle
bool make_map_bf16_128(CUtensorMap* m, const void* base, uint64_t rows, uint32_t box_rows) {
  const cuuint64_t dims[2] = {128, rows};
  const cuuint64_t strides[1] = {256};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ---------------------------------------------------------------- index call

struct IndexPlan {
  bool pool, hsi;
  int BQ, qg, hb;
  int hist_every;      // 1: exact score histogram; 8: every 8th tile (many queries per MMA group)
  int64_t n_elems, nblk;
  int64_t ld, bld;     // score row strides (multiples of 4 for 16-byte loads)
  // counter region (histograms): zeroed at the start of every call; data
  // region (scores): no precondition
  size_t off_hist, off_bhist, off_ctr, zero_bytes;
  size_t off_scores, off_bscores, data_bytes;
  size_t total;
};

csa2_status validate_index(const csa2_index_args* a) {
  if (!a) return CSA2_ERR_ARG;
  if (a->mode != CSA2_FULL && a->mode != CSA2_REINDEX && a->mode != CSA2_REINDEX_POOL) return CSA2_ERR_ARG;
  if (a->B < 1 || a->Q < 1 || static_cast<int64_t>(a->B) * a->Q > CSA2_MAX_BQ || a->K < 1 || a->K > CSA2_MAX_K ||
      a->N < 1)
    return CSA2_ERR_SHAPE;
  if (static_cast<int64_t>(a->B) * a->N >= (static_cast<int64_t>(1) << 31)) return CSA2_ERR_SHAPE;
  if (!a->qI || !a->w || !a->kI || !a->n_vis || !a->idx) return CSA2_ERR_ARG;
  const bool hsi = a->mode == CSA2_FULL && a->hsi_blocks > 0;
  if (a->hsi_blocks < 0 || a->hsi_blocks > CSA2_MAX_K) return CSA2_ERR_SHAPE;
  if (hsi || a->mode == CSA2_REINDEX_POOL) {
    if (a->hsi_block != CSA2_HSI_BLOCK) return CSA2_ERR_SHAPE;
    if (a->hsi_blocks < 1) return CSA2_ERR_SHAPE;
  }
  if (hsi && !a->pool_out) return CSA2_ERR_ARG;
  if (a->mode == CSA2_REINDEX_POOL && !a->pool_in) return CSA2_ERR_ARG;
  if (a->k_format != CSA2_FMT_BF16 && a->k_format != CSA2_FMT_MXFP4) return CSA2_ERR_ARG;
  if (a->k_format == CSA2_FMT_MXFP4 && (a->N & 3)) return CSA2_ERR_SHAPE;   // 16-byte aligned raw tiles
  // a pool block of MXFP4 entries is fetched whole (8 x 68 B by one bulk
  // copy, which has no bounds check): the blocks must tile each row
  if (a->k_format == CSA2_FMT_MXFP4 && (hsi || a->mode == CSA2_REINDEX_POOL) && (a->N & 7)) return CSA2_ERR_SHAPE;
  if (!aligned16(a->qI) || !aligned16(a->w) || !aligned16(a->kI) || !aligned16(a->n_vis) || !aligned16(a->idx) ||
      (a->scores && !aligned16(a->scores)) || (hsi && !aligned16(a->pool_out)) ||
      (a->mode == CSA2_REINDEX_POOL && !aligned16(a->pool_in)))
    return CSA2_ERR_ALIGN;
  return CSA2_OK;
}

IndexPlan plan_index(const csa2_index_args* a) {
  IndexPlan P;
  P.pool = a->mode == CSA2_REINDEX_POOL;
  P.hsi = a->mode == CSA2_FULL && a->hsi_blocks > 0;
  P.BQ = a->B * a->Q;
  P.qg = P.pool ? 1 : std::min(a->Q, a->k_format == CSA2_FMT_MXFP4 ? kF4MaxQG : 8);
  // score histogram bits: 4096 bins per query for 1-2 queries per MMA group,
  // 2048 for 4-8 (1024 with HSI, whose block histogram needs the room too)
  P.hb = (P.qg <= 2) ? 12 : (P.hsi ? 10 : 11);
  // with 4+ queries per group the histogram increments cost a quarter of the
  // scan: count one tile in 8 and let the top-K verify its threshold
  P.hist_every = (P.qg >= 4 && !P.hsi) ? 8 : 1;
  P.n_elems = P.pool ? static_cast<int64_t>(a->hsi_blocks) * 8 : a->N;
  P.nblk = P.hsi ? (a->N + 7) / 8 : 0;
  P.ld = (P.n_elems + 3) & ~static_cast<int64_t>(3);
  P.bld = (P.nblk + 3) & ~static_cast<int64_t>(3);
  const size_t nb = static_cast<size_t>(1) << P.hb;
  size_t off = 0;
  P.off_hist = off;    off = up256(off + static_cast<size_t>(P.BQ) * nb * 4);
  P.off_bhist = off;   off = up256(off + (P.hsi ? static_cast<size_t>(P.BQ) * nb * 4 : 0));
  // tile claims of the one-query-per-group scan, one counter per query
  P.off_ctr = off;     off = up256(off + (P.qg == 1 ? static_cast<size_t>(P.BQ) * 4 : 0));
  P.zero_bytes = off;
  off = 0;
  P.off_scores = off;  off = up256(off + static_cast<size_t>(P.BQ) * P.ld * 4);
  P.off_bscores = off; off = up256(off + static_cast<size_t>(P.BQ) * P.bld * 4);
  P.data_bytes = off;
  P.total = P.zero_bytes + P.data_bytes;
  return P;
}

// One cluster of topk_cluster_size() CTAs per selection problem.
cudaError_t launch_topk(const TopkParams& tp, int problems, const DeviceInfo& dev, cudaStream_t st) {
  const int C = topk_cluster_size(tp.n_elems, problems, dev.sms, dev.topk_max_cluster);
  trace_pre(kKTopk, st);
  const cudaError_t e = launch_ex(topk_select_kernel, dim3(static_cast<unsigned>(C), static_cast<unsigned>(problems)),
                                  dim3(kTopkThreads), topk_smem_bytes(), st, static_cast<unsigned>(C), tp);
  trace_post(st);
  return e;
}

// CTAs sharing one MMA group's tile range: the split whose waves of one
// CTA per SM finish first, counting about four tiles of set-up per CTA.
// Few groups (decode) get one wave over every SM; many groups (prefill) get
// pieces that keep the last wave nearly full.
int scan_ctas_per_group(int groups, int tiles, int sms, int setup_tiles = 4) {
  int best = 1;
  int64_t best_cost = INT64_MAX;
  for (int c = 1; c <= std::min(tiles, 4096); ++c) {
    const int64_t waves = (static_cast<int64_t>(groups) * c + sms - 1) / sms;
    const int64_t cost = waves * ((tiles + c - 1) / c + setup_tiles);
    if (cost < best_cost) { best_cost = cost; best = c; }
  }
  return best;
}

// zero: the call's counter region (already zeroed); data: its data region
// kv_prefetch: optional FP4 cache whose selected rows are pulled into L2 as
// the top-K writes their indices (the group call's attention reads them next)
// early_q: index-Q and w are complete when the scan starts (the caller's,
// not a result of the kernel before it)
csa2_status run_index(const csa2_index_args* a, const DeviceInfo& dev, void* zero, void* data, cudaStream_t st,
                      const void* kv_prefetch = nullptr, bool early_q = true) {
  const IndexPlan P = plan_index(a);
  uint8_t* z = static_cast<uint8_t*>(zero);
  uint8_t* w = static_cast<uint8_t*>(data);

  ScanParams sp;
  memset(&sp, 0, sizeof(sp));
  sp.pool_mode = P.pool;
  sp.B = a->B; sp.Q = a->Q; sp.qg = P.qg; sp.N = a->N; sp.n_elems = P.n_elems; sp.ld = P.ld; sp.bld = P.bld;
  sp.n_vis = a->n_vis; sp.w = a->w;
  sp.pool = P.pool ? a->pool_in : nullptr;
  sp.pool_blocks = P.pool ? a->hsi_blocks : 0;
  sp.scores = reinterpret_cast<float*>(w + P.off_scores);
  sp.bscores = P.hsi ? reinterpret_cast<float*>(w + P.off_bscores) : nullptr;
  sp.nblk = P.nblk;
  sp.hist = reinterpret_cast<uint32_t*>(z + P.off_hist);
  sp.bhist = P.hsi ? reinterpret_cast<uint32_t*>(z + P.off_bhist) : nullptr;
  sp.tile_ctr = reinterpret_cast<int*>(z + P.off_ctr);
  sp.hb = P.hb;
  sp.hist_every = P.hist_every;
  sp.qblocks = P.pool ? 1 : (a->Q + P.qg - 1) / P.qg;
  sp.groups = P.pool ? P.BQ : a->B * sp.qblocks;
  const bool kf4 = a->k_format == CSA2_FMT_MXFP4;
  const int smem_room = kMaxDynSmem - 1024;
  sp.early_q = early_q ? 1 : 0;
  if (P.qg == 1) {
    // one query per group (decode, or the HSI pool re-score): the scan with
    // the entries on the MMA's N side, 256 per instruction
    const int tile_t = scan_t_tile(kf4);
    sp.tiles_per_group = static_cast<int>((P.n_elems + tile_t - 1) / tile_t);
    sp.ctas_per_group = scan_ctas_per_group(sp.groups, sp.tiles_per_group, dev.sms, 2);
    int raw = 0;
    if (kf4) {
      // 6 raw tiles (13 KB each) in flight: 12 measured no faster, the
      // tensor pipe (two block-scale copies and two MMAs per tile) sets the pace
      sp.k4 = static_cast<const uint8_t*>(a->kI);
      sp.stages = 4;
      raw = 6;
      while (raw > 2 && static_cast<int>(scan_t_smem_layout(sp.stages, P.hb, P.hsi, true, raw).total) > smem_room) --raw;
    } else {
      sp.stages = 2;                                // 2 x 64 KB in flight
    }
    sp.raw_stages = raw;
    const ScanTSmem L = scan_t_smem_layout(sp.stages, P.hb, P.hsi, kf4, raw);
    if (static_cast<int>(L.total) > smem_room) return CSA2_ERR_SHAPE;
    sp.tmem_cols = scan_t_tmem_cols(kf4, sp.stages);
    CUtensorMap tk, tq;
    if (!make_map_bf16_128(&tq, a->qI, static_cast<uint64_t>(P.BQ) * 32, 32)) return CSA2_ERR_CUDA;
    if (kf4) tk = tq;                               // not read: index-K arrives by bulk copies
    else if (!make_map_bf16_128(&tk, a->kI, static_cast<uint64_t>(a->B) * a->N, P.pool ? 8 : tile_t))
      return CSA2_ERR_CUDA;
    const unsigned grid = static_cast<unsigned>(sp.groups * sp.ctas_per_group);
    trace_pre(kKIndexScan, st);
    const cudaError_t es = launch_scan_t1(P.hsi, kf4, grid, L.total + 1024, st, tk, tq, sp);
    trace_post(st);
    if (es != cudaSuccess) return CSA2_ERR_CUDA;
  } else {
    sp.tiles_per_group = static_cast<int>((P.n_elems + kTileRows - 1) / kTileRows);
    sp.ctas_per_group = scan_ctas_per_group(sp.groups, sp.tiles_per_group, dev.sms);
    const int QG = scan_qg(P.qg);
    const uint32_t n_mma = 32u * QG;
    int raw = 0;
    if (kf4) {
      // MXFP4 index-K: up to kF4RawStages raw tiles (8.5 KB each) in flight
      // and 4 repacked stages (9 KB each) for the MMA
      sp.k4 = static_cast<const uint8_t*>(a->kI);
      sp.stages = 4;
      raw = kF4RawStages;
      while (raw > 2 && static_cast<int>(scan_smem_layout(sp.stages, QG, P.hb, P.hsi, raw).total) > smem_room) --raw;
    } else {
      // three 32 KB stages per SM measured fastest (fewer bytes in flight per
      // stream keep DRAM pages open longer; 2, 4 and 6 stages were slower)
      const ScanSmem L0 = scan_smem_layout(0, QG, P.hb, P.hsi, 0);
      sp.stages = std::min(kScanStages, static_cast<int>((smem_room - L0.total) / (kStageBytes + 16)));
      if (sp.stages < 2) return CSA2_ERR_SHAPE;
    }
    sp.raw_stages = raw;
    const ScanSmem L = scan_smem_layout(sp.stages, QG, P.hb, P.hsi, raw);
    if (static_cast<int>(L.total) > smem_room) return CSA2_ERR_SHAPE;
    sp.tmem_cols = scan_tmem_cols(QG, kf4, sp.stages);
    CUtensorMap tk, tq;
    if (!make_map_bf16_128(&tq, a->qI, static_cast<uint64_t>(P.BQ) * 32, n_mma)) return CSA2_ERR_CUDA;
    if (kf4) tk = tq;                                 // not read: index-K arrives by bulk copies
    else if (!make_map_bf16_128(&tk, a->kI, static_cast<uint64_t>(a->B) * a->N, P.pool ? 8 : kTileRows))
      return CSA2_ERR_CUDA;

    const unsigned grid = static_cast<unsigned>(sp.groups * sp.ctas_per_group);
    trace_pre(kKIndexScan, st);
    const cudaError_t es = launch_scan(QG, P.hsi, kf4, grid, L.total + 1024, st, tk, tq, sp);
    trace_post(st);
    if (es != cudaSuccess) return CSA2_ERR_CUDA;
  }

  TopkParams tp;
  memset(&tp, 0, sizeof(tp));
  tp.scores = sp.scores;
  tp.ld = P.ld;
  tp.n_elems = P.n_elems;
  tp.n_vis = P.pool ? nullptr : a->n_vis;
  tp.vis_div = 1;
  tp.pool = sp.pool;
  tp.pool_blocks = sp.pool_blocks;
  tp.hist = sp.hist;
  tp.hb = P.hb;
  tp.hist_sample = P.hist_every;
  tp.K = a->K;
  tp.out_idx = a->idx;
  tp.out_scores = a->scores;
  tp.prefetch_kv = static_cast<const uint8_t*>(kv_prefetch);
  tp.prefetch_N = a->N;
  tp.Q = a->Q;
  if (launch_topk(tp, P.BQ, dev, st) != cudaSuccess) return CSA2_ERR_CUDA;

  if (P.hsi) {
    TopkParams bp = tp;
    bp.scores = sp.bscores;
    bp.ld = P.bld;
    bp.n_elems = P.nblk;
    bp.n_vis = a->n_vis;
    bp.vis_div = 8;
    bp.pool = nullptr;
    bp.hist = sp.bhist;
    bp.hist_sample = 1;
    bp.K = a->hsi_blocks;
    bp.out_idx = a->pool_out;
    bp.out_scores = nullptr;
    bp.prefetch_kv = nullptr;
    if (launch_topk(bp, P.BQ, dev, st) != cudaSuccess) return CSA2_ERR_CUDA;
  }
  return CSA2_OK;
}

// ---------------------------------------------------------------- attention call
csa2_status validate_attn(const csa2_attn_args* a) {
  if (!a) return CSA2_ERR_ARG;
  if (a->B < 1 || a->Q < 1 || static_cast<int64_t>(a->B) * a->Q > CSA2_MAX_BQ || a->K < 0 || a->K > CSA2_MAX_K ||
      a->W < 0 || a->W > CSA2_MAX_W ||
      a->K + a->W < 1 || a->N < 1 || a->swa_step < 0)
    return CSA2_ERR_SHAPE;
  if (a->swa_format != CSA2_FMT_BF16 && a->swa_format != CSA2_FMT_FP8) return CSA2_ERR_ARG;
  if (a->q_format != CSA2_FMT_BF16 && a->q_format != CSA2_FMT_NVFP4) return CSA2_ERR_ARG;
  if (!a->q || !a->out || (a->K > 0 && (!a->kv_fp4 || !a->idx)) || (a->W > 0 && !a->swa)) return CSA2_ERR_ARG;
  if (a->W > 0 && a->swa_format == CSA2_FMT_FP8 && !a->swa_scale) return CSA2_ERR_ARG;
  if (a->W > 0 && static_cast<int64_t>(a->Q - 1) * a->swa_step + a->W > a->swa_rows) return CSA2_ERR_SHAPE;
  if (!aligned16(a->q) || !aligned16(a->out) || (a->kv_fp4 && !aligned16(a->kv_fp4)) || (a->idx && !aligned16(a->idx)) ||
      (a->swa && !aligned16(a->swa)) || (a->lse && !aligned16(a->lse)) ||
      (a->swa_scale && (reinterpret_cast<uintptr_t>(a->swa_scale) & 3)))
    return CSA2_ERR_ALIGN;
  return CSA2_OK;
}

inline int attn_kv_slices(const csa2_attn_args* a) { return (a->K + kTcAttnKeys - 1) / kTcAttnKeys; }
inline int attn_slices(const csa2_attn_args* a) {
  return attn_kv_slices(a) + (a->W + kTcAttnKeys - 1) / kTcAttnKeys;
}

// bf16 [rows][512] matrix as a 2-D TMA map with 128-byte swizzle, box 64 x box_rows
bool make_map_bf16_512(CUtensorMap* m, const void* base, uint64_t rows, uint32_t box_rows) {
  const cuuint64_t dims[2] = {512, rows};
  const cuuint64_t strides[1] = {1024};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// With this many queries one CTA per query (all its slices in turn, final
// output) fills the GPU; fewer queries split their slices over CTAs and
// merge fp32 partials in sparse_attn_combine_kernel.
constexpr int64_t kAttnPerQueryMinBQ = 128;
inline bool attn_per_query(const csa2_attn_args* a) {
  return static_cast<int64_t>(a->B) * a->Q >= kAttnPerQueryMinBQ;
}

// Split mode with few enough slices: the slice CTAs of a query form one
// cluster and merge over distributed shared memory (no partials, no merge
// kernel).
inline bool attn_cluster_merge(const csa2_attn_args* a) {
  return !attn_per_query(a) && attn_slices(a) <= kTcMaxClusterSlices;
}

size_t attn_ws_bytes(const csa2_attn_args* a) {
  // unused in these modes; the size query stays non-zero for valid arguments
  if (attn_per_query(a) || attn_cluster_merge(a)) return 256;
  const size_t bq = static_cast<size_t>(a->B) * a->Q, s = attn_slices(a);
  return up256(bq * s * 64 * 512 * 4) + up256(bq * s * 64 * 2 * 4);
}

// early_inputs: the attention follows a kernel of this library in the same
// call (group), so q and the window rows are already complete
csa2_status run_attn(const csa2_attn_args* a, void* ws, cudaStream_t st, bool early_inputs = false) {
  const float scale = a->scale > 0.0f ? a->scale : 1.0f / sqrtf(512.0f);
  const size_t bq = static_cast<size_t>(a->B) * a->Q;
  const int slices = attn_slices(a);
  float* opart = static_cast<float*>(ws);
  float* ml = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + up256(bq * slices * 64 * 512 * 4));

  TcAttnParams t;
  t.B = a->B; t.Q = a->Q; t.K = a->K; t.W = a->W; t.N = a->N;
  t.kv = static_cast<const uint8_t*>(a->kv_fp4);
  t.idx = a->idx;
  t.swa_rows = a->swa_rows; t.swa_step = a->swa_step;
  t.kv_slices = attn_kv_slices(a);
  t.slices = slices;
  t.scale_log2 = scale * 1.4426950408889634f;
  const bool per_query = attn_per_query(a);
  const bool cluster = attn_cluster_merge(a);
  t.per_query = per_query ? 1 : 0;
  t.cluster_merge = cluster ? 1 : 0;
  t.early_inputs = early_inputs ? 1 : 0;
  t.opart = (per_query || cluster) ? nullptr : opart;
  t.ml = (per_query || cluster) ? nullptr : ml;
  t.out = static_cast<__nv_bfloat16*>(a->out);
  t.lse = a->lse;
  t.swa_fp8 = (a->W > 0 && a->swa_format == CSA2_FMT_FP8) ? 1 : 0;
  t.q_fp4 = a->q_format == CSA2_FMT_NVFP4 ? 1 : 0;
  t.q4 = static_cast<const uint8_t*>(a->q);
  t.swa8 = static_cast<const uint8_t*>(a->swa);
  t.swa_scale = a->swa_scale;
  CUtensorMap tq, tw;
  if (t.q_fp4) {
    // Q arrives by one bulk copy of FP4 rows; the map is never read
    if (!make_map_bf16_512(&tq, a->out, bq * 64, 64)) return CSA2_ERR_CUDA;
  } else if (!make_map_bf16_512(&tq, a->q, bq * 64, 64)) {
    return CSA2_ERR_CUDA;
  }
  if (a->W > 0 && !t.swa_fp8) {
    if (!make_map_bf16_512(&tw, a->swa, static_cast<uint64_t>(a->B) * a->swa_rows, kTcAttnKeys)) return CSA2_ERR_CUDA;
  } else {
    tw = tq;                                    // no window slices: never used
  }
  trace_pre(kKAttnSlice, st);
  const cudaError_t e1 = launch_ex(sparse_attn_tc_kernel, dim3(per_query ? 1 : slices, static_cast<unsigned>(bq)),
                                   dim3(kTcAttnThreads), kTcAttnSmem, st, cluster ? static_cast<unsigned>(slices) : 0u,
                                   tq, tw, t);
  trace_post(st);
  if (e1 != cudaSuccess) return CSA2_ERR_CUDA;
  if (per_query || cluster) return CSA2_OK;

  AttnParams p;
  p.slices = slices;
  p.opart = opart;
  p.ml = ml;
  p.out = static_cast<__nv_bfloat16*>(a->out);
  p.lse = a->lse;
  trace_pre(kKAttnCombine, st);
  const cudaError_t e2 = launch_ex(sparse_attn_combine_kernel, dim3(static_cast<unsigned>(bq * 64)), dim3(128), 0, st, 0, p);
  trace_post(st);
  if (e2 != cudaSuccess) return CSA2_ERR_CUDA;
  return CSA2_OK;
}

// ---------------------------------------------------------------- group call
// cur_pool: the pool REINDEX_POOL layers read at this point of the group
// (the call's own pool once a FULL layer built it, else pool_in)
csa2_index_args layer_index_args(const csa2_group_args* g, const csa2_layer& L, const int32_t* cur_pool) {
  csa2_index_args a;
  memset(&a, 0, sizeof(a));
  a.mode = L.mode; a.B = g->B; a.Q = g->Q; a.K = g->K; a.N = g->N;
  a.qI = L.qI; a.w = L.w; a.kI = g->kI; a.n_vis = g->n_vis;
  a.idx = L.idx; a.scores = L.scores;
  a.k_format = g->index_k_format;
  a.hsi_blocks = (L.mode == CSA2_FULL || L.mode == CSA2_REINDEX_POOL) ? g->hsi_blocks : 0;
  a.hsi_block = g->hsi_block;
  a.pool_out = (L.mode == CSA2_FULL && g->hsi_blocks > 0) ? g->pool : nullptr;
  a.pool_in = (L.mode == CSA2_REINDEX_POOL) ? cur_pool : nullptr;
  return a;
}

csa2_attn_args layer_attn_args(const csa2_group_args* g, const csa2_layer& L, const int32_t* idx) {
  csa2_attn_args a;
  memset(&a, 0, sizeof(a));
  a.B = g->B; a.Q = g->Q; a.K = g->K; a.W = g->W; a.N = g->N;
  a.q = L.q; a.kv_fp4 = g->kv_fp4; a.idx = idx; a.swa = L.swa;
  a.swa_rows = g->swa_rows; a.swa_step = g->swa_step; a.scale = g->scale;
  a.out = L.out; a.lse = L.lse;
  a.swa_format = g->swa_format; a.swa_scale = L.swa_scale;
  a.q_format = g->q_format;
  return a;
}

csa2_status validate_group(const csa2_group_args* g, size_t* index_zero, size_t* index_ws, size_t* attn_ws) {
  if (!g || !g->layers || g->n_layers < 1 || g->n_layers > 64) return CSA2_ERR_ARG;
  if (g->flags & ~(CSA2_GROUP_INPUTS_READY | CSA2_GROUP_SERIAL)) return CSA2_ERR_ARG;
  if (g->n_new < 0) return CSA2_ERR_SHAPE;
  if (g->n_new > 0 && (!g->kv_new || !g->new_rows || !g->kv_fp4)) return CSA2_ERR_ARG;
  if (g->n_new > 0 && (!aligned16(g->kv_new) || !aligned16(g->kv_fp4) || !aligned16(g->new_rows))) return CSA2_ERR_ALIGN;
  if (g->pool_in && !aligned16(g->pool_in)) return CSA2_ERR_ALIGN;
  size_t iz = 0, idata = 0;
  bool have_idx = false;
  const int32_t* cur_pool = g->pool_in;
  for (int i = 0; i < g->n_layers; ++i) {
    const csa2_layer& L = g->layers[i];
    if (L.mode == CSA2_REUSE) {
      if (!have_idx) return CSA2_ERR_ARG;
    } else {
      if (L.mode == CSA2_REINDEX_POOL && !cur_pool) return CSA2_ERR_ARG;
      const csa2_index_args a = layer_index_args(g, L, cur_pool);
      const csa2_status s = validate_index(&a);
      if (s != CSA2_OK) return s;
      const IndexPlan P = plan_index(&a);
      iz += P.zero_bytes;
      idata = std::max(idata, P.data_bytes);
      have_idx = true;
      if (L.mode == CSA2_FULL && g->hsi_blocks > 0) cur_pool = g->pool;
    }
    const csa2_attn_args aa = layer_attn_args(g, L, L.idx ? L.idx : g->layers[0].idx);
    const csa2_status s = validate_attn(&aa);
    if (s != CSA2_OK) return s;
  }
  const csa2_layer& L0 = g->layers[0];
  const csa2_attn_args a0 = layer_attn_args(g, L0, L0.idx);
  *index_zero = iz;
  *index_ws = iz + up256(idata);
  *attn_ws = attn_ws_bytes(&a0);
  return CSA2_OK;
}

// Validation of a group beyond validate_group: every indexing layer has an
// output index buffer.  *need = workspace bytes.
csa2_status check_group(const csa2_group_args* g, size_t* iz, size_t* iw, size_t* need) {
  size_t aw = 0;
  const csa2_status s = validate_group(g, iz, iw, &aw);
  if (s != CSA2_OK) return s;
  for (int i = 0; i < g->n_layers; ++i)
    if (g->layers[i].mode != CSA2_REUSE && !g->layers[i].idx) return CSA2_ERR_ARG;
  *need = *iw + aw;
  return CSA2_OK;
}

// ---------------------------------------------------------------- overlapped host copies
// The copy streams and events of csa2_*_decode_io, one set per device,
// created on first use and kept for the life of the process.
struct IoDevice {
  cudaStream_t h2d = nullptr, d2h = nullptr;
  std::vector<cudaEvent_t> ev;
};
IoDevice g_io[kMaxDevices];

csa2_status validate_copies(const csa2_copy* c, int32_t n, int n_layers) {
  if (n < 0 || (n > 0 && !c)) return CSA2_ERR_ARG;
  int prev = 0;
  for (int i = 0; i < n; ++i) {
    if (!c[i].dst || !c[i].src || c[i].layer < 0 || c[i].layer >= n_layers || c[i].layer < prev) return CSA2_ERR_ARG;
    prev = c[i].layer;
  }
  return CSA2_OK;
}

csa2_status validate_io(const csa2_io* io, int n_layers) {
  if (!io) return CSA2_ERR_ARG;
  const csa2_status s = validate_copies(io->in, io->n_in, n_layers);
  return s != CSA2_OK ? s : validate_copies(io->out, io->n_out, n_layers);
}

// One io call: which layers have copies, their events, and the hooks the
// group runner calls around each layer.  Event 0 marks the call's start on
// the caller's stream, events 1 and 2 the ends of the two copy streams,
// then one per layer with input copies and one per layer with outputs.
struct IoRun {
  const csa2_io* io = nullptr;
  IoDevice* d = nullptr;
  cudaStream_t st = nullptr;
  std::vector<int> ev_in, ev_out;   // per layer: event index, -1 if none
  std::vector<char> waited;
};

cudaError_t io_fail(cudaError_t e) {
  if (e != cudaSuccess) g_last_cuda_error = e;
  return e;
}

// Resources, then every input copy in order on the H2D stream (each layer's
// last copy followed by that layer's event).
csa2_status io_begin(IoRun* r, const csa2_io* io, int n_layers, cudaStream_t st) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return CSA2_ERR_CUDA;
  r->io = io;
  r->st = st;
  r->ev_in.assign(n_layers, -1);
  r->ev_out.assign(n_layers, -1);
  r->waited.assign(n_layers, 0);
  int n_ev = 3;
  for (int i = 0; i < io->n_in; ++i)
    if (r->ev_in[io->in[i].layer] < 0) r->ev_in[io->in[i].layer] = n_ev++;
  for (int i = 0; i < io->n_out; ++i)
    if (r->ev_out[io->out[i].layer] < 0) r->ev_out[io->out[i].layer] = n_ev++;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    IoDevice& d = g_io[dev];
    if (!d.h2d && io_fail(cudaStreamCreateWithFlags(&d.h2d, cudaStreamNonBlocking)) != cudaSuccess) return CSA2_ERR_CUDA;
    if (!d.d2h && io_fail(cudaStreamCreateWithFlags(&d.d2h, cudaStreamNonBlocking)) != cudaSuccess) return CSA2_ERR_CUDA;
    while (static_cast<int>(d.ev.size()) < n_ev) {
      cudaEvent_t e;
      if (io_fail(cudaEventCreateWithFlags(&e, cudaEventDisableTiming)) != cudaSuccess) return CSA2_ERR_CUDA;
      d.ev.push_back(e);
    }
    r->d = &d;
  }
  IoDevice& d = *r->d;
  if (io_fail(cudaEventRecord(d.ev[0], st)) != cudaSuccess ||
      io_fail(cudaStreamWaitEvent(d.h2d, d.ev[0], 0)) != cudaSuccess ||
      io_fail(cudaStreamWaitEvent(d.d2h, d.ev[0], 0)) != cudaSuccess)
    return CSA2_ERR_CUDA;
  for (int i = 0; i < io->n_in; ++i) {
    const csa2_copy& c = io->in[i];
    if (c.bytes > 0 && io_fail(cudaMemcpyAsync(c.dst, c.src, c.bytes, cudaMemcpyHostToDevice, d.h2d)) != cudaSuccess)
      return CSA2_ERR_CUDA;
    if ((i + 1 == io->n_in || io->in[i + 1].layer != c.layer) &&
        io_fail(cudaEventRecord(d.ev[r->ev_in[c.layer]], d.h2d)) != cudaSuccess)
      return CSA2_ERR_CUDA;
  }
  return CSA2_OK;
}

// Before layer l's first kernel: its input copies have landed.
csa2_status io_before_layer(IoRun* r, int l) {
  if (!r || r->ev_in[l] < 0 || r->waited[l]) return CSA2_OK;
  r->waited[l] = 1;
  return io_fail(cudaStreamWaitEvent(r->st, r->d->ev[r->ev_in[l]], 0)) == cudaSuccess ? CSA2_OK : CSA2_ERR_CUDA;
}

// After layer l's attention: its output copies go out on the D2H stream.
csa2_status io_after_layer(IoRun* r, int l) {
  if (!r || r->ev_out[l] < 0) return CSA2_OK;
  IoDevice& d = *r->d;
  const cudaEvent_t e = d.ev[r->ev_out[l]];
  if (io_fail(cudaEventRecord(e, r->st)) != cudaSuccess || io_fail(cudaStreamWaitEvent(d.d2h, e, 0)) != cudaSuccess)
    return CSA2_ERR_CUDA;
  for (int i = 0; i < r->io->n_out; ++i) {
    const csa2_copy& c = r->io->out[i];
    if (c.layer == l && c.bytes > 0 &&
        io_fail(cudaMemcpyAsync(c.dst, c.src, c.bytes, cudaMemcpyDeviceToHost, d.d2h)) != cudaSuccess)
      return CSA2_ERR_CUDA;
  }
  return CSA2_OK;
}

// Both copy streams join the caller's stream (also after a failure, so
// that no copy stream is left forked from a capture).
csa2_status io_end(IoRun* r) {
  if (!r->d) return CSA2_OK;
  IoDevice& d = *r->d;
  const bool ok = io_fail(cudaEventRecord(d.ev[1], d.h2d)) == cudaSuccess &&
                  io_fail(cudaEventRecord(d.ev[2], d.d2h)) == cudaSuccess &&
                  io_fail(cudaStreamWaitEvent(r->st, d.ev[1], 0)) == cudaSuccess &&
                  io_fail(cudaStreamWaitEvent(r->st, d.ev[2], 0)) == cudaSuccess;
  return ok ? CSA2_OK : CSA2_ERR_CUDA;
}

// Enqueue one validated group on `st` (workspace already large enough).
// first_early: the first layer's inputs were complete before the call
// (false for a group of a stack after the first: its first layer follows
// the previous group's last layer in model order)
// io / layer_base: the overlapped copies of an io call and the index of the
// group's first layer among the call's layers (nullptr / 0 otherwise)
csa2_status run_group(const csa2_group_args* g, size_t iz, size_t iw, const DeviceInfo& dev, void* ws,
                      cudaStream_t st, bool first_early = true, IoRun* io = nullptr, int layer_base = 0) {
  struct SerialScope {                             // CSA2_GROUP_SERIAL: plain stream order for this call
    bool prev;
    explicit SerialScope(bool on) : prev(g_serial_launch) { if (on) g_serial_launch = true; }
    ~SerialScope() { g_serial_launch = prev; }
  } serial((g->flags & CSA2_GROUP_SERIAL) != 0);
  const bool inputs_ready = (g->flags & CSA2_GROUP_INPUTS_READY) != 0;
  uint8_t* zws = static_cast<uint8_t*>(ws);     // one counter region per indexing layer
  uint8_t* dws = zws + iz;                         // data region shared by the layers in turn
  uint8_t* aws = zws + iw;
  if (cudaMemsetAsync(zws, 0, iz, st) != cudaSuccess) return CSA2_ERR_CUDA;
  if (io_before_layer(io, layer_base) != CSA2_OK) return CSA2_ERR_CUDA;    // the new entries
  if (g->n_new > 0) {
    if (launch_quantize(g->kv_new, g->n_new, 512, g->kv_fp4, g->new_rows, 0, st) != cudaSuccess) return CSA2_ERR_CUDA;
  }
  const int32_t* last_idx = nullptr;
  const int32_t* cur_pool = g->pool_in;
  for (int i = 0; i < g->n_layers; ++i) {
    const csa2_layer& L = g->layers[i];
    // the first layer's inputs precede the call; a later layer's are, in a
    // model, the previous layer's results unless the caller says otherwise
    const bool early = inputs_ready || (i == 0 && first_early);
    if (io_before_layer(io, layer_base + i) != CSA2_OK) return CSA2_ERR_CUDA;
    if (L.mode != CSA2_REUSE) {
      const csa2_index_args a = layer_index_args(g, L, cur_pool);
      const csa2_status s = run_index(&a, dev, zws, dws, st, g->kv_fp4, early);
      if (s != CSA2_OK) return s;
      zws += plan_index(&a).zero_bytes;
      last_idx = L.idx;
      if (L.mode == CSA2_FULL && g->hsi_blocks > 0) cur_pool = g->pool;
    }
    const csa2_attn_args aa = layer_attn_args(g, L, last_idx);
    const csa2_status s = run_attn(&aa, aws, st, early);
    if (s != CSA2_OK) return s;
    if (io_after_layer(io, layer_base + i) != CSA2_OK) return CSA2_ERR_CUDA;
  }
  return CSA2_OK;
}

csa2_status validate_stack(const csa2_stack_args* sa, size_t* need) {
  if (!sa || !sa->groups || sa->n_groups < 1 || sa->n_groups > 64) return CSA2_ERR_ARG;
  size_t mx = 0;
  for (int i = 0; i < sa->n_groups; ++i) {
    size_t iz = 0, iw = 0, n = 0;
    const csa2_status s = check_group(&sa->groups[i], &iz, &iw, &n);
    if (s != CSA2_OK) return s;
    mx = std::max(mx, n);
  }
  *need = mx;
  return CSA2_OK;
}

// ---------------------------------------------------------------- no-allocation variant
// Scratch of csa2_index_score_topk_noalloc: one file-scope device array.
// Every GPU that loads the library holds it until the process exits, and
// every call of that entry point on a device shares it.  In host code the
// symbol is only a stand-in: the kernels get the device address that
// cudaGetSymbolAddress returns for the current device.
constexpr size_t kNoAllocScratchBytes = static_cast<size_t>(CSA2_NOALLOC_SCRATCH_BYTES);
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];
// the address and the CUDA context it belongs to, per device: a context
// destroyed and re-created (cudaDeviceReset) reloads the module, and the
// array may then sit elsewhere
struct NoAllocAddr {
  CUcontext ctx = nullptr;
  void* addr = nullptr;
};
NoAllocAddr g_noalloc_addr[kMaxDevices];
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
CtxGetCurrentFn g_ctx_get_current = nullptr;

CUcontext current_context() {
  if (!g_ctx_get_current) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
      return nullptr;
    g_ctx_get_current = reinterpret_cast<CtxGetCurrentFn>(fn);
  }
  CUcontext c = nullptr;
  if (g_ctx_get_current(&c) != CUDA_SUCCESS) return nullptr;
  return c;
}

// Device address of the scratch array on the current device, looked up on
// the first call in each device context (without a context handle, on
// every call).
csa2_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return CSA2_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  NoAllocAddr& slot = g_noalloc_addr[dev];
  CUcontext ctx = current_context();
  if (!ctx || ctx != slot.ctx || !slot.addr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return CSA2_ERR_CUDA;
    slot.addr = p;
    slot.ctx = current_context();                  // the lookup made the device's context current
  }
  *out = slot.addr;
  return CSA2_OK;
}

}  // namespace
}  // namespace csa2

using namespace csa2;

extern "C" {

csa2_status csa2_quantize_kv_fp4(const void* x, int64_t n, int64_t ld_x, void* kv_fp4, const int64_t* dst_rows,
                                 int64_t row_offset, void* stream) {
  if (n < 0 || ld_x < 512 || (ld_x & 7) || row_offset < 0) return CSA2_ERR_SHAPE;
  if (n == 0) return CSA2_OK;
  if (!x || !kv_fp4) return CSA2_ERR_ARG;
  if (!aligned16(x) || !aligned16(kv_fp4) || (dst_rows && (reinterpret_cast<uintptr_t>(dst_rows) & 7))) return CSA2_ERR_ALIGN;
  DeviceInfo* dev = nullptr;
  const csa2_status s = device_info(&dev);
  if (s != CSA2_OK) return s;
  return launch_quantize(x, n, ld_x, kv_fp4, dst_rows, row_offset, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? CSA2_OK : CSA2_ERR_CUDA;
}

csa2_status csa2_quantize_window_fp8(const void* x, int64_t n, int64_t ld_x, void* codes, float* scales,
                                     const int64_t* dst_rows, int64_t row_offset, void* stream) {
  if (n < 0 || ld_x < 512 || (ld_x & 7) || row_offset < 0) return CSA2_ERR_SHAPE;
  if (n == 0) return CSA2_OK;
  if (!x || !codes || !scales) return CSA2_ERR_ARG;
  if (!aligned16(x) || !aligned16(codes) || (reinterpret_cast<uintptr_t>(scales) & 3) ||
      (dst_rows && (reinterpret_cast<uintptr_t>(dst_rows) & 7)))
    return CSA2_ERR_ALIGN;
  DeviceInfo* dev = nullptr;
  const csa2_status s = device_info(&dev);
  if (s != CSA2_OK) return s;
  return launch_quantize_window(x, n, ld_x, codes, scales, dst_rows, row_offset, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess ? CSA2_OK : CSA2_ERR_CUDA;
}

csa2_status csa2_compress_rope_quantize_kv_fp4(const csa2_compress_args* a, void* stream) {
  if (!a) return CSA2_ERR_ARG;
  if (a->n_entries < 0 || a->ld_x < 512 || (a->ld_x & 7) || a->r < 1 || a->r > 16 || a->row_offset < 0 ||
      (a->w_stride != 0 && a->w_stride != static_cast<int64_t>(a->r) * 512))
    return CSA2_ERR_SHAPE;
  if (a->n_entries == 0) return CSA2_OK;
  if (!a->x || !a->w || !a->cos || !a->sin || !a->kv_fp4) return CSA2_ERR_ARG;
  if (!aligned16(a->x) || !aligned16(a->w) || !aligned16(a->kv_fp4) ||
      (reinterpret_cast<uintptr_t>(a->cos) & 3) || (reinterpret_cast<uintptr_t>(a->sin) & 3) ||
      (a->dst_rows && (reinterpret_cast<uintptr_t>(a->dst_rows) & 7)))
    return CSA2_ERR_ALIGN;
  DeviceInfo* dev = nullptr;
  const csa2_status s = device_info(&dev);
  if (s != CSA2_OK) return s;
  return launch_compress_rope_quantize(a->x, a->n_entries, a->ld_x, a->r, a->w, a->w_stride, a->cos, a->sin, a->kv_fp4,
                                       a->dst_rows, a->row_offset, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? CSA2_OK : CSA2_ERR_CUDA;
}

csa2_status csa2_quantize_index_k_mxfp4(const void* x, int64_t n, int64_t ld_x, void* out, const int64_t* dst_rows,
                                        int64_t row_offset, void* stream) {
  if (n < 0 || ld_x < 128 || (ld_x & 3) || row_offset < 0) return CSA2_ERR_SHAPE;
  if (n == 0) return CSA2_OK;
  if (!x || !out) return CSA2_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(x) & 7) || (reinterpret_cast<uintptr_t>(out) & 3) ||
      (dst_rows && (reinterpret_cast<uintptr_t>(dst_rows) & 7)))
    return CSA2_ERR_ALIGN;
  DeviceInfo* dev = nullptr;
  const csa2_status s = device_info(&dev);
  if (s != CSA2_OK) return s;
  return launch_quantize_index_k(x, n, ld_x, out, dst_rows, row_offset, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess ? CSA2_OK : CSA2_ERR_CUDA;
}

csa2_status csa2_index_score_topk(const csa2_index_args* a, void* ws, size_t ws_bytes, void* stream) {
  csa2_status s = validate_index(a);
  if (s != CSA2_OK) return s;
  const IndexPlan P = plan_index(a);
  if (!ws || ws_bytes < P.total || !aligned16(ws)) return CSA2_ERR_WORKSPACE;
  DeviceInfo* dev = nullptr;
  s = device_info(&dev);
  if (s != CSA2_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(ws, 0, P.zero_bytes, st) != cudaSuccess) return CSA2_ERR_CUDA;
  return run_index(a, *dev, ws, static_cast<uint8_t*>(ws) + P.zero_bytes, st);
}

csa2_status csa2_index_score_topk_noalloc(const csa2_index_args* a, void* stream) {
  csa2_status s = validate_index(a);
  if (s != CSA2_OK) return s;
  const IndexPlan P = plan_index(a);
  if (P.total > kNoAllocScratchBytes) return CSA2_ERR_WORKSPACE;
  DeviceInfo* dev = nullptr;
  s = device_info(&dev);
  if (s != CSA2_OK) return s;
  void* ws = nullptr;
  s = noalloc_scratch(&ws);
  if (s != CSA2_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the array keeps the previous call's contents: clear the counter region
  if (cudaMemsetAsync(ws, 0, P.zero_bytes, st) != cudaSuccess) return CSA2_ERR_CUDA;
  return run_index(a, *dev, ws, static_cast<uint8_t*>(ws) + P.zero_bytes, st);
}

csa2_status csa2_sparse_attn(const csa2_attn_args* a, void* ws, size_t ws_bytes, void* stream) {
  csa2_status s = validate_attn(a);
  if (s != CSA2_OK) return s;
  if (!ws || ws_bytes < attn_ws_bytes(a) || !aligned16(ws)) return CSA2_ERR_WORKSPACE;
  DeviceInfo* dev = nullptr;
  s = device_info(&dev);
  if (s != CSA2_OK) return s;
  return run_attn(a, ws, static_cast<cudaStream_t>(stream));
}


csa2_status csa2_group_decode(const csa2_group_args* g, void* ws, size_t ws_bytes, void* stream) {
  size_t iz = 0, iw = 0, need = 0;
  csa2_status s = check_group(g, &iz, &iw, &need);
  if (s != CSA2_OK) return s;
  if (!ws || ws_bytes < need || !aligned16(ws)) return CSA2_ERR_WORKSPACE;
  DeviceInfo* dev = nullptr;
  s = device_info(&dev);
  if (s != CSA2_OK) return s;
  return run_group(g, iz, iw, *dev, ws, static_cast<cudaStream_t>(stream));
}

csa2_status csa2_stack_decode(const csa2_stack_args* sa, void* ws, size_t ws_bytes, void* stream) {
  size_t need = 0;
  csa2_status s = validate_stack(sa, &need);
  if (s != CSA2_OK) return s;
  if (!ws || ws_bytes < need || !aligned16(ws)) return CSA2_ERR_WORKSPACE;
  DeviceInfo* dev = nullptr;
  s = device_info(&dev);
  if (s != CSA2_OK) return s;
  for (int i = 0; i < sa->n_groups; ++i) {
    size_t iz = 0, iw = 0, n = 0;
    check_group(&sa->groups[i], &iz, &iw, &n);
    s = run_group(&sa->groups[i], iz, iw, *dev, ws, static_cast<cudaStream_t>(stream), i == 0);
    if (s != CSA2_OK) return s;
  }
  return CSA2_OK;
}

csa2_status csa2_group_decode_io(const csa2_group_args* g, const csa2_io* io, void* ws, size_t ws_bytes,
                                 void* stream) {
  size_t iz = 0, iw = 0, need = 0;
  csa2_status s = check_group(g, &iz, &iw, &need);
  if (s != CSA2_OK) return s;
  s = validate_io(io, g->n_layers);
  if (s != CSA2_OK) return s;
  if (!ws || ws_bytes < need || !aligned16(ws)) return CSA2_ERR_WORKSPACE;
  DeviceInfo* dev = nullptr;
  s = device_info(&dev);
  if (s != CSA2_OK) return s;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  IoRun r;
  s = io_begin(&r, io, g->n_layers, st);
  if (s == CSA2_OK) s = run_group(g, iz, iw, *dev, ws, st, true, &r, 0);
  const csa2_status e = io_end(&r);
  return s != CSA2_OK ? s : e;
}

csa2_status csa2_stack_decode_io(const csa2_stack_args* sa, const csa2_io* io, void* ws, size_t ws_bytes,
                                 void* stream) {
  size_t need = 0;
  csa2_status s = validate_stack(sa, &need);
  if (s != CSA2_OK) return s;
  int n_layers = 0;
  for (int i = 0; i < sa->n_groups; ++i) n_layers += sa->groups[i].n_layers;
  s = validate_io(io, n_layers);
  if (s != CSA2_OK) return s;
  if (!ws || ws_bytes < need || !aligned16(ws)) return CSA2_ERR_WORKSPACE;
  DeviceInfo* dev = nullptr;
  s = device_info(&dev);
  if (s != CSA2_OK) return s;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  IoRun r;
  s = io_begin(&r, io, n_layers, st);
  for (int i = 0, base = 0; s == CSA2_OK && i < sa->n_groups; base += sa->groups[i].n_layers, ++i) {
    size_t iz = 0, iw = 0, n = 0;
    check_group(&sa->groups[i], &iz, &iw, &n);
    s = run_group(&sa->groups[i], iz, iw, *dev, ws, st, i == 0, &r, base);
  }
  const csa2_status e = io_end(&r);
  return s != CSA2_OK ? s : e;
}

size_t csa2_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

size_t csa2_workspace_size(const void* args, int32_t which) {
  if (!args) return 0;
  if (which == CSA2_WS_INDEX) {
    const csa2_index_args* a = static_cast<const csa2_index_args*>(args);
    return validate_index(a) == CSA2_OK ? plan_index(a).total : 0;
  }
  if (which == CSA2_WS_ATTN) {
    const csa2_attn_args* a = static_cast<const csa2_attn_args*>(args);
    return validate_attn(a) == CSA2_OK ? attn_ws_bytes(a) : 0;
  }
  if (which == CSA2_WS_GROUP) {
    size_t iz = 0, iw = 0, need = 0;
    return check_group(static_cast<const csa2_group_args*>(args), &iz, &iw, &need) == CSA2_OK ? need : 0;
  }
  if (which == CSA2_WS_STACK) {
    size_t need = 0;
    return validate_stack(static_cast<const csa2_stack_args*>(args), &need) == CSA2_OK ? need : 0;
  }
  return 0;
}

csa2_status csa2_device_status(int32_t* code, void* stream) {
  int v = 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyFromSymbolAsync(&v, g_device_error, sizeof(int), 0, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return CSA2_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return CSA2_ERR_CUDA;
  if (code) *code = v;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbolAsync(g_device_error, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
      return CSA2_ERR_CUDA;
    return CSA2_ERR_DEVICE;
  }
  return CSA2_OK;
}

const char* csa2_cuda_error_string(void) { return cudaGetErrorString(g_last_cuda_error); }

const char* csa2_status_string(int32_t s) {
  switch (s) {
    case CSA2_OK: return "ok";
    case CSA2_ERR_ARG: return "invalid argument";
    case CSA2_ERR_SHAPE: return "unsupported shape";
    case CSA2_ERR_ALIGN: return "misaligned pointer or stride";
    case CSA2_ERR_WORKSPACE: return "workspace missing or too small";
    case CSA2_ERR_CUDA: return "CUDA error";
    case CSA2_ERR_DEVICE: return "device-side failure recorded";
    case CSA2_ERR_ARCH: return "device is not sm_100";
    default: return "unknown status";
  }
}

int32_t csa2_version(void) { return 107; }

csa2_status csa2_trace_begin(int32_t max_launches) {
  if (max_launches < 1 || max_launches > (1 << 20)) return CSA2_ERR_SHAPE;
  csa2_trace_end();
  g_trace.ev = new cudaEvent_t[2 * static_cast<size_t>(max_launches)];
  g_trace.kid = new int[max_launches];
  for (int i = 0; i < 2 * max_launches; ++i) {
    if (cudaEventCreate(&g_trace.ev[i]) != cudaSuccess) {
      for (int j = 0; j < i; ++j) cudaEventDestroy(g_trace.ev[j]);
      delete[] g_trace.ev; delete[] g_trace.kid;
      g_trace.ev = nullptr; g_trace.kid = nullptr;
      return CSA2_ERR_CUDA;
    }
  }
  g_trace.max = max_launches;
  g_trace.n = 0;
  g_trace.on = true;
  return CSA2_OK;
}

csa2_status csa2_trace_stop(void) {
  g_trace.on = false;
  return CSA2_OK;
}

csa2_status csa2_trace_end(void) {
  g_trace.on = false;
  if (g_trace.ev) {
    for (int i = 0; i < 2 * g_trace.max; ++i) cudaEventDestroy(g_trace.ev[i]);
    delete[] g_trace.ev;
    delete[] g_trace.kid;
  }
  g_trace = LaunchTrace();
  return CSA2_OK;
}

int32_t csa2_trace_count(void) { return g_trace.n; }

csa2_status csa2_trace_get(int32_t i, int32_t* kernel, float* ms) {
  if (i < 0 || i >= g_trace.n || !kernel || !ms) return CSA2_ERR_ARG;
  if (cudaEventSynchronize(g_trace.ev[2 * i + 1]) != cudaSuccess) return CSA2_ERR_CUDA;
  if (cudaEventElapsedTime(ms, g_trace.ev[2 * i], g_trace.ev[2 * i + 1]) != cudaSuccess) return CSA2_ERR_CUDA;
  *kernel = g_trace.kid[i];
  return CSA2_OK;
}

const char* csa2_kernel_name(int32_t kernel) {
  switch (kernel) {
    case kKQuantize: return "quantize_kv_fp4_kernel";
    case kKIndexScan: return "index_scan_kernel";
    case kKTopk: return "topk_select_kernel";
    case kKAttnSlice: return "sparse_attn_tc_kernel";
    case kKAttnCombine: return "sparse_attn_combine_kernel";
    case kKQuantizeWindow: return "quantize_window_fp8_kernel";
    case kKQuantizeIndexK: return "quantize_index_k_mxfp4_kernel";
    case kKCompressRope: return "compress_rope_quantize_kernel";
    default: return "unknown";
  }
}

}  // extern "C"
