// Host launcher of the tcgen05 GEMM template, shared by the dense and group-sparse paths.
#pragma once
#include <algorithm>
#include <cmath>

#include "swf_internal.h"
#include "swf_tc_gemm.cuh"

namespace swf {

inline int cdiv(int64_t a, int64_t b) { return (int)((a + b - 1) / b); }

// Launches tc_gemm_kernel on min(tiles, SMs) persistent CTAs, bracketed for profiling as `kind`.
template <int BN, bool A_MN, bool B_MN, bool B_DUAL, int EPI, int MODE = kModeDense,
          bool TMA_EPI = false, int GATHER = kGatherNone>
swf_status launch_tc(int kind, const CUtensorMap& ta, const CUtensorMap& tb0,
                     const CUtensorMap& tb1, TcGemmArgs args, cudaStream_t st,
                     const EpiMaps& em = EpiMaps{}) {
  DevCtx ctx;
  swf_status s = get_ctx(&ctx);
  if (s != SWF_OK) return s;
  const int64_t tiles = (int64_t)args.num_m_blk * args.num_n_blk *
                        (MODE == kModeKGrouped ? args.n_groups : 1);
  if (tiles == 0) return SWF_OK;
  if (tiles > INT32_MAX) return SWF_ERR_UNSUPPORTED;
  args.status = ctx.status;
  if (args.wait_limit_ns == 0) args.wait_limit_ns = kDefaultWaitNs;
  args.raster = std::max(1, std::min(args.raster, args.num_m_blk));
  auto kern = tc_gemm_kernel<BN, A_MN, B_MN, B_DUAL, EPI, MODE, false, TMA_EPI, GATHER>;
  constexpr int smem = TcSmem<BN, false, epi_smem_bytes<EPI, TMA_EPI, false>()>::kBytes;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return SWF_ERR_LAUNCH;
  const int64_t units = args.unit > 1 ? (tiles + args.unit - 1) / args.unit : tiles;
  const int grid = (int)std::min<int64_t>(units, ctx.num_sms);
  ProfScope prof(kind, st);
  kern<<<grid, gemm_threads<GATHER>(), smem, st>>>(ta, tb0, tb1, em, args);
  return cudaGetLastError() == cudaSuccess ? SWF_OK : SWF_ERR_LAUNCH;
}

// Launches the pair-mode (cta_group::2) dense GEMM as clusters of two CTAs: min(tiles, SMs / 2)
// clusters, each walking 256 x BN tiles.  TMA_EPI: the epilogue moves its tiles with TMA through
// the maps in `em`.
template <int BN, bool A_MN, bool B_MN, bool B_DUAL, int EPI, bool TMA_EPI = false>
swf_status launch_tc_pair(int kind, const CUtensorMap& ta, const CUtensorMap& tb0,
                          const CUtensorMap& tb1, const EpiMaps& em, TcGemmArgs args,
                          cudaStream_t st) {
  DevCtx ctx;
  swf_status s = get_ctx(&ctx);
  if (s != SWF_OK) return s;
  const int64_t tiles = (args.tile_count > 0 ? (int64_t)args.tile_count
                                              : (int64_t)args.num_m_blk * args.num_n_blk - args.tile_offset) *
                        std::max(1, args.ksplit);
  if (tiles <= 0) return SWF_OK;
  if (tiles > INT32_MAX) return SWF_ERR_UNSUPPORTED;
  args.status = ctx.status;
  if (args.wait_limit_ns == 0) args.wait_limit_ns = kDefaultWaitNs;
  args.raster = std::max(1, std::min(args.raster, args.num_m_blk));
  auto kern = tc_gemm_kernel<BN, A_MN, B_MN, B_DUAL, EPI, kModeDense, true, TMA_EPI>;
  constexpr int smem = TcSmem<BN, true, epi_smem_bytes<EPI, TMA_EPI, true>()>::kBytes;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return SWF_ERR_LAUNCH;
  const int clusters = (int)std::min<int64_t>(tiles, ctx.num_sms / 2);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * clusters, 1, 1);
  cfg.blockDim = dim3(kGemmThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  ProfScope prof(kind, st);
  if (cudaLaunchKernelEx(&cfg, kern, ta, tb0, tb1, em, args) != cudaSuccess) return SWF_ERR_LAUNCH;
  return cudaGetLastError() == cudaSuccess ? SWF_OK : SWF_ERR_LAUNCH;
}

// K splits of a pair-mode GEMM with `tiles` output tiles of kb_total k-blocks whose fp32 partial
// planes hold out_elems elements each: the split that minimises (waves x k-blocks per split) of
// the GEMM plus the partials' extra HBM traffic, on the 74 clusters of a 148-SM B200 (a host
// planning constant: the launch itself uses the device's SM count).
inline int choose_ksplit(int64_t tiles, int kb_total, int64_t out_elems) {
  constexpr double kClusters = 74.0, kKblockUs = 0.27, kBytesPerUs = 5.0e6;
  int best = 1;
  double best_us = std::ceil(tiles / kClusters) * kb_total * kKblockUs;
  for (int ks = 2; ks <= 16 && kb_total / ks >= 8; ++ks) {
    const double per = std::ceil((double)kb_total / ks);
    const double us = std::ceil(tiles * ks / kClusters) * per * kKblockUs +
                      (8.0 * ks * out_elems + 2.0 * out_elems) / kBytesPerUs;
    if (us < best_us) {
      best_us = us;
      best = ks;
    }
  }
  return best;
}

// Arguments of a dense GEMM of M x N (N-blocks of n_blk_cols columns) over K, with M-blocks of
// m_tile rows (256 in pair mode).
inline TcGemmArgs base_args(int64_t M, int64_t N, int n_blk_cols, int64_t K, int m_tile = kTileM) {
  TcGemmArgs a{};
  a.M = (int)M;
  a.N = (int)N;
  a.num_m_blk = cdiv(M, m_tile);
  a.num_n_blk = cdiv(N, n_blk_cols);
  a.raster = 8;
  a.kb_total = cdiv(K, kTileK);
  a.kb_seg0 = a.kb_total;
  a.row_split = (int)M;
  return a;
}

}  // namespace swf
