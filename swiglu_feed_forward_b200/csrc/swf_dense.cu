// Dense SwiGLU FFN: host launchers of the tcgen05 (bf16) and CUDA-core (fp32) GEMM chains.
//
// Training forward (flash-swiglu-mlp overview, "Fused train forward" + "Down projection"):
//   K1  [g|u] = x [W_g|W_u]^T, epilogue h, a, b         (gate|up dual tile, K = d_model)
//   K2  y = h W_d^T                                        (K = d_ff)
// Backward ("Activation gradients", "Weight gradients", "Input gradient"; parameter-golf
// PR 1105 "Fused MLP Kernels" for the epilogue multiply by the stored factor):
//   K3  dH = dY W_d, epilogue dG = dH*a, dU = dH*b -> dGU = [dG | dU]   (K = d_model)
//   K4  dx = dGU [W_g ; W_u]                               (K = 2 d_ff, two B segments)
//   K5  [dW_g ; dW_u] = dGU^T x                            (K = M)
//   K6  dW_d = dY^T h                                      (K = M)
#include <algorithm>

#include "swf_internal.h"
#include "swf_launch.cuh"
#include "swf_simt.cuh"

namespace swf {

namespace {
// Tensor map of a TMA epilogue's output or factor plane: 32-row boxes of 32 columns (64-byte
// swizzle) or 64 columns (128-byte swizzle), as the epilogue's staging boxes are laid out.
bool epi_map(CUtensorMap* m, const void* base, int64_t cols, int64_t rows, int64_t row_elems,
             int box_cols = 32) {
  return encode_tmap_bf16(m, base, cols, rows, row_elems, box_cols, 32, box_cols == 64 ? 128 : 64);
}

// out[m, n] = bf16(sum over splits s = 0, 1, ... of part[s][m][n]) in that fixed order; rows at
// or past row_split go to out1 (row - row_split).  8 elements per thread.
__global__ void splitk_reduce_kernel(const float4* __restrict__ part, int64_t plane4, int ks,
                                     int64_t rows, int64_t cols, int64_t row_split,
                                     __nv_bfloat16* __restrict__ out0,
                                     __nv_bfloat16* __restrict__ out1) {
  const int64_t n8 = rows * cols / 8;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8;
       i += (int64_t)gridDim.x * blockDim.x) {
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int s = 0; s < ks; ++s) {
      const float4 a = part[s * plane4 + 2 * i], b = part[s * plane4 + 2 * i + 1];
      acc[0] += a.x, acc[1] += a.y, acc[2] += a.z, acc[3] += a.w;
      acc[4] += b.x, acc[5] += b.y, acc[6] += b.z, acc[7] += b.w;
    }
    const int64_t e = 8 * i, m = e / cols, n = e - m * cols;
    __nv_bfloat16* dst = m < row_split ? out0 + m * cols + n : out1 + (m - row_split) * cols + n;
    *reinterpret_cast<uint4*>(dst) = make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                                                pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
  }
}

// How a weight-gradient GEMM of rows x cols over K (pair tiles 256 x BN) is scheduled:
//   uniform K split into ks planes (ks = 1: direct bf16 stores), or
//   hybrid: the first `head` output tiles (whole waves of the 74 clusters) with direct stores,
//   and the remaining ones in a second launch split ks ways along K into fp32 partial planes,
//   summed per tile by splitk_reduce_tiles_kernel.
// A persistent launch of n tiles takes ceil(n / 74) tile times, so 344 tiles take 5 where 4.65
// would do; splitting only the last, partial wave recovers most of that without the partial
// traffic of a uniform split.  Costs are the same model as choose_ksplit (k-block time, partial
// bytes at HBM speed), plus a launch for the tail and its reduction.
struct DwPlan {
  int ks;    // uniform split (hybrid: the tail's split)
  int head;  // hybrid: output tiles of the first launch (0: uniform)
  int tiles, bn;
};

DwPlan dw_plan(int64_t rows, int64_t cols, int64_t K) {
  constexpr double kClusters = 74.0, kKblockUs = 0.27, kBytesPerUs = 5.0e6, kLaunchUs = 6.0;
  DwPlan p{};
  p.bn = cols <= 128 ? 128 : 256;
  p.tiles = cdiv(rows, 2 * kTileM) * cdiv(cols, p.bn);
  const int kb = cdiv(K, kTileK);
  const int ks = choose_ksplit(p.tiles, kb, rows * cols);
  p.ks = ks > 1 ? cdiv(kb, cdiv(kb, ks)) : 1;  // no empty trailing split
  p.head = 0;
  auto uniform_us = [&](int k) {
    const double per = std::ceil((double)kb / k);
    const double us = std::ceil(p.tiles * k / kClusters) * per * kKblockUs;
    return k > 1 ? us + (8.0 * k * rows * cols + 2.0 * rows * cols) / kBytesPerUs + kLaunchUs : us;
  };
  double best = uniform_us(p.ks);
  const int waves = (int)(p.tiles / kClusters), tail = p.tiles - waves * (int)kClusters;
  if (waves >= 1 && tail > 0) {
    const double tile_elems = 2.0 * kTileM * p.bn;
    for (int k = 2; k <= 16 && kb / k >= 8; ++k) {
      const double per = std::ceil((double)kb / k);
      const double us = waves * kb * kKblockUs + std::ceil(tail * k / kClusters) * per * kKblockUs +
                        (8.0 * k * tail * tile_elems + 2.0 * tail * tile_elems) / kBytesPerUs + 2 * kLaunchUs;
      if (us < best) {
        best = us;
        p.ks = k;
        p.head = waves * (int)kClusters;
      }
    }
  }
  return p;
}

// The tail tiles [tile0, tile0 + ntiles) of a hybrid weight-gradient GEMM (pair tiles of 256 x BN,
// raster order as the GEMM's): out = bf16(sum over splits s = 0, 1, ... of part[s]) in that order;
// rows at or past row_split go to out1 (row - row_split).  8 elements per thread.
__global__ void splitk_reduce_tiles_kernel(const float* __restrict__ part, int64_t plane, int ks, int64_t rows,
                                           int64_t cols, int64_t row_split, __nv_bfloat16* __restrict__ out0,
                                           __nv_bfloat16* __restrict__ out1, int num_m_blk, int num_n_blk,
                                           int raster, int tile0, int ntiles, int bn) {
  const int per_tile = 2 * kTileM * bn / 8;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < (int64_t)ntiles * per_tile;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int lt = (int)(i / per_tile), e = (int)(i - (int64_t)lt * per_tile) * 8;
    int mb, nb;
    tile_coords(tile0 + lt, num_m_blk, num_n_blk, raster, mb, nb);
    const int64_t m = (int64_t)mb * 2 * kTileM + e / bn, n = (int64_t)nb * bn + e % bn;
    if (m >= rows || n >= cols) continue;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    const float* src = part + m * cols + n;
    for (int s0 = 0; s0 < ks; s0 += 4) {  // the loads of up to four splits in flight, summed in order
      float4 a[4], b[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const bool in = s0 + j < ks;
        const float4* p4 = reinterpret_cast<const float4*>(src + (int64_t)(in ? s0 + j : s0) * plane);
        a[j] = in ? p4[0] : make_float4(0.f, 0.f, 0.f, 0.f);
        b[j] = in ? p4[1] : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (s0 + j >= ks) break;
        acc[0] += a[j].x, acc[1] += a[j].y, acc[2] += a[j].z, acc[3] += a[j].w;
        acc[4] += b[j].x, acc[5] += b[j].y, acc[6] += b[j].z, acc[7] += b[j].w;
      }
    }
    __nv_bfloat16* dst = m < row_split ? out0 + m * cols + n : out1 + (m - row_split) * cols + n;
    *reinterpret_cast<uint4*>(dst) = make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                                                pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
  }
}

}  // namespace

swf_status splitk_reduce(const float* part, int ks, int64_t rows, int64_t cols, int64_t row_split,
                         void* out0, void* out1, cudaStream_t st);

// Weight-gradient GEMM (both operands MN-major, K = tokens), scheduled as dw_plan says: direct
// stores, a uniform K split into fp32 partial planes plus a fixed-order reduction, or the hybrid
// of the two (whole waves direct, the last partial wave split).
template <int BN>
swf_status launch_dw_bn(int kind, const CUtensorMap& ta, const CUtensorMap& tb, int64_t rows, int64_t cols,
                        int64_t K, void* out0, void* out1, int64_t row_split, float* part, const DwPlan& p,
                        cudaStream_t st) {
  TcGemmArgs a = base_args(rows, cols, BN, K, 2 * kTileM);
  a.out0 = out0;
  a.out1 = out1;
  a.row_split = (int)row_split;
  a.ld_out = cols;
  if (p.ks <= 1) return launch_tc_pair<BN, true, true, false, kEpiStore>(kind, ta, tb, tb, EpiMaps{}, a, st);
  swf_status s = SWF_OK;
  if (p.head > 0) {  // whole waves: direct stores
    a.tile_count = p.head;
    if ((s = launch_tc_pair<BN, true, true, false, kEpiStore>(kind, ta, tb, tb, EpiMaps{}, a, st)) != SWF_OK) return s;
    a.tile_offset = p.head;
    a.tile_count = p.tiles - p.head;
  }
  a.ksplit = p.ks;
  a.kb_per_split = cdiv(a.kb_total, p.ks);
  a.part = part;
  a.part_plane = rows * cols;
  if ((s = launch_tc_pair<BN, true, true, false, kEpiPartialF32>(kind, ta, tb, tb, EpiMaps{}, a, st)) != SWF_OK)
    return s;
  if (p.head == 0) return splitk_reduce(part, p.ks, rows, cols, row_split, out0, out1, st);
  ProfScope prof(SWF_K_SPLITK_REDUCE, st);
  const int ntail = p.tiles - p.head;
  const int64_t work = (int64_t)ntail * 2 * kTileM * BN / 8;
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>((work + 255) / 256, 148 * 16));
  splitk_reduce_tiles_kernel<<<grid, 256, 0, st>>>(part, rows * cols, p.ks, rows, cols, row_split,
                                                   static_cast<__nv_bfloat16*>(out0),
                                                   static_cast<__nv_bfloat16*>(out1), a.num_m_blk, a.num_n_blk,
                                                   std::max(1, std::min(a.raster, a.num_m_blk)), p.head, ntail, BN);
  return cudaGetLastError() == cudaSuccess ? SWF_OK : SWF_ERR_LAUNCH;
}

swf_status launch_dw(int kind, const CUtensorMap& ta, const CUtensorMap& tb, int64_t rows,
                     int64_t cols, int64_t K, void* out0, void* out1, int64_t row_split,
                     float* part, cudaStream_t st) {
  const DwPlan p = dw_plan(rows, cols, K);
  if (p.bn == 128)  // narrow outputs: pair tiles of 256 x 128
    return launch_dw_bn<128>(kind, ta, tb, rows, cols, K, out0, out1, row_split, part, p, st);
  return launch_dw_bn<256>(kind, ta, tb, rows, cols, K, out0, out1, row_split, part, p, st);
}

swf_status splitk_reduce(const float* part, int ks, int64_t rows, int64_t cols, int64_t row_split,
                         void* out0, void* out1, cudaStream_t st) {
  ProfScope prof(SWF_K_SPLITK_REDUCE, st);
  const int64_t n8 = rows * cols / 8;
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>((n8 + 255) / 256, 148 * 16));
  splitk_reduce_kernel<<<grid, 256, 0, st>>>(reinterpret_cast<const float4*>(part), rows * cols / 4,
                                             ks, rows, cols, row_split,
                                             static_cast<__nv_bfloat16*>(out0),
                                             static_cast<__nv_bfloat16*>(out1));
  return cudaGetLastError() == cudaSuccess ? SWF_OK : SWF_ERR_LAUNCH;
}

int64_t part_elems(int64_t rows, int64_t cols, int64_t K) {
  const DwPlan p = dw_plan(rows, cols, K);
  return p.ks > 1 ? p.ks * rows * cols : 0;
}

int64_t dense_bwd_part_elems(int64_t M, int64_t d, int64_t f) {
  return std::max(part_elems(2 * f, d, M), part_elems(d, f, M));
}

int64_t mlp2_bwd_part_elems(int64_t M, int64_t d, int64_t f) {
  return std::max(part_elems(f, d, M), part_elems(d, f, M));
}

int64_t dense_gemm_tiles(int op, int64_t M, int64_t d, int64_t f) {
  auto t = [](int64_t m, int64_t n, int64_t bn) { return (int64_t)cdiv(m, kTileM) * cdiv(n, bn); };
  // pair-mode tiles of 256 rows
  if (op == SWF_OP_FWD || op == SWF_OP_FWD_INFER) return (t(M, f, 128) + t(M, d, 256) + 1) / 2;
  if (op == SWF_OP_BWD) return (t(M, f, 256) + t(M, d, 256) + t(2 * f, d, 256) + t(d, f, 256) + 1) / 2;
  return 0;
}

swf_status dense_fwd_bf16(const void* x, const void* wg, const void* wu, const void* wd, void* y,
                          void* h, void* a, void* b, int64_t M, int64_t d, int64_t f, bool infer,
                          cudaStream_t st) {
  CUtensorMap tx, twg, twu, th, twd;
  if (!encode_tmap_bf16(&tx, x, d, M, d, 64, 128) || !encode_tmap_bf16(&twg, wg, d, f, d, 64, 128) ||
      !encode_tmap_bf16(&twu, wu, d, f, d, 64, 128) || !encode_tmap_bf16(&th, h, f, M, f, 64, 128) ||
      !encode_tmap_bf16(&twd, wd, f, d, f, 64, 128))
    return SWF_ERR_LAUNCH;
  // K1: gate|up dual tile, 128 columns of each per tile
  TcGemmArgs k1 = base_args(M, f, 128, d, 2 * kTileM);
  k1.out0 = h;
  k1.ld_out = f;
  k1.aux0 = a;
  k1.aux1 = b;
  k1.ld_aux = f;
  // h (and a, b) leave through per-warp staging boxes and TMA stores
  EpiMaps e1{};
  if (!epi_map(&e1.o[0], h, f, M, f) ||
      (!infer && (!epi_map(&e1.o[1], a, f, M, f) || !epi_map(&e1.o[2], b, f, M, f))))
    return SWF_ERR_LAUNCH;
  swf_status s =
      infer ? launch_tc_pair<256, false, false, true, kEpiSwiGLUInf, true>(SWF_K_GATE_UP_INFER, tx, twg, twu, e1, k1, st)
            : launch_tc_pair<256, false, false, true, kEpiSwiGLU, true>(SWF_K_GATE_UP, tx, twg, twu, e1, k1, st);
  if (s != SWF_OK) return s;
  // K2: y = h W_d^T
  TcGemmArgs k2 = base_args(M, d, 256, f, 2 * kTileM);
  k2.out0 = y;
  k2.ld_out = d;
  return launch_tc_pair<256, false, false, false, kEpiStore>(SWF_K_DOWN, th, twd, twd, EpiMaps{}, k2, st);
}

swf_status dense_bwd_bf16(const void* dy, const void* x, const void* wg, const void* wu,
                          const void* wd, const void* h, const void* a, const void* b, void* dx,
                          void* dwg, void* dwu, void* dwd, void* dgu, float* part, int64_t M,
                          int64_t d, int64_t f, cudaStream_t st) {
  swf_status s;
  {  // K3: dH = dY W_d (B = W_d viewed [K=d rows, N=f cols], MN-major), epilogue * a, * b
    CUtensorMap tdy, twd;
    if (!encode_tmap_bf16(&tdy, dy, d, M, d, 64, 128) || !encode_tmap_bf16(&twd, wd, f, d, f, 64, 64))
      return SWF_ERR_LAUNCH;
    // TMA epilogue (measured: 1.05 -> 0.67 ms at 32768 x 2048 x 5504): a and b come in by TMA,
    // dG and dU leave by TMA through two views of dGU (each [M, f], rows 2f apart)
    EpiMaps e3{};
    const __nv_bfloat16* dgu_b = static_cast<const __nv_bfloat16*>(dgu);
    constexpr int kBc = tma_epi_cols<kEpiDGate>();
    if (!epi_map(&e3.o[0], dgu_b, f, M, 2 * f, kBc) || !epi_map(&e3.o[1], dgu_b + f, f, M, 2 * f, kBc) ||
        !epi_map(&e3.o[2], a, f, M, f, kBc) || !epi_map(&e3.o[3], b, f, M, f, kBc))
      return SWF_ERR_LAUNCH;
    TcGemmArgs k3 = base_args(M, f, 256, d, 2 * kTileM);
    s = launch_tc_pair<256, false, true, false, kEpiDGate, true>(SWF_K_DGATE, tdy, twd, twd, e3, k3, st);
    if (s != SWF_OK) return s;
  }
  {  // K4: dx = dG W_g + dU W_u: A = dGU (K-major, K = 2f), B segments W_g / W_u (MN-major)
    CUtensorMap tdgu, twg, twu;
    if (!encode_tmap_bf16(&tdgu, dgu, 2 * f, M, 2 * f, 64, 128) ||
        !encode_tmap_bf16(&twg, wg, d, f, d, 64, 64) || !encode_tmap_bf16(&twu, wu, d, f, d, 64, 64))
      return SWF_ERR_LAUNCH;
    TcGemmArgs k4 = base_args(M, d, 256, 0, 2 * kTileM);
    k4.kb_seg0 = cdiv(f, kTileK);
    k4.kb_total = 2 * k4.kb_seg0;
    k4.a_koff1 = (int)f;
    k4.out0 = dx;
    k4.ld_out = d;
    s = launch_tc_pair<256, false, true, false, kEpiStore>(SWF_K_DX, tdgu, twg, twu, EpiMaps{}, k4, st);
    if (s != SWF_OK) return s;
  }
  {  // K5: [dW_g ; dW_u] = dGU^T x: A = dGU viewed [K=M rows, 2f cols] (MN-major), B = x (MN)
    CUtensorMap tdgu, tx;
    if (!encode_tmap_bf16(&tdgu, dgu, 2 * f, M, 2 * f, 64, 64) || !encode_tmap_bf16(&tx, x, d, M, d, 64, 64))
      return SWF_ERR_LAUNCH;
    s = launch_dw(SWF_K_DW_GATE_UP, tdgu, tx, 2 * f, d, M, dwg, dwu, f, part, st);
    if (s != SWF_OK) return s;
  }
  {  // K6: dW_d = dY^T h: A = dY viewed [K=M rows, d cols] (MN), B = h [K=M rows, f cols] (MN)
    CUtensorMap tdy, th;
    if (!encode_tmap_bf16(&tdy, dy, d, M, d, 64, 64) || !encode_tmap_bf16(&th, h, f, M, f, 64, 64))
      return SWF_ERR_LAUNCH;
    s = launch_dw(SWF_K_DW_DOWN, tdy, th, d, f, M, dwd, dwd, d, part, st);
  }
  return s;
}

// ------------------------------------------------------------------ fp32 (CUDA cores)
namespace {
template <int EPI, bool DUAL>
swf_status launch_simt(const SimtArgs& a, cudaStream_t st) {
  if (a.M == 0 || a.N == 0) return SWF_OK;
  dim3 grid(cdiv(a.N, kSimtTile), cdiv(a.M, kSimtTile));
  ProfScope prof(SWF_K_F32_GEMM, st);
  simt_gemm_f32<EPI, DUAL><<<grid, 256, 0, st>>>(a);
  return cudaGetLastError() == cudaSuccess ? SWF_OK : SWF_ERR_LAUNCH;
}
SimtArgs simt_base(int64_t M, int64_t N, int64_t K) {
  SimtArgs a{};
  a.M = (int)M;
  a.N = (int)N;
  a.K = (int)K;
  a.k_split = (int)K;
  a.row_split = (int)M;
  return a;
}
}  // namespace

swf_status dense_fwd_f32(const float* x, const float* wg, const float* wu, const float* wd,
                         float* y, float* h, float* a, float* b, int64_t M, int64_t d, int64_t f,
                         bool infer, cudaStream_t st) {
  SimtArgs k1 = simt_base(M, f, d);
  k1.A = x, k1.sam = d, k1.sak = 1;
  k1.B0 = wg, k1.B1 = wu, k1.sbn = d, k1.sbk = 1;
  k1.out0 = h, k1.ld_out = f, k1.aux0 = a, k1.aux1 = b, k1.ld_aux = f;
  swf_status s = infer ? launch_simt<kSimtSwiGLUInf, true>(k1, st) : launch_simt<kSimtSwiGLU, true>(k1, st);
  if (s != SWF_OK) return s;
  SimtArgs k2 = simt_base(M, d, f);
  k2.A = h, k2.sam = f, k2.sak = 1;
  k2.B0 = wd, k2.B1 = wd, k2.sbn = f, k2.sbk = 1;
  k2.out0 = y, k2.ld_out = d;
  return launch_simt<kSimtStore, false>(k2, st);
}

swf_status dense_bwd_f32(const float* dy, const float* x, const float* wg, const float* wu,
                         const float* wd, const float* h, const float* a, const float* b,
                         float* dx, float* dwg, float* dwu, float* dwd, float* dgu, int64_t M,
                         int64_t d, int64_t f, cudaStream_t st) {
  SimtArgs k3 = simt_base(M, f, d);  // dH[m, n] = sum_k dY[m, k] W_d[k, n]
  k3.A = dy, k3.sam = d, k3.sak = 1;
  k3.B0 = wd, k3.B1 = wd, k3.sbn = 1, k3.sbk = f;
  k3.out0 = dgu, k3.ld_out = 2 * f, k3.aux0 = const_cast<float*>(a), k3.aux1 = const_cast<float*>(b);
  k3.ld_aux = f, k3.d_ff = (int)f;
  swf_status s = launch_simt<kSimtDGate, false>(k3, st);
  if (s != SWF_OK) return s;
  SimtArgs k4 = simt_base(M, d, 2 * f);  // dx[m, n] = sum_k dGU[m, k] [W_g ; W_u][k, n]
  k4.A = dgu, k4.sam = 2 * f, k4.sak = 1;
  k4.B0 = wg, k4.B1 = wu, k4.sbn = 1, k4.sbk = d, k4.k_split = (int)f;
  k4.out0 = dx, k4.ld_out = d;
  if ((s = launch_simt<kSimtStore, false>(k4, st)) != SWF_OK) return s;
  SimtArgs k5 = simt_base(2 * f, d, M);  // [dW_g ; dW_u][i, n] = sum_m dGU[m, i] x[m, n]
  k5.A = dgu, k5.sam = 1, k5.sak = 2 * f;
  k5.B0 = x, k5.B1 = x, k5.sbn = 1, k5.sbk = d;
  k5.out0 = dwg, k5.out1 = dwu, k5.row_split = (int)f, k5.ld_out = d;
  if ((s = launch_simt<kSimtStore, false>(k5, st)) != SWF_OK) return s;
  SimtArgs k6 = simt_base(d, f, M);  // dW_d[i, n] = sum_m dY[m, i] h[m, n]
  k6.A = dy, k6.sam = 1, k6.sak = d;
  k6.B0 = h, k6.B1 = h, k6.sbn = 1, k6.sbk = f;
  k6.out0 = dwd, k6.ld_out = f;
  return launch_simt<kSimtStore, false>(k6, st);
}

}  // namespace swf

// ------------------------------------------------------------------ LeakyReLU(0.5)^2 MLP
// parameter-golf PR 1105, "Fused MLP Kernels":
//   U1  pre = x W_up^T, epilogue post = LeakyReLU(0.5)(pre)^2, act_grad    (K = d_model)
//   U2  y = post W_down^T                                                   (K = hidden)
//   U3  dpre = (dY W_down) * act_grad, the multiply in the epilogue         (K = d_model)
//   U4  dx = dpre W_up                                                      (K = hidden)
//   U5  dW_up = dpre^T x;  U6  dW_down = dY^T post                          (K = M)
namespace swf {

swf_status mlp2_fwd_bf16(const void* x, const void* wu, const void* wd, void* y, void* post,
                         void* act_grad, int64_t M, int64_t d, int64_t f, cudaStream_t st) {
  CUtensorMap tx, twu, tpost, twd;
  if (!encode_tmap_bf16(&tx, x, d, M, d, 64, 128) || !encode_tmap_bf16(&twu, wu, d, f, d, 64, 128) ||
      !encode_tmap_bf16(&tpost, post, f, M, f, 64, 128) || !encode_tmap_bf16(&twd, wd, f, d, f, 64, 128))
    return SWF_ERR_LAUNCH;
  // post and act_grad leave through TMA stores (K = d_model is short, the epilogue dominates)
  EpiMaps e1{};
  if (!epi_map(&e1.o[0], post, f, M, f, tma_epi_cols<kEpiLeakySq>()) ||
      !epi_map(&e1.o[1], act_grad, f, M, f, tma_epi_cols<kEpiLeakySq>()))
    return SWF_ERR_LAUNCH;
  TcGemmArgs u1 = base_args(M, f, 256, d, 2 * kTileM);
  swf_status s = launch_tc_pair<256, false, false, false, kEpiLeakySq, true>(SWF_K_MLP2_UP, tx, twu, twu, e1, u1, st);
  if (s != SWF_OK) return s;
  TcGemmArgs u2 = base_args(M, d, 256, f, 2 * kTileM);
  u2.out0 = y;
  u2.ld_out = d;
  return launch_tc_pair<256, false, false, false, kEpiStore>(SWF_K_DOWN, tpost, twd, twd, EpiMaps{}, u2, st);
}

swf_status mlp2_bwd_bf16(const void* dy, const void* x, const void* wu, const void* wd,
                         const void* post, const void* act_grad, void* dx, void* dwu, void* dwd,
                         void* dpre, float* part, int64_t M, int64_t d, int64_t f, cudaStream_t st) {
  swf_status s;
  {  // U3: dpost = dY W_down (B = W_down viewed [K=d rows, N=hidden cols]); * act_grad by TMA epilogue
    CUtensorMap tdy, twd;
    EpiMaps e{};
    if (!encode_tmap_bf16(&tdy, dy, d, M, d, 64, 128) || !encode_tmap_bf16(&twd, wd, f, d, f, 64, 64) ||
        !epi_map(&e.o[0], dpre, f, M, f, tma_epi_cols<kEpiScale>()) ||
        !epi_map(&e.o[2], act_grad, f, M, f, tma_epi_cols<kEpiScale>()))
      return SWF_ERR_LAUNCH;
    TcGemmArgs u3 = base_args(M, f, 256, d, 2 * kTileM);
    s = launch_tc_pair<256, false, true, false, kEpiScale, true>(SWF_K_MLP2_DPRE, tdy, twd, twd, e, u3, st);
    if (s != SWF_OK) return s;
  }
  {  // U4: dx = dpre W_up (B = W_up viewed [K=hidden rows, N=d cols], MN-major)
    CUtensorMap tdp, twu;
    if (!encode_tmap_bf16(&tdp, dpre, f, M, f, 64, 128) || !encode_tmap_bf16(&twu, wu, d, f, d, 64, 64))
      return SWF_ERR_LAUNCH;
    TcGemmArgs u4 = base_args(M, d, 256, f, 2 * kTileM);
    u4.out0 = dx;
    u4.ld_out = d;
    s = launch_tc_pair<256, false, true, false, kEpiStore>(SWF_K_MLP2_DX, tdp, twu, twu, EpiMaps{}, u4, st);
    if (s != SWF_OK) return s;
  }
  {  // U5: dW_up = dpre^T x (both MN-major)
    CUtensorMap tdp, tx;
    if (!encode_tmap_bf16(&tdp, dpre, f, M, f, 64, 64) || !encode_tmap_bf16(&tx, x, d, M, d, 64, 64))
      return SWF_ERR_LAUNCH;
    s = launch_dw(SWF_K_MLP2_DW_UP, tdp, tx, f, d, M, dwu, dwu, f, part, st);
    if (s != SWF_OK) return s;
  }
  {  // U6: dW_down = dY^T post
    CUtensorMap tdy, tpost;
    if (!encode_tmap_bf16(&tdy, dy, d, M, d, 64, 64) || !encode_tmap_bf16(&tpost, post, f, M, f, 64, 64))
      return SWF_ERR_LAUNCH;
    s = launch_dw(SWF_K_DW_DOWN, tdy, tpost, d, f, M, dwd, dwd, d, part, st);
  }
  return s;
}

swf_status mlp2_fwd_f32(const float* x, const float* wu, const float* wd, float* y, float* post,
                        float* act_grad, int64_t M, int64_t d, int64_t f, cudaStream_t st) {
  SimtArgs u1 = simt_base(M, f, d);
  u1.A = x, u1.sam = d, u1.sak = 1;
  u1.B0 = wu, u1.B1 = wu, u1.sbn = d, u1.sbk = 1;
  u1.out0 = post, u1.ld_out = f, u1.aux0 = act_grad, u1.ld_aux = f;
  swf_status s = launch_simt<kSimtLeakySq, false>(u1, st);
  if (s != SWF_OK) return s;
  SimtArgs u2 = simt_base(M, d, f);
  u2.A = post, u2.sam = f, u2.sak = 1;
  u2.B0 = wd, u2.B1 = wd, u2.sbn = f, u2.sbk = 1;
  u2.out0 = y, u2.ld_out = d;
  return launch_simt<kSimtStore, false>(u2, st);
}

swf_status mlp2_bwd_f32(const float* dy, const float* x, const float* wu, const float* wd,
                        const float* post, const float* act_grad, float* dx, float* dwu,
                        float* dwd, float* dpre, int64_t M, int64_t d, int64_t f, cudaStream_t st) {
  SimtArgs u3 = simt_base(M, f, d);  // dpre[m, n] = sum_k dY[m, k] W_d[k, n] * act_grad[m, n]
  u3.A = dy, u3.sam = d, u3.sak = 1;
  u3.B0 = wd, u3.B1 = wd, u3.sbn = 1, u3.sbk = f;
  u3.out0 = dpre, u3.ld_out = f, u3.aux0 = const_cast<float*>(act_grad), u3.ld_aux = f;
  swf_status s = launch_simt<kSimtScale, false>(u3, st);
  if (s != SWF_OK) return s;
  SimtArgs u4 = simt_base(M, d, f);  // dx[m, n] = sum_k dpre[m, k] W_u[k, n]
  u4.A = dpre, u4.sam = f, u4.sak = 1;
  u4.B0 = wu, u4.B1 = wu, u4.sbn = 1, u4.sbk = d;
  u4.out0 = dx, u4.ld_out = d;
  if ((s = launch_simt<kSimtStore, false>(u4, st)) != SWF_OK) return s;
  SimtArgs u5 = simt_base(f, d, M);  // dW_u[i, n] = sum_m dpre[m, i] x[m, n]
  u5.A = dpre, u5.sam = 1, u5.sak = f;
  u5.B0 = x, u5.B1 = x, u5.sbn = 1, u5.sbk = d;
  u5.out0 = dwu, u5.ld_out = d;
  if ((s = launch_simt<kSimtStore, false>(u5, st)) != SWF_OK) return s;
  SimtArgs u6 = simt_base(d, f, M);  // dW_d[i, n] = sum_m dY[m, i] post[m, n]
  u6.A = dy, u6.sam = 1, u6.sak = d;
  u6.B0 = post, u6.B1 = post, u6.sbn = 1, u6.sbk = f;
  u6.out0 = dwd, u6.ld_out = f;
  return launch_simt<kSimtStore, false>(u6, st);
}

}  // namespace swf
