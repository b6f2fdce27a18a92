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
#include "swf_internal.h"
#include "swf_launch.cuh"
#include "swf_simt.cuh"

namespace swf {

namespace {
// 32 x 32 box with 64-byte swizzle: the staging box of the TMA epilogue.
bool epi_map(CUtensorMap* m, const void* base, int64_t cols, int64_t rows, int64_t row_elems) {
  return encode_tmap_bf16(m, base, cols, rows, row_elems, 32, 32, 64);
}
}  // namespace

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
  swf_status s =
      infer ? launch_tc_pair<256, false, false, true, kEpiSwiGLUInf>(SWF_K_GATE_UP_INFER, tx, twg, twu, EpiMaps{}, k1, st)
            : launch_tc_pair<256, false, false, true, kEpiSwiGLU>(SWF_K_GATE_UP, tx, twg, twu, EpiMaps{}, k1, st);
  if (s != SWF_OK) return s;
  // K2: y = h W_d^T
  TcGemmArgs k2 = base_args(M, d, 256, f, 2 * kTileM);
  k2.out0 = y;
  k2.ld_out = d;
  return launch_tc_pair<256, false, false, false, kEpiStore>(SWF_K_DOWN, th, twd, twd, EpiMaps{}, k2, st);
}

swf_status dense_bwd_bf16(const void* dy, const void* x, const void* wg, const void* wu,
                          const void* wd, const void* h, const void* a, const void* b, void* dx,
                          void* dwg, void* dwu, void* dwd, void* dgu, int64_t M, int64_t d,
                          int64_t f, cudaStream_t st) {
  swf_status s;
  {  // K3: dH = dY W_d (B = W_d viewed [K=d rows, N=f cols], MN-major), epilogue * a, * b
    CUtensorMap tdy, twd;
    if (!encode_tmap_bf16(&tdy, dy, d, M, d, 64, 128) || !encode_tmap_bf16(&twd, wd, f, d, f, 64, 64))
      return SWF_ERR_LAUNCH;
    // TMA epilogue (measured: 1.05 -> 0.67 ms at 32768 x 2048 x 5504): a and b come in by TMA,
    // dG and dU leave by TMA through two views of dGU (each [M, f], rows 2f apart)
    EpiMaps e3{};
    const __nv_bfloat16* dgu_b = static_cast<const __nv_bfloat16*>(dgu);
    if (!epi_map(&e3.o[0], dgu_b, f, M, 2 * f) || !epi_map(&e3.o[1], dgu_b + f, f, M, 2 * f) ||
        !epi_map(&e3.o[2], a, f, M, f) || !epi_map(&e3.o[3], b, f, M, f))
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
    TcGemmArgs k5 = base_args(2 * f, d, 256, M, 2 * kTileM);
    k5.out0 = dwg;
    k5.out1 = dwu;
    k5.row_split = (int)f;
    k5.ld_out = d;
    s = launch_tc_pair<256, true, true, false, kEpiStore>(SWF_K_DW_GATE_UP, tdgu, tx, tx, EpiMaps{}, k5, st);
    if (s != SWF_OK) return s;
  }
  {  // K6: dW_d = dY^T h: A = dY viewed [K=M rows, d cols] (MN), B = h [K=M rows, f cols] (MN)
    CUtensorMap tdy, th;
    if (!encode_tmap_bf16(&tdy, dy, d, M, d, 64, 64) || !encode_tmap_bf16(&th, h, f, M, f, 64, 64))
      return SWF_ERR_LAUNCH;
    TcGemmArgs k6 = base_args(d, f, 256, M, 2 * kTileM);
    k6.out0 = dwd;
    k6.ld_out = f;
    s = launch_tc_pair<256, true, true, false, kEpiStore>(SWF_K_DW_DOWN, tdy, th, th, EpiMaps{}, k6, st);
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
