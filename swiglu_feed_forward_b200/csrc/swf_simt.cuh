// fp32 GEMM on the CUDA cores (FFMA) with the same fused epilogues as the tensor-core path.
// Used when the caller's tensors are fp32: tf32 tensor-core inputs keep 10 mantissa bits,
// about 1e-3 relative, while fp32 results are expected to 1e-4.
//
//   C[m, n] = sum_k A(m, k) * B(n, k),   A(m, k) = A[m*sam + k*sak],
//   B(n, k) = B0[n*sbn + k*sbk] for k < k_split, else B1[n*sbn + (k - k_split)*sbk]
//   (kDual: a second accumulator C1 = sum_k A(m,k) * B1(n,k) over all k, for gate|up)
#pragma once
#include <cstdint>

namespace swf {

enum : int {
  kSimtStore = 0,
  kSimtSwiGLU = 1,
  kSimtSwiGLUInf = 2,
  kSimtDGate = 3,
  kSimtLeakySq = 4,  // out0 = LeakyReLU(0.5)(C)^2, aux0 = its derivative (2 C or 0.5 C)
  kSimtScale = 5     // out0 = C * aux0
};

struct SimtArgs {
  int M, N, K;
  const float* A;
  int64_t sam, sak;
  const float* B0;
  const float* B1;
  int64_t sbn, sbk;
  int k_split;
  float* out0;
  float* out1;
  int64_t ld_out;
  int row_split;
  float* aux0;  // SwiGLU: saved_a out; DGate: saved_a in
  float* aux1;  // SwiGLU: saved_b out; DGate: saved_b in
  int64_t ld_aux;
  int d_ff;     // DGate: column offset of dU
};

constexpr int kSimtTile = 64;
constexpr int kSimtKT = 16;

template <int EPI, bool DUAL>
__global__ void __launch_bounds__(256) simt_gemm_f32(const SimtArgs a) {
  __shared__ float As[kSimtKT][kSimtTile + 4];
  __shared__ float Bs[kSimtKT][kSimtTile + 4];
  __shared__ float Cs[DUAL ? kSimtKT : 1][kSimtTile + 4];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int m0 = blockIdx.y * kSimtTile, n0 = blockIdx.x * kSimtTile;
  float acc[4][4] = {}, acc1[4][4] = {};
  for (int k0 = 0; k0 < a.K; k0 += kSimtKT) {
    for (int i = threadIdx.x; i < kSimtKT * kSimtTile; i += 256) {
      const int kk = i / kSimtTile, r = i % kSimtTile;
      const int k = k0 + kk;
      const int m = m0 + r, n = n0 + r;
      As[kk][r] = (m < a.M && k < a.K) ? a.A[m * a.sam + k * a.sak] : 0.f;
      float b = 0.f, b1 = 0.f;
      if (n < a.N && k < a.K) {
        if (DUAL) {
          b = a.B0[n * a.sbn + k * a.sbk];
          b1 = a.B1[n * a.sbn + k * a.sbk];
        } else {
          b = k < a.k_split ? a.B0[n * a.sbn + k * a.sbk]
                            : a.B1[n * a.sbn + (int64_t)(k - a.k_split) * a.sbk];
        }
      }
      Bs[kk][r] = b;
      if (DUAL) Cs[kk][r] = b1;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kSimtKT; ++kk) {
      float av[4], bv[4], cv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        av[i] = As[kk][ty * 4 + i];
        bv[i] = Bs[kk][tx * 4 + i];
        if (DUAL) cv[i] = Cs[kk][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
          if (DUAL) acc1[i][j] = fmaf(av[i], cv[j], acc1[i][j]);
        }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= a.M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n >= a.N) continue;
      const float c = acc[i][j];
      if constexpr (EPI == kSimtStore) {
        if (m < a.row_split) a.out0[m * a.ld_out + n] = c;
        else a.out1[(int64_t)(m - a.row_split) * a.ld_out + n] = c;
      } else if constexpr (EPI == kSimtSwiGLU || EPI == kSimtSwiGLUInf) {
        const float g = c, u = acc1[i][j];
        const float s = 1.0f / (1.0f + expf(-g));
        a.out0[m * a.ld_out + n] = g * s * u;
        if constexpr (EPI == kSimtSwiGLU) {
          a.aux0[m * a.ld_aux + n] = u * s * (1.0f + g * (1.0f - s));
          a.aux1[m * a.ld_aux + n] = g * s;
        }
      } else if constexpr (EPI == kSimtLeakySq) {
        const float lk = c > 0.f ? c : 0.5f * c;
        a.out0[m * a.ld_out + n] = lk * lk;
        a.aux0[m * a.ld_aux + n] = c > 0.f ? 2.f * c : 0.5f * c;
      } else if constexpr (EPI == kSimtScale) {
        a.out0[m * a.ld_out + n] = c * a.aux0[m * a.ld_aux + n];
      } else if constexpr (EPI == kSimtDGate) {
        a.out0[m * a.ld_out + n] = c * a.aux0[m * a.ld_aux + n];
        a.out0[m * a.ld_out + a.d_ff + n] = c * a.aux1[m * a.ld_aux + n];
      }
    }
  }
}

}  // namespace swf
