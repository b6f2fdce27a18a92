// Host-side internals shared by the library's translation units.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

#include "../../include/swiglu_ffn.h"

namespace swf {

struct DevCtx {
  int device;
  int num_sms;
  int* status;  // device address of the status word
};

// Current device's context (SM count, status word address); cached per device.
swf_status get_ctx(DevCtx* out);

// 2-D bf16 tensor map with 128-byte (or 64- or 32-byte) swizzle over a row-major matrix of
// `rows` x `cols` elements whose rows are `row_elems` apart; box of box_cols x box_rows.
// Out-of-range elements of a box read as zero.
bool encode_tmap_bf16(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows,
                      uint64_t row_elems, uint32_t box_cols, uint32_t box_rows,
                      int swizzle_bytes = 128);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Brackets one kernel launch with CUDA events while profiling is enabled (swf_profile_*).
class ProfScope {
 public:
  ProfScope(int kind, cudaStream_t st);
  ~ProfScope();
 private:
  int kind_;
  cudaStream_t st_;
  cudaEvent_t ev0_ = nullptr;
};

// Default bound on a single in-kernel wait (ns).
constexpr uint64_t kDefaultWaitNs = 2000000000ull;

// ---- dense path (swf_dense.cu) ----
swf_status dense_fwd_bf16(const void* x, const void* wg, const void* wu, const void* wd, void* y,
                          void* h, void* a, void* b, int64_t M, int64_t d, int64_t f, bool infer,
                          cudaStream_t st);
swf_status dense_bwd_bf16(const void* dy, const void* x, const void* wg, const void* wu,
                          const void* wd, const void* h, const void* a, const void* b, void* dx,
                          void* dwg, void* dwu, void* dwd, void* dgu, float* part, int64_t M,
                          int64_t d, int64_t f, cudaStream_t st);
swf_status dense_fwd_f32(const float* x, const float* wg, const float* wu, const float* wd,
                         float* y, float* h, float* a, float* b, int64_t M, int64_t d, int64_t f,
                         bool infer, cudaStream_t st);
swf_status dense_bwd_f32(const float* dy, const float* x, const float* wg, const float* wu,
                         const float* wd, const float* h, const float* a, const float* b,
                         float* dx, float* dwg, float* dwu, float* dwd, float* dgu, int64_t M,
                         int64_t d, int64_t f, cudaStream_t st);

// ---- LeakyReLU(0.5)^2 MLP (swf_dense.cu) ----
swf_status mlp2_fwd_bf16(const void* x, const void* wu, const void* wd, void* y, void* post,
                         void* act_grad, int64_t M, int64_t d, int64_t f, cudaStream_t st);
swf_status mlp2_bwd_bf16(const void* dy, const void* x, const void* wu, const void* wd,
                         const void* post, const void* act_grad, void* dx, void* dwu, void* dwd,
                         void* dpre, float* part, int64_t M, int64_t d, int64_t f, cudaStream_t st);
swf_status mlp2_fwd_f32(const float* x, const float* wu, const float* wd, float* y, float* post,
                        float* act_grad, int64_t M, int64_t d, int64_t f, cudaStream_t st);
swf_status mlp2_bwd_f32(const float* dy, const float* x, const float* wu, const float* wd,
                        const float* post, const float* act_grad, float* dx, float* dwu,
                        float* dwd, float* dpre, int64_t M, int64_t d, int64_t f, cudaStream_t st);

// Weight-gradient GEMM out = A^T B of rows x cols over K (tokens), both operands MN-major (maps
// with 64 x 64 boxes), as pair tiles of 256 x 256; split-K into `part` (part_elems(...) fp32) and
// a fixed-order reduction when the planner finds too few tiles (of the whole GEMM, or of its last
// partial wave only).  Rows >= row_split go to out1.
swf_status launch_dw(int kind, const CUtensorMap& ta, const CUtensorMap& tb, int64_t rows,
                     int64_t cols, int64_t K, void* out0, void* out1, int64_t row_split,
                     float* part, cudaStream_t st);
int64_t part_elems(int64_t rows, int64_t cols, int64_t K);

// fp32 elements of the split-K partial planes the bf16 backward passes need (0: no split).
int64_t dense_bwd_part_elems(int64_t M, int64_t d, int64_t f);
int64_t mlp2_bwd_part_elems(int64_t M, int64_t d, int64_t f);

// Tile count and launch shape of the dense bf16 GEMMs (for swf_plan).
int64_t dense_gemm_tiles(int op, int64_t M, int64_t d, int64_t f);

}  // namespace swf
