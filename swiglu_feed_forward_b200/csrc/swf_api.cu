// C ABI of the SwiGLU FFN library: argument validation, workspace sizing, planning, and
// dispatch to the bf16 tensor-core or fp32 CUDA-core launchers.  Nothing here allocates
// device memory or synchronises, except swf_device_status (documented).
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "swf_internal.h"
#include "swf_ptx.cuh"
#include "swf_sparse.h"

// Per-device status word: kernels whose bounded waits run out write SWF_ERR_TIMEOUT here.
__device__ int g_swf_status_word;

namespace swf {

namespace {

constexpr int kMaxDevices = 64;
struct CtxCache {
  bool ready = false;
  DevCtx ctx{};
};
CtxCache g_ctx[kMaxDevices];
std::mutex g_ctx_mu;

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

void load_encode() {
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
}

}  // namespace

swf_status get_ctx(DevCtx* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SWF_ERR_LAUNCH;
  std::lock_guard<std::mutex> lock(g_ctx_mu);
  CtxCache& c = g_ctx[dev];
  if (!c.ready) {
    DevCtx ctx{};
    ctx.device = dev;
    if (cudaDeviceGetAttribute(&ctx.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return SWF_ERR_LAUNCH;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_swf_status_word) != cudaSuccess) return SWF_ERR_LAUNCH;
    ctx.status = static_cast<int*>(p);
    c.ctx = ctx;
    c.ready = true;
  }
  *out = c.ctx;
  return SWF_OK;
}

bool encode_tmap_bf16(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows,
                      uint64_t row_elems, uint32_t box_cols, uint32_t box_rows, int swizzle_bytes) {
  std::call_once(g_encode_once, load_encode);
  if (!g_encode) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {row_elems * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle_bytes == 32   ? CU_TENSOR_MAP_SWIZZLE_32B
                  : swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                        : CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ------------------------------------------------------------------ validation
namespace {

inline size_t esize(swf_dtype dt) { return dt == SWF_BF16 ? 2 : 4; }

swf_status check_dense(int64_t M, int64_t d, int64_t f, swf_dtype dt) {
  if (dt != SWF_BF16 && dt != SWF_F32) return SWF_ERR_INVALID_ARG;
  if (M <= 0 || d <= 0 || f <= 0) return SWF_ERR_INVALID_ARG;
  if (M > INT32_MAX / 2 || d > (1 << 20) || f > (1 << 20)) return SWF_ERR_UNSUPPORTED;
  if (dt == SWF_BF16 && (d % 16 != 0 || f % 16 != 0)) return SWF_ERR_UNSUPPORTED;
  return SWF_OK;
}

bool all_aligned(std::initializer_list<const void*> ps) {
  for (const void* p : ps)
    if (!aligned16(p)) return false;
  return true;
}
bool any_null(std::initializer_list<const void*> ps) {
  for (const void* p : ps)
    if (p == nullptr) return true;
  return false;
}

}  // namespace

swf_status check_sparse_shape(int64_t M, int64_t d, int64_t f, int32_t G, int32_t K, swf_dtype dt) {
  swf_status s = check_dense(M, d, f, dt);
  if (s != SWF_OK) return s;
  if (G <= 0 || K <= 0) return SWF_ERR_INVALID_ARG;
  if (dt != SWF_BF16) return SWF_ERR_UNSUPPORTED;
  if (G < 16 || G > 64 || (G & (G - 1)) != 0) return SWF_ERR_UNSUPPORTED;
  if (f % G != 0 || f / G < 2) return SWF_ERR_UNSUPPORTED;
  if (K > f / G) return SWF_ERR_UNSUPPORTED;
  if (M * (int64_t)K >= (int64_t(1) << 31)) return SWF_ERR_UNSUPPORTED;
  return SWF_OK;
}

}  // namespace swf

using namespace swf;

// ------------------------------------------------------------------ queries
extern "C" const char* swf_status_string(swf_status s) {
  switch (s) {
    case SWF_OK: return "SWF_OK";
    case SWF_ERR_INVALID_ARG: return "SWF_ERR_INVALID_ARG: null pointer, non-positive size or bad enum";
    case SWF_ERR_UNSUPPORTED: return "SWF_ERR_UNSUPPORTED: shape or dtype outside the supported rules";
    case SWF_ERR_ALIGNMENT: return "SWF_ERR_ALIGNMENT: pointer not 16-byte aligned";
    case SWF_ERR_WORKSPACE: return "SWF_ERR_WORKSPACE: workspace or saved buffer too small";
    case SWF_ERR_LAUNCH: return "SWF_ERR_LAUNCH: the CUDA runtime refused a launch or query";
    case SWF_ERR_TIMEOUT: return "SWF_ERR_TIMEOUT: a bounded in-kernel wait ran out";
  }
  return "unknown swf_status";
}

extern "C" swf_status swf_supported(swf_op op, int64_t M, int64_t d, int64_t f, int32_t G,
                                    int32_t K, int32_t spg, swf_dtype dt) {
  switch (op) {
    case SWF_OP_FWD:
    case SWF_OP_FWD_INFER:
    case SWF_OP_BWD:
      return check_dense(M, d, f, dt);
    case SWF_OP_SELECT: {
      swf_status s = check_sparse_shape(M, d, f, G, K, dt);
      if (s != SWF_OK) return s;
      if (spg < 0 || spg > G) return SWF_ERR_UNSUPPORTED;
      return SWF_OK;
    }
    case SWF_OP_SPARSE_FWD:
    case SWF_OP_SPARSE_BWD:
      return check_sparse_shape(M, d, f, G, K, dt);
    case SWF_OP_MLP2_FWD:
    case SWF_OP_MLP2_BWD:
      return check_dense(M, d, f, dt);
    case SWF_OP_BUCKETS:
      if (M <= 0 || K <= 0 || G <= 0) return SWF_ERR_INVALID_ARG;
      if (K > G || M * (int64_t)K >= (int64_t(1) << 31)) return SWF_ERR_UNSUPPORTED;
      return SWF_OK;
  }
  return SWF_ERR_INVALID_ARG;
}

extern "C" size_t swf_workspace_bytes(swf_op op, int64_t M, int64_t d, int64_t f, int32_t G,
                                      int32_t K, swf_dtype dt) {
  const int32_t spg_probe = G > 0 ? 1 : 0;
  if (swf_supported(op, M, d, f, G, K, spg_probe, dt) != SWF_OK) return 0;
  switch (op) {
    case SWF_OP_FWD: return 0;
    case SWF_OP_FWD_INFER: return round_up((size_t)M * f * esize(dt), 256);
    case SWF_OP_BWD:  // [dG | dU], then the split-K partial planes of the weight gradients
      return round_up((size_t)M * 2 * f * esize(dt), 256) +
             (dt == SWF_BF16 ? round_up((size_t)dense_bwd_part_elems(M, d, f) * 4, 256) : 0);
    case SWF_OP_SELECT: return select_workspace_bytes(M, d, f, G, K);
    case SWF_OP_SPARSE_FWD: return sparse_fwd_workspace_bytes(M, d, f, G, K);
    case SWF_OP_SPARSE_BWD: return sparse_bwd_workspace_bytes(M, d, f, G, K);
    case SWF_OP_BUCKETS: return buckets_workspace_bytes(M, K, G);
    case SWF_OP_MLP2_FWD: return 0;
    case SWF_OP_MLP2_BWD:  // dpre, then the split-K partial planes
      return round_up((size_t)M * f * esize(dt), 256) +
             (dt == SWF_BF16 ? round_up((size_t)mlp2_bwd_part_elems(M, d, f) * 4, 256) : 0);
  }
  return 0;
}

extern "C" size_t swf_sparse_saved_bytes(int64_t M, int64_t d, int64_t f, int32_t G, int32_t K,
                                         swf_dtype dt) {
  if (check_sparse_shape(M, d, f, G, K, dt) != SWF_OK) return 0;
  return sparse_saved_bytes(M, d, f, G, K);
}

extern "C" swf_status swf_plan(swf_op op, int64_t M, int64_t d, int64_t f, int32_t G, int32_t K,
                               int32_t spg, swf_dtype dt, swf_plan_info* out) {
  if (!out) return SWF_ERR_INVALID_ARG;
  swf_status s = swf_supported(op, M, d, f, G, K, spg, dt);
  if (s != SWF_OK) return s;
  swf_plan_info p{};
  p.path = dt == SWF_BF16 ? 1 : 0;
  p.tile_m = dt == SWF_BF16 ? 128 : 64;
  p.tile_n = dt == SWF_BF16 ? 256 : 64;
  p.tile_k = dt == SWF_BF16 ? 64 : 16;
  p.stages = dt == SWF_BF16 ? 4 : 1;
  p.grid = 148;
  p.deterministic = 1;
  p.workspace_bytes = swf_workspace_bytes(op, M, d, f, G, K, dt);
  switch (op) {
    case SWF_OP_FWD:
    case SWF_OP_FWD_INFER:
      p.num_kernels = 2;
      p.flops = 6 * M * d * f;
      p.gemm_tiles = dense_gemm_tiles(op, M, d, f);
      break;
    case SWF_OP_BWD:
      p.num_kernels = 4;
      p.flops = 12 * M * d * f;
      p.gemm_tiles = dense_gemm_tiles(op, M, d, f);
      break;
    case SWF_OP_MLP2_FWD:
      p.num_kernels = 2;
      p.flops = 4 * M * d * f;
      break;
    case SWF_OP_MLP2_BWD:
      p.num_kernels = 4;
      p.flops = 8 * M * d * f;
      break;
    default:
      sparse_plan(op, M, d, f, G, K, spg, &p);
      break;
  }
  *out = p;
  return SWF_OK;
}

// ------------------------------------------------------------------ dense entry points
extern "C" swf_status swiglu_ffn_fwd(const void* x, const void* w_gate, const void* w_up,
                                     const void* w_down, void* y, void* saved_h, void* saved_a,
                                     void* saved_b, int64_t M, int64_t d, int64_t f,
                                     swf_dtype dt, void* stream) {
  if (any_null({x, w_gate, w_up, w_down, y, saved_h, saved_a, saved_b})) return SWF_ERR_INVALID_ARG;
  swf_status s = check_dense(M, d, f, dt);
  if (s != SWF_OK) return s;
  if (!all_aligned({x, w_gate, w_up, w_down, y, saved_h, saved_a, saved_b})) return SWF_ERR_ALIGNMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dt == SWF_BF16)
    return dense_fwd_bf16(x, w_gate, w_up, w_down, y, saved_h, saved_a, saved_b, M, d, f, false, st);
  return dense_fwd_f32((const float*)x, (const float*)w_gate, (const float*)w_up, (const float*)w_down,
                       (float*)y, (float*)saved_h, (float*)saved_a, (float*)saved_b, M, d, f, false, st);
}

extern "C" swf_status swiglu_ffn_fwd_infer(const void* x, const void* w_gate, const void* w_up,
                                           const void* w_down, void* y, void* workspace,
                                           size_t ws_bytes, int64_t M, int64_t d, int64_t f,
                                           swf_dtype dt, void* stream) {
  if (any_null({x, w_gate, w_up, w_down, y, workspace})) return SWF_ERR_INVALID_ARG;
  swf_status s = check_dense(M, d, f, dt);
  if (s != SWF_OK) return s;
  if (!all_aligned({x, w_gate, w_up, w_down, y, workspace})) return SWF_ERR_ALIGNMENT;
  if (ws_bytes < swf_workspace_bytes(SWF_OP_FWD_INFER, M, d, f, 0, 0, dt)) return SWF_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dt == SWF_BF16)
    return dense_fwd_bf16(x, w_gate, w_up, w_down, y, workspace, nullptr, nullptr, M, d, f, true, st);
  return dense_fwd_f32((const float*)x, (const float*)w_gate, (const float*)w_up, (const float*)w_down,
                       (float*)y, (float*)workspace, nullptr, nullptr, M, d, f, true, st);
}

extern "C" swf_status swiglu_ffn_bwd(const void* dy, const void* x, const void* w_gate,
                                     const void* w_up, const void* w_down, const void* saved_h,
                                     const void* saved_a, const void* saved_b, void* dx,
                                     void* dw_gate, void* dw_up, void* dw_down, void* workspace,
                                     size_t ws_bytes, int64_t M, int64_t d, int64_t f,
                                     swf_dtype dt, void* stream) {
  if (any_null({dy, x, w_gate, w_up, w_down, saved_h, saved_a, saved_b, dx, dw_gate, dw_up, dw_down,
                workspace}))
    return SWF_ERR_INVALID_ARG;
  swf_status s = check_dense(M, d, f, dt);
  if (s != SWF_OK) return s;
  if (!all_aligned({dy, x, w_gate, w_up, w_down, saved_h, saved_a, saved_b, dx, dw_gate, dw_up,
                    dw_down, workspace}))
    return SWF_ERR_ALIGNMENT;
  if (ws_bytes < swf_workspace_bytes(SWF_OP_BWD, M, d, f, 0, 0, dt)) return SWF_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dt == SWF_BF16)
    return dense_bwd_bf16(dy, x, w_gate, w_up, w_down, saved_h, saved_a, saved_b, dx, dw_gate, dw_up,
                          dw_down, workspace,
                          reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                                   round_up((size_t)M * 2 * f * 2, 256)),
                          M, d, f, st);
  return dense_bwd_f32((const float*)dy, (const float*)x, (const float*)w_gate, (const float*)w_up,
                       (const float*)w_down, (const float*)saved_h, (const float*)saved_a,
                       (const float*)saved_b, (float*)dx, (float*)dw_gate, (float*)dw_up,
                       (float*)dw_down, (float*)workspace, M, d, f, st);
}

// ------------------------------------------------------------------ LeakyReLU(0.5)^2 MLP
extern "C" swf_status leaky_relu_sq_mlp_fwd(const void* x, const void* w_up, const void* w_down,
                                            void* y, void* post, void* act_grad, int64_t M,
                                            int64_t d, int64_t f, swf_dtype dt, void* stream) {
  if (any_null({x, w_up, w_down, y, post, act_grad})) return SWF_ERR_INVALID_ARG;
  swf_status s = check_dense(M, d, f, dt);
  if (s != SWF_OK) return s;
  if (!all_aligned({x, w_up, w_down, y, post, act_grad})) return SWF_ERR_ALIGNMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dt == SWF_BF16) return mlp2_fwd_bf16(x, w_up, w_down, y, post, act_grad, M, d, f, st);
  return mlp2_fwd_f32((const float*)x, (const float*)w_up, (const float*)w_down, (float*)y,
                      (float*)post, (float*)act_grad, M, d, f, st);
}

extern "C" swf_status leaky_relu_sq_mlp_bwd(const void* dy, const void* x, const void* w_up,
                                            const void* w_down, const void* post,
                                            const void* act_grad, void* dx, void* dw_up,
                                            void* dw_down, void* workspace, size_t ws_bytes,
                                            int64_t M, int64_t d, int64_t f, swf_dtype dt,
                                            void* stream) {
  if (any_null({dy, x, w_up, w_down, post, act_grad, dx, dw_up, dw_down, workspace}))
    return SWF_ERR_INVALID_ARG;
  swf_status s = check_dense(M, d, f, dt);
  if (s != SWF_OK) return s;
  if (!all_aligned({dy, x, w_up, w_down, post, act_grad, dx, dw_up, dw_down, workspace}))
    return SWF_ERR_ALIGNMENT;
  if (ws_bytes < swf_workspace_bytes(SWF_OP_MLP2_BWD, M, d, f, 0, 0, dt)) return SWF_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dt == SWF_BF16)
    return mlp2_bwd_bf16(dy, x, w_up, w_down, post, act_grad, dx, dw_up, dw_down, workspace,
                         reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                                  round_up((size_t)M * f * 2, 256)),
                         M, d, f, st);
  return mlp2_bwd_f32((const float*)dy, (const float*)x, (const float*)w_up, (const float*)w_down,
                      (const float*)post, (const float*)act_grad, (float*)dx, (float*)dw_up,
                      (float*)dw_down, (float*)workspace, M, d, f, st);
}

// ------------------------------------------------------------------ status and self test
extern "C" swf_status swf_device_status(void* stream) {
  DevCtx ctx;
  swf_status s = get_ctx(&ctx);
  if (s != SWF_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return SWF_ERR_LAUNCH;
  int word = 0;
  if (cudaMemcpyFromSymbol(&word, g_swf_status_word, sizeof(int)) != cudaSuccess) return SWF_ERR_LAUNCH;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_swf_status_word, &zero, sizeof(int)) != cudaSuccess) return SWF_ERR_LAUNCH;
  return word == 0 ? SWF_OK : static_cast<swf_status>(word);
}

namespace swf {
// Waits on a barrier that nothing ever completes; the bounded wait runs out, records the
// timeout and the kernel returns.
__global__ void selftest_wait_kernel(int* status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    WaitCtl ctl{&abort_flag, status, limit_ns};
    mbar_wait(&bar, 0, ctl);
  }
  __syncthreads();
}
}  // namespace swf

extern "C" swf_status swf_selftest_wait_timeout(int32_t limit_us, void* stream) {
  if (limit_us < 1 || limit_us > 1000000) return SWF_ERR_INVALID_ARG;
  DevCtx ctx;
  swf_status s = get_ctx(&ctx);
  if (s != SWF_OK) return s;
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(ctx.status,
                                                                       (uint64_t)limit_us * 1000ull);
  return cudaGetLastError() == cudaSuccess ? SWF_OK : SWF_ERR_LAUNCH;
}
