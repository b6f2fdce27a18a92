// Inference forward that allocates nothing and needs no caller workspace.
//
// Some callers cannot hand the library a workspace: a host program that reaches the library
// only through the C ABI and owns no device allocator of its own, or a plug-in inside a runtime
// that forbids device allocation on its execution path.  For them this entry point keeps the
// intermediate h = SiLU(x W_gate^T) * (x W_up^T) in a fixed, file-scope device array instead.
// Its first call on a device looks up the array's device address with that device current;
// make that first call before any stream capture on the device.
//
// The array lives in every GPU that loads the library, until the process exits.  All calls
// share it and it keeps the last call's contents; nothing in it needs to start at zero (the
// gate|up kernel writes every element of h that the down projection reads, and rows past M are
// outside the tensor map, so the hardware reads them as zero).  Two calls whose kernels overlap
// on the GPU (different streams, or different host threads on the same device) race on it.
#include <mutex>

#include "swf_internal.h"

namespace {

// The scratch h: [M, d_ff] in the call's dtype, at most SWF_NOALLOC_SCRATCH_BYTES.
static __device__ __align__(256) unsigned char g_noalloc_scratch[SWF_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array for the current device.  In host code the array's name
// is only a host-side stand-in, so the address comes from cudaGetSymbolAddress, once per
// device, with that device current.
swf_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SWF_ERR_LAUNCH;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return SWF_ERR_LAUNCH;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return SWF_OK;
}

}  // namespace

extern "C" swf_status swiglu_ffn_fwd_infer_noalloc(const void* x, const void* w_gate,
                                                   const void* w_up, const void* w_down, void* y,
                                                   int64_t M, int64_t d_model, int64_t d_ff,
                                                   swf_dtype dtype, void* stream) {
  if (!x || !w_gate || !w_up || !w_down || !y) return SWF_ERR_INVALID_ARG;
  const swf_status ok = swf_supported(SWF_OP_FWD_INFER, M, d_model, d_ff, 0, 0, 0, dtype);
  if (ok != SWF_OK) return ok;
  for (const void* p : {x, w_gate, w_up, w_down, static_cast<const void*>(y)})
    if (!swf::aligned16(p)) return SWF_ERR_ALIGNMENT;
  const size_t esz = dtype == SWF_BF16 ? 2 : 4;
  if ((uint64_t)M * (uint64_t)d_ff * esz > (uint64_t)SWF_NOALLOC_SCRATCH_BYTES)
    return SWF_ERR_WORKSPACE;
  void* h = nullptr;
  const swf_status s = scratch_address(&h);
  if (s != SWF_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == SWF_BF16)
    return swf::dense_fwd_bf16(x, w_gate, w_up, w_down, y, h, nullptr, nullptr, M, d_model, d_ff,
                               true, st);
  return swf::dense_fwd_f32(static_cast<const float*>(x), static_cast<const float*>(w_gate),
                            static_cast<const float*>(w_up), static_cast<const float*>(w_down),
                            static_cast<float*>(y), static_cast<float*>(h), nullptr, nullptr, M,
                            d_model, d_ff, true, st);
}
