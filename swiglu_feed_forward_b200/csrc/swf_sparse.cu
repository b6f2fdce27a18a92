// Group-sparse SwiGLU FFN (eugen_sparse README): subsample index, grouped top-k selection,
// group bucketing, sparse forward and backward.
#include <vector>

#include "swf_sparse.h"

namespace swf {

size_t select_workspace_bytes(int64_t, int64_t, int64_t, int32_t, int32_t) { return 0; }
size_t sparse_fwd_workspace_bytes(int64_t, int64_t, int64_t, int32_t, int32_t) { return 0; }
size_t sparse_bwd_workspace_bytes(int64_t, int64_t, int64_t, int32_t, int32_t) { return 0; }
size_t buckets_workspace_bytes(int64_t, int32_t, int32_t) { return 0; }
size_t sparse_saved_bytes(int64_t, int64_t, int64_t, int32_t, int32_t) { return 0; }
void sparse_plan(int, int64_t, int64_t, int64_t, int32_t, int32_t, int32_t, swf_plan_info* p) {
  p->num_kernels = 0;
}

}  // namespace swf

using namespace swf;

// splitmix64 (Steele, Lea & Flood, OOPSLA 2014): one output per call.
static inline uint64_t splitmix64_next(uint64_t& state) {
  state += 0x9E3779B97F4A7C15ull;
  uint64_t z = state;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

extern "C" swf_status swf_make_subsample_index(int64_t d_ff, int32_t G, int32_t spg, uint64_t seed,
                                               int32_t* out) {
  if (!out || d_ff <= 0 || G <= 0 || spg <= 0) return SWF_ERR_INVALID_ARG;
  if (d_ff % G != 0 || spg > G || d_ff / G < 1 || d_ff > INT32_MAX) return SWF_ERR_UNSUPPORTED;
  const int64_t ng = d_ff / G;
  uint64_t state = seed;
  std::vector<int32_t> perm((size_t)G);
  for (int64_t c = 0; c < ng; ++c) {
    for (int32_t i = 0; i < G; ++i) perm[i] = i;
    for (int32_t i = 0; i < spg; ++i) {
      const uint64_t r = splitmix64_next(state);
      const int32_t j = i + (int32_t)(r % (uint64_t)(G - i));
      const int32_t t = perm[i];
      perm[i] = perm[j];
      perm[j] = t;
    }
    // ascending order of the chosen offsets (insertion sort; spg <= G is small)
    for (int32_t i = 1; i < spg; ++i) {
      const int32_t v = perm[i];
      int32_t k = i - 1;
      while (k >= 0 && perm[k] > v) { perm[k + 1] = perm[k]; --k; }
      perm[k + 1] = v;
    }
    for (int32_t i = 0; i < spg; ++i) out[c * spg + i] = (int32_t)(c * G + perm[i]);
  }
  return SWF_OK;
}

extern "C" swf_status grouped_topk_select(const void*, const void*, const int32_t*, int32_t,
                                          const float*, int32_t, int32_t, int32_t*, float*, void*,
                                          size_t, int64_t, int64_t, int64_t, swf_dtype, void*) {
  return SWF_ERR_UNSUPPORTED;
}
extern "C" swf_status swf_group_buckets(const int32_t*, int64_t, int32_t, int32_t, int32_t*,
                                        int32_t*, void*, size_t, void*) {
  return SWF_ERR_UNSUPPORTED;
}
extern "C" swf_status sparse_swiglu_ffn_fwd(const void*, const void*, const void*, const void*,
                                            const int32_t*, int32_t, int32_t, void*, void*, size_t,
                                            void*, size_t, int64_t, int64_t, int64_t, swf_dtype,
                                            void*) {
  return SWF_ERR_UNSUPPORTED;
}
extern "C" swf_status sparse_swiglu_ffn_bwd(const void*, const void*, const void*, const void*,
                                            const void*, const int32_t*, const void*, size_t, void*,
                                            void*, void*, void*, void*, size_t, int64_t, int64_t,
                                            int64_t, int32_t, int32_t, swf_dtype, void*) {
  return SWF_ERR_UNSUPPORTED;
}
