// Per-kernel event timing (profiling aid behind swf_profile_enable / swf_profile_read).
#include <mutex>
#include <vector>

#include "swf_internal.h"

namespace swf {
namespace {

struct Pending {
  int kind;
  cudaEvent_t ev0, ev1;
};

std::mutex g_mu;
bool g_enabled = false;
std::vector<cudaEvent_t> g_pool;
std::vector<Pending> g_pending;

cudaEvent_t take_event() {
  if (!g_pool.empty()) {
    cudaEvent_t e = g_pool.back();
    g_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

void recycle_pending() {
  for (const Pending& p : g_pending) {
    g_pool.push_back(p.ev0);
    g_pool.push_back(p.ev1);
  }
  g_pending.clear();
}

const char* const kNames[SWF_K_NUM_KINDS] = {
    "gate_up_swiglu",  "gate_up_swiglu_infer", "down_proj",     "dgate",         "dx",
    "dw_gate_up",      "dw_down",              "f32_gemm",      "select_gather", "select_score",
    "select_topk",     "buckets",              "sparse_gather", "sparse_up",     "sparse_down",
    "sparse_dgate",    "sparse_dx",            "sparse_dw",     "elementwise",   "pair_sum",
    "balance",         "mlp2_up",              "mlp2_dpre",     "mlp2_dx",       "mlp2_dw_up",
    "splitk_reduce", "mhffn_fwd", "mhffn_prologue", "mhffn_bwd", "mhffn_bwd_dw",
    "mhffn_bwd_dr"};

}  // namespace

ProfScope::ProfScope(int kind, cudaStream_t st) : kind_(kind), st_(st) {
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_enabled) return;
  ev0_ = take_event();
  if (ev0_ && cudaEventRecord(ev0_, st_) != cudaSuccess) {
    g_pool.push_back(ev0_);
    ev0_ = nullptr;
  }
}

ProfScope::~ProfScope() {
  if (!ev0_) return;
  std::lock_guard<std::mutex> lock(g_mu);
  cudaEvent_t ev1 = take_event();
  if (!ev1 || cudaEventRecord(ev1, st_) != cudaSuccess) {
    g_pool.push_back(ev0_);
    if (ev1) g_pool.push_back(ev1);
    return;
  }
  g_pending.push_back({kind_, ev0_, ev1});
}

}  // namespace swf

using namespace swf;

extern "C" swf_status swf_profile_enable(int32_t enable) {
  std::lock_guard<std::mutex> lock(g_mu);
  for (const Pending& p : g_pending) cudaEventSynchronize(p.ev1);
  recycle_pending();
  g_enabled = enable != 0;
  return SWF_OK;
}

extern "C" int32_t swf_profile_read(int32_t max_kinds, int64_t* launches, double* total_ms) {
  if (max_kinds < 0 || (max_kinds > 0 && (!launches || !total_ms))) return -1;
  std::lock_guard<std::mutex> lock(g_mu);
  for (int k = 0; k < max_kinds; ++k) {
    launches[k] = 0;
    total_ms[k] = 0.0;
  }
  int32_t rc = SWF_K_NUM_KINDS;
  for (const Pending& p : g_pending) {
    float ms = 0.f;
    if (cudaEventSynchronize(p.ev1) != cudaSuccess || cudaEventElapsedTime(&ms, p.ev0, p.ev1) != cudaSuccess) {
      rc = -1;
      continue;
    }
    if (p.kind >= 0 && p.kind < max_kinds) {
      launches[p.kind] += 1;
      total_ms[p.kind] += ms;
    }
  }
  recycle_pending();
  return rc;
}

extern "C" const char* swf_kernel_name(int32_t kind) {
  return (kind >= 0 && kind < SWF_K_NUM_KINDS) ? kNames[kind] : "?";
}
