// Host-side interface of the group-sparse path (selection, bucketing, sparse FFN).
#pragma once
#include "swf_internal.h"

namespace swf {

swf_status check_sparse_shape(int64_t M, int64_t d, int64_t f, int32_t G, int32_t K, swf_dtype dt);
size_t select_workspace_bytes(int64_t M, int64_t d, int64_t f, int32_t G, int32_t K);
size_t sparse_fwd_workspace_bytes(int64_t M, int64_t d, int64_t f, int32_t G, int32_t K);
size_t sparse_bwd_workspace_bytes(int64_t M, int64_t d, int64_t f, int32_t G, int32_t K);
size_t buckets_workspace_bytes(int64_t M, int32_t K, int32_t ng);
size_t sparse_saved_bytes(int64_t M, int64_t d, int64_t f, int32_t G, int32_t K);
void sparse_plan(int op, int64_t M, int64_t d, int64_t f, int32_t G, int32_t K, int32_t spg,
                 swf_plan_info* p);

}  // namespace swf
