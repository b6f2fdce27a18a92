/*
 * swiglu_ffn.h -- C ABI of the SwiGLU feed-forward library for NVIDIA B200 (sm_100a).
 *
 * The block is y = (SiLU(x W_gate^T) * (x W_up^T)) W_down^T with SiLU(z) = z * sigmoid(z)
 * (flash-swiglu-mlp overview: fused gate/up projections with SiLU gating, then the down
 * projection; training saves intermediates, inference does not), plus the group-sparse
 * variant of the eugen_sparse README ("What it does": grouped_topk_select picks, per token,
 * the num_active_groups groups of group_size FFN rows with the largest energy
 * sum |SiLU(x W_gate^T)|, optionally on a fixed row subsample and with a balancing bias;
 * sparse_swiglu_ffn computes only the selected groups, forward and backward).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every tensor pointer is a DEVICE pointer owned by the caller, row-major and contiguous,
 *    16-byte aligned (SWF_ERR_ALIGNMENT otherwise).  Weights use the nn.Linear layout:
 *    w_gate, w_up are [d_ff, d_model]; w_down is [d_model, d_ff].  Activations are
 *    [M, d_model] with M the number of tokens.
 *  - `dtype` (swf_dtype) is the element type of every floating tensor except the balancing
 *    bias and the energies, which are always fp32.  bf16 runs on the tcgen05 tensor cores with
 *    fp32 accumulation; fp32 runs in full fp32 on the CUDA cores.
 *  - `stream` is a cudaStream_t (passed as void*).  Calls only enqueue work on it and return;
 *    nothing allocates device memory, nothing synchronises.  Buffers that the work needs
 *    beyond its inputs and outputs come from the caller's `workspace` of `workspace_bytes`
 *    bytes (size it with swf_workspace_bytes; SWF_ERR_WORKSPACE if too small).
 *  - Argument errors are detected on the host before anything is enqueued; then no work is
 *    launched and outputs are untouched.  There is never a CPU or library fallback: a shape
 *    outside the rules returns SWF_ERR_UNSUPPORTED.
 *  - Weight gradients are overwritten, not accumulated.
 *  - Every wait inside a kernel is bounded in time; a wait that runs out records
 *    SWF_ERR_TIMEOUT in a per-device status word (read with swf_device_status) and the kernel
 *    returns instead of hanging.
 *
 * Shape rules (eugen_sparse README, "Parameters and how to choose them" and "Pitfalls"):
 *  - bf16: d_model and d_ff multiples of 16 (TMA rows must be 16-byte multiples).
 *  - fp32: any positive d_model, d_ff.
 *  - sparse / selection: group_size a power of two in [16, 64]; d_ff a multiple of group_size
 *    with at least 2 groups; 1 <= num_active_groups <= d_ff / group_size; 1 <= samples_per_group
 *    <= group_size; M * num_active_groups < 2^31.
 */
#ifndef SWIGLU_FFN_H
#define SWIGLU_FFN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum swf_status {
  SWF_OK = 0,
  SWF_ERR_INVALID_ARG = 1,  /* null pointer, non-positive size, bad enum */
  SWF_ERR_UNSUPPORTED = 2,  /* shape or dtype outside the rules above */
  SWF_ERR_ALIGNMENT = 3,    /* a pointer not 16-byte aligned */
  SWF_ERR_WORKSPACE = 4,    /* workspace (or sparse saved buffer) smaller than required */
  SWF_ERR_LAUNCH = 5,       /* the CUDA runtime refused a launch or a query */
  SWF_ERR_TIMEOUT = 6       /* a bounded in-kernel wait ran out (see swf_device_status) */
} swf_status;

typedef enum swf_dtype { SWF_F32 = 0, SWF_BF16 = 1 } swf_dtype;

typedef enum swf_op {
  SWF_OP_FWD = 0,         /* swiglu_ffn_fwd */
  SWF_OP_FWD_INFER = 1,   /* swiglu_ffn_fwd_infer */
  SWF_OP_BWD = 2,         /* swiglu_ffn_bwd */
  SWF_OP_SELECT = 3,      /* grouped_topk_select */
  SWF_OP_SPARSE_FWD = 4,  /* sparse_swiglu_ffn_fwd */
  SWF_OP_SPARSE_BWD = 5,  /* sparse_swiglu_ffn_bwd */
  SWF_OP_BUCKETS = 6,     /* swf_group_buckets */
  SWF_OP_MLP2_FWD = 7,    /* leaky_relu_sq_mlp_fwd (d_ff = hidden) */
  SWF_OP_MLP2_BWD = 8     /* leaky_relu_sq_mlp_bwd (d_ff = hidden) */
} swf_op;

/* How an operation will run (eugen_sparse README: plan() reports how the work is split,
 * without touching the GPU).  Filled by swf_plan. */
typedef struct swf_plan_info {
  int32_t path;            /* 0 = fp32 CUDA cores, 1 = bf16 tcgen05 tensor cores */
  int32_t tile_m, tile_n, tile_k;
  int32_t stages;          /* shared-memory pipeline depth of the GEMM kernels */
  int32_t grid;            /* CTAs of the persistent GEMM kernels (<= number of SMs) */
  int32_t num_kernels;     /* kernels one call launches */
  int32_t deterministic;   /* 1 if repeated calls give bitwise-identical results */
  int64_t gemm_tiles;      /* output tiles over all GEMMs of the call */
  int64_t flops;           /* algorithmic FLOPs of the call */
  size_t workspace_bytes;  /* = swf_workspace_bytes(...) */
  size_t saved_bytes;      /* sparse forward: = swf_sparse_saved_bytes(...), else 0 */
} swf_plan_info;

/* ------------------------------------------------------------------ dense SwiGLU FFN */

/* Training forward (flash-swiglu-mlp overview, "Fused train forward" storing intermediates;
 * parameter-golf PR 1105 "Fused MLP Kernels": store the activation gradient, not the
 * pre-activation).  Computes g = x W_gate^T, u = x W_up^T (fp32 accumulation, never written
 * to memory), and writes
 *   saved_h = SiLU(g) * u,  saved_a = u * SiLU'(g),  saved_b = SiLU(g)   (each [M, d_ff]),
 *   y = saved_h W_down^T                                                   ([M, d_model]).
 * saved_* are outputs the caller keeps for swiglu_ffn_bwd.  No workspace. */
swf_status swiglu_ffn_fwd(const void* x, const void* w_gate, const void* w_up, const void* w_down,
                          void* y, void* saved_h, void* saved_a, void* saved_b,
                          int64_t M, int64_t d_model, int64_t d_ff, swf_dtype dtype, void* stream);

/* Inference forward (flash-swiglu-mlp overview: "inference skips saving gate/up activations").
 * Same y as swiglu_ffn_fwd; the product h lives only in `workspace`
 * (swf_workspace_bytes(SWF_OP_FWD_INFER, ...) bytes). */
swf_status swiglu_ffn_fwd_infer(const void* x, const void* w_gate, const void* w_up,
                                const void* w_down, void* y, void* workspace,
                                size_t workspace_bytes, int64_t M, int64_t d_model, int64_t d_ff,
                                swf_dtype dtype, void* stream);

/* Backward of the training forward (flash-swiglu-mlp: activation-gradient, weight-gradient and
 * input-gradient steps; parameter-golf "Fused MLP Kernels": the down-projection gradient is
 * multiplied by the stored activation-gradient factor inside the GEMM epilogue):
 *   dH = dy W_down;  dG = dH * saved_a;  dU = dH * saved_b        (workspace, [M, 2 d_ff])
 *   dx = dG W_gate + dU W_up;  dw_gate = dG^T x;  dw_up = dU^T x;  dw_down = dy^T saved_h.
 * dx [M, d_model]; dw_gate, dw_up [d_ff, d_model]; dw_down [d_model, d_ff] (overwritten).  When
 * a weight gradient has too few output tiles to fill the GPU, its sum over the tokens is split
 * into fp32 partial sums (in the workspace) that are added in a fixed order, so the result stays
 * deterministic. */
swf_status swiglu_ffn_bwd(const void* dy, const void* x, const void* w_gate, const void* w_up,
                          const void* w_down, const void* saved_h, const void* saved_a,
                          const void* saved_b, void* dx, void* dw_gate, void* dw_up,
                          void* dw_down, void* workspace, size_t workspace_bytes, int64_t M,
                          int64_t d_model, int64_t d_ff, swf_dtype dtype, void* stream);

/* Size of the fixed device scratch used by swiglu_ffn_fwd_infer_noalloc (32 MiB). */
#define SWF_NOALLOC_SCRATCH_BYTES (32u << 20)

/* Inference forward that allocates nothing and takes no workspace.  The pages have no
 * counterpart: it exists for callers that cannot provide device memory for the intermediate
 * h, such as a host program that reaches the library only through this ABI and has no device
 * allocator, or a plug-in inside a runtime that forbids allocation on its execution path.
 * Computes the same y as
 * swiglu_ffn_fwd_infer, keeping h [M, d_ff] in a file-scope device array of
 * SWF_NOALLOC_SCRATCH_BYTES that every GPU loading the library holds until the process exits.
 *  - Returns SWF_ERR_WORKSPACE, launching nothing, when M * d_ff * element size exceeds
 *    SWF_NOALLOC_SCRATCH_BYTES (e.g. at most 3048 tokens for bf16 with d_ff = 5504).
 *  - The first call on each device looks up the array's device address (with that device
 *    current); make that first call before any stream capture on the device.
 *  - All calls share the array and it keeps the last call's contents (nothing in it needs to
 *    start at zero).  Calls whose kernels overlap on the GPU, e.g. on two streams, race on it:
 *    serialise them.
 *  - Calls no cudaMalloc, cudaFree or allocating library routine. */
swf_status swiglu_ffn_fwd_infer_noalloc(const void* x, const void* w_gate, const void* w_up,
                                        const void* w_down, void* y, int64_t M, int64_t d_model,
                                        int64_t d_ff, swf_dtype dtype, void* stream);

/* ------------------------------------------------------------------ LeakyReLU(0.5)^2 MLP */

/* The MLP of parameter-golf PR 1105 ("Fused MLP Kernels"): an up projection, LeakyReLU with
 * slope 0.5, a square, and a down projection, with the activation gradient stored in the
 * forward pass instead of the pre-activation:
 *   pre = x W_up^T (fp32 accumulation, never written to memory),
 *   saved_post = LeakyReLU(0.5)(pre)^2,  saved_act_grad = 2 pre if pre > 0 else 0.5 pre,
 *   y = saved_post W_down^T.
 * w_up [hidden, d_model], w_down [d_model, hidden] (nn.Linear layout); saved_* [M, hidden] are
 * outputs the caller keeps for the backward.  Same dtype and shape rules as the dense SwiGLU
 * entry points (hidden in place of d_ff).  No workspace. */
swf_status leaky_relu_sq_mlp_fwd(const void* x, const void* w_up, const void* w_down, void* y,
                                 void* saved_post, void* saved_act_grad, int64_t M,
                                 int64_t d_model, int64_t hidden, swf_dtype dtype, void* stream);

/* Backward of the MLP above (the page's branch-free backward: the multiply by the stored
 * activation gradient happens in the GEMM epilogue):
 *   dpre = (dy W_down) * saved_act_grad      (workspace, [M, hidden])
 *   dx = dpre W_up;  dw_up = dpre^T x;  dw_down = dy^T saved_post   (overwritten). */
swf_status leaky_relu_sq_mlp_bwd(const void* dy, const void* x, const void* w_up,
                                 const void* w_down, const void* saved_post,
                                 const void* saved_act_grad, void* dx, void* dw_up, void* dw_down,
                                 void* workspace, size_t workspace_bytes, int64_t M,
                                 int64_t d_model, int64_t hidden, swf_dtype dtype, void* stream);

/* ------------------------------------------------------------------ FlashFFN multi-head FFN */

/* Multi-head FFN forward ("FlashFFN: Multi-Head Decomposition Enables I/O-Aware Feed-Forward
 * Networks", section "Overview"): for every token t and head h,
 *   o[t,h,:] = sum_e router[t,h,e] * (SiLU(q[t,h,:] K_{h,e}^T) (.) (q[t,h,:] U_{h,e}^T)) V_{h,e}
 * with K_{h,e}, U_{h,e}, V_{h,e} the [sub_dim, head_dim] blocks of w_k, w_u, w_v.
 *   q        [T, num_heads * head_dim]   the heads' normalised input projections (head-minor)
 *   w_k/u/v  [num_heads * num_sub * sub_dim, head_dim], rows ordered (head, sub-network, row)
 *   router   [T, num_heads, num_sub] fp32 sub-network weights
 *   o        [T, num_heads * head_dim]   (overwritten)
 * One fused kernel: the [T, num_sub * sub_dim] activations of a head stay on chip (TMEM and
 * shared memory) and never reach HBM.  Device pointers, caller-owned, 16-byte aligned (else
 * SWF_ERR_ALIGNMENT); asynchronous on `stream`; nothing allocates.  Supported: dtype SWF_BF16
 * (fp32 accumulation), head_dim 128 (the page's d_h), sub_dim a multiple of 64; anything else
 * returns SWF_ERR_UNSUPPORTED (there is no fallback). */
swf_status flash_mhffn_fwd(const void* q, const void* w_k, const void* w_u, const void* w_v,
                           const float* router, void* o, int64_t T, int32_t num_heads,
                           int32_t head_dim, int32_t num_sub, int32_t sub_dim, swf_dtype dtype,
                           void* stream);

/* Backward of flash_mhffn_fwd: gradients of L = sum(d_o * o) with respect to q, w_k, w_u, w_v
 * and router (same shapes as those inputs; all overwritten, drouter fp32).  With dA = d_o_h V_e^T,
 * act = SiLU(g) u (g = q_h K_e^T, u = q_h U_e^T) and r the sub-network's router weight:
 *   drouter = sum over the sub-network's columns of dA act;  dS_g = dA r u SiLU'(g);
 *   dS_u = dA r SiLU(g);  P = r act;  dq_h = sum_e dS_g K_e + dS_u U_e;
 *   [dw_k ; dw_u]_e = [dS_g | dS_u]^T q_h;  dw_v_e = P^T d_o_h.
 * One fused tcgen05 kernel per group of up to four heads recomputes g and u, forms dA on chip
 * (never stored), accumulates dq and writes dS_g | dS_u and P (bf16) to `workspace`; split-K
 * tcgen05 GEMMs then reduce them over the tokens into the weight gradients.  Workspace:
 * flash_mhffn_bwd_workspace_bytes bytes (about 6 * min(num_heads, 4) * T * num_sub * sub_dim).
 * Device pointers, caller-owned, 16-byte aligned; asynchronous on `stream`; deterministic.
 * Supported: dtype SWF_BF16, head_dim 128, sub_dim a multiple of 128; else SWF_ERR_UNSUPPORTED.
 * Workspace missing or too small: SWF_ERR_WORKSPACE. */
swf_status flash_mhffn_bwd(const void* q, const void* w_k, const void* w_u, const void* w_v,
                           const float* router, const void* d_o, void* dq, void* dw_k,
                           void* dw_u, void* dw_v, float* drouter, void* workspace,
                           size_t workspace_bytes, int64_t T, int32_t num_heads,
                           int32_t head_dim, int32_t num_sub, int32_t sub_dim, swf_dtype dtype,
                           void* stream);
/* Bytes of flash_mhffn_bwd's workspace (0 for rejected arguments). */
size_t flash_mhffn_bwd_workspace_bytes(int64_t T, int32_t num_heads, int32_t head_dim,
                                       int32_t num_sub, int32_t sub_dim, swf_dtype dtype);

/* The multi-head block's prologue (same page, "Overview": Q is the heads' RMS-normalised
 * projection of the input, R the sigmoid-normalised router weights):
 *   q[t, h*head_dim + i] = z[t,h,i] / sqrt(mean_i z[t,h,i]^2 + eps) * q_gain[i],  z = x w_q^T
 *   router[t, h, e] = sigmoid(l[t,h,e]) / sum_e' sigmoid(l[t,h,e']),         l = x w_r^T
 *   x [T, d_model]; w_q [num_heads * head_dim, d_model]; q_gain [head_dim] fp32 or NULL (no
 *   gain); w_r [num_heads * num_sub, d_model]; q [T, num_heads * head_dim] (the input of
 *   flash_mhffn_fwd); router [T, num_heads, num_sub] fp32.  Outputs are overwritten.
 * Two tcgen05 GEMMs with the normalisations fused into their epilogues.  Device pointers,
 * caller-owned, 16-byte aligned; asynchronous on `stream`; nothing allocates.  Supported:
 * dtype SWF_BF16, head_dim 128, d_model a multiple of 16, num_heads * num_sub <= 256; else
 * SWF_ERR_UNSUPPORTED.  eps < 0 or NaN: SWF_ERR_INVALID_ARG. */
swf_status flash_mhffn_prologue(const void* x, const void* w_q, const float* q_gain,
                                const void* w_r, void* q, float* router, int64_t T,
                                int64_t d_model, int32_t num_heads, int32_t head_dim,
                                int32_t num_sub, float eps, swf_dtype dtype, void* stream);

/* Backward of flash_mhffn_prologue given dq [T, num_heads * head_dim] (bf16) and drouter
 * [T, num_heads, num_sub] (fp32): dx [T, d_model], dw_q, dw_r (shapes of w_q, w_r) and, when
 * both q_gain and dq_gain are given, dq_gain [head_dim] fp32 (dq_gain alone: written as zeros).
 * The projection and router GEMMs are recomputed with the normalisations' backward in their
 * epilogues; then dx = [dz | dl] [w_q ; w_r] and [dw_q ; dw_r] = [dz | dl]^T x.  Workspace:
 * flash_mhffn_prologue_bwd_workspace_bytes bytes.  Same support rules and error codes as the
 * forward; outputs overwritten; deterministic. */
swf_status flash_mhffn_prologue_bwd(const void* x, const void* w_q, const float* q_gain,
                                    const void* w_r, const void* dq, const float* drouter,
                                    void* dx, void* dw_q, float* dq_gain, void* dw_r,
                                    void* workspace, size_t workspace_bytes, int64_t T,
                                    int64_t d_model, int32_t num_heads, int32_t head_dim,
                                    int32_t num_sub, float eps, swf_dtype dtype, void* stream);
size_t flash_mhffn_prologue_bwd_workspace_bytes(int64_t T, int64_t d_model, int32_t num_heads,
                                                int32_t head_dim, int32_t num_sub, swf_dtype dtype);

/* ------------------------------------------------------------------ group-sparse variant */

/* Subsample index (eugen_sparse README, make_subsample_index; drawn once per layer).  HOST
 * function, no GPU work.  Writes out[c * spg + i], c < d_ff / group_size, i < spg: the absolute
 * gate-row ids of group c's sample, ascending, drawn by a partial Fisher-Yates shuffle of the
 * group's offsets driven by one splitmix64 stream seeded with `seed` (groups in order). */
swf_status swf_make_subsample_index(int64_t d_ff, int32_t group_size, int32_t samples_per_group,
                                    uint64_t seed, int32_t* out);

/* Grouped top-k selection (eugen_sparse README, grouped_topk_select; hard top-k, no gradient,
 * deterministic).  For token t and group c (rows [c*G, (c+1)*G) of w_gate):
 *   s[t,c] = sum_{j in S_c} |SiLU(x_t . w_gate[j])|  (+ load_balance_bias[c] when non-null)
 * where S_c is the group's subsample subsample_idx[c*spg .. c*spg+spg) (absolute row ids, as
 * written by swf_make_subsample_index), or all G rows when subsample_idx is NULL (then
 * samples_per_group is ignored).  The bias is additive and affects selection only.
 * group_idx [M, K] int32 receives each token's K best groups (ties: lower group index wins),
 * ascending within the row.  energies, if non-null, receives s [M, d_ff/G] fp32. */
swf_status grouped_topk_select(const void* x, const void* w_gate, const int32_t* subsample_idx,
                               int32_t samples_per_group, const float* load_balance_bias,
                               int32_t group_size, int32_t num_active_groups, int32_t* group_idx,
                               float* energies, void* workspace, size_t workspace_bytes,
                               int64_t M, int64_t d_model, int64_t d_ff, swf_dtype dtype,
                               void* stream);

/* Group-major bucketing of the (token, group) pairs (eugen_sparse README, "Pitfalls": the
 * CSR bucketing is deterministic).  offsets [num_groups + 1] int32 and tokens [M * K] int32:
 * tokens[offsets[c] .. offsets[c+1]) are the ids of the tokens whose group_idx row holds c, in
 * ascending order.  group_idx rows must hold distinct in-range groups: slots out of range or
 * repeating an earlier slot of the row are dropped (checked only in debug mode, swf_set_debug). */
swf_status swf_group_buckets(const int32_t* group_idx, int64_t M, int32_t num_active_groups,
                             int32_t num_groups, int32_t* offsets, int32_t* tokens,
                             void* workspace, size_t workspace_bytes, void* stream);

/* Sparse forward (eugen_sparse README, sparse_swiglu_ffn):
 *   y[t] = sum over c in group_idx[t] of (SiLU(x_t W_gate[c]^T) * x_t W_up[c]^T) W_down[:, c]^T
 * with W_*[c] the group's G rows.  Each (token, group) contribution is computed in fp32 and
 * stored in `dtype`; a token's contributions are then summed in fp32 in the order of its
 * group_idx slots, so y is bitwise deterministic (the README's kernel uses fp32 atomics
 * instead).  The GEMMs gather the token rows of x themselves (from L2); no gathered copy of x
 * is written.  `saved` (swf_sparse_saved_bytes bytes) receives what the backward needs: the
 * bucketing and the compact per-pair h, a, b; the caller keeps it for sparse_swiglu_ffn_bwd,
 * together with x and the group_idx (the backward reads both again). */
swf_status sparse_swiglu_ffn_fwd(const void* x, const void* w_gate, const void* w_up,
                                 const void* w_down, const int32_t* group_idx, int32_t group_size,
                                 int32_t num_active_groups, void* y, void* saved,
                                 size_t saved_bytes, void* workspace, size_t workspace_bytes,
                                 int64_t M, int64_t d_model, int64_t d_ff, swf_dtype dtype,
                                 void* stream);

/* Sparse backward: gradients to x and all three weights of L = sum(dy * y) for the forward
 * above.  Only selected groups get weight gradients; rows (dw_gate, dw_up) and columns
 * (dw_down) of groups no token selected are written as exact zeros (eugen_sparse README,
 * "Hard selection").  dx is reduced like y in the forward; every output is deterministic. */
swf_status sparse_swiglu_ffn_bwd(const void* dy, const void* x, const void* w_gate,
                                 const void* w_up, const void* w_down, const int32_t* group_idx,
                                 const void* saved, size_t saved_bytes, void* dx, void* dw_gate,
                                 void* dw_up, void* dw_down, void* workspace,
                                 size_t workspace_bytes, int64_t M, int64_t d_model, int64_t d_ff,
                                 int32_t group_size, int32_t num_active_groups, swf_dtype dtype,
                                 void* stream);

/* Group-usage frequency of one batch (eugen_sparse README, "What it does": the balancing step
 * uses the current usage of each group): freq[c] = (number of tokens whose group_idx row holds c)
 * / M, fp32 [num_groups].  The frequencies sum to num_active_groups.  Entries that are out of
 * range or repeat an earlier slot of the same row are not counted. */
swf_status swf_group_frequency(const int32_t* group_idx, int64_t M, int32_t num_active_groups,
                               int32_t num_groups, float* freq, void* stream);

/* Auxiliary-loss-free load balancing, called once per optimizer step (eugen_sparse README,
 * update_load_balance_bias, "in the style of DeepSeek-V3"; defaults gamma 1e-3, bias_max 0.5,
 * momentum 0.99, target_freq = num_active_groups / num_groups).  In place on the device, per
 * group c:  freq_ema[c] = momentum * freq_ema[c] + (1 - momentum) * current_freq[c];
 *           bias[c] = clamp(bias[c] + gamma * sign(target_freq - freq_ema[c]), -bias_max, bias_max)
 * (the README gives no formula; this is the plainest reading of it).  All arrays fp32
 * [num_groups]; bias and freq_ema are the caller's persistent buffers. */
swf_status update_load_balance_bias(float* bias, float* freq_ema, const float* current_freq,
                                    float target_freq, float gamma, float bias_max,
                                    float momentum, int32_t num_groups, void* stream);

/* ------------------------------------------------------------------ group_idx checks */

/* The eugen_sparse README ("Pitfalls and limitations") leaves group_idx unchecked: it must come
 * from grouped_topk_select, and nothing validates the input beyond the shape rules.  This
 * library's kernels never index out of bounds on a bad group_idx -- a slot whose group is out of
 * [0, num_groups) or repeats an earlier slot of its row is dropped by the bucketing -- but the
 * result then differs from what the caller meant.  These calls find such slots.
 *
 * swf_validate_group_idx counts the invalid slots of group_idx [M, num_active_groups] on
 * `stream`, WAITS for the count (it synchronises the stream) and writes it to *bad_slots when
 * non-null.  Returns SWF_OK when every slot is valid, SWF_ERR_INVALID_ARG when any is not; never
 * traps.  Uses one device counter per GPU: concurrent validations on one device are serialised
 * by the library (host mutex held across the synchronisation). */
swf_status swf_validate_group_idx(const int32_t* group_idx, int64_t M, int32_t num_active_groups,
                                  int32_t num_groups, int64_t* bad_slots, void* stream);

/* Debug mode (default: on when the environment variable SWF_DEBUG is set and not "0" at the
 * first query).  While it is on, every entry point that reads group_idx (swf_group_buckets,
 * swf_group_frequency, sparse_swiglu_ffn_fwd, sparse_swiglu_ffn_bwd) first runs
 * swf_validate_group_idx on its stream -- so it synchronises that stream -- and returns
 * SWF_ERR_INVALID_ARG, having launched nothing else and left its outputs untouched, if any slot
 * is invalid.  swf_set_debug(0 or 1) overrides the environment (else SWF_ERR_INVALID_ARG);
 * swf_get_debug returns the mode in effect. */
swf_status swf_set_debug(int32_t enable);
int32_t swf_get_debug(void);

/* ------------------------------------------------------------------ planning and queries */

/* Workspace bytes `op` needs (0 if none).  group_size / num_active_groups are ignored by the
 * dense ops; returns 0 for arguments that swf_supported rejects. */
size_t swf_workspace_bytes(swf_op op, int64_t M, int64_t d_model, int64_t d_ff,
                           int32_t group_size, int32_t num_active_groups, swf_dtype dtype);

/* Bytes of the `saved` buffer of sparse_swiglu_ffn_fwd / _bwd (0 for rejected arguments). */
size_t swf_sparse_saved_bytes(int64_t M, int64_t d_model, int64_t d_ff, int32_t group_size,
                              int32_t num_active_groups, swf_dtype dtype);

/* SWF_OK if `op` runs for these sizes, else the status the op would return (eugen_sparse
 * README, kernel_supported).  Host only. */
swf_status swf_supported(swf_op op, int64_t M, int64_t d_model, int64_t d_ff, int32_t group_size,
                         int32_t num_active_groups, int32_t samples_per_group, swf_dtype dtype);

/* How `op` will run (eugen_sparse README, plan): fills *out.  Host only. */
swf_status swf_plan(swf_op op, int64_t M, int64_t d_model, int64_t d_ff, int32_t group_size,
                    int32_t num_active_groups, int32_t samples_per_group, swf_dtype dtype,
                    swf_plan_info* out);

/* Synchronises `stream`, then reads and clears the current device's status word: SWF_OK, or
 * SWF_ERR_TIMEOUT if a kernel's bounded wait ran out since the last read. */
swf_status swf_device_status(void* stream);

/* Failure-detection self test: launches one kernel that waits on a barrier that nothing
 * completes, with a limit of `limit_us` microseconds (1 .. 1000000), so that the wait runs
 * out and the kernel records SWF_ERR_TIMEOUT and returns.  Returns the launch status. */
swf_status swf_selftest_wait_timeout(int32_t limit_us, void* stream);

/* ------------------------------------------------------------------ profiling aid */

/* Kernel kinds the library launches (indices of swf_profile_read's arrays). */
typedef enum swf_kernel_kind {
  SWF_K_GATE_UP = 0,       /* training forward: x [W_g|W_u]^T with the SwiGLU epilogue */
  SWF_K_GATE_UP_INFER = 1, /* inference forward: same, h only */
  SWF_K_DOWN = 2,          /* y = h W_d^T */
  SWF_K_DGATE = 3,         /* dH = dY W_d with the gating epilogue -> [dG | dU] */
  SWF_K_DX = 4,            /* dx = [dG | dU] [W_g ; W_u] */
  SWF_K_DW_GATE_UP = 5,    /* [dW_g ; dW_u] = [dG | dU]^T x */
  SWF_K_DW_DOWN = 6,       /* dW_d = dY^T h */
  SWF_K_F32_GEMM = 7,      /* fp32 CUDA-core GEMM (any dense step) */
  SWF_K_SELECT_GATHER = 8, /* gather of the subsampled gate rows */
  SWF_K_SELECT_SCORE = 9,  /* scoring GEMM with the energy epilogue */
  SWF_K_SELECT_TOPK = 10,  /* warp-level grouped top-k */
  SWF_K_BUCKETS = 11,      /* group bucketing (count, scan, place) */
  SWF_K_SPARSE_GATHER = 12,/* gather of token rows into group-major order */
  SWF_K_SPARSE_UP = 13,    /* sparse gate|up GEMM with the SwiGLU epilogue */
  SWF_K_SPARSE_DOWN = 14,  /* sparse down GEMM: per-pair contributions to y */
  SWF_K_SPARSE_DGATE = 15, /* sparse dH GEMM with the gating epilogue */
  SWF_K_SPARSE_DX = 16,    /* sparse dx GEMM: per-pair contributions to dx */
  SWF_K_SPARSE_DW = 17,    /* sparse weight-gradient GEMMs */
  SWF_K_ELEMENTWISE = 18,  /* fills */
  SWF_K_PAIR_SUM = 19,     /* per-token sum of the per-pair contributions (y, dx) */
  SWF_K_BALANCE = 20,      /* group frequency and balancing-bias update */
  SWF_K_MLP2_UP = 21,      /* LeakyReLU^2 MLP: x W_up^T with the post / act_grad epilogue */
  SWF_K_MLP2_DPRE = 22,    /* LeakyReLU^2 MLP: (dY W_down) * act_grad */
  SWF_K_MLP2_DX = 23,      /* LeakyReLU^2 MLP: dpre W_up */
  SWF_K_MLP2_DW_UP = 24,   /* LeakyReLU^2 MLP: dpre^T x */
  SWF_K_SPLITK_REDUCE = 25,/* fixed-order sum of split-K weight-gradient partials */
  SWF_K_MHFFN_FWD = 26,    /* FlashFFN multi-head FFN forward (fused, one kernel) */
  SWF_K_MHFFN_PROLOGUE = 27, /* FlashFFN prologue: head-normalised projection, router */
  SWF_K_MHFFN_BWD = 28,    /* FlashFFN backward, fused per token tile: dA, dS_g | dS_u, P, dQ */
  SWF_K_MHFFN_BWD_DW = 29, /* FlashFFN backward: dK, dU, dV */
  SWF_K_MHFFN_BWD_DR = 30, /* FlashFFN backward: router-gradient sums */
  SWF_K_NUM_KINDS = 31
} swf_kernel_kind;

/* While enabled, every kernel the library launches is bracketed by a pair of CUDA events on
 * its stream (events are created by the library on first use and reused).  Enabling or
 * disabling clears the accumulated statistics.  Not thread-safe against concurrent calls of
 * the other entry points. */
swf_status swf_profile_enable(int32_t enable);

/* Waits for the recorded events, then adds each bracketed launch to launches[kind] and its
 * duration (ms) to total_ms[kind] for kind < max_kinds (both arrays zeroed by the call),
 * and forgets the events.  Returns the number of kinds (SWF_K_NUM_KINDS) or -1 on error. */
int32_t swf_profile_read(int32_t max_kinds, int64_t* launches, double* total_ms);

/* Static name of a kernel kind ("?" when out of range). */
const char* swf_kernel_name(int32_t kind);

/* Static, human-readable name of a status code. */
const char* swf_status_string(swf_status status);

#ifdef __cplusplus
}
#endif

#endif /* SWIGLU_FFN_H */
