// FlashFFN multi-head feed-forward block, forward, as one fused tcgen05 kernel.
//
// "FlashFFN: Multi-Head Decomposition Enables I/O-Aware Feed-Forward Networks", section
// "Overview": per head h (d_h = 128),
//     O_h = sum_e R_e * ((SiLU(Q K_e^T) (.) (Q U_e^T)) V_e),
// with Q the head's RMS-normalised input projection and R_e the sigmoid-normalised router weights
// (both inputs here).  The page's point is that a head's accumulator (128 tokens x d_h fp32) fits
// on chip, so the [tokens, E*d_e] intermediate never reaches HBM.  On B200 it lives in TMEM and
// shared memory:
//
//   per work unit (head h, 128-token tile), for each 64-column chunk c of the head's E*d_e
//   sub-network columns:
//     [S_g | S_u] = Q [K_c ; U_c]^T     (tcgen05, M=128 N=128 K=128, fp32 in TMEM, two buffers)
//     P   = SiLU(S_g) * S_u * R_e       (epilogue warps, bf16 into shared memory, two buffers)
//     O  += P V_c                       (tcgen05, M=128 N=128 K=64, A from shared memory)
//   then O (128 TMEM columns) -> bf16 -> HBM.
//
// Warp roles: warp 0 lane 0 issues TMA loads (Q once per unit, then a ring of K|U|V chunk
// stages); warp 1 owns TMEM and lane 0 issues every MMA, running the S products two chunks ahead
// of the PV products; warps 2..9 turn S into P and drain O as two sets of four warps (one per
// TMEM lane quadrant) that take alternate chunks, so two chunks' epilogues are in flight.
// Every wait is bounded (status word + abort flag, as in the GEMM template).
#include <algorithm>
#include <initializer_list>

#include "swf_internal.h"
#include "swf_ptx.cuh"

namespace swf {
namespace {

constexpr int kMhTile = 128;     // tokens per unit
constexpr int kMhDh = 128;       // head width d_h
constexpr int kMhChunk = 64;     // sub-network columns per chunk
constexpr int kMhKuStages = 3;   // K|U chunk stages (free once the chunk's S products are done)
constexpr int kMhVStages = 4;    // V chunk stages (free once its PV product is done)
constexpr int kMhEpiWarps = 8;  // two sets of four (one warp per TMEM lane quadrant each)
constexpr int kMhThreads = 64 + 32 * kMhEpiWarps;
constexpr int kMhEpiThreads = 32 * kMhEpiWarps;
constexpr int kMhBox = 64 * 64 * 2;                 // one 64 x 64 bf16 TMA box (8 KB)
constexpr int kMhQBytes = 2 * kMhTile * 64 * 2;     // Q tile: two 128 x 64 boxes
constexpr int kMhKuBytes = 4 * kMhBox;              // K and U chunks: two boxes each
constexpr int kMhVBytes = 2 * kMhBox;               // V chunk: two boxes
constexpr int kMhPBytes = kMhTile * kMhChunk * 2;   // one P buffer (128 x 64 bf16)
constexpr int kMhKuOff = kMhQBytes;
constexpr int kMhVOff = kMhKuOff + kMhKuStages * kMhKuBytes;
constexpr int kMhPOff = kMhVOff + kMhVStages * kMhVBytes;
constexpr int kMhBarOff = kMhPOff + 2 * kMhPBytes;
constexpr int kMhSmemBytes = kMhBarOff + 256 + 1024;  // barriers + alignment slack
static_assert(kMhSmemBytes <= 232448, "shared memory per CTA");
constexpr int kMhTmemCols = 512;                      // O [0,128); S buffers at 128, 256

struct MhArgs {
  int T, H, E, de;
  int n_tt;         // 128-token tiles
  int n_units;      // n_tt * H, head-major
  int nch;          // 64-column chunks per head (E * de / 64)
  int ch_per_sub;   // chunks per sub-network (de / 64)
  const float* r;   // [T][H][E]
  __nv_bfloat16* o; // [T][H * 128]
  int* status;
  uint64_t wait_limit_ns;
};

// P tile element (row, column 8*c16 .. 8*c16+7) in the 128-byte-swizzled K-major layout the UMMA
// descriptor reads: row r at r*128 bytes, its 16-byte chunk c16 at position c16 ^ (r & 7).
__device__ __forceinline__ uint32_t p_offset(int row, int c16) {
  return static_cast<uint32_t>(row * 128 + ((c16 ^ (row & 7)) << 4));
}

// SiLU(z) = z * sigmoid(z) with sigmoid(z) = (1 + tanh(z / 2)) / 2: one MUFU operation
// (tanh.approx.f32, relative error about 2^-11) instead of an exponential and a reciprocal.  The
// epilogue is bound by the MUFU pipe, and P is rounded to bf16 (2^-9) right after.
__device__ __forceinline__ float silu_tanh(float z) {
  const float hz = 0.5f * z;
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(hz));
  return fmaf(hz, t, hz);
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}

__global__ void __launch_bounds__(kMhThreads, 1)
    mhffn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmU, const __grid_constant__ CUtensorMap tmV,
                     const MhArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kMhBarOff);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* ku_full = bars + 2;               // [kMhKuStages]
  uint64_t* ku_empty = ku_full + kMhKuStages;  // [kMhKuStages]
  uint64_t* v_full = ku_empty + kMhKuStages;   // [kMhVStages]
  uint64_t* v_empty = v_full + kMhVStages;     // [kMhVStages]
  uint64_t* s_full = v_empty + kMhVStages;     // [2]
  uint64_t* s_empty = s_full + 2;        // [2]
  uint64_t* p_full = s_empty + 2;        // [2]
  uint64_t* p_empty = p_full + 2;        // [2]
  uint64_t* o_full = p_empty + 2;
  uint64_t* o_empty = o_full + 1;
  uint64_t* drain = o_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < kMhKuStages; ++s) {
      mbar_init(&ku_full[s], 1);
      mbar_init(&ku_empty[s], 1);
    }
    for (int s = 0; s < kMhVStages; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&s_empty[b], 128);  // one epilogue set per buffer
      mbar_init(&p_full[b], 128);
      mbar_init(&p_empty[b], 1);
    }
    mbar_init(o_full, 1);
    mbar_init(o_empty, kMhEpiThreads);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmU);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kMhTmemCols);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const WaitCtl ctl{abort_flag, args.status, args.wait_limit_ns};
  const int rows_per_head = args.E * args.de;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t gc = 0;  // chunks loaded so far (all units)
      int lu = 0;       // units so far
      bool ok = true;
      for (int unit = blockIdx.x; ok && unit < args.n_units; unit += gridDim.x, ++lu) {
        const int h = unit / args.n_tt, tt = unit - h * args.n_tt;
        if (!mbar_wait(q_empty, (lu & 1) ^ 1u, ctl)) { ok = false; break; }
        mbar_arrive_expect_tx(q_full, kMhQBytes);
        tma_load_2d(smem, &tmQ, h * kMhDh, tt * kMhTile, q_full);
        tma_load_2d(smem + kMhQBytes / 2, &tmQ, h * kMhDh + 64, tt * kMhTile, q_full);
        for (int c = 0; c < args.nch; ++c, ++gc) {
          const int row = h * rows_per_head + c * kMhChunk;
          const int s = gc % kMhKuStages;
          if (!mbar_wait(&ku_empty[s], ((gc / kMhKuStages) & 1u) ^ 1u, ctl)) { ok = false; break; }
          uint8_t* ku = smem + kMhKuOff + s * kMhKuBytes;
          mbar_arrive_expect_tx(&ku_full[s], kMhKuBytes);
          // [K | U] rows of the chunk per 64-wide d_h half: one N = 128 B operand for both
          tma_load_2d(ku + 0 * kMhBox, &tmK, 0, row, &ku_full[s]);
          tma_load_2d(ku + 1 * kMhBox, &tmU, 0, row, &ku_full[s]);
          tma_load_2d(ku + 2 * kMhBox, &tmK, 64, row, &ku_full[s]);
          tma_load_2d(ku + 3 * kMhBox, &tmU, 64, row, &ku_full[s]);
          const int sv = gc % kMhVStages;
          if (!mbar_wait(&v_empty[sv], ((gc / kMhVStages) & 1u) ^ 1u, ctl)) { ok = false; break; }
          uint8_t* vs = smem + kMhVOff + sv * kMhVBytes;
          mbar_arrive_expect_tx(&v_full[sv], kMhVBytes);
          tma_load_2d(vs, &tmV, 0, row, &v_full[sv]);
          tma_load_2d(vs + kMhBox, &tmV, 64, row, &v_full[sv]);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ UMMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdescS = idesc_bf16(kMhTile, 2 * kMhChunk, 0, 0);  // [g | u]
      constexpr uint32_t kIdescPV = idesc_bf16(kMhTile, kMhDh, 0, 1);
      const uint32_t q_addr = smem_u32(smem);
      const uint32_t p_addr = smem_u32(smem + kMhPOff);
      const uint32_t ku_addr = smem_u32(smem + kMhKuOff);
      const uint32_t v_addr = smem_u32(smem + kMhVOff);
      uint32_t gc = 0;
      int lu = 0;
      bool ok = true, issued = false;
      // O += P_g V_g for global chunk g (first: the unit's first chunk, which starts O afresh)
      auto pv = [&](uint32_t g, bool first, int unit_local) -> bool {
        const uint32_t pb = g & 1u;
        if (!mbar_wait(&p_full[pb], (g >> 1) & 1u, ctl)) return false;
        if (first && !mbar_wait(o_empty, (unit_local & 1) ^ 1u, ctl)) return false;
        const uint32_t sv = g % kMhVStages;
        if (!mbar_wait(&v_full[sv], (g / kMhVStages) & 1u, ctl)) return false;
        tc_fence_after();
        const uint32_t vst = v_addr + sv * kMhVBytes;
#pragma unroll
        for (int k = 0; k < kMhChunk / 16; ++k)
          umma_bf16(tmem_base, smem_desc_sw128(p_addr + pb * kMhPBytes + k * 32, 16, 1024),
                    smem_desc_sw128(vst + k * 2048, kMhBox, 1024), kIdescPV,
                    (!first || k != 0) ? 1u : 0u);
        umma_commit(&p_empty[pb]);
        umma_commit(&v_empty[sv]);
        return true;
      };
      for (int unit = blockIdx.x; ok && unit < args.n_units; unit += gridDim.x, ++lu) {
        if (!mbar_wait(q_full, lu & 1, ctl)) { ok = false; break; }
        tc_fence_after();
        const uint32_t gcb = gc;
        for (int c = 0; c < args.nch; ++c, ++gc) {
          const uint32_t s = gc % kMhKuStages;
          if (!mbar_wait(&ku_full[s], (gc / kMhKuStages) & 1u, ctl)) { ok = false; break; }
          const uint32_t sb = gc & 1u;
          if (!mbar_wait(&s_empty[sb], ((gc >> 1) & 1u) ^ 1u, ctl)) { ok = false; break; }
          tc_fence_after();
          const uint32_t kst = ku_addr + s * kMhKuBytes;
          const uint32_t d_s = tmem_base + 128 + sb * 128;
#pragma unroll
          for (int kb = 0; kb < 2; ++kb) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint64_t qd = smem_desc_sw128(q_addr + kb * (kMhQBytes / 2) + k * 32, 16, 1024);
              umma_bf16(d_s, qd, smem_desc_sw128(kst + kb * 2 * kMhBox + k * 32, 16, 1024), kIdescS,
                        (kb | k) != 0 ? 1u : 0u);
            }
          }
          umma_commit(&s_full[sb]);
          umma_commit(&ku_empty[s]);
          if (c == args.nch - 1) umma_commit(q_empty);  // Q no longer read in this unit
          issued = true;
          if (c >= 2 && !pv(gc - 2, c == 2, lu)) { ok = false; break; }
        }
        if (!ok) break;
        for (int c = args.nch >= 2 ? args.nch - 2 : 0; c < args.nch; ++c)
          if (!pv(gcb + c, c == 0, lu)) { ok = false; break; }
        if (!ok) break;
        umma_commit(o_full);
      }
      if (!ok && issued) {
        umma_commit(drain);
        WaitCtl quick{abort_flag, args.status, 100000000ull};
        volatile int no_abort = 0;
        quick.abort = &no_abort;
        mbar_wait(drain, 0, quick);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue warps 2..9
    const int q = warp & 3;            // TMEM lane quadrant this warp may access
    const int set = (warp - 2) >> 2;   // chunks with (global chunk index & 1) == set; O columns
    const int row = q * 32 + lane;
    const uint32_t t_lane = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    const uint32_t pbuf = smem_u32(smem + kMhPOff) + set * kMhPBytes;
    const int64_t o_ld = (int64_t)args.H * kMhDh;
    uint32_t gc = 0;
    int lu = 0;
    bool ok = true;
    for (int unit = blockIdx.x; ok && unit < args.n_units; unit += gridDim.x, ++lu) {
      const int h = unit / args.n_tt, tt = unit - h * args.n_tt;
      const int token = tt * kMhTile + row;
      const bool tok_ok = token < args.T;
      const float* rrow = args.r + ((int64_t)(tok_ok ? token : 0) * args.H + h) * args.E;
      for (int c = 0; c < args.nch; ++c, ++gc) {
        if ((int)(gc & 1u) != set) continue;
        const uint32_t use = gc >> 1;
        const bool ready = mbar_wait(&s_full[set], use & 1u, ctl);
        __syncwarp();  // tcgen05.ld is warp-collective: reconverge after the per-thread wait
        if (!__all_sync(0xffffffffu, ready)) { ok = false; break; }
        tc_fence_after();
        const uint32_t ts = t_lane + 128 + set * 128;
        const float rv = tok_ok ? rrow[c / args.ch_per_sub] : 0.f;
        uint32_t w[32];  // this row's 64 P values as bf16 pairs
        float g[32], u[32];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          tmem_ld32(ts + hh * 32, g);
          tmem_ld32(ts + kMhChunk + hh * 32, u);
          tmem_ld_wait_regs(g);
          pin_regs(u);
          if (hh == 1) {
            tc_fence_before();
            mbar_arrive(&s_empty[set]);  // the whole S buffer is in registers or P
          }
#pragma unroll
          for (int j = 0; j < 16; ++j)
            w[hh * 16 + j] = pack_bf16x2(silu_tanh(g[2 * j]) * u[2 * j] * rv,
                                         silu_tanh(g[2 * j + 1]) * u[2 * j + 1] * rv);
        }
        if (!mbar_wait(&p_empty[set], (use & 1u) ^ 1u, ctl)) { ok = false; break; }
#pragma unroll
        for (int c16 = 0; c16 < 8; ++c16)
          st_shared_v4(pbuf + p_offset(row, c16), w[4 * c16], w[4 * c16 + 1], w[4 * c16 + 2],
                       w[4 * c16 + 3]);
        fence_proxy_async_smem();  // make P visible to the tensor core's reads
        mbar_arrive(&p_full[set]);
      }
      if (!ok) break;
      const bool ready = mbar_wait(o_full, lu & 1, ctl);
      __syncwarp();
      if (!__all_sync(0xffffffffu, ready)) { ok = false; break; }
      tc_fence_after();
      __nv_bfloat16* orow = args.o + (int64_t)token * o_ld + h * kMhDh;
#pragma unroll 1
      for (int cc = set * 64; cc < set * 64 + 64; cc += 32) {
        float ov[32];
        tmem_ld32(t_lane + cc, ov);
        tmem_ld_wait_regs(ov);
        if (tok_ok) {
#pragma unroll
          for (int v = 0; v < 4; ++v)
            *reinterpret_cast<uint4*>(orow + cc + 8 * v) =
                make_uint4(pack_bf16x2(ov[8 * v], ov[8 * v + 1]), pack_bf16x2(ov[8 * v + 2], ov[8 * v + 3]),
                           pack_bf16x2(ov[8 * v + 4], ov[8 * v + 5]), pack_bf16x2(ov[8 * v + 6], ov[8 * v + 7]));
        }
      }
      tc_fence_before();
      mbar_arrive(o_empty);
    }
  }

  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, kMhTmemCols);
  }
}

}  // namespace
}  // namespace swf

// ------------------------------------------------------------------ host side

using namespace swf;

extern "C" swf_status flash_mhffn_fwd(const void* q, const void* w_k, const void* w_u,
                                      const void* w_v, const float* router, void* o, int64_t T,
                                      int32_t num_heads, int32_t head_dim, int32_t num_sub,
                                      int32_t sub_dim, swf_dtype dtype, void* stream) {
  if (!q || !w_k || !w_u || !w_v || !router || !o) return SWF_ERR_INVALID_ARG;
  if (T <= 0 || num_heads <= 0 || head_dim <= 0 || num_sub <= 0 || sub_dim <= 0)
    return SWF_ERR_INVALID_ARG;
  if (dtype != SWF_BF16 && dtype != SWF_F32) return SWF_ERR_INVALID_ARG;
  if (dtype != SWF_BF16 || head_dim != kMhDh || sub_dim % kMhChunk != 0) return SWF_ERR_UNSUPPORTED;
  const int64_t rows = (int64_t)num_heads * num_sub * sub_dim;  // K, U, V rows
  if (T > INT32_MAX / 2 || rows > INT32_MAX / 2 || (int64_t)num_heads * kMhDh > (1 << 20) ||
      (int64_t)num_sub * sub_dim > (1 << 24) || T * (int64_t)num_heads > INT32_MAX / 2)
    return SWF_ERR_UNSUPPORTED;
  for (const void* p : std::initializer_list<const void*>{q, w_k, w_u, w_v, router, o})
    if (!aligned16(p)) return SWF_ERR_ALIGNMENT;
  DevCtx ctx;
  swf_status s = get_ctx(&ctx);
  if (s != SWF_OK) return s;
  CUtensorMap tq, tk, tu, tv;
  const uint64_t qcols = (uint64_t)num_heads * kMhDh;
  if (!encode_tmap_bf16(&tq, q, qcols, T, qcols, 64, kMhTile) ||
      !encode_tmap_bf16(&tk, w_k, kMhDh, rows, kMhDh, 64, 64) ||
      !encode_tmap_bf16(&tu, w_u, kMhDh, rows, kMhDh, 64, 64) ||
      !encode_tmap_bf16(&tv, w_v, kMhDh, rows, kMhDh, 64, 64))
    return SWF_ERR_LAUNCH;
  MhArgs a{};
  a.T = (int)T;
  a.H = num_heads;
  a.E = num_sub;
  a.de = sub_dim;
  a.n_tt = (int)((T + kMhTile - 1) / kMhTile);
  a.n_units = a.n_tt * num_heads;
  a.nch = num_sub * sub_dim / kMhChunk;
  a.ch_per_sub = sub_dim / kMhChunk;
  a.r = router;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.status = ctx.status;
  a.wait_limit_ns = kDefaultWaitNs;
  if (cudaFuncSetAttribute(mhffn_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           kMhSmemBytes) != cudaSuccess)
    return SWF_ERR_LAUNCH;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int grid = std::min(a.n_units, ctx.num_sms);
  ProfScope prof(SWF_K_MHFFN_FWD, st);
  mhffn_fwd_kernel<<<grid, kMhThreads, kMhSmemBytes, st>>>(tq, tk, tu, tv, a);
  return cudaGetLastError() == cudaSuccess ? SWF_OK : SWF_ERR_LAUNCH;
}
