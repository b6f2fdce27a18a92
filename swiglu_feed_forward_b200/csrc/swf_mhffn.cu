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
//   per work unit (head h, 256 tokens on a pair of CTAs), for each 64-column chunk c of the
//   head's E*d_e sub-network columns:
//     [S_g | S_u] = Q [K_c ; U_c]^T   (tcgen05 cta_group::2, M=256 N=128 K=128, fp32 in TMEM)
//     P   = SiLU(S_g) * S_u * R_e     (epilogue warps, bf16 into shared memory, two buffers)
//     O  += P V_c                     (tcgen05 cta_group::2, M=256 N=128 K=64, A from smem)
//   then O (128 TMEM columns per CTA) -> bf16 -> HBM.
//
// Pair mode: the two CTAs of a cluster each hold 128 tokens of Q and of P and half of each B
// operand (the even CTA the K rows and V's first 64 d_h columns, the odd CTA the U rows and V's
// other 64), so each SM stages half of the weight bytes; the even CTA issues every MMA, both
// CTAs' TMA loads complete on its barriers, and the MMA commits arrive on both CTAs' barriers.
// Warp roles per CTA: warp 0 lane 0 issues the TMA loads of Q (once per unit) and of the K|U
// chunk ring, warp 3 lane 0 those of the V chunk ring; warp 1 owns TMEM and, in the even CTA,
// lane 0 issues the S products; warp 2 lane 0 (even CTA) issues the PV products; warps 4..11
// turn S into P and drain O as two sets of four
// warps (one per TMEM lane quadrant) that take alternate chunks.  A thread issues about one
// tcgen05.mma per 60-90 cycles, close to the 64 tensor cycles of each product here, so the S and
// PV products come from two threads.  No TMA load uses multicast.  Every wait is bounded (status word + abort flag, as in the GEMM template).
#include <algorithm>
#include <initializer_list>

#include "swf_internal.h"
#include "swf_launch.cuh"
#include "swf_ptx.cuh"

namespace swf {
namespace {

constexpr int kMhTile = 128;     // tokens per CTA and unit
constexpr int kMhDh = 128;       // head width d_h
constexpr int kMhChunk = 64;     // sub-network columns per chunk
constexpr int kMhKuStages = 4;   // K|U chunk stages (free once the chunk's S products are done)
constexpr int kMhVStages = 6;    // V chunk stages (free once its PV product is done)
constexpr int kMhEpiWarps = 8;   // two sets of four (one warp per TMEM lane quadrant each)
constexpr int kMhThreads = 128 + 32 * kMhEpiWarps;  // 2 producers, S and PV issuers, epilogue
constexpr int kMhBox = 64 * 64 * 2;                 // one 64 x 64 bf16 TMA box (8 KB)
constexpr int kMhQBytes = 2 * kMhTile * 64 * 2;     // Q tile: two 128 x 64 boxes
constexpr int kMhKuBytes = 2 * kMhBox;              // this CTA's half of [K; U]: two d_h boxes
constexpr int kMhVBytes = kMhBox;                   // this CTA's 64 d_h columns of V
constexpr int kMhPBytes = kMhTile * kMhChunk * 2;   // one P buffer (128 x 64 bf16)
constexpr int kMhKuOff = kMhQBytes;
constexpr int kMhVOff = kMhKuOff + kMhKuStages * kMhKuBytes;
constexpr int kMhPOff = kMhVOff + kMhVStages * kMhVBytes;
constexpr int kMhPBufs = 4;                         // P buffers: two per epilogue set
constexpr int kMhBarOff = kMhPOff + kMhPBufs * kMhPBytes;
constexpr int kMhSmemBytes = kMhBarOff + 512 + 1024;  // barriers + alignment slack
static_assert(kMhSmemBytes <= 232448, "shared memory per CTA");
constexpr int kMhSBufs = 3;                           // S buffers (TMEM: O 128 + 3 x 128 = 512)
constexpr int kMhTmemCols = 512;                      // O [0,128); S buffers at 128, 256, 384

struct MhArgs {
  int T, H, E, de;
  int n_tt;         // 128-token tiles
  int n_pt;         // pairs of token tiles (one per cluster and unit)
  int n_units;      // n_pt * H, head-major
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

__device__ constexpr float2 kHalf2 = {0.5f, 0.5f};
__device__ constexpr float2 kMinusHalf2 = {-0.5f, -0.5f};

// SiLU(g) * u * r for two columns, as bf16x2.  SiLU(g) = g sigmoid(g) with sigmoid(g) =
// (1 + tanh(g / 2)) / 2, i.e. h + h tanh(h) with h = g / 2: one MUFU operation (tanh.approx.f32,
// relative error about 2^-11) instead of an exponential and a reciprocal, the rest in Blackwell's
// paired fp32 operations (mul/fma .f32x2, IEEE round-to-nearest like the scalar forms).  The
// result is rounded to bf16 (2^-9) right after.
__device__ __forceinline__ uint32_t silu_mul_pair(float ga, float gb, float ua, float ub, float2 r2) {
  const float2 h2 = __fmul2_rn(make_float2(ga, gb), kHalf2);
  float2 th;
  asm("tanh.approx.f32 %0, %1;" : "=f"(th.x) : "f"(h2.x));
  asm("tanh.approx.f32 %0, %1;" : "=f"(th.y) : "f"(h2.y));
  const float2 v = __fmul2_rn(__fmul2_rn(__ffma2_rn(h2, th, h2), make_float2(ua, ub)), r2);
  return pack_bf16x2(v.x, v.y);
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}

// One arrival per warp on `bar` of the even CTA (locally there, remotely from the odd CTA), after
// every lane of the warp has reached this point (its TMEM reads waited, its P stores fenced).
// Every signal sent this way releases data of the arriving CTA's own SM (see mbar_arrive_remote).
__device__ __forceinline__ void warp_arrive_lead(uint64_t* bar, uint32_t rank, int lane) {
  __syncwarp();
  if (lane == 0) {
    if (rank == 0) mbar_arrive(bar);
    else mbar_arrive_remote(map_to_rank(smem_u32(bar), 0));
  }
}

// UMMA shared-memory descriptor (sm_100 format) of a K-major operand in the 32-byte-swizzle
// layout: rows of 32 bytes (16 bf16 of K, one K16 step), 16-byte chunk c of row r at chunk
// position c ^ ((r >> 2) & 1), 8-row groups `sbo_bytes` apart (layout type 6 at bits 61..63; the
// leading byte offset is not used by swizzled K-major layouts).  Tiles are 256-byte aligned so
// the swizzle phase is that of the address.
__device__ __forceinline__ uint64_t smem_desc_sw32(uint32_t saddr, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(1u) << 16;
  d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= 1ull << 46;
  d |= 6ull << 61;
  return d;
}

// 32 lanes x 16 consecutive fp32 columns (thread i gets lane taddr.lane + i), and the wait that
// ties three such loads' registers to it.
__device__ __forceinline__ void tmem_ld16x(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_wait16x3(float (&x)[16], float (&y)[16], float (&z)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int j = 0; j < 16; ++j) asm volatile("" : "+f"(x[j]), "+f"(y[j]), "+f"(z[j])::"memory");
}

// UMMA shared-memory descriptor moved by `bytes` (a multiple of 16): the start address is the
// low 14-bit field in 16-byte units, which stays below 2^14 for any address in the 227 KB.
__device__ __forceinline__ uint64_t desc_add(uint64_t desc, uint32_t bytes) { return desc + (bytes >> 4); }

// After an aborted wait: lets this thread's MMAs in flight finish (bounded) before the CTA leaves.
__device__ __forceinline__ void drain_mma(uint64_t* bar, volatile int* abort_flag, int* status) {
  umma_commit_pair(bar, 1);
  WaitCtl quick{abort_flag, status, 100000000ull};
  volatile int no_abort = 0;
  quick.abort = &no_abort;
  mbar_wait(bar, 0, quick);
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
  uint64_t* ku_full = bars + 2;                // [kMhKuStages]
  uint64_t* ku_empty = ku_full + kMhKuStages;  // [kMhKuStages]
  uint64_t* v_full = ku_empty + kMhKuStages;   // [kMhVStages]
  uint64_t* v_empty = v_full + kMhVStages;     // [kMhVStages]
  uint64_t* s_full = v_empty + kMhVStages;     // [kMhSBufs]
  uint64_t* s_empty = s_full + kMhSBufs;       // [kMhSBufs]
  uint64_t* p_full = s_empty + kMhSBufs;       // [kMhPBufs]
  uint64_t* p_empty = p_full + kMhPBufs;       // [kMhPBufs]
  uint64_t* o_full = p_empty + kMhPBufs;
  uint64_t* o_empty = o_full + 1;
  uint64_t* drain = o_empty + 1;  // [2]: one per issuing thread
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  static_assert((2 + 2 * kMhKuStages + 2 * kMhVStages + 2 * kMhSBufs + 2 * kMhPBufs + 4) * 8 + 8 <= 512,
                "barrier block");

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int cl = static_cast<int>(blockIdx.x >> 1), n_cl = static_cast<int>(gridDim.x >> 1);
  if (threadIdx.x == 0) {
    // arrival counts are those of the even CTA's barriers, the only ones waited on with them
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
    for (int b = 0; b < kMhSBufs; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&s_empty[b], 2 * 4);  // one arrival per warp of a set, in both CTAs
    }
    for (int b = 0; b < kMhPBufs; ++b) {
      mbar_init(&p_full[b], 2 * 4);
      mbar_init(&p_empty[b], 1);
    }
    mbar_init(o_full, 1);
    mbar_init(o_empty, 2 * kMhEpiWarps);
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(rank == 0 ? &tmK : &tmU);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, kMhTmemCols);
    tmem_relinquish_pair();
  }
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before any remote signal
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const WaitCtl ctl{abort_flag, args.status, args.wait_limit_ns};
  const int rows_per_head = args.E * args.de;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      const uint32_t q_full_lead = map_to_rank(smem_u32(q_full), 0);
      const uint32_t ku_full_lead = map_to_rank(smem_u32(ku_full), 0);
      const CUtensorMap* tm_b = rank == 0 ? &tmK : &tmU;  // this CTA's half of [K; U]
      uint32_t gc = 0;  // chunks loaded so far (all units)
      int lu = 0;       // units so far
      bool ok = true;
      for (int unit = cl; ok && unit < args.n_units; unit += n_cl, ++lu) {
        const int h = unit / args.n_pt, pt = unit - h * args.n_pt;
        const int tt = 2 * pt + static_cast<int>(rank);  // may lie past the last tile: zero rows
        if (!mbar_wait(q_empty, (lu & 1) ^ 1u, ctl)) { ok = false; break; }
        if (rank == 0) mbar_arrive_expect_tx(q_full, 2 * kMhQBytes);
        tma_load_2d_pair(smem, &tmQ, h * kMhDh, tt * kMhTile, q_full_lead);
        tma_load_2d_pair(smem + kMhQBytes / 2, &tmQ, h * kMhDh + 64, tt * kMhTile, q_full_lead);
        for (int c = 0; c < args.nch; ++c, ++gc) {
          const int row = h * rows_per_head + c * kMhChunk;
          const int s = gc % kMhKuStages;
          if (!mbar_wait(&ku_empty[s], ((gc / kMhKuStages) & 1u) ^ 1u, ctl)) { ok = false; break; }
          uint8_t* ku = smem + kMhKuOff + s * kMhKuBytes;
          if (rank == 0) mbar_arrive_expect_tx(&ku_full[s], 2 * kMhKuBytes);
          tma_load_2d_pair(ku, tm_b, 0, row, ku_full_lead + s * 8);
          tma_load_2d_pair(ku + kMhBox, tm_b, 64, row, ku_full_lead + s * 8);
        }
      }
    }
  } else if (warp == 3) {
    // ------------------------------------------------------------ V producer (both CTAs)
    // A ring of its own: V chunks wait only for the PV products, K|U chunks only for the S
    // products, so neither ring holds the other back.
    if (lane == 0) {
      const uint32_t v_full_lead = map_to_rank(smem_u32(v_full), 0);
      uint32_t gc = 0;
      bool ok = true;
      for (int unit = cl; ok && unit < args.n_units; unit += n_cl) {
        const int h = unit / args.n_pt;
        for (int c = 0; c < args.nch; ++c, ++gc) {
          const int row = h * rows_per_head + c * kMhChunk;
          const int sv = gc % kMhVStages;
          if (!mbar_wait(&v_empty[sv], ((gc / kMhVStages) & 1u) ^ 1u, ctl)) { ok = false; break; }
          if (rank == 0) mbar_arrive_expect_tx(&v_full[sv], 2 * kMhVBytes);
          tma_load_2d_pair(smem + kMhVOff + sv * kMhVBytes, &tmV, static_cast<int>(rank) * 64, row,
                           v_full_lead + sv * 8);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ S issuer (even CTA)
    if (lane == 0 && rank == 0) {
      constexpr uint32_t kIdescS = idesc_bf16(2 * kMhTile, 2 * kMhChunk, 0, 0);  // [g | u]
      // descriptors of the first stage of each operand; every MMA moves them by a constant
      const uint64_t q_desc = smem_desc_sw128(smem_u32(smem), 16, 1024);
      const uint64_t ku_desc = smem_desc_sw128(smem_u32(smem + kMhKuOff), 16, 1024);
      uint32_t gc = 0;
      int lu = 0;
      bool ok = true, issued = false;
      for (int unit = cl; ok && unit < args.n_units; unit += n_cl, ++lu) {
        if (!mbar_wait(q_full, lu & 1, ctl)) { ok = false; break; }
        tc_fence_after();
        for (int c = 0; c < args.nch; ++c, ++gc) {
          const uint32_t s = gc % kMhKuStages;
          if (!mbar_wait(&ku_full[s], (gc / kMhKuStages) & 1u, ctl)) { ok = false; break; }
          const uint32_t sb = gc % kMhSBufs;
          if (!mbar_wait(&s_empty[sb], ((gc / kMhSBufs) & 1u) ^ 1u, ctl)) { ok = false; break; }
          tc_fence_after();
          const uint64_t kd = desc_add(ku_desc, s * kMhKuBytes);
          const uint32_t d_s = tmem_base + 128 + sb * 128;
#pragma unroll
          for (int kb = 0; kb < 2; ++kb) {
#pragma unroll
            for (int k = 0; k < 4; ++k)
              umma_bf16_pair(d_s, desc_add(q_desc, kb * (kMhQBytes / 2) + k * 32),
                             desc_add(kd, kb * kMhBox + k * 32), kIdescS, (kb | k) != 0 ? 1u : 0u);
          }
          umma_commit_pair(&s_full[sb], 3);
          umma_commit_pair(&ku_empty[s], 3);
          if (c == args.nch - 1) umma_commit_pair(q_empty, 3);  // Q no longer read in this unit
          issued = true;
        }
      }
      if (!ok && issued) drain_mma(&drain[0], abort_flag, args.status);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ PV issuer (even CTA)
    // Issues O += P_c V_c as soon as the epilogue has written P_c; its products write only O and
    // read only P and V, so the two issuing threads share no state.
    if (lane == 0 && rank == 0) {
      constexpr uint32_t kIdescPV = idesc_bf16(2 * kMhTile, kMhDh, 0, 1);
      const uint64_t p_desc = smem_desc_sw128(smem_u32(smem + kMhPOff), 16, 1024);
      const uint64_t v_desc = smem_desc_sw128(smem_u32(smem + kMhVOff), kMhBox, 1024);
      uint32_t gc = 0;
      int lu = 0;
      bool ok = true, issued = false;
      for (int unit = cl; ok && unit < args.n_units; unit += n_cl, ++lu) {
        for (int c = 0; c < args.nch; ++c, ++gc) {
          const uint32_t pb = gc % kMhPBufs;
          if (!mbar_wait(&p_full[pb], (gc / kMhPBufs) & 1u, ctl)) { ok = false; break; }
          if (c == 0 && !mbar_wait(o_empty, (lu & 1) ^ 1u, ctl)) { ok = false; break; }
          const uint32_t sv = gc % kMhVStages;
          if (!mbar_wait(&v_full[sv], (gc / kMhVStages) & 1u, ctl)) { ok = false; break; }
          tc_fence_after();
          const uint64_t pd = desc_add(p_desc, pb * kMhPBytes);
          const uint64_t vd = desc_add(v_desc, sv * kMhVBytes);
#pragma unroll
          for (int k = 0; k < kMhChunk / 16; ++k)
            umma_bf16_pair(tmem_base, desc_add(pd, k * 32), desc_add(vd, k * 2048), kIdescPV,
                           (c != 0 || k != 0) ? 1u : 0u);
          umma_commit_pair(&p_empty[pb], 3);
          umma_commit_pair(&v_empty[sv], 3);
          issued = true;
        }
        if (!ok) break;
        umma_commit_pair(o_full, 3);
      }
      if (!ok && issued) drain_mma(&drain[1], abort_flag, args.status);
    }
  } else {
    // ------------------------------------------------------------ epilogue warps 4..11
    const int q = warp & 3;            // TMEM lane quadrant this warp may access
    const int set = (warp - 4) >> 2;   // chunks with (global chunk index & 1) == set; O columns
    const int row = q * 32 + lane;
    const uint32_t t_lane = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    const uint32_t p_base = smem_u32(smem + kMhPOff);
    const int64_t o_ld = (int64_t)args.H * kMhDh;
    uint32_t gc = 0;
    int lu = 0;
    bool ok = true;
    for (int unit = cl; ok && unit < args.n_units; unit += n_cl, ++lu) {
      const int h = unit / args.n_pt, pt = unit - h * args.n_pt;
      const int token = (2 * pt + static_cast<int>(rank)) * kMhTile + row;
      const bool tok_ok = token < args.T;
      const float* rrow = args.r + ((int64_t)(tok_ok ? token : 0) * args.H + h) * args.E;
      for (int c = 0; c < args.nch; ++c, ++gc) {
        if ((int)(gc & 1u) != set) continue;
        const uint32_t pb = gc % kMhPBufs;  // the set's two buffers in turn
        const uint32_t sb = gc % kMhSBufs;
        const bool ready = mbar_wait(&s_full[sb], (gc / kMhSBufs) & 1u, ctl);
        __syncwarp();  // tcgen05.ld is warp-collective: reconverge after the per-thread wait
        if (!__all_sync(0xffffffffu, ready)) { ok = false; break; }
        tc_fence_after();
        const uint32_t ts = t_lane + 128 + sb * 128;
        const float rv = tok_ok ? rrow[c / args.ch_per_sub] : 0.f;
        uint32_t w[32];  // this row's 64 P values as bf16 pairs
        float g0[32], u0[32], g1[32], u1[32];
        tmem_ld32(ts, g0);
        tmem_ld32(ts + kMhChunk, u0);
        tmem_ld32(ts + 32, g1);
        tmem_ld32(ts + kMhChunk + 32, u1);
        tmem_ld_wait_regs(g0);
        pin_regs(u0);
        pin_regs(g1);
        pin_regs(u1);
        tc_fence_before();
        warp_arrive_lead(&s_empty[sb], rank, lane);  // the S buffer is in registers
        const float2 rv2 = make_float2(rv, rv);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          w[j] = silu_mul_pair(g0[2 * j], g0[2 * j + 1], u0[2 * j], u0[2 * j + 1], rv2);
          w[16 + j] = silu_mul_pair(g1[2 * j], g1[2 * j + 1], u1[2 * j], u1[2 * j + 1], rv2);
        }
        const bool p_free = mbar_wait(&p_empty[pb], ((gc / kMhPBufs) & 1u) ^ 1u, ctl);
        if (!__all_sync(0xffffffffu, p_free)) { ok = false; break; }  // warp-uniform exit
#pragma unroll
        for (int c16 = 0; c16 < 8; ++c16)
          st_shared_v4(p_base + pb * kMhPBytes + p_offset(row, c16), w[4 * c16], w[4 * c16 + 1], w[4 * c16 + 2],
                       w[4 * c16 + 3]);
        fence_proxy_async_smem();  // make P visible to the tensor core's reads
        warp_arrive_lead(&p_full[pb], rank, lane);
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
      warp_arrive_lead(o_empty, rank, lane);
    }
  }

  __syncthreads();
  cluster_sync();  // the pair's MMAs and TMEM reads are all done
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kMhTmemCols);
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
  a.n_pt = (a.n_tt + 1) / 2;
  a.n_units = a.n_pt * num_heads;
  a.nch = num_sub * sub_dim / kMhChunk;
  a.ch_per_sub = sub_dim / kMhChunk;
  a.r = router;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.status = ctx.status;
  a.wait_limit_ns = kDefaultWaitNs;
  if (cudaFuncSetAttribute(mhffn_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           kMhSmemBytes) != cudaSuccess)
    return SWF_ERR_LAUNCH;
  const int clusters = std::min(a.n_units, ctx.num_sms / 2);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * clusters, 1, 1);
  cfg.blockDim = dim3(kMhThreads, 1, 1);
  cfg.dynamicSmemBytes = kMhSmemBytes;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  ProfScope prof(SWF_K_MHFFN_FWD, cfg.stream);
  if (cudaLaunchKernelEx(&cfg, mhffn_fwd_kernel, tq, tk, tu, tv, a) != cudaSuccess)
    return SWF_ERR_LAUNCH;
  return cudaGetLastError() == cudaSuccess ? SWF_OK : SWF_ERR_LAUNCH;
}

namespace swf {
namespace {

// Router rows of the block's prologue ("Overview": sigmoid-normalised router weights).  The
// router GEMM leaves s = sigmoid(logits) in each token's row of N = H * E values; one warp per
// token stages the row in shared memory, one lane per head sums its E values in index order, and
// the row goes back out with coalesced accesses.
constexpr int kRouterRows = 8;  // tokens (warps) per block

//   R = s / sum_e s, in place
__global__ void router_norm_kernel(float* __restrict__ r, int64_t T, int N, int E) {
  __shared__ float sv[kRouterRows][256];
  __shared__ float inv[kRouterRows][256];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t t = (int64_t)blockIdx.x * kRouterRows + w;
  if (t >= T) return;  // warp-uniform; the block never synchronises
  float* row = r + t * N;
  for (int j = lane; j < N; j += 32) sv[w][j] = row[j];
  __syncwarp();
  for (int h = lane; h < N / E; h += 32) {
    float sum = 0.f;
    for (int e = 0; e < E; ++e) sum += sv[w][h * E + e];
    inv[w][h] = 1.0f / sum;
  }
  __syncwarp();
  for (int j = lane; j < N; j += 32) row[j] = sv[w][j] * inv[w][j / E];
}

//   dl = s (1 - s) (dR - sum_e dR R) / S  with S = sum_e s, R = s / S  -> bf16 out (row stride
//   ld_out), from s (rows of `sig`, N values) and dR (rows of N values)
__global__ void router_bwd_kernel(const float* __restrict__ sig, const float* __restrict__ dr, int64_t T,
                                  int N, int E, __nv_bfloat16* __restrict__ out, int64_t ld_out) {
  __shared__ float sv[kRouterRows][256];
  __shared__ float dv[kRouterRows][256];
  __shared__ float hinv[kRouterRows][256];
  __shared__ float hdot[kRouterRows][256];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t t = (int64_t)blockIdx.x * kRouterRows + w;
  if (t >= T) return;  // warp-uniform; the block never synchronises
  for (int j = lane; j < N; j += 32) {
    sv[w][j] = sig[t * N + j];
    dv[w][j] = dr[t * N + j];
  }
  __syncwarp();
  for (int h = lane; h < N / E; h += 32) {
    float sum = 0.f;
    for (int e = 0; e < E; ++e) sum += sv[w][h * E + e];
    const float invS = 1.0f / sum;
    float cdot = 0.f;
    for (int e = 0; e < E; ++e) cdot = fmaf(dv[w][h * E + e], sv[w][h * E + e] * invS, cdot);
    hinv[w][h] = invS;
    hdot[w][h] = cdot;
  }
  __syncwarp();
  __nv_bfloat16* orow = out + t * ld_out;
  for (int j = lane; j < N; j += 32) {
    const float s_ = sv[w][j];
    orow[j] = __float2bfloat16_rn(s_ * (1.f - s_) * (dv[w][j] - hdot[w][j / E]) * hinv[w][j / E]);
  }
}

}  // namespace
}  // namespace swf

// The block's prologue ("Overview": Q is the per-head RMS-normalised projection of the input, R
// the sigmoid-normalised router weights), as two tcgen05 GEMMs with fused epilogues:
//   q[t, h*128 + i] = z_h[i] / sqrt(mean_i z_h[i]^2 + eps) * q_gain[i],  z = x w_q^T
//   router[t, h, e] = sigmoid(l[h*E + e]) / sum_e' sigmoid(l[h*E + e']),  l = x w_r^T
extern "C" swf_status flash_mhffn_prologue(const void* x, const void* w_q, const float* q_gain,
                                           const void* w_r, void* q, float* router, int64_t T,
                                           int64_t d_model, int32_t num_heads, int32_t head_dim,
                                           int32_t num_sub, float eps, swf_dtype dtype,
                                           void* stream) {
  if (!x || !w_q || !w_r || !q || !router) return SWF_ERR_INVALID_ARG;
  if (T <= 0 || d_model <= 0 || num_heads <= 0 || head_dim <= 0 || num_sub <= 0 || !(eps >= 0.f))
    return SWF_ERR_INVALID_ARG;
  if (dtype != SWF_BF16 && dtype != SWF_F32) return SWF_ERR_INVALID_ARG;
  if (dtype != SWF_BF16 || head_dim != kMhDh || d_model % 16 != 0 || num_heads * num_sub > 256 ||
      T > INT32_MAX / 2 || d_model > (1 << 20) || (int64_t)num_heads * kMhDh > (1 << 20))
    return SWF_ERR_UNSUPPORTED;
  for (const void* p : std::initializer_list<const void*>{x, w_q, w_r, q, router, q_gain})
    if (p && !aligned16(p)) return SWF_ERR_ALIGNMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t nq = (int64_t)num_heads * kMhDh, nr = (int64_t)num_heads * num_sub;
  CUtensorMap tx, tq, tr;
  if (!encode_tmap_bf16(&tx, x, d_model, T, d_model, 64, 128) ||
      !encode_tmap_bf16(&tq, w_q, d_model, nq, d_model, 64, 128) ||  // 128 rows: a CTA's half
      !encode_tmap_bf16(&tr, w_r, d_model, nr, d_model, 64, 256))
    return SWF_ERR_LAUNCH;
  // projection: with an even head count, pair (cta_group::2) tiles of 256 tokens x 256 columns
  // (two heads per epilogue row); otherwise one-CTA tiles of one head
  const bool pair = nq % 256 == 0;
  TcGemmArgs a = pair ? base_args(T, nq, 256, d_model, 2 * kTileM) : base_args(T, nq, 128, d_model);
  a.out0 = q;
  a.ld_out = nq;
  a.bias = q_gain;
  a.eps = eps;
  swf_status s =
      pair ? launch_tc_pair<256, false, false, false, kEpiHeadNorm>(SWF_K_MHFFN_PROLOGUE, tx, tq, tq,
                                                                    EpiMaps{}, a, st)
           : launch_tc<128, false, false, false, kEpiHeadNorm>(SWF_K_MHFFN_PROLOGUE, tx, tq, tq, a, st);
  if (s != SWF_OK) return s;
  TcGemmArgs b = base_args(T, nr, 256, d_model);
  b.out0 = router;
  b.ld_out = nr;
  b.group_size = num_sub;
  if ((s = launch_tc<256, false, false, false, kEpiRouter>(SWF_K_MHFFN_PROLOGUE, tx, tr, tr, b, st)) != SWF_OK)
    return s;
  ProfScope prof(SWF_K_MHFFN_PROLOGUE, st);
  router_norm_kernel<<<(unsigned)((T + kRouterRows - 1) / kRouterRows), 32 * kRouterRows, 0, st>>>(
      router, T, (int)nr, num_sub);
  return cudaGetLastError() == cudaSuccess ? SWF_OK : SWF_ERR_LAUNCH;
}

// ------------------------------------------------------------------ backward (fused per token tile)
// Gradients of L = sum(dO * O) for the block above ("Overview" formula, chain rule), per head:
//   dA  = dO V_e^T                      (the gradient reaching R_e * act)
//   dR_e = sum over the sub-network's d_e columns of dA * act,   act = SiLU(S_g) * S_u
//   dS_g = R_e dA S_u SiLU'(S_g),  dS_u = R_e dA SiLU(S_g),  P = R_e act
//   dQ  = sum_e dS_g K_e + dS_u U_e,  dK_e = dS_g^T Q,  dU_e = dS_u^T Q,  dV_e = P^T dO.
// One kernel does everything that is local to a token tile: per work unit (head, 256 tokens on a
// pair of CTAs) and per 64-column chunk c of the head's E*d_e columns it
//   recomputes [S_g | S_u] = Q [K_c ; U_c]^T and dA = dO V_c^T   (tcgen05 pair, into one of two
//     192-column TMEM buffers: S_g 64 | S_u 64 | dA 64),
//   forms dS_g, dS_u, P and the router-gradient sums in the epilogue warps (dS_g, dS_u into
//     shared memory in the operand layout, 64-byte swizzled K-major atoms; P into a staging tile),
//   accumulates dQ += dS_g K_c + dS_u U_c in TMEM (128 columns) with dS from shared memory,
//   and sends dS_g, dS_u and P to HBM by TMA stores from those shared-memory tiles (each warp its
//     own 32 x 32 boxes; per-thread global stores of rows 11 KB apart were the bottleneck).
// dA never leaves the chip; the [T, E*d_e] planes that reach HBM are dS_g | dS_u and P, the A
// operands of the weight gradients (a reduction over all tokens, run after it as split-K GEMMs).
//
// Operand placement.  The S products split each weight chunk across the pair by rows (even CTA
// K_c, odd CTA U_c, as in the forward); the dQ products split it by d_h columns (even CTA
// K_c[:, :64] and U_c[:, :64], odd CTA the other halves), so the chunk is staged twice: a ring for
// the S products and a ring for the dQ products, each 16 KB per CTA and stage.  V_c is split by
// rows (32 per CTA) for dA.  Shared memory: Q and dO 64 KB, S ring 2 x 16, V ring 2 x 8, dQ ring
// 2 x 16, two dS buffers of 32 KB, P staging 16 KB = 224 KB.
//
// Threads (640 per CTA): warp 0 lane 0 loads Q, dO (once per unit) and the S ring; warp 3 lane 0
// the V ring; warp 2 lane 0 the dQ ring and, in the even CTA, issues the dQ products; warp 1 owns
// TMEM and, in the even CTA, issues the S and dA products (a thread issues about one tcgen05.mma
// per 60-90 cycles, so the dQ products come from a second thread); warps 4..19 form dS_g, dS_u, P
// for every chunk (warp (q, qc): token rows 32q..32q+31, the chunk's columns 16qc..16qc+15;
// chunk c uses TMEM buffer c & 1 and dS buffer c & 1), and at the end of a unit they drain dQ.
// Every wait is bounded.
namespace swf {
namespace {

constexpr int kBwSuStages = 2;
constexpr int kBwVStages = 2;
constexpr int kBwDqStages = 2;
constexpr int kBwVBox = 32 * 64 * 2;          // 32 V rows x 64 d_h (4 KB)
constexpr int kBwVBytes = 2 * kBwVBox;        // this CTA's 32 rows of V_c
constexpr int kBwEpiWarps = 16;              // four per TMEM lane quadrant, 16 columns each
constexpr int kBwVWarp = 3;                  // the V-ring producer
constexpr int kBwThreads = 128 + 32 * kBwEpiWarps;
constexpr int kBwCols = kMhChunk / 4;         // columns of a chunk per epilogue warp
constexpr int kBwDsAtom = 128 * kBwCols * 2;  // 128 rows x 16 bf16 (32-byte rows): one K16 atom
constexpr int kBwDsBytes = 8 * kBwDsAtom;     // dS_g and dS_u of one chunk (2 x 128 x 64 bf16)
constexpr int kBwDoOff = kMhQBytes;
constexpr int kBwSuOff = 2 * kMhQBytes;
constexpr int kBwVOff = kBwSuOff + kBwSuStages * kMhKuBytes;
constexpr int kBwDqOff = kBwVOff + kBwVStages * kBwVBytes;
constexpr int kBwDsOff = kBwDqOff + kBwDqStages * kMhKuBytes;
constexpr int kBwPOff = kBwDsOff + 2 * kBwDsBytes;  // P staging: 4 atoms of 128 x 16 bf16
constexpr int kBwBarOff = kBwPOff + 4 * kBwDsAtom;
constexpr int kBwSmemBytes = kBwBarOff + 512 + 1024;
static_assert(kBwSmemBytes <= 232448, "shared memory per CTA");
constexpr int kBwBufCols = 192;               // S_g 64 | S_u 64 | dA 64 per TMEM buffer
static_assert(kMhDh + 2 * kBwBufCols == kMhTmemCols, "TMEM: dQ + two buffers");

struct MhBwArgs {
  int T, H, E, de;
  int h0;            // first head of this launch
  int n_pt;          // pairs of 128-token tiles
  int n_units;       // n_pt * heads of this launch, head-major
  int nch;           // 64-column chunks per head (even: d_e is a multiple of 128)
  int ch_per_sub;    // chunks per sub-network
  int F;             // E * d_e
  int tp;            // rows per head in the dS / P planes (n_pt * 256)
  const float* r;    // [T][H][E]
  __nv_bfloat16* dq; // [T][H * 128]
  float* dr_part;    // [T][H][E][4]: partial sums of the four column quarters
  int* status;
  uint64_t wait_limit_ns;
};

__global__ void __launch_bounds__(kBwThreads, 1)
    mhffn_bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                     const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmU,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDS,
                     const __grid_constant__ CUtensorMap tmP, const MhBwArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBwBarOff);
  uint64_t* q_full = bars + 0;                 // Q and dO of a unit
  uint64_t* q_empty = bars + 1;
  uint64_t* su_full = bars + 2;                // [kBwSuStages]
  uint64_t* su_empty = su_full + kBwSuStages;  // [kBwSuStages]
  uint64_t* v_full = su_empty + kBwSuStages;   // [kBwVStages]
  uint64_t* v_empty = v_full + kBwVStages;     // [kBwVStages]
  uint64_t* w_full = v_empty + kBwVStages;     // [kBwDqStages] dQ operand stages
  uint64_t* w_empty = w_full + kBwDqStages;    // [kBwDqStages]
  uint64_t* s_full = w_empty + kBwDqStages;    // [2] TMEM buffers
  uint64_t* s_empty = s_full + 2;              // [2]
  uint64_t* ds_full = s_empty + 2;             // [2] dS shared-memory buffers
  uint64_t* ds_empty = ds_full + 2;            // [2]
  uint64_t* dq_full = ds_empty + 2;
  uint64_t* dq_empty = dq_full + 1;
  uint64_t* drain = dq_empty + 1;              // [3]: one per issuing thread
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 3);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  static_assert((2 + 2 * kBwSuStages + 2 * kBwVStages + 2 * kBwDqStages + 8 + 5) * 8 + 8 <= 512,
                "barrier block");

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int cl = static_cast<int>(blockIdx.x >> 1), n_cl = static_cast<int>(gridDim.x >> 1);
  if (threadIdx.x == 0) {
    // arrival counts are those of the even CTA's barriers, the only ones waited on with them
    // (the dQ-ring and dS barriers are also waited on in the odd CTA: commit arrivals only)
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);  // released by the S / dA issuer
    for (int s = 0; s < kBwSuStages; ++s) {
      mbar_init(&su_full[s], 1);
      mbar_init(&su_empty[s], 1);
    }
    for (int s = 0; s < kBwVStages; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int s = 0; s < kBwDqStages; ++s) {
      mbar_init(&w_full[s], 1);
      mbar_init(&w_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);                   // the S and dA products of a chunk
      mbar_init(&s_empty[b], 2 * kBwEpiWarps);    // one arrival per epilogue warp, both CTAs
      mbar_init(&ds_full[b], 2 * kBwEpiWarps);
      mbar_init(&ds_empty[b], 1);
    }
    mbar_init(dq_full, 1);
    mbar_init(dq_empty, 2 * kBwEpiWarps);
    for (int d = 0; d < 3; ++d) mbar_init(&drain[d], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmDO);
    tma_prefetch_desc(rank == 0 ? &tmK : &tmU);
  }
  if (warp == kBwVWarp && lane == 0) tma_prefetch_desc(&tmV);
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&tmDS);
    tma_prefetch_desc(&tmP);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, kMhTmemCols);
    tmem_relinquish_pair();
  }
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before any remote signal
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const WaitCtl ctl{abort_flag, args.status, args.wait_limit_ns};
  const int rows_per_head = args.F;

  if (warp == 0) {
    // ------------------------------------------------------------ Q, dO and S-ring producer
    if (lane == 0) {
      const uint32_t q_full_lead = map_to_rank(smem_u32(q_full), 0);
      const uint32_t su_full_lead = map_to_rank(smem_u32(su_full), 0);
      const CUtensorMap* tm_b = rank == 0 ? &tmK : &tmU;  // this CTA's half of [K_c; U_c]
      uint32_t gc = 0;
      int lu = 0;
      bool ok = true;
      for (int unit = cl; ok && unit < args.n_units; unit += n_cl, ++lu) {
        const int hl = unit / args.n_pt, pt = unit - hl * args.n_pt;
        const int h = args.h0 + hl;
        const int tt = 2 * pt + static_cast<int>(rank);  // may lie past the last tile: zero rows
        if (!mbar_wait(q_empty, (lu & 1) ^ 1u, ctl)) { ok = false; break; }
        if (rank == 0) mbar_arrive_expect_tx(q_full, 4 * kMhQBytes);  // Q and dO of both CTAs
        tma_load_2d_pair(smem, &tmQ, h * kMhDh, tt * kMhTile, q_full_lead);
        tma_load_2d_pair(smem + kMhQBytes / 2, &tmQ, h * kMhDh + 64, tt * kMhTile, q_full_lead);
        tma_load_2d_pair(smem + kBwDoOff, &tmDO, h * kMhDh, tt * kMhTile, q_full_lead);
        tma_load_2d_pair(smem + kBwDoOff + kMhQBytes / 2, &tmDO, h * kMhDh + 64, tt * kMhTile,
                         q_full_lead);
        for (int c = 0; c < args.nch; ++c, ++gc) {
          const int row = h * rows_per_head + c * kMhChunk;
          const int s = gc % kBwSuStages;
          if (!mbar_wait(&su_empty[s], ((gc / kBwSuStages) & 1u) ^ 1u, ctl)) { ok = false; break; }
          uint8_t* su = smem + kBwSuOff + s * kMhKuBytes;
          if (rank == 0) mbar_arrive_expect_tx(&su_full[s], 2 * kMhKuBytes);
          tma_load_2d_pair(su, tm_b, 0, row, su_full_lead + s * 8);
          tma_load_2d_pair(su + kMhBox, tm_b, 64, row, su_full_lead + s * 8);
        }
      }
    }
  } else if (warp == kBwVWarp) {
    // ------------------------------------------------------------ V-ring producer (both CTAs)
    // A thread of its own, so the loads run ahead as soon as the dA products free a stage (an
    // issuing thread that also refilled the ring waited a whole load latency every chunk).
    if (lane == 0) {
      const uint32_t v_full_lead = map_to_rank(smem_u32(v_full), 0);
      uint32_t gc = 0;
      bool ok = true;
      for (int unit = cl; ok && unit < args.n_units; unit += n_cl) {
        const int h = args.h0 + unit / args.n_pt;
        for (int c = 0; c < args.nch; ++c, ++gc) {
          const int row = h * rows_per_head + c * kMhChunk + static_cast<int>(rank) * 32;
          const uint32_t sv = gc % kBwVStages;
          if (!mbar_wait(&v_empty[sv], ((gc / kBwVStages) & 1u) ^ 1u, ctl)) { ok = false; break; }
          uint8_t* vb = smem + kBwVOff + sv * kBwVBytes;
          if (rank == 0) mbar_arrive_expect_tx(&v_full[sv], 2 * kBwVBytes);
          tma_load_2d_pair(vb, &tmV, 0, row, v_full_lead + sv * 8);
          tma_load_2d_pair(vb + kBwVBox, &tmV, 64, row, v_full_lead + sv * 8);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ S and dA issuer (even CTA)
    // 16 products per chunk from one thread (about 1600 cycles of issue against a chunk's 3000 or
    // more), so the V ring can have a producer thread of its own.
    if (lane == 0 && rank == 0) {
      constexpr uint32_t kIdescS = idesc_bf16(2 * kMhTile, 2 * kMhChunk, 0, 0);  // [g | u]
      const uint64_t q_desc = smem_desc_sw128(smem_u32(smem), 16, 1024);
      const uint64_t su_desc = smem_desc_sw128(smem_u32(smem + kBwSuOff), 16, 1024);
      uint32_t gc = 0;
      int lu = 0;
      bool ok = true, issued = false;
      for (int unit = cl; ok && unit < args.n_units; unit += n_cl, ++lu) {
        if (!mbar_wait(q_full, lu & 1, ctl)) { ok = false; break; }
        tc_fence_after();
        for (int c = 0; c < args.nch; ++c, ++gc) {
          const uint32_t s = gc % kBwSuStages, b = gc & 1u;
          if (!mbar_wait(&su_full[s], (gc / kBwSuStages) & 1u, ctl)) { ok = false; break; }
          if (!mbar_wait(&s_empty[b], ((gc >> 1) & 1u) ^ 1u, ctl)) { ok = false; break; }
          tc_fence_after();
          const uint32_t d = tmem_base + kMhDh + b * kBwBufCols;
          const uint64_t sd = desc_add(su_desc, s * kMhKuBytes);
#pragma unroll
          for (int kb = 0; kb < 2; ++kb) {
#pragma unroll
            for (int k = 0; k < 4; ++k)
              umma_bf16_pair(d, desc_add(q_desc, kb * (kMhQBytes / 2) + k * 32),
                             desc_add(sd, kb * kMhBox + k * 32), kIdescS, (kb | k) != 0 ? 1u : 0u);
          }
          {
            constexpr uint32_t kIdescA = idesc_bf16(2 * kMhTile, kMhChunk, 0, 0);
            const uint64_t do_desc = smem_desc_sw128(smem_u32(smem + kBwDoOff), 16, 1024);
            const uint64_t v_desc = smem_desc_sw128(smem_u32(smem + kBwVOff), 16, 1024);
            const uint32_t sv = gc % kBwVStages;
            if (!mbar_wait(&v_full[sv], (gc / kBwVStages) & 1u, ctl)) { ok = false; break; }
            tc_fence_after();
            const uint64_t vd = desc_add(v_desc, sv * kBwVBytes);
#pragma unroll
            for (int kb = 0; kb < 2; ++kb) {
#pragma unroll
              for (int k = 0; k < 4; ++k)
                umma_bf16_pair(d + 2 * kMhChunk, desc_add(do_desc, kb * (kMhQBytes / 2) + k * 32),
                               desc_add(vd, kb * kBwVBox + k * 32), kIdescA, (kb | k) != 0 ? 1u : 0u);
            }
            umma_commit_pair(&v_empty[sv], 3);
          }
          umma_commit_pair(&s_full[b], 3);
          umma_commit_pair(&su_empty[s], 3);
          if (c == args.nch - 1) umma_commit_pair(q_empty, 3);  // Q no longer read in this unit
          issued = true;
        }
      }
      if (!ok && issued) drain_mma(&drain[0], abort_flag, args.status);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ dQ ring and dQ issuer
    // The loads run at most kBwDqStages - 1 chunks ahead of the products: a stage is free once
    // the dQ products of the chunk that used it are done, and in the even CTA this same thread
    // issues those products (it refills a stage after issuing the next chunk's products).
    if (lane == 0) {
      const uint32_t w_full_lead = map_to_rank(smem_u32(w_full), 0);
      const int my_units = cl < args.n_units ? (args.n_units - cl + n_cl - 1) / n_cl : 0;
      const uint32_t total = static_cast<uint32_t>(my_units) * static_cast<uint32_t>(args.nch);
      uint32_t nl = 0;  // chunks whose dQ operands were requested
      bool ok = true, issued = false;
      auto load_next = [&]() -> bool {
        const int unit = cl + static_cast<int>(nl / args.nch) * n_cl;
        const int c = static_cast<int>(nl % args.nch);
        const int row = (args.h0 + unit / args.n_pt) * rows_per_head + c * kMhChunk;
        const uint32_t st = nl % kBwDqStages;
        if (!mbar_wait(&w_empty[st], ((nl / kBwDqStages) & 1u) ^ 1u, ctl)) return false;
        uint8_t* wb = smem + kBwDqOff + st * kMhKuBytes;
        if (rank == 0) mbar_arrive_expect_tx(&w_full[st], 2 * kMhKuBytes);
        tma_load_2d_pair(wb, &tmK, static_cast<int>(rank) * 64, row, w_full_lead + st * 8);
        tma_load_2d_pair(wb + kMhBox, &tmU, static_cast<int>(rank) * 64, row, w_full_lead + st * 8);
        ++nl;
        return true;
      };
      if (rank != 0) {
        while (ok && nl < total) ok = load_next();
      } else {
        constexpr uint32_t kIdescDQ = idesc_bf16(2 * kMhTile, kMhDh, 0, 1);
        const uint64_t ds_desc = smem_desc_sw32(smem_u32(smem + kBwDsOff), 256);
        const uint64_t w_desc = smem_desc_sw128(smem_u32(smem + kBwDqOff), kMhBox, 1024);
        while (ok && nl < total && nl < static_cast<uint32_t>(kBwDqStages)) ok = load_next();
        int lu = -1;
        for (uint32_t i = 0; ok && i < total; ++i) {
          const int c = static_cast<int>(i % args.nch);
          if (c == 0) {
            ++lu;
            if (!mbar_wait(dq_empty, (lu & 1) ^ 1u, ctl)) { ok = false; break; }
          }
          const uint32_t b = i & 1u, st = i % kBwDqStages;
          if (!mbar_wait(&ds_full[b], (i >> 1) & 1u, ctl)) { ok = false; break; }
          if (!mbar_wait(&w_full[st], (i / kBwDqStages) & 1u, ctl)) { ok = false; break; }
          tc_fence_after();
          const uint64_t ad = desc_add(ds_desc, b * kBwDsBytes);
          const uint64_t bd = desc_add(w_desc, st * kMhKuBytes);
#pragma unroll
          for (int seg = 0; seg < 2; ++seg) {  // dS_g with K_c, then dS_u with U_c
#pragma unroll
            for (int k = 0; k < kMhChunk / 16; ++k)  // one K16 step per 32-byte atom
              umma_bf16_pair(tmem_base, desc_add(ad, seg * 4 * kBwDsAtom + k * kBwDsAtom),
                             desc_add(bd, seg * kMhBox + k * 2048), kIdescDQ,
                             (c | seg | k) != 0 ? 1u : 0u);
          }
          umma_commit_pair(&ds_empty[b], 3);
          umma_commit_pair(&w_empty[st], 3);
          if (c == args.nch - 1) umma_commit_pair(dq_full, 3);
          issued = true;
          // refill after issuing: the stage of chunk i + kBwDqStages - 1 waits only for the
          // products of chunk i - 1, issued a chunk ago
          while (ok && nl < total && nl < i + kBwDqStages) ok = load_next();
        }
        if (!ok && issued) drain_mma(&drain[1], abort_flag, args.status);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue warps 4..19
    // Every chunk goes through all sixteen warps: warp (q, qc) takes TMEM lane quadrant q and the
    // chunk's columns [16 qc, 16 qc + 16), so each thread loads its 48 values (g, u, dA) with one
    // round of tcgen05 loads and frees the TMEM buffer at once, and four warps per SM sub-partition
    // hide each other's latencies.  dS and P tiles are stored K-major in 32-byte swizzled atoms of
    // 16 columns (atom qc belongs to the warps of column quarter qc), so each warp sends its own
    // 32-row boxes to HBM.
    const int q = warp & 3;           // TMEM lane quadrant this warp may access
    const int qc = (warp - 4) >> 2;   // column quarter of every chunk
    const int row = q * 32 + lane;
    const int swz = (lane >> 2) & 1;  // 32-byte swizzle phase of this thread's row
    const uint32_t t_lane = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    const uint32_t ds_row = smem_u32(smem + kBwDsOff) + qc * kBwDsAtom + row * (2 * kBwCols);
    const int64_t q_ld = (int64_t)args.H * kMhDh;
    uint32_t gc = 0;
    int lu = 0;
    bool ok = true;
    for (int unit = cl; ok && unit < args.n_units; unit += n_cl, ++lu) {
      const int hl = unit / args.n_pt, pt = unit - hl * args.n_pt;
      const int h = args.h0 + hl;
      const int tile_row0 = (2 * pt + static_cast<int>(rank)) * kMhTile;
      const int token = tile_row0 + row;
      const bool tok_ok = token < args.T;
      const float* rrow = args.r + ((int64_t)(tok_ok ? token : 0) * args.H + h) * args.E;
      float2 dr2 = make_float2(0.f, 0.f);     // router-gradient sum (even | odd columns)
      float rv_next = tok_ok ? rrow[0] : 0.f;  // router weight of the next chunk (loaded ahead)
      for (int c = 0; c < args.nch; ++c, ++gc) {
        const uint32_t b = gc & 1u;
        const int e = c / args.ch_per_sub;
        const float2 rv2 = make_float2(rv_next, rv_next);
        if (c + 1 < args.nch) rv_next = tok_ok ? rrow[(c + 1) / args.ch_per_sub] : 0.f;
        const bool ready = mbar_wait(&s_full[b], (gc >> 1) & 1u, ctl);
        __syncwarp();  // tcgen05.ld is warp-collective: reconverge after the per-thread wait
        if (!__all_sync(0xffffffffu, ready)) { ok = false; break; }
        tc_fence_after();
        const uint32_t tb = t_lane + kMhDh + b * kBwBufCols + qc * kBwCols;
        float g[16], u[16], a[16];
        tmem_ld16x(tb, g);
        tmem_ld16x(tb + kMhChunk, u);
        tmem_ld16x(tb + 2 * kMhChunk, a);
        tmem_wait16x3(g, u, a);
        tc_fence_before();
        warp_arrive_lead(&s_empty[b], rank, lane);  // the TMEM buffer is in registers
        // dS buffer b is free once this warp's TMA stores from it (two chunks ago) have read it
        // and the dQ products of that chunk are done; the P staging once the previous chunk's
        // stores have read it
        if (lane == 0) bulk_wait_read<0>();
        __syncwarp();
        const bool free_ds = mbar_wait(&ds_empty[b], ((gc >> 1) & 1u) ^ 1u, ctl);
        if (!__all_sync(0xffffffffu, free_ds)) { ok = false; break; }
        const uint32_t dsg = ds_row + b * kBwDsBytes;
        const uint32_t dsu = dsg + 4 * kBwDsAtom;
        const uint32_t pst = ds_row + (kBwPOff - kBwDsOff);
#pragma unroll
        for (int c8 = 0; c8 < 2; ++c8) {
          uint32_t wg[4], wu[4], wp[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            // two columns at a time with Blackwell's paired fp32 operations (fma/mul .f32x2,
            // IEEE round-to-nearest like the scalar forms); sigmoid(g) = (1 + tanh(g / 2)) / 2 is
            // one MUFU operation (tanh.approx.f32, relative error about 2^-11), and every result
            // is rounded to bf16 (2^-9) after
            const int k = c8 * 8 + 2 * j;
            const float2 g2 = make_float2(g[k], g[k + 1]);
            const float2 u2 = make_float2(u[k], u[k + 1]);
            const float2 a2 = make_float2(a[k], a[k + 1]);
            const float2 h2 = __fmul2_rn(g2, kHalf2);
            float2 th;
            asm("tanh.approx.f32 %0, %1;" : "=f"(th.x) : "f"(h2.x));
            asm("tanh.approx.f32 %0, %1;" : "=f"(th.y) : "f"(h2.y));
            const float2 sg = __ffma2_rn(th, kHalf2, kHalf2);           // sigmoid
            const float2 silu = __ffma2_rn(h2, th, h2);                  // g sigmoid(g)
            const float2 dsilu = __ffma2_rn(silu, __ffma2_rn(th, kMinusHalf2, kHalf2), sg);  // s + SiLU (1 - s)
            const float2 act = __fmul2_rn(silu, u2);
            const float2 dact = __fmul2_rn(rv2, a2);
            dr2 = __ffma2_rn(a2, act, dr2);
            const float2 vp = __fmul2_rn(rv2, act);
            const float2 vu = __fmul2_rn(dact, silu);
            const float2 vg = __fmul2_rn(__fmul2_rn(dact, u2), dsilu);
            wg[j] = pack_bf16x2(vg.x, vg.y);
            wu[j] = pack_bf16x2(vu.x, vu.y);
            wp[j] = pack_bf16x2(vp.x, vp.y);
          }
          const uint32_t off = static_cast<uint32_t>((c8 ^ swz) << 4);
          st_shared_v4(dsg + off, wg[0], wg[1], wg[2], wg[3]);
          st_shared_v4(dsu + off, wu[0], wu[1], wu[2], wu[3]);
          st_shared_v4(pst + off, wp[0], wp[1], wp[2], wp[3]);
        }
        fence_proxy_async_smem();  // dS and P visible to the tensor core and to the TMA stores
        __syncwarp();
        if (lane == 0) {
          const int prow0 = hl * args.tp + tile_row0 + q * 32;
          const int col = c * kMhChunk + qc * kBwCols;
          uint8_t* box = smem + kBwDsOff + b * kBwDsBytes + qc * kBwDsAtom + q * 32 * (2 * kBwCols);
          tma_store_2d(&tmDS, col, prow0, box);
          tma_store_2d(&tmDS, args.F + col, prow0, box + 4 * kBwDsAtom);
          tma_store_2d(&tmP, col, prow0, smem + kBwPOff + qc * kBwDsAtom + q * 32 * (2 * kBwCols));
          bulk_commit();
        }
        warp_arrive_lead(&ds_full[b], rank, lane);
        if (c == (e + 1) * args.ch_per_sub - 1) {  // last chunk of sub-network e
          if (tok_ok) args.dr_part[(((int64_t)token * args.H + h) * args.E + e) * 4 + qc] = dr2.x + dr2.y;
          dr2 = make_float2(0.f, 0.f);
        }
      }
      if (!ok) break;
      const bool ready = mbar_wait(dq_full, lu & 1, ctl);
      __syncwarp();
      if (!__all_sync(0xffffffffu, ready)) { ok = false; break; }
      tc_fence_after();
      __nv_bfloat16* dqrow = args.dq + (int64_t)(tok_ok ? token : 0) * q_ld + h * kMhDh;
#pragma unroll 1
      for (int cc = qc * 32; cc < qc * 32 + 32; cc += 32) {
        float ov[32];
        tmem_ld32(t_lane + cc, ov);
        tmem_ld_wait_regs(ov);
        if (tok_ok) {
#pragma unroll
          for (int v = 0; v < 4; ++v)
            *reinterpret_cast<uint4*>(dqrow + cc + 8 * v) =
                make_uint4(pack_bf16x2(ov[8 * v], ov[8 * v + 1]), pack_bf16x2(ov[8 * v + 2], ov[8 * v + 3]),
                           pack_bf16x2(ov[8 * v + 4], ov[8 * v + 5]), pack_bf16x2(ov[8 * v + 6], ov[8 * v + 7]));
        }
      }
      tc_fence_before();
      warp_arrive_lead(dq_empty, rank, lane);
    }
    if (lane == 0) bulk_wait_all();  // the TMA stores are done before the CTA leaves
  }

  __syncthreads();
  cluster_sync();  // the pair's MMAs and TMEM reads are all done
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kMhTmemCols);
  }
}

__global__ void mh_dr_reduce_kernel(const float* __restrict__ part, int64_t n, float* __restrict__ dr) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    dr[i] = (part[4 * i] + part[4 * i + 1]) + (part[4 * i + 2] + part[4 * i + 3]);  // fixed order
}

constexpr int kMhBwdHeads = 4;  // heads per fused launch: sizes the dS / P planes of the workspace

struct MhBwdWs {
  __nv_bfloat16 *dsgu, *p;  // [hg][tp][2F], [hg][tp][F]
  float *dr_part, *split;
  int64_t tp;
  int hg;
};

MhBwdWs mh_bwd_ws(void* base, int64_t T, int64_t H, int64_t E, int64_t F, size_t* bytes) {
  size_t off = 0;
  auto take = [&](size_t n) {
    off = round_up(off, 256);
    char* p = base ? static_cast<char*>(base) + off : nullptr;
    off += n;
    return p;
  };
  MhBwdWs w;
  const int64_t n_pt = ((T + kMhTile - 1) / kMhTile + 1) / 2;
  w.tp = n_pt * 2 * kMhTile;
  w.hg = static_cast<int>(std::min<int64_t>(H, kMhBwdHeads));
  w.dsgu = reinterpret_cast<__nv_bfloat16*>(take((size_t)w.hg * w.tp * 2 * F * 2));
  w.p = reinterpret_cast<__nv_bfloat16*>(take((size_t)w.hg * w.tp * F * 2));
  w.dr_part = reinterpret_cast<float*>(take((size_t)T * H * E * 4 * 4));
  const int64_t part = std::max(part_elems(2 * F, kMhDh, T), part_elems(F, kMhDh, T));
  w.split = reinterpret_cast<float*>(take((size_t)std::max<int64_t>(part, 4) * 4));
  if (bytes) *bytes = off;
  return w;
}

swf_status check_mh_bwd(int64_t T, int32_t H, int32_t dh, int32_t E, int32_t de, swf_dtype dt) {
  if (T <= 0 || H <= 0 || dh <= 0 || E <= 0 || de <= 0) return SWF_ERR_INVALID_ARG;
  if (dt != SWF_BF16 && dt != SWF_F32) return SWF_ERR_INVALID_ARG;
  if (dt != SWF_BF16 || dh != kMhDh || de % 128 != 0) return SWF_ERR_UNSUPPORTED;
  if (T > INT32_MAX / 4 || (int64_t)E * de > (1 << 20) || (int64_t)H * E * de > INT32_MAX / 4 ||
      (int64_t)H * kMhDh > (1 << 20) || (int64_t)kMhBwdHeads * (T + 2 * kMhTile) > INT32_MAX / 2)
    return SWF_ERR_UNSUPPORTED;
  return SWF_OK;
}

}  // namespace
}  // namespace swf

extern "C" size_t flash_mhffn_bwd_workspace_bytes(int64_t T, int32_t num_heads, int32_t head_dim,
                                                  int32_t num_sub, int32_t sub_dim, swf_dtype dtype) {
  if (check_mh_bwd(T, num_heads, head_dim, num_sub, sub_dim, dtype) != SWF_OK) return 0;
  size_t need = 0;
  mh_bwd_ws(nullptr, T, num_heads, num_sub, (int64_t)num_sub * sub_dim, &need);
  return need;
}

extern "C" swf_status flash_mhffn_bwd(const void* q, const void* w_k, const void* w_u,
                                      const void* w_v, const float* router, const void* d_o,
                                      void* dq, void* dw_k, void* dw_u, void* dw_v,
                                      float* drouter, void* workspace, size_t workspace_bytes,
                                      int64_t T, int32_t num_heads, int32_t head_dim,
                                      int32_t num_sub, int32_t sub_dim, swf_dtype dtype,
                                      void* stream) {
  for (const void* p : std::initializer_list<const void*>{q, w_k, w_u, w_v, router, d_o, dq, dw_k,
                                                          dw_u, dw_v, drouter})
    if (!p) return SWF_ERR_INVALID_ARG;
  swf_status s = check_mh_bwd(T, num_heads, head_dim, num_sub, sub_dim, dtype);
  if (s != SWF_OK) return s;
  for (const void* p : std::initializer_list<const void*>{q, w_k, w_u, w_v, router, d_o, dq, dw_k,
                                                          dw_u, dw_v, drouter, workspace})
    if (p && !aligned16(p)) return SWF_ERR_ALIGNMENT;
  const int64_t H = num_heads, E = num_sub, de = sub_dim, F = E * de, ld = H * kMhDh;
  size_t need = 0;
  const MhBwdWs w = mh_bwd_ws(workspace, T, H, E, F, &need);
  if (!workspace || workspace_bytes < need) return SWF_ERR_WORKSPACE;
  DevCtx ctx;
  if ((s = get_ctx(&ctx)) != SWF_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  using bf = __nv_bfloat16;
  const int64_t rows = H * F;
  CUtensorMap tq, tdo, tk, tu, tv;
  if (!encode_tmap_bf16(&tq, q, ld, T, ld, 64, kMhTile) ||
      !encode_tmap_bf16(&tdo, d_o, ld, T, ld, 64, kMhTile) ||
      !encode_tmap_bf16(&tk, w_k, kMhDh, rows, kMhDh, 64, 64) ||
      !encode_tmap_bf16(&tu, w_u, kMhDh, rows, kMhDh, 64, 64) ||
      !encode_tmap_bf16(&tv, w_v, kMhDh, rows, kMhDh, 64, 32))
    return SWF_ERR_LAUNCH;
  if (cudaFuncSetAttribute(mhffn_bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           kBwSmemBytes) != cudaSuccess)
    return SWF_ERR_LAUNCH;
  MhBwArgs a{};
  a.T = (int)T;
  a.H = num_heads;
  a.E = num_sub;
  a.de = sub_dim;
  a.n_pt = (int)(w.tp / (2 * kMhTile));
  a.nch = (int)(F / kMhChunk);
  a.ch_per_sub = (int)(de / kMhChunk);
  a.F = (int)F;
  a.tp = (int)w.tp;
  a.r = router;
  a.dq = static_cast<bf*>(dq);
  a.dr_part = w.dr_part;
  a.status = ctx.status;
  a.wait_limit_ns = kDefaultWaitNs;
  for (int64_t h0 = 0; h0 < H; h0 += w.hg) {
    const int g = (int)std::min<int64_t>(w.hg, H - h0);
    {  // fused: dA, [S_g | S_u], dS_g | dS_u and P planes, router-gradient partials, dQ
      CUtensorMap tds, tp;  // dS_g | dS_u and P planes of this launch's heads, 16 x 32 boxes
      if (!encode_tmap_bf16(&tds, w.dsgu, 2 * F, (uint64_t)g * w.tp, 2 * F, kBwCols, 32, 32) ||
          !encode_tmap_bf16(&tp, w.p, F, (uint64_t)g * w.tp, F, kBwCols, 32, 32))
        return SWF_ERR_LAUNCH;
      a.h0 = (int)h0;
      a.n_units = a.n_pt * g;
      const int clusters = std::min(a.n_units, ctx.num_sms / 2);
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(2 * clusters, 1, 1);
      cfg.blockDim = dim3(kBwThreads, 1, 1);
      cfg.dynamicSmemBytes = kBwSmemBytes;
      cfg.stream = st;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      ProfScope prof(SWF_K_MHFFN_BWD, st);
      if (cudaLaunchKernelEx(&cfg, mhffn_bwd_kernel, tq, tdo, tk, tu, tv, tds, tp, a) != cudaSuccess)
        return SWF_ERR_LAUNCH;
    }
    for (int hl = 0; hl < g; ++hl) {
      const int64_t h = h0 + hl;
      const bf* qh = static_cast<const bf*>(q) + h * kMhDh;
      const bf* doh = static_cast<const bf*>(d_o) + h * kMhDh;
      const bf* dsgu_h = w.dsgu + (int64_t)hl * w.tp * 2 * F;
      const bf* p_h = w.p + (int64_t)hl * w.tp * F;
      {  // [dK_h ; dU_h] = [dS_g | dS_u]^T Q_h
        CUtensorMap ta, tb;
        if (!encode_tmap_bf16(&ta, dsgu_h, 2 * F, T, 2 * F, 64, 64) ||
            !encode_tmap_bf16(&tb, qh, kMhDh, T, ld, 64, 64))
          return SWF_ERR_LAUNCH;
        if ((s = launch_dw(SWF_K_MHFFN_BWD_DW, ta, tb, 2 * F, kMhDh, T, static_cast<bf*>(dw_k) + h * F * kMhDh,
                           static_cast<bf*>(dw_u) + h * F * kMhDh, F, w.split, st)) != SWF_OK)
          return s;
      }
      {  // dV_h = P^T dO_h
        CUtensorMap ta, tb;
        if (!encode_tmap_bf16(&ta, p_h, F, T, F, 64, 64) || !encode_tmap_bf16(&tb, doh, kMhDh, T, ld, 64, 64))
          return SWF_ERR_LAUNCH;
        bf* dv = static_cast<bf*>(dw_v) + h * F * kMhDh;
        if ((s = launch_dw(SWF_K_MHFFN_BWD_DW, ta, tb, F, kMhDh, T, dv, dv, F, w.split, st)) != SWF_OK) return s;
      }
    }
  }
  ProfScope prof(SWF_K_MHFFN_BWD_DR, st);
  const int64_t n = T * H * E;
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>((n + 255) / 256, 148 * 16));
  mh_dr_reduce_kernel<<<grid, 256, 0, st>>>(w.dr_part, n, drouter);
  return cudaGetLastError() == cudaSuccess ? SWF_OK : SWF_ERR_LAUNCH;
}

// ------------------------------------------------------------------ prologue backward
// Gradients of the prologue given dq and drouter: the projection and router GEMMs are recomputed
// with epilogues that apply the normalisations' backward (kEpiHeadNormBwd: dz and the gain's
// partial sums; the router's sigmoid, then a row kernel for dl), writing dz | dl side by side;
// then dx = [dz | dl] [W_q ; W_r]
// (two K segments) and [dW_q ; dW_r] = [dz | dl]^T x (split-K weight-gradient GEMM); one kernel
// sums the gain partials in a fixed order.
namespace swf {
namespace {

// Column sums of the [rows][128] gain-gradient partials in a fixed order: block b of
// kGainBlocks sums its contiguous range of rows (one thread per column), then one block sums
// the kGainBlocks results in block order.
constexpr int kGainBlocks = 256;
__global__ void dgain_partial_kernel(const float* __restrict__ part, int64_t rows, float* __restrict__ out) {
  const int i = threadIdx.x;  // 128 columns
  const int64_t per = (rows + kGainBlocks - 1) / kGainBlocks;
  const int64_t r0 = blockIdx.x * per, r1 = r0 + per < rows ? r0 + per : rows;
  float s = 0.f;
  for (int64_t r = r0; r < r1; ++r) s += part[r * 128 + i];
  out[blockIdx.x * 128 + i] = s;
}
__global__ void dgain_reduce_kernel(const float* __restrict__ part2, float* __restrict__ dgain) {
  const int i = threadIdx.x;
  float s = 0.f;
  for (int b = 0; b < kGainBlocks; ++b) s += part2[b * 128 + i];
  dgain[i] = s;
}

struct ProBwdWs {
  __nv_bfloat16* dzl;
  float *sig, *gain_part, *gain_part2, *split;
  int64_t ld;
};

ProBwdWs pro_bwd_ws(void* base, int64_t T, int64_t d_model, int64_t H, int64_t E, size_t* bytes) {
  size_t off = 0;
  auto take = [&](size_t n) {
    off = round_up(off, 256);
    char* p = base ? static_cast<char*>(base) + off : nullptr;
    off += n;
    return p;
  };
  const int64_t nq = H * kMhDh, nr = H * E;
  ProBwdWs w;
  w.ld = (int64_t)round_up(nq + nr, 8);
  w.dzl = reinterpret_cast<__nv_bfloat16*>(take((size_t)T * w.ld * 2));
  w.sig = reinterpret_cast<float*>(take((size_t)T * nr * 4));
  w.gain_part = reinterpret_cast<float*>(take((size_t)round_up(T, 256) / 32 * H * 128 * 4));
  w.gain_part2 = reinterpret_cast<float*>(take((size_t)kGainBlocks * 128 * 4));
  w.split = reinterpret_cast<float*>(take((size_t)std::max<int64_t>(part_elems(nq + nr, d_model, T), 4) * 4));
  if (bytes) *bytes = off;
  return w;
}

swf_status check_pro(int64_t T, int64_t d_model, int32_t H, int32_t dh, int32_t E, float eps, swf_dtype dt) {
  if (T <= 0 || d_model <= 0 || H <= 0 || dh <= 0 || E <= 0 || !(eps >= 0.f)) return SWF_ERR_INVALID_ARG;
  if (dt != SWF_BF16 && dt != SWF_F32) return SWF_ERR_INVALID_ARG;
  if (dt != SWF_BF16 || dh != kMhDh || d_model % 16 != 0 || (int64_t)H * E > 256 || T > INT32_MAX / 2 ||
      d_model > (1 << 20) || (int64_t)H * kMhDh > (1 << 20))
    return SWF_ERR_UNSUPPORTED;
  return SWF_OK;
}

}  // namespace
}  // namespace swf

extern "C" size_t flash_mhffn_prologue_bwd_workspace_bytes(int64_t T, int64_t d_model,
                                                           int32_t num_heads, int32_t head_dim,
                                                           int32_t num_sub, swf_dtype dtype) {
  if (check_pro(T, d_model, num_heads, head_dim, num_sub, 0.f, dtype) != SWF_OK) return 0;
  size_t need = 0;
  pro_bwd_ws(nullptr, T, d_model, num_heads, num_sub, &need);
  return need;
}

extern "C" swf_status flash_mhffn_prologue_bwd(
    const void* x, const void* w_q, const float* q_gain, const void* w_r, const void* dq,
    const float* drouter, void* dx, void* dw_q, float* dq_gain, void* dw_r, void* workspace,
    size_t workspace_bytes, int64_t T, int64_t d_model, int32_t num_heads, int32_t head_dim,
    int32_t num_sub, float eps, swf_dtype dtype, void* stream) {
  for (const void* p : std::initializer_list<const void*>{x, w_q, w_r, dq, drouter, dx, dw_q, dw_r})
    if (!p) return SWF_ERR_INVALID_ARG;
  swf_status s = check_pro(T, d_model, num_heads, head_dim, num_sub, eps, dtype);
  if (s != SWF_OK) return s;
  for (const void* p : std::initializer_list<const void*>{x, w_q, q_gain, w_r, dq, drouter, dx, dw_q,
                                                          dq_gain, dw_r, workspace})
    if (p && !aligned16(p)) return SWF_ERR_ALIGNMENT;
  const int64_t H = num_heads, E = num_sub, nq = H * kMhDh, nr = H * E;
  size_t need = 0;
  const ProBwdWs w = pro_bwd_ws(workspace, T, d_model, H, E, &need);
  if (!workspace || workspace_bytes < need) return SWF_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  CUtensorMap tx, tq, tr;
  if (!encode_tmap_bf16(&tx, x, d_model, T, d_model, 64, 128) ||
      !encode_tmap_bf16(&tq, w_q, d_model, nq, d_model, 64, 128) ||
      !encode_tmap_bf16(&tr, w_r, d_model, nr, d_model, 64, 256))
    return SWF_ERR_LAUNCH;
  {  // dz from the recomputed projection (one-CTA tiles of one head; the gain partials are per
     // 32-row slab and head)
    // with an even head count, pair (cta_group::2) tiles of 256 tokens x 256 columns (two heads
    // per epilogue row), as in the forward; otherwise one-CTA tiles of one head
    const bool pair = nq % 256 == 0;
    TcGemmArgs a = pair ? base_args(T, nq, 256, d_model, 2 * kTileM) : base_args(T, nq, 128, d_model);
    a.aux0 = dq;
    a.ld_aux = nq;
    a.bias = q_gain;
    a.eps = eps;
    a.out0 = w.dzl;
    a.ld_out = w.ld;
    a.dgain_part = (q_gain && dq_gain) ? w.gain_part : nullptr;
    a.heads = num_heads;
    s = pair ? launch_tc_pair<256, false, false, false, kEpiHeadNormBwd>(SWF_K_MHFFN_PROLOGUE, tx, tq, tq,
                                                                        EpiMaps{}, a, st)
             : launch_tc<128, false, false, false, kEpiHeadNormBwd>(SWF_K_MHFFN_PROLOGUE, tx, tq, tq, a, st);
    if (s != SWF_OK) return s;
  }
  {  // dl from the recomputed router logits, into the columns after dz
    TcGemmArgs a = base_args(T, nr, 256, d_model);
    a.out0 = w.sig;
    a.ld_out = nr;
    if ((s = launch_tc<256, false, false, false, kEpiRouter>(SWF_K_MHFFN_PROLOGUE, tx, tr, tr, a, st)) != SWF_OK)
      return s;
    ProfScope prof(SWF_K_MHFFN_PROLOGUE, st);
    router_bwd_kernel<<<(unsigned)((T + kRouterRows - 1) / kRouterRows), 32 * kRouterRows, 0, st>>>(
        w.sig, drouter, T, (int)nr, num_sub, w.dzl + nq, w.ld);
    if (cudaGetLastError() != cudaSuccess) return SWF_ERR_LAUNCH;
  }
  {  // dx = dz W_q + dl W_r: A = [dz | dl] (K = nq + nr), B segments W_q, W_r (MN-major)
    CUtensorMap ta, tbq, tbr;
    if (!encode_tmap_bf16(&ta, w.dzl, nq + nr, T, w.ld, 64, 128) ||
        !encode_tmap_bf16(&tbq, w_q, d_model, nq, d_model, 64, 64) ||
        !encode_tmap_bf16(&tbr, w_r, d_model, nr, d_model, 64, 64))
      return SWF_ERR_LAUNCH;
    TcGemmArgs a = base_args(T, d_model, 256, 0, 2 * kTileM);
    a.kb_seg0 = (int)(nq / kTileK);
    a.kb_total = a.kb_seg0 + cdiv(nr, kTileK);
    a.a_koff1 = (int)nq;
    a.out0 = dx;
    a.ld_out = d_model;
    if ((s = launch_tc_pair<256, false, true, false, kEpiStore>(SWF_K_MHFFN_PROLOGUE, ta, tbq, tbr, EpiMaps{},
                                                              a, st)) != SWF_OK)
      return s;
  }
  {  // [dW_q ; dW_r] = [dz | dl]^T x
    CUtensorMap ta, tb;
    if (!encode_tmap_bf16(&ta, w.dzl, nq + nr, T, w.ld, 64, 64) || !encode_tmap_bf16(&tb, x, d_model, T, d_model, 64, 64))
      return SWF_ERR_LAUNCH;
    if ((s = launch_dw(SWF_K_MHFFN_PROLOGUE, ta, tb, nq + nr, d_model, T, dw_q, dw_r, nq, w.split, st)) != SWF_OK)
      return s;
  }
  if (q_gain && dq_gain) {
    ProfScope prof(SWF_K_MHFFN_PROLOGUE, st);
    dgain_partial_kernel<<<kGainBlocks, 128, 0, st>>>(w.gain_part, (int64_t)cdiv(T, 128) * 4 * H,
                                                      w.gain_part2);
    dgain_reduce_kernel<<<1, 128, 0, st>>>(w.gain_part2, dq_gain);
    if (cudaGetLastError() != cudaSuccess) return SWF_ERR_LAUNCH;
  } else if (dq_gain) {
    if (cudaMemsetAsync(dq_gain, 0, 128 * sizeof(float), st) != cudaSuccess) return SWF_ERR_LAUNCH;
  }
  return SWF_OK;
}
