// Persistent, warp-specialised tcgen05 GEMM for sm_100a with fused SwiGLU epilogues.
//
//   C[m, n] = sum_k A(m, k) * B(n, k)      bf16 operands, fp32 accumulation in TMEM
//
// One CTA per SM walks a static list of 128 x BN output tiles.  Warp 0 streams A/B tiles
// into a ring of shared-memory stages with TMA (128-byte swizzle), warp 1 allocates TMEM and
// one of its threads issues tcgen05.mma (M=128, N=BN, K=16) into one of two TMEM accumulators,
// warps 2..5 drain the other accumulator with tcgen05.ld, apply the epilogue in fp32
// registers and store to global memory, so the epilogue of tile i overlaps the main loop of
// tile i+1.  Either operand may be K-major (rows of K contiguous) or MN-major (rows of M or N
// contiguous); the tensor-core descriptors read both layouts, so no transposes are needed.
//
// Tile modes:
//   kModeDense       one GEMM; tiles rasterised in groups of `raster` M-blocks
//   kModeRowGrouped  the rows are group-major padded segments (group-sparse path): M-block mb
//                    belongs to group tile_group[mb] (-1: unused, skipped), whose B tile sits
//                    at n + g*grp_b_n, k + g*grp_b_k
//   kModeKGrouped    one small GEMM per group g over the rows [seg_start[g], +seg_rows[g]) of
//                    the group-major buffers (weight gradients of the group-sparse path)
//
// Epilogues (flash-swiglu-mlp overview; parameter-golf PR 1105 "Fused MLP Kernels";
// eugen_sparse README "What it does" and "Pitfalls and limitations"):
//   kEpiStore      C -> bf16, row m < row_split to out0 else out1 (two weight-gradient halves)
//   kEpiSwiGLU     gate|up dual tile: h = SiLU(g)*u, a = u*SiLU'(g), b = SiLU(g) -> bf16
//   kEpiSwiGLUInf  same, h only
//   kEpiDGate      C = dH: dG = dH*a -> out0[:, n], dU = dH*b -> out0[:, d_ff + n]; columns
//                  [N, pad_cols) of both halves are written as zeros
//   kEpiEnergy     per group of energy_p columns: sum |SiLU(C)| -> fp32 out0 (no bias: the top-k
//                  step adds it)
//   kEpiGroupDWgu  per-group [dG|dU]^T X: rows [0,G) -> out0 rows g*G.., [64,64+G) -> out1
//   kEpiGroupDWd   per-group dY^T h: columns [0,G) -> out0[:, g*G ..]
//   kEpiLeakySq    C = pre: post = LeakyReLU(0.5)(pre)^2 -> out0, act_grad (2 pre or 0.5 pre)
//                  -> aux0 (parameter-golf PR 1105, "Fused MLP Kernels")
//   kEpiScale      C * aux -> out0 (the stored activation gradient applied to dpost)
//   kEpiPartialF32 fp32 C of K-split ks -> part[ks][m][n] (split-K weight gradients; a separate
//                  kernel sums the splits in a fixed order)
//   kEpiHeadNorm   BN a multiple of 128, heads of 128 columns: C / sqrt(mean(C^2) + eps) * gain
//                  -> bf16 out0 (FlashFFN's per-head RMS-normalised projection Q)
//   kEpiRouter     N <= BN = 256 columns: sigmoid(C) -> fp32 out0 (FlashFFN's router; a row kernel
//                  then divides each head's values by their sum, or applies that step's backward)
//   kEpiHeadNormBwd C = z (the projection), heads of 128 columns, with dq (aux0, ld_aux) and the
//                  gain (bias, nullable): dz = inv (dn - n mean(dn n)), n = z inv, dn = dq gain,
//                  inv = 1 / sqrt(mean(z^2) + eps) -> bf16 out0; if dgain_part, per 32-row slab
//                  and head the column sums of dq n -> dgain_part[(m / 32) * heads + h][i]
//   kEpiEnergyTopK the energies of a CTA's 128 tokens kept in shared memory; once the CTA has
//                  scored every group of them (it owns all N-blocks of an M-block, `unit` =
//                  num_n_blk) each epilogue thread adds the bias to its token's energies (-> out0
//                  if not null) and picks the top-k groups -> sel_idx (ascending; larger energy
//                  first, lower group index among equal energies; NaN never chosen, -1 fills
//                  what cannot be chosen)
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "swf_ptx.cuh"

namespace swf {

enum : int {
  kEpiStore = 0,
  kEpiSwiGLU = 1,
  kEpiSwiGLUInf = 2,
  kEpiDGate = 3,
  kEpiEnergy = 4,
  kEpiGroupDWgu = 5,
  kEpiGroupDWd = 6,
  kEpiLeakySq = 7,
  kEpiScale = 8,
  kEpiPartialF32 = 9,
  kEpiEnergyTopK = 10,
  kEpiHeadNorm = 11,
  kEpiRouter = 12,
  kEpiHeadNormBwd = 14
};
constexpr int kTopKMaxGroups = 64;  // kEpiEnergyTopK: groups held in registers per token
enum : int { kModeDense = 0, kModeRowGrouped = 1, kModeKGrouped = 2 };

constexpr int kTileM = 128;
constexpr int kTileK = 64;  // one 128-byte swizzle row of bf16
constexpr int kUmmaK = 16;
constexpr int kGemmThreads = 192;

// Operands whose rows are gathered from token rows (group-sparse path) instead of loaded by TMA:
//   kGatherA  row-grouped mode: the K-major A tile's 128 rows (padded pair rows); per-group-K
//             mode: the MN-major A tile's 64 K rows
//   kGatherB  per-group-K mode: the MN-major B tile's 64 K rows
// Padded row r holds token gather_token[r] of gather_src (-1: a zero row).  kGatherWarps extra
// warps (6 ..) copy the rows 16 bytes at a time with cp.async into the stage's 128-byte-swizzled
// layout, each warp taking every kGatherWarps-th k-block; the token rows (x or dY) come from L2.
enum : int { kGatherNone = 0, kGatherA = 1, kGatherB = 2 };
constexpr int kGatherWarps = 4;
template <int GATHER>
constexpr int gemm_threads() {
  return GATHER != kGatherNone ? kGemmThreads + 32 * kGatherWarps : kGemmThreads;
}

struct TcGemmArgs {
  int M;            // rows of C (kModeKGrouped: rows of each group's C)
  int N;            // columns of C that exist (kEpiSwiGLU*: d_ff; sparse: group_size)
  int num_m_blk, num_n_blk;
  int raster;       // m-blocks per raster group
  int kb_seg0;      // 64-wide k-blocks in K segment 0
  int kb_total;     // k-blocks in total (segment 1 = the rest)
  int a_koff1;      // A's K coordinate where segment 1 starts
  // epilogue
  void* out0;
  void* out1;
  int64_t ld_out;   // elements
  int row_split;    // kEpiStore: rows >= row_split go to out1 (row - row_split)
  const void* aux0; // kEpiSwiGLU: saved_a out; kEpiDGate: saved_a in
  const void* aux1; // kEpiSwiGLU: saved_b out; kEpiDGate: saved_b in
  int64_t ld_aux;
  int d_ff;         // kEpiDGate: column offset of dU in out0
  int pad_cols;     // kEpiDGate: zero-filled columns up to here
  // group-sparse modes
  const int* tile_group;  // kModeRowGrouped
  const int* seg_start;   // kModeKGrouped: first padded row of each group
  const int* seg_rows;    // kModeKGrouped: padded rows of each group (multiple of 128)
  int grp_b_n, grp_b_k;   // kModeRowGrouped: B coordinate offsets per group
  int group_size;
  const float* bias;      // kEpiEnergy (nullable)
  int energy_p;           // kEpiEnergy: columns per group
  int n_groups;           // kEpiEnergy: groups (columns of out0)
  int64_t ld_grp;         // kEpiEnergy*: stride of out0 between groups (0: 1); ld_out is the
                          //   stride between tokens (1 with ld_grp = M: group-major energies)
  float eps;              // kEpiHeadNorm
  float* dgain_part;      // kEpiHeadNormBwd (nullable): [M / 32 * heads][128] gain-gradient partials
  int heads;
  int32_t* sel_idx;       // kEpiEnergyTopK: [M][sel_k] chosen groups
  int sel_k;
  int unit;               // tiles a CTA takes back to back (<= 1: one); tile ids are unit-major
  int ksplit;             // kModeDense: K splits per output tile (1: none)
  int tile_offset;        // kModeDense: first output tile (raster order) of this launch
  int tile_count;         //   output tiles of this launch (0: all from tile_offset)
  int kb_per_split;       //   k-blocks of each split (the last may be shorter)
  float* part;            // kEpiPartialF32: [ksplit][M][N] fp32 partial sums
  int64_t part_plane;     //   elements per split (M * N)
  int* status;            // device status word
  uint64_t wait_limit_ns;
  // gathered operand (GATHER != kGatherNone)
  const int32_t* gather_token;  // token of each padded row (-1: zero row)
  const void* gather_src;       // bf16 token rows [tokens][gather_ld]
  int64_t gather_ld;            // elements between token rows
  int gather_cols;              // columns that exist (the rest of a tile reads as zero)
};

// Epilogues that move their tiles with TMA: bf16 outputs staged per warp in shared memory
// (32-row boxes, 32 or 64 columns wide: see tma_epi_cols) and, for kEpiDGate and kEpiScale,
// the factor tiles loaded by TMA into the same kind of buffers.  Pair-mode (dense) kernels keep one box per output, which a warp
// overwrites once the previous chunk's store has read it (the chunk's TMEM load and arithmetic
// cover that); this leaves the gate|up kernel its six ring stages.  Measured with a %clock64
// probe of the MMA issuer on B200, its k-blocks then take about 605 cycles, against about 690
// with per-thread 16-byte row stores and 613 with two boxes per output and five stages.  The
// 1-CTA row-grouped tiles of the sparse path keep two boxes per output (one box: sparse dx
// 6% slower).
template <int EPI>
constexpr int tma_epi_outputs() {
  return EPI == kEpiSwiGLU ? 3 : ((EPI == kEpiDGate || EPI == kEpiLeakySq) ? 2 : 1);
}
template <int EPI>
constexpr int tma_epi_aux() {
  return EPI == kEpiDGate ? 2 : (EPI == kEpiScale ? 1 : 0);
}
constexpr int kEpiAuxMap = 2;  // first tensor map of the factors a TMA epilogue loads
// Buffers per epilogue warp for the factor boxes a TMA epilogue loads: kEpiScale's short-K tiles
// (the activation gradient of a 512-deep product) prefetch two 64-column chunks ahead.
template <int EPI>
constexpr int tma_epi_aux_bufs() {
  return EPI == kEpiScale ? 3 : 2;
}
template <bool PAIR>
constexpr int tma_epi_out_bufs() {
  return PAIR ? 1 : 2;
}
// Columns of one output (and factor) staging box (rows: 32, one per lane).  The plain-store
// epilogue of the row-grouped sparse GEMMs and the LeakyReLU^2 up / activation-gradient
// epilogues move 64 columns per chunk through 32 x 64 boxes (128-byte swizzle): their K is one,
// two or eight k-blocks, so each tile is mostly epilogue, and half the chunks means half the
// TMEM-load waits, proxy fences and TMA copies (sparse down 84 -> 62 us, LeakyReLU^2 up 186 ->
// 167 us on B200).  The others keep 32 x 32 boxes (64-byte swizzle).
//
// kEpiDGate works in place: its two factor boxes (a, b: 32 rows x 64 columns, 128-byte swizzle)
// receive dG = dH a and dU = dH b and are stored from there, so it needs no output boxes and
// moves whole 128-byte rows.  Measured with a %clock64 probe of the MMA issuer on B200, the dH
// kernel's k-blocks take about 544 cycles when its epilogue moves nothing and 620-650 with the
// factor loads and output stores of 32-column chunks: the epilogue's TMA operations delay the
// operand loads of the main loop (the same at 74, 48 and 32 clusters, so not a DRAM limit).
template <int EPI>
constexpr int tma_epi_cols() {
  return (EPI == kEpiStore || EPI == kEpiLeakySq || EPI == kEpiScale || EPI == kEpiDGate) ? 64 : 32;
}
template <int EPI>
constexpr bool tma_epi_in_place() {
  return EPI == kEpiDGate;
}
template <int EPI, bool TMA_EPI, bool PAIR>
constexpr int epi_smem_bytes() {
  return EPI == kEpiEnergyTopK
             ? kTopKMaxGroups * kTileM * 4
             : (TMA_EPI ? 4 * ((tma_epi_in_place<EPI>() ? 0 : tma_epi_out_bufs<PAIR>() * tma_epi_outputs<EPI>()) *
                                   64 * tma_epi_cols<EPI>() +
                               tma_epi_aux_bufs<EPI>() * tma_epi_aux<EPI>() * 64 * tma_epi_cols<EPI>())
                        : 0);
}

// Tensor maps of a TMA epilogue: outputs in o[0..], then the factors it loads by TMA from
// o[kEpiAuxMap] on (kEpiDGate's a/b in o[2], o[3]; kEpiScale's in o[2]).
struct EpiMaps {
  CUtensorMap o[4];
};

// Shared-memory plan of one CTA.  In pair mode (cta_group::2) each CTA holds 128 rows of A and
// BN/2 rows of B; the pair computes a 256 x BN tile.  The stage ring takes what the epilogue
// staging buffers and the barrier block leave of the 227 KB.
template <int BN, bool PAIR = false, int EPI_BYTES = 0>
struct TcSmem {
  static constexpr int kBRows = PAIR ? BN / 2 : BN;
  static constexpr int kABytes = kTileM * kTileK * 2;
  static constexpr int kBBytes = kBRows * kTileK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  // Without epilogue staging the ring stays at 192 KB (6 pair stages): measured on B200, a
  // deeper ring that fills the 227 KB slowed the direct-store epilogues by 3-4%.
  static constexpr int kBudget = EPI_BYTES == 0 ? 196608 : 232448 - 1024 - 512 - EPI_BYTES;
  static constexpr int kStages = (kBudget / kStageBytes) < 8 ? (kBudget / kStageBytes) : 8;
  static constexpr int kTileBytes = kStages * kStageBytes;
  static constexpr int kEpiOffset = kTileBytes;
  static constexpr int kBarOffset = kTileBytes + EPI_BYTES;
  static constexpr int kBytes = kBarOffset + 512 + 1024;  // barriers + alignment slack
};

__device__ __forceinline__ void tile_coords(int tile, int num_m, int num_n, int raster, int& mb,
                                            int& nb) {
  const int per_group = raster * num_n;
  const int g = tile / per_group;
  const int r = tile - g * per_group;
  const int m0 = g * raster;
  const int gm = min(raster, num_m - m0);
  mb = m0 + r % gm;
  nb = r / gm;
}

// The i-th tile of a persistent CTA: units of `unit` consecutive tile ids, dealt out round robin.
__device__ __forceinline__ int sched_tile(int i, int tile0, int step, int unit) {
  if (unit <= 1) return tile0 + i * step;
  const int u = i / unit;
  return (tile0 + u * step) * unit + (i - u * unit);
}

// What one tile computes: output block (mb, nb), group (-1: skip), TMA coordinates of its first
// k-block, and its number of k-blocks.
struct Tile {
  int mb, nb, grp;
  int a_m, a_k, b_n, b_k;
  int kb;
  int ks;  // K split (split-K GEMMs)
};

template <int BN, bool B_DUAL, int MODE>
__device__ __forceinline__ Tile decode_tile(int tile, const TcGemmArgs& a) {
  Tile t;
  if constexpr (MODE == kModeKGrouped) {
    const int per = a.num_m_blk * a.num_n_blk;
    t.grp = tile / per;
    const int r = tile - t.grp * per;
    t.mb = r % a.num_m_blk;
    t.nb = r / a.num_m_blk;
    const int s0 = a.seg_start[t.grp];
    t.a_m = t.mb * kTileM;
    t.a_k = s0;
    t.b_n = t.nb * BN;
    t.b_k = s0;
    t.kb = a.seg_rows[t.grp] / kTileK;
  } else {
    t.ks = 0;
    if (MODE == kModeDense && a.ksplit > 1) {  // consecutive tiles are the splits of one block
      t.ks = tile % a.ksplit;
      tile /= a.ksplit;
    }
    if (MODE == kModeDense) tile += a.tile_offset;
    tile_coords(tile, a.num_m_blk, a.num_n_blk, a.raster, t.mb, t.nb);
    t.grp = MODE == kModeRowGrouped ? a.tile_group[t.mb] : 0;
    const int g = t.grp < 0 ? 0 : t.grp;
    const int k0 = t.ks * a.kb_per_split * kTileK;
    t.a_m = t.mb * kTileM;
    t.a_k = k0;
    t.b_n = t.nb * (B_DUAL ? BN / 2 : BN) + g * a.grp_b_n;
    t.b_k = g * a.grp_b_k + k0;
    t.kb = a.ksplit > 1 ? min(a.kb_per_split, a.kb_total - t.ks * a.kb_per_split) : a.kb_total;
  }
  return t;
}

// Adds the bias (if any) to one token's n_groups (<= kTopKMaxGroups) energies e_row[g * stride]
// (writing the sums to e_out[g * out_stride] if e_out), then selects the top k of them as k rounds of an argmax that
// prefers the larger energy and, among equal energies, the lower group; NaN is never chosen.  The
// energies become order-preserving int keys (NaN, chosen and absent slots: INT_MIN, below -inf),
// and each round is a pairwise tree over the 64 slots (left = lower groups; the right side wins
// only with a strictly larger key), so its compares are independent.  The chosen groups go out in
// ascending order, then -1 for rounds that found nothing.
__device__ __forceinline__ void topk_row(const float* e_row, int64_t stride, int n_groups,
                                         const float* bias, float* e_out, int64_t out_stride,
                                         int k, int32_t* out) {
  const float kNaN = __int_as_float(0x7fc00000);
  float e[kTopKMaxGroups];
#pragma unroll
  for (int j = 0; j < kTopKMaxGroups; ++j) e[j] = ld_if(e_row + j * stride, j < n_groups, kNaN);
  if (bias) {
#pragma unroll
    for (int j = 0; j < kTopKMaxGroups; ++j) e[j] += ld_if(bias + j, j < n_groups, 0.f);
  }
  if (e_out) {
#pragma unroll
    for (int j = 0; j < kTopKMaxGroups; ++j) st_if(e_out + j * out_stride, e[j], j < n_groups);
  }
  int key[kTopKMaxGroups];
#pragma unroll
  for (int j = 0; j < kTopKMaxGroups; ++j) {
    const int b = __float_as_int(e[j] + 0.0f);  // -0 -> +0: equal energies get equal keys
    key[j] = e[j] != e[j] ? INT32_MIN : (b >= 0 ? b : b ^ 0x7fffffff);
  }
  uint64_t taken = 0;
  for (int r = 0; r < k; ++r) {
    int v[kTopKMaxGroups / 2];
    int ix[kTopKMaxGroups / 2];
#pragma unroll
    for (int i = 0; i < kTopKMaxGroups / 2; ++i) {
      const bool right = key[2 * i + 1] > key[2 * i];
      v[i] = right ? key[2 * i + 1] : key[2 * i];
      ix[i] = right ? 2 * i + 1 : 2 * i;
    }
#pragma unroll
    for (int w = kTopKMaxGroups / 4; w >= 1; w >>= 1) {
#pragma unroll
      for (int i = 0; i < w; ++i) {
        const bool right = v[2 * i + 1] > v[2 * i];
        v[i] = right ? v[2 * i + 1] : v[2 * i];
        ix[i] = right ? ix[2 * i + 1] : ix[2 * i];
      }
    }
    if (v[0] == INT32_MIN) break;  // only NaN, chosen or absent slots are left
    const int win = ix[0];
    taken |= 1ull << win;
#pragma unroll
    for (int j = 0; j < kTopKMaxGroups; ++j) key[j] = j == win ? INT32_MIN : key[j];
  }
  int p = 0;
#pragma unroll
  for (int j = 0; j < kTopKMaxGroups; ++j) {
    const bool bit = (taken >> j) & 1ull;
    st_if(out + p, j, bit);
    p += bit;
  }
  for (; p < k; ++p) out[p] = -1;
}

// ep[(g0 + q) * lg] = v[q] for the NG group sums of a chunk that exist (g0 + q < n_groups).
template <int NG>
__device__ __forceinline__ void store_group_sums(float* ep, int64_t lg, int g0, int n_groups,
                                                 const float (&v)[32]) {
#pragma unroll
  for (int q = 0; q < NG; ++q) st_if(ep + (g0 + q) * lg, v[q], g0 + q < n_groups);
}

// 16-byte vector store of 8 bf16 values held as 4 packed words.
__device__ __forceinline__ void st_v4(void* p, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  *reinterpret_cast<uint4*>(p) = make_uint4(a, b, c, d);
}

// CW consecutive fp32 columns of this thread's TMEM lane (CW = 16 or 32).
template <int CW>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, float (&v)[32]) {
  if constexpr (CW == 32) {
    tmem_ld32(taddr, v);
  } else {
    tmem_ld16(taddr, v);
  }
}

__device__ __forceinline__ void store_bf16x8(__nv_bfloat16* p, const float* v) {
  st_v4(p, pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
        pack_bf16x2(v[6], v[7]));
}

// PAIR: launched as clusters of 2 CTAs; the even CTA issues tcgen05.mma.cta_group::2 over both
// CTAs' shared memory, each CTA keeps its 128 rows of the 256 x BN accumulator in its own TMEM
// and runs its own epilogue.  Both CTAs' TMA loads complete on the even CTA's stage barrier,
// and the MMA commits arrive on the stage and accumulator barriers of both CTAs.
template <int BN, bool A_MN, bool B_MN, bool B_DUAL, int EPI, int MODE = kModeDense,
          bool PAIR = false, bool TMA_EPI = false, int GATHER = kGatherNone>
__global__ void __launch_bounds__(gemm_threads<GATHER>(), 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                   const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ EpiMaps emaps,
                   const TcGemmArgs args) {
  using L = TcSmem<BN, PAIR, epi_smem_bytes<EPI, TMA_EPI, PAIR>()>;
  constexpr int S = L::kStages;
  constexpr uint32_t kIdesc = idesc_bf16(PAIR ? 2 * kTileM : kTileM, BN, A_MN ? 1 : 0, B_MN ? 1 : 0);
  // A pair tile whose N-block holds at most BN / 2 columns of the output (the last block of an N
  // that is not a multiple of BN, e.g. d_ff = 5504 in 256-column blocks) is computed with N = BN / 2:
  // each CTA stages BN / 4 of its columns (the odd CTA the second quarter, not the second half),
  // and half the MMA work of an all-zero half is not spent.
  constexpr bool kHalfTiles = PAIR && !B_DUAL && MODE == kModeDense && BN % 64 == 0;
  constexpr uint32_t kIdescHalf = idesc_bf16(2 * kTileM, BN / 2, A_MN ? 1 : 0, B_MN ? 1 : 0);
  auto half_tile = [&](const Tile& t_) {
    return kHalfTiles && t_.nb == args.num_n_blk - 1 && args.N - t_.nb * BN <= BN / 2;
  };
  constexpr int kTmemCols = 2 * BN < 32 ? 32 : 2 * BN;  // two accumulators
  constexpr int kBRows = L::kBRows;
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "UMMA N");
  static_assert(!B_MN || kBRows % 64 == 0, "MN-major B tiles are whole 64-column boxes");
  static_assert(!PAIR || (MODE == kModeDense && BN % 32 == 0), "pair mode: dense tiles");
  static_assert(GATHER == kGatherNone ||
                    (!PAIR && ((GATHER == kGatherA && MODE == kModeRowGrouped && !A_MN) ||
                               (GATHER == kGatherA && MODE == kModeKGrouped && A_MN) ||
                               (GATHER == kGatherB && MODE == kModeKGrouped && B_MN))),
                "gathered operands: K-major A of row-grouped tiles, MN-major A or B of per-group-K tiles");
  static_assert(!TMA_EPI || (MODE == kModeDense && (EPI == kEpiStore || EPI == kEpiSwiGLU ||
                                                    EPI == kEpiSwiGLUInf || EPI == kEpiDGate ||
                                                    EPI == kEpiScale || EPI == kEpiLeakySq)) ||
                    (MODE == kModeRowGrouped && (EPI == kEpiStore || EPI == kEpiSwiGLU || EPI == kEpiDGate)),
                "TMA epilogue: dense bf16 outputs, or row-grouped plain / SwiGLU / gating stores");
  // each gather warp owns whole ring stages: more warps than stages would let two of them wait on
  // the same stage's barriers one phase apart
  static_assert(GATHER == kGatherNone || S >= kGatherWarps, "a ring stage per gather warp");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOffset);
  uint64_t* empty = full + S;
  uint64_t* tfull = empty + S;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* auxbar = drain + 1;  // [4 epilogue warps][up to 4 buffers]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(auxbar + 16);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int num_tiles = MODE == kModeKGrouped
                            ? args.num_m_blk * args.num_n_blk * args.n_groups
                            : (args.tile_count > 0 ? args.tile_count : args.num_m_blk * args.num_n_blk - args.tile_offset) *
                                  (args.ksplit > 1 ? args.ksplit : 1);
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const int tile0 = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int tile_step = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
  const int unit_ = args.unit > 1 ? args.unit : 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      // gathered operand: one arrival per lane of the gathering warp after its copies land
      mbar_init(&full[s], GATHER != kGatherNone ? 33 : 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], PAIR ? 256 : 128);
    }
    mbar_init(drain, 1);
    for (int i = 0; i < 16; ++i) mbar_init(&auxbar[i], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB0);
    if (B_DUAL || args.kb_seg0 < args.kb_total) tma_prefetch_desc(&tmB1);
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc_pair(tmem_slot, kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, kTmemCols);
      tmem_relinquish();
    }
  }
  __syncthreads();
  if constexpr (PAIR) cluster_sync();  // both CTAs' barriers exist before any remote signal
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const WaitCtl ctl{abort_flag, args.status, args.wait_limit_ns};

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      // pair mode: every stage completes on the even CTA's barrier
      const uint32_t full_lead = PAIR ? map_to_rank(smem_u32(full), 0) : 0u;
      for (int i_ = 0, tile = tile0 * unit_; ok && tile < num_tiles; tile = sched_tile(++i_, tile0, tile_step, unit_)) {
        Tile t = decode_tile<BN, B_DUAL, MODE>(tile, args);
        if (t.grp < 0) continue;
        if (PAIR) t.a_m = t.mb * 2 * kTileM + (int)rank * kTileM;
        for (int kb = 0; kb < t.kb; ++kb, ++it) {
          const int s = it % S;
          const uint32_t ph = (it / S) & 1u;
          if (!mbar_wait(&empty[s], ph ^ 1u, ctl)) { ok = false; break; }
          uint8_t* sA = smem + s * L::kStageBytes;
          uint8_t* sB = sA + L::kABytes;
          if (!PAIR)
            mbar_arrive_expect_tx(&full[s], GATHER == kGatherA   ? L::kBBytes
                                            : GATHER == kGatherB ? L::kABytes
                                                                 : L::kStageBytes);
          else if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * L::kStageBytes);
          auto load = [&](void* dst, const CUtensorMap* m, int c0, int c1) {
            if constexpr (PAIR) tma_load_2d_pair(dst, m, c0, c1, full_lead + s * 8);
            else tma_load_2d(dst, m, c0, c1, &full[s]);
          };
          const bool seg1 = kb >= args.kb_seg0;
          const int kk = (seg1 ? kb - args.kb_seg0 : kb) * kTileK;  // K inside the segment
          const int ka = t.a_k + (seg1 ? args.a_koff1 + kk : kk);
          if (GATHER == kGatherA) {
            // rows copied by the gather warps
          } else if (A_MN) {
            load(sA, &tmA, t.a_m, ka);
            load(sA + 8192, &tmA, t.a_m + 64, ka);
          } else {
            load(sA, &tmA, ka, t.a_m);
          }
          const CUtensorMap* mapB = seg1 ? &tmB1 : &tmB0;
          const int b_n = t.b_n + (PAIR && !B_DUAL ? (int)rank * (half_tile(t) ? kBRows / 2 : kBRows) : 0);
          if (B_DUAL) {
            if constexpr (PAIR) {
              load(sB, rank ? &tmB1 : &tmB0, t.b_k + kk, t.b_n);  // even CTA: gate rows, odd: up
            } else {
              load(sB, &tmB0, t.b_k + kk, t.b_n);
              load(sB + (BN / 2) * 128, &tmB1, t.b_k + kk, t.b_n);
            }
          } else if (GATHER == kGatherB) {
            // rows copied by the gather warps
          } else if (B_MN) {
#pragma unroll
            for (int j = 0; j < kBRows / 64; ++j) load(sB + j * 8192, mapB, b_n + j * 64, t.b_k + kk);
          } else {
            load(sB, mapB, t.b_k + kk, b_n);
          }
        }
      }
      if (!ok) {
        // Let copies already in flight land before the CTA leaves (bounded).
        WaitCtl quick{abort_flag, args.status, 100000000ull};
        volatile int no_abort = 0;
        quick.abort = &no_abort;
        const uint32_t first = it > (uint32_t)S ? it - S : 0;
        for (uint32_t j = first; j < it; ++j) mbar_wait(&full[j % S], (j / S) & 1u, quick);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ UMMA issuer
    // This one thread's issue loop bounds the dense GEMMs (a %clock64 probe on B200: precomputed
    // descriptors took dx from 542 to 528 cycles per k-block), so it does as little as it can:
    // the smem descriptors of stage 0 are built once and a stage / K step adds its byte offset
    // / 16 to the address field (the whole ring lies below 256 KB, so the 14-bit field cannot
    // carry), and the stage index and phase advance by increment.
    if (lane == 0 && rank == 0) {
      int s = 0;        // ring stage of the next k-block
      uint32_t ph = 0;  // parity of its full barrier
      int local = 0;
      bool ok = true;
      bool issued = false;
      const uint32_t sbase = smem_u32(smem);
      const uint64_t a_desc0 = A_MN ? smem_desc_sw128(sbase, 8192, 1024) : smem_desc_sw128(sbase, 16, 1024);
      const uint64_t b_desc0 = B_MN ? smem_desc_sw128(sbase + L::kABytes, 8192, 1024)
                                    : smem_desc_sw128(sbase + L::kABytes, 16, 1024);
      constexpr uint64_t kAStep = A_MN ? 2048 / 16 : 32 / 16;  // one K step of 16
      constexpr uint64_t kBStep = B_MN ? 2048 / 16 : 32 / 16;
      static_assert(L::kTileBytes + 2048 < (1 << 18), "descriptor address field");
      for (int i_ = 0, tile = tile0 * unit_; ok && tile < num_tiles; tile = sched_tile(++i_, tile0, tile_step, unit_)) {
        const Tile t = decode_tile<BN, B_DUAL, MODE>(tile, args);
        if (t.grp < 0) continue;
        const int buf = local & 1;
        const uint32_t use = static_cast<uint32_t>(local >> 1);
        ++local;
        if (!mbar_wait(&tempty[buf], (use & 1u) ^ 1u, ctl)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * BN;
        const uint32_t idesc = half_tile(t) ? kIdescHalf : kIdesc;
        for (int kb = 0; kb < t.kb; ++kb) {
          if (!mbar_wait(&full[s], ph, ctl)) { ok = false; break; }
          // gathered rows were written by cp.async (generic proxy); the barrier made them
          // visible to this thread, the fence orders them before the MMAs' async-proxy reads
          if constexpr (GATHER != kGatherNone) fence_proxy_async_smem();
          tc_fence_after();
          const uint64_t so = static_cast<uint64_t>(s) * (L::kStageBytes / 16);
#pragma unroll
          for (int k = 0; k < kTileK / kUmmaK; ++k) {
            const uint64_t ad = a_desc0 + so + k * kAStep;
            const uint64_t bd = b_desc0 + so + k * kBStep;
            if constexpr (PAIR) umma_bf16_pair(d_tmem, ad, bd, idesc, (kb | k) != 0 ? 1u : 0u);
            else umma_bf16(d_tmem, ad, bd, kIdesc, (kb | k) != 0 ? 1u : 0u);
          }
          if constexpr (PAIR) umma_commit_pair(&empty[s], 3);
          else umma_commit(&empty[s]);
          if (++s == S) {
            s = 0;
            ph ^= 1u;
          }
          issued = true;
        }
        if (!ok) break;
        if (t.kb > 0) {
          if constexpr (PAIR) umma_commit_pair(&tfull[buf], 3);
          else umma_commit(&tfull[buf]);
        } else {
          mbar_arrive(&tfull[buf]);
          if constexpr (PAIR) mbar_arrive_cluster(map_to_rank(smem_u32(&tfull[buf]), 1));
        }
      }
      if (!ok && issued) {
        if constexpr (PAIR) umma_commit_pair(drain, 1);
        else umma_commit(drain);
        WaitCtl quick{abort_flag, args.status, 100000000ull};
        volatile int no_abort = 0;
        quick.abort = &no_abort;
        mbar_wait(drain, 0, quick);
      }
    }
  } else if (GATHER != kGatherNone && warp >= 6) {
    // ------------------------------------------------------------ gather warps 6 ..
    if constexpr (GATHER != kGatherNone) {
      constexpr bool kKGrp = MODE == kModeKGrouped;
      constexpr int kRows = kKGrp ? kTileK : kTileM;          // rows of the gathered tile
      constexpr int kBlocks = GATHER == kGatherA ? (kKGrp ? 2 : 1) : kBRows / 64;  // 64-col blocks
      constexpr int kPerLane = kRows / 4;                     // rows per lane (4 rows per warp step)
      constexpr uint32_t kOpOff = GATHER == kGatherA ? 0u : (uint32_t)L::kABytes;
      const int gw = warp - 6;
      const int ch = lane & 7;     // 16-byte chunk of a 128-byte row piece
      const int rsub = lane >> 3;  // row of the warp's 4-row step
      const char* src = static_cast<const char*>(args.gather_src);
      const int64_t ld_bytes = args.gather_ld * 2;
      const uint32_t sbase = smem_u32(smem) + kOpOff;
      uint32_t it = 0;
      bool ok = true;
      int tok[kPerLane];
      for (int i_ = 0, tile = tile0 * unit_; ok && tile < num_tiles; tile = sched_tile(++i_, tile0, tile_step, unit_)) {
        const Tile t = decode_tile<BN, B_DUAL, MODE>(tile, args);
        if (t.grp < 0) continue;
        if constexpr (!kKGrp) {  // the tile's 128 padded rows are its M rows: same for every k-block
#pragma unroll
          for (int i = 0; i < kPerLane; ++i) tok[i] = args.gather_token[t.a_m + rsub + 4 * i];
        }
        for (int kb = 0; kb < t.kb; ++kb, ++it) {
          if ((int)(it % kGatherWarps) != gw) continue;
          const int s = (int)(it % S);
          const uint32_t ph = (it / S) & 1u;
          const bool got = mbar_wait(&empty[s], ph ^ 1u, ctl);
          if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
          int col0;
          if constexpr (kKGrp) {  // the K rows change with every k-block
            const int r0 = (GATHER == kGatherA ? t.a_k : t.b_k) + kb * kTileK;
#pragma unroll
            for (int i = 0; i < kPerLane; ++i) tok[i] = args.gather_token[r0 + rsub + 4 * i];
            col0 = GATHER == kGatherA ? t.a_m : t.b_n;
          } else {
            col0 = t.a_k + kb * kTileK;
          }
          const uint32_t sop = sbase + (uint32_t)s * L::kStageBytes;
#pragma unroll
          for (int j = 0; j < kBlocks; ++j) {
            const int col = col0 + j * 64 + ch * 8;
            const bool col_ok = col < args.gather_cols;
#pragma unroll
            for (int i = 0; i < kPerLane; ++i) {
              const int r = rsub + 4 * i;
              const uint32_t dst = sop + (uint32_t)(j * kRows * 128 + r * 128 + ((ch ^ (r & 7)) << 4));
              const bool v = col_ok && tok[i] >= 0;
              cp_async16(dst, src + (v ? (int64_t)tok[i] * ld_bytes + (int64_t)col * 2 : 0), v);
            }
          }
          cp_async_arrive_noinc(&full[s]);
        }
      }
      cp_async_wait_all();  // copies still in flight land before the CTA leaves
    }
  } else if constexpr (TMA_EPI) {
    // ------------------------------------------------------------ epilogue warps 2..5 (TMA I/O)
    constexpr int NOUT = tma_epi_outputs<EPI>();
    constexpr int NAUX = tma_epi_aux<EPI>();
    constexpr bool kGLU = EPI == kEpiSwiGLU || EPI == kEpiSwiGLUInf;
    constexpr bool kDual = kGLU;  // [g | u] accumulator halves
    constexpr int CWO = tma_epi_cols<EPI>();  // output columns per chunk
    constexpr bool kInPlace = tma_epi_in_place<EPI>();
    static_assert(CWO == 32 || (CWO == 64 && !kDual && (NAUX <= 1 || kInPlace)), "64-column chunks");
    constexpr int kOutBox = 64 * CWO;         // bytes of one 32-row output (or factor) box
    constexpr int NCH = (kDual ? BN / 2 : BN) / CWO;
    static_assert((kDual ? BN / 2 : BN) % CWO == 0, "whole chunks");
    const int q = warp & 3;  // TMEM lane quadrant this warp may access
    const int ew = warp - 2;
    constexpr int AB = tma_epi_aux_bufs<EPI>();
    constexpr int OB = tma_epi_out_bufs<PAIR>();
    constexpr int kOutBoxes = kInPlace ? 0 : OB * NOUT;
    uint8_t* ebase = smem + L::kEpiOffset + ew * (kOutBoxes + AB * NAUX) * kOutBox;  // boxes [NOUT][OB]
    uint8_t* abase = ebase + kOutBoxes * kOutBox;  // aux buffers [AB][NAUX]
    uint64_t* abar = auxbar + ew * AB;
    const uint32_t tempty_lead = PAIR ? map_to_rank(smem_u32(tempty), 0) : 0u;
    const int swz = (lane >> 1) & 3;  // 64-byte swizzle phase of this lane's staging row
    uint32_t aux_issued = 0, aux_done = 0, chunks = 0;
    int local = 0;
    bool ok = true;
    for (int i_ = 0, tile = tile0 * unit_; ok && tile < num_tiles; tile = sched_tile(++i_, tile0, tile_step, unit_)) {
      Tile t = decode_tile<BN, B_DUAL, MODE>(tile, args);
      if (t.grp < 0) continue;
      if (PAIR) t.a_m = t.mb * 2 * kTileM + (int)rank * kTileM;
      const int buf = local & 1;
      const uint32_t use = static_cast<uint32_t>(local >> 1);
      ++local;
      const int m_slab = t.a_m + q * 32;
      const int n_base = t.nb * (kDual ? BN / 2 : BN);
      auto issue_aux = [&](int c) {
        if constexpr (NAUX > 0) {
          if (lane == 0) {
            const int db = aux_issued % AB;
            mbar_arrive_expect_tx(&abar[db], NAUX * kOutBox);
            tma_load_2d(abase + (db * NAUX) * kOutBox, &emaps.o[kEpiAuxMap], n_base + c * CWO, m_slab,
                        &abar[db]);
            if constexpr (NAUX > 1)
              tma_load_2d(abase + (db * NAUX + 1) * kOutBox, &emaps.o[3], n_base + c * CWO, m_slab, &abar[db]);
          }
          ++aux_issued;
        }
      };
      // the factors do not depend on the accumulator: fetch the first chunks' early (in place:
      // once the stores of the chunk that last used the buffer have read it)
      if (kInPlace && lane == 0) bulk_wait_read<AB - 2>();
      __syncwarp();
      for (int c = 0; c < AB - 1 && c < NCH; ++c) issue_aux(c);
      const bool ready = mbar_wait(&tfull[buf], use & 1u, ctl);
      __syncwarp();
      if (!__all_sync(0xffffffffu, ready)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t t_acc = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + buf * BN;
      const bool have_acc = t.kb > 0;
#pragma unroll 1
      for (int c = 0; c < NCH; ++c) {
        const uint8_t* aux = nullptr;
        if constexpr (NAUX > 0) {
          if (c + AB - 1 < NCH) {
            if (kInPlace && lane == 0) bulk_wait_read<AB - 2>();  // that buffer's stores have read it
            __syncwarp();
            issue_aux(c + AB - 1);
          }
          const int db = aux_done % AB;
          const bool got = mbar_wait(&abar[db], (aux_done / AB) & 1u, ctl);
          __syncwarp();
          if (!__all_sync(0xffffffffu, got)) {
            ok = false;
            break;
          }
          ++aux_done;
          aux = abase + (db * NAUX) * kOutBox;
        }
        float v0[32], v1[32];  // kDual: g | u columns; 64-column chunks: the chunk's two halves
        if (have_acc) {
          tmem_ld32(t_acc + c * CWO, v0);
          if constexpr (kDual) tmem_ld32(t_acc + BN / 2 + c * 32, v1);
          else if constexpr (CWO == 64) tmem_ld32(t_acc + c * CWO + 32, v1);
          tmem_ld_wait_regs(v0);
          if constexpr (kDual || CWO == 64) pin_regs(v1);
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) v0[j] = v1[j] = 0.f;
        }
        uint32_t w[NOUT][CWO / 2];
        if constexpr (EPI == kEpiStore) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            w[0][i] = pack_bf16x2(v0[2 * i], v0[2 * i + 1]);
            w[0][16 + i] = pack_bf16x2(v1[2 * i], v1[2 * i + 1]);
          }
        } else if constexpr (kGLU) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            // two columns per f32x2 multiply / FMA (2.2% fewer cycles per k-block on B200: the
            // epilogue shares an issue slot with the MMA-issuing warp)
            const float2 g2 = make_float2(v0[2 * i], v0[2 * i + 1]);
            const float2 u2 = make_float2(v1[2 * i], v1[2 * i + 1]);
            const float2 s2 = make_float2(sigmoidf_(g2.x), sigmoidf_(g2.y));
            const float2 b2 = __fmul2_rn(g2, s2);
            const float2 h2 = __fmul2_rn(b2, u2);
            w[0][i] = pack_bf16x2(h2.x, h2.y);
            if constexpr (EPI == kEpiSwiGLU) {
              const float2 oms = __ffma2_rn(s2, make_float2(-1.f, -1.f), make_float2(1.f, 1.f));
              const float2 a2 = __fmul2_rn(u2, __ffma2_rn(b2, oms, s2));  // u (s + SiLU(g) (1 - s))
              w[1][i] = pack_bf16x2(a2.x, a2.y);
              w[2][i] = pack_bf16x2(b2.x, b2.y);
            }
          }
        } else if constexpr (EPI == kEpiLeakySq) {
#pragma unroll
          for (int i = 0; i < CWO / 2; ++i) {
            const float* vh = i < 16 ? v0 : v1;  // resolved at compile time (unrolled)
            float post[2], ag[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const float pre = vh[2 * (i & 15) + e];
              const float lk = pre > 0.f ? pre : 0.5f * pre;
              post[e] = lk * lk;
              ag[e] = pre > 0.f ? 2.f * pre : 0.5f * pre;
            }
            w[0][i] = pack_bf16x2(post[0], post[1]);
            w[1][i] = pack_bf16x2(ag[0], ag[1]);
          }
        } else if constexpr (EPI == kEpiScale) {
#pragma unroll
          for (int c4 = 0; c4 < CWO / 8; ++c4) {  // 16-byte pieces of the factor row
            const int phys = CWO == 64 ? (c4 ^ (lane & 7)) : (c4 ^ swz);
            const uint4 av = *reinterpret_cast<const uint4*>(aux + lane * (2 * CWO) + phys * 16);
            const uint32_t aw[4] = {av.x, av.y, av.z, av.w};
            const float* vh = c4 < 4 ? v0 : v1;  // resolved at compile time (unrolled)
#pragma unroll
            for (int p = 0; p < 4; ++p)
              w[0][c4 * 4 + p] = pack_bf16x2(vh[(c4 & 3) * 8 + p * 2] * bf16_lo(aw[p]),
                                             vh[(c4 & 3) * 8 + p * 2 + 1] * bf16_hi(aw[p]));
          }
        } else if constexpr (EPI == kEpiDGate) {
          // in place: each 16-byte piece of this lane's factor rows becomes the same piece of dG, dU
          uint8_t* fa = const_cast<uint8_t*>(aux);
#pragma unroll
          for (int c8 = 0; c8 < CWO / 8; ++c8) {
            const int off = lane * (2 * CWO) + ((c8 ^ (lane & 7)) * 16);
            const uint4 av = *reinterpret_cast<const uint4*>(fa + off);
            const uint4 bv = *reinterpret_cast<const uint4*>(fa + kOutBox + off);
            const uint32_t aw[4] = {av.x, av.y, av.z, av.w};
            const uint32_t bw[4] = {bv.x, bv.y, bv.z, bv.w};
            const float* vh = c8 < 4 ? v0 : v1;  // resolved at compile time (unrolled)
            uint32_t gw[4], uw[4];
#pragma unroll
            for (int p = 0; p < 4; ++p) {
              const float d0 = vh[(c8 & 3) * 8 + p * 2], d1 = vh[(c8 & 3) * 8 + p * 2 + 1];
              gw[p] = pack_bf16x2(d0 * bf16_lo(aw[p]), d1 * bf16_hi(aw[p]));
              uw[p] = pack_bf16x2(d0 * bf16_lo(bw[p]), d1 * bf16_hi(bw[p]));
            }
            *reinterpret_cast<uint4*>(fa + off) = make_uint4(gw[0], gw[1], gw[2], gw[3]);
            *reinterpret_cast<uint4*>(fa + kOutBox + off) = make_uint4(uw[0], uw[1], uw[2], uw[3]);
          }
        }
        // stage this warp's 32-row box of every output, then one lane stores them with TMA
        const int db = OB > 1 ? static_cast<int>(chunks & 1u) : 0;
        if constexpr (!kInPlace) {
          if (lane == 0) bulk_wait_read<OB - 1>();  // the store that last used box db has read it
          __syncwarp();
#pragma unroll
          for (int o = 0; o < NOUT; ++o) {
            uint8_t* ob = ebase + (o * OB + db) * kOutBox;
#pragma unroll
            for (int c4 = 0; c4 < CWO / 8; ++c4) {  // 16-byte pieces of this lane's row, swizzled
              const int phys = CWO == 64 ? (c4 ^ (lane & 7)) : (c4 ^ swz);
              *reinterpret_cast<uint4*>(ob + lane * (2 * CWO) + phys * 16) =
                  make_uint4(w[o][c4 * 4], w[o][c4 * 4 + 1], w[o][c4 * 4 + 2], w[o][c4 * 4 + 3]);
            }
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        const int n0 = n_base + c * CWO;
        // A box that starts inside its tensor is clipped by TMA at the far edges; boxes that
        // start past the last row or column are not issued at all.
        if (lane == 0 && m_slab < args.M && n0 < args.N) {
          if constexpr (EPI == kEpiStore) {
            if (m_slab < args.row_split) tma_store_2d(&emaps.o[0], n0, m_slab, ebase + db * kOutBox);
            else tma_store_2d(&emaps.o[1], n0, m_slab - args.row_split, ebase + db * kOutBox);
          } else {
#pragma unroll
            for (int o = 0; o < NOUT; ++o)
              tma_store_2d(&emaps.o[o], n0, m_slab,
                           kInPlace ? aux + o * kOutBox : ebase + (o * OB + db) * kOutBox);
          }
          bulk_commit();
        }
        ++chunks;
      }
      if (!ok) break;
      tc_fence_before();
      if (PAIR && rank != 0) mbar_arrive_remote(tempty_lead + buf * 8);  // TMEM read: own SM
      else mbar_arrive(&tempty[buf]);
    }
    if (lane == 0) {
      // factor loads still in flight after an abort land before the CTA leaves (bounded)
      WaitCtl quick{abort_flag, args.status, 100000000ull};
      volatile int no_abort = 0;
      quick.abort = &no_abort;
      for (; aux_done < aux_issued; ++aux_done) mbar_wait(&abar[aux_done % AB], (aux_done / AB) & 1u, quick);
      bulk_wait_all();
    }
  } else {
    // ------------------------------------------------------------ epilogue warps 2..5
    const int q = warp & 3;  // TMEM lane quadrant this warp may access
    const int row = q * 32 + lane;
    const uint32_t tempty_lead = PAIR ? map_to_rank(smem_u32(tempty), 0) : 0u;
    int local = 0;
    for (int i_ = 0, tile = tile0 * unit_; tile < num_tiles; tile = sched_tile(++i_, tile0, tile_step, unit_)) {
      Tile t = decode_tile<BN, B_DUAL, MODE>(tile, args);
      if (t.grp < 0) continue;
      if (PAIR) t.a_m = t.mb * 2 * kTileM + (int)rank * kTileM;
      const int buf = local & 1;
      const uint32_t use = static_cast<uint32_t>(local >> 1);
      ++local;
      const bool ready = mbar_wait(&tfull[buf], use & 1u, ctl);
      __syncwarp();  // tcgen05.ld is warp-collective: reconverge after the per-thread wait
      if (!__all_sync(0xffffffffu, ready)) break;
      tc_fence_after();
      const uint32_t t_acc = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + buf * BN;
      const bool have_acc = t.kb > 0;
      const int m = t.a_m + row;
      const bool row_ok = m < args.M;

      if constexpr (EPI == kEpiSwiGLU || EPI == kEpiSwiGLUInf) {
        constexpr int CW = BN / 2 < 32 ? BN / 2 : 32;
#pragma unroll 1
        for (int c = 0; c < BN / 2; c += CW) {
          float g[32], u[32];
          if (have_acc) {
            tmem_ld_cols<CW>(t_acc + c, g);
            tmem_ld_cols<CW>(t_acc + BN / 2 + c, u);
            tmem_ld_wait();
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) g[j] = u[j] = 0.f;
          }
          const int n0 = t.nb * (BN / 2) + c;
          if (row_ok) {
            __nv_bfloat16* hp = static_cast<__nv_bfloat16*>(args.out0) + (int64_t)m * args.ld_out + n0;
            __nv_bfloat16* ap = static_cast<__nv_bfloat16*>(const_cast<void*>(args.aux0)) +
                                (int64_t)m * args.ld_aux + n0;
            __nv_bfloat16* bp = static_cast<__nv_bfloat16*>(const_cast<void*>(args.aux1)) +
                                (int64_t)m * args.ld_aux + n0;
#pragma unroll
            for (int v = 0; v < CW / 8; ++v) {
              if (n0 + v * 8 + 8 <= args.N) {
                float hv[8], av[8], bv[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                  const int j = v * 8 + e;
                  const float s = sigmoidf_(g[j]);
                  bv[e] = g[j] * s;
                  hv[e] = bv[e] * u[j];
                  av[e] = u[j] * s * (1.f + g[j] * (1.f - s));
                }
                store_bf16x8(hp + v * 8, hv);
                if constexpr (EPI == kEpiSwiGLU) {
                  store_bf16x8(ap + v * 8, av);
                  store_bf16x8(bp + v * 8, bv);
                }
              }
            }
          }
        }
      } else if constexpr (EPI == kEpiHeadNorm) {
        static_assert(BN % 128 == 0, "whole heads per tile");
#pragma unroll 1
        for (int hd = 0; hd < BN / 128; ++hd) {  // each head: 128 columns of this row
          float v[4][32];
#pragma unroll
          for (int c = 0; c < 4; ++c) tmem_ld32(t_acc + hd * 128 + c * 32, v[c]);
          tmem_ld_wait_regs(v[0]);
          pin_regs(v[1]);
          pin_regs(v[2]);
          pin_regs(v[3]);
          const int n0 = t.nb * BN + hd * 128;
          if (row_ok && n0 < args.N) {
            float ss = 0.f;
#pragma unroll
            for (int c = 0; c < 4; ++c)
#pragma unroll
              for (int j = 0; j < 32; ++j) ss = fmaf(v[c][j], v[c][j], ss);
            const float inv = rsqrtf(ss * (1.0f / 128.0f) + args.eps);
            __nv_bfloat16* op = static_cast<__nv_bfloat16*>(args.out0) + (int64_t)m * args.ld_out + n0;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              float o[32];
#pragma unroll
              for (int j = 0; j < 32; ++j) o[j] = v[c][j] * inv * (args.bias ? args.bias[c * 32 + j] : 1.f);
#pragma unroll
              for (int q8 = 0; q8 < 4; ++q8) store_bf16x8(op + c * 32 + q8 * 8, o + q8 * 8);
            }
          }
        }
      } else if constexpr (EPI == kEpiHeadNormBwd) {
        // three passes over the head's 128 columns, 32 at a time (z re-read from TMEM, dq from
        // global memory): the mean square, then sum(dn n), then dz and the gain partials; the
        // sums run in the same column order as one pass would
        static_assert(BN % 128 == 0, "whole heads per tile");
#pragma unroll 1
        for (int hd = 0; hd < BN / 128; ++hd) {
          const int n0 = t.nb * BN + hd * 128;
          if (n0 >= args.N) continue;  // warp-uniform
          const uint32_t tz = t_acc + hd * 128;
          const __nv_bfloat16* dqp = static_cast<const __nv_bfloat16*>(args.aux0) + (int64_t)m * args.ld_aux + n0;
          auto load_dq = [&](int c, uint32_t (&w)[16]) {
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              const uint4 d4 = row_ok ? *reinterpret_cast<const uint4*>(dqp + c * 32 + v * 8) : make_uint4(0u, 0u, 0u, 0u);
              w[v * 4] = d4.x, w[v * 4 + 1] = d4.y, w[v * 4 + 2] = d4.z, w[v * 4 + 3] = d4.w;
            }
          };
          float ss = 0.f;
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            float z[32];
            tmem_ld32(tz + c * 32, z);
            tmem_ld_wait_regs(z);
#pragma unroll
            for (int j = 0; j < 32; ++j) ss = fmaf(z[j], z[j], ss);
          }
          const float inv = rsqrtf(ss * (1.0f / 128.0f) + args.eps);
          float dot = 0.f;
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            float z[32];
            uint32_t dqw[16];
            tmem_ld32(tz + c * 32, z);
            load_dq(c, dqw);
            tmem_ld_wait_regs(z);
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const float dq = (j & 1) ? bf16_hi(dqw[j >> 1]) : bf16_lo(dqw[j >> 1]);
              const float dn = dq * (args.bias ? args.bias[c * 32 + j] : 1.f);
              dot = fmaf(dn, z[j] * inv, dot);
            }
          }
          const float mdot = dot * (1.0f / 128.0f);
          __nv_bfloat16* op = static_cast<__nv_bfloat16*>(args.out0) + (int64_t)m * args.ld_out + n0;
          float* gp = args.dgain_part
                          ? args.dgain_part + ((int64_t)((t.a_m + (warp & 3) * 32) / 32) * args.heads + n0 / 128) * 128
                          : nullptr;
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            float z[32];
            uint32_t dqw[16];
            tmem_ld32(tz + c * 32, z);
            load_dq(c, dqw);
            tmem_ld_wait_regs(z);
            float o[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const float dq = (j & 1) ? bf16_hi(dqw[j >> 1]) : bf16_lo(dqw[j >> 1]);
              const float nv = z[j] * inv;
              const float dn = dq * (args.bias ? args.bias[c * 32 + j] : 1.f);
              o[j] = inv * (dn - nv * mdot);
            }
            if (row_ok) {
#pragma unroll
              for (int q8 = 0; q8 < 4; ++q8) store_bf16x8(op + c * 32 + q8 * 8, o + q8 * 8);
            }
            if (gp) {  // column sums of dq * n over the warp's 32 rows (fixed order)
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                const float dq = (j & 1) ? bf16_hi(dqw[j >> 1]) : bf16_lo(dqw[j >> 1]);
                float v = dq * z[j] * inv;
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
                if (lane == j) gp[c * 32 + j] = v;
              }
            }
          }
        }
      } else if constexpr (EPI == kEpiRouter) {
        // sigmoid of each logit into this token's output row
        float* rp = static_cast<float*>(args.out0) + (int64_t)m * args.ld_out;
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          float z[32];
          tmem_ld32(t_acc + c, z);
          tmem_ld_wait_regs(z);
          if (row_ok) {
#pragma unroll
            for (int j = 0; j < 32; ++j) st_if(rp + c + j, sigmoidf_(z[j]), c + j < args.N);
          }
        }
      } else if constexpr (EPI == kEpiEnergy || EPI == kEpiEnergyTopK) {
        // |SiLU| of each column, summed over aligned runs of P = energy_p = 2^lp columns (lp <= 6),
        // stored at ep[g * lg] (the bias is added by the top-k step, which reads every energy).  Columns arrive 32 at a time from TMEM (the
        // next 32 load while these are reduced); pairwise sums pack a chunk's group sums into
        // v[0 .. 32/P); a 64-column group spans two chunks.
        // kEpiEnergyTopK keeps the energies of its 128 tokens in shared memory, group-major
        float* ep = EPI == kEpiEnergyTopK
                        ? reinterpret_cast<float*>(smem + L::kEpiOffset) + row
                        : static_cast<float*>(args.out0) + (int64_t)m * args.ld_out;
        const int64_t lg = EPI == kEpiEnergyTopK ? kTileM : (args.ld_grp ? args.ld_grp : 1);
        const int lp = __ffs(args.energy_p) - 1;
        const int lv = lp < 5 ? lp : 5;
        float run = 0.f;
        float nxt[32];
        if (have_acc) tmem_ld32(t_acc, nxt);
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          float v[32];
          if (have_acc) {
            tmem_ld_wait_regs(nxt);
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = nxt[j];
            if (c + 32 < BN) tmem_ld32(t_acc + c + 32, nxt);  // warp-uniform: before any row test
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = 0.f;
          }
          if (!row_ok) continue;
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = fabsf(v[j] * sigmoidf_(v[j]));
#pragma unroll
          for (int l = 1, w = 16; l <= 5; ++l, w >>= 1) {
            if (l <= lv) {
#pragma unroll
              for (int j = 0; j < w; ++j) v[j] = v[2 * j] + v[2 * j + 1];
            }
          }
          const int n0 = t.nb * BN + c;
          const int g0 = n0 >> lp;
          if (lp == 6) {
            if ((n0 & 32) == 0) {
              run = v[0];
            } else if (g0 < args.n_groups) {
              ep[g0 * lg] = run + v[0];
            }
          } else {
            switch (lv) {  // a fixed number of group sums per chunk for each group width
              case 0: store_group_sums<32>(ep, lg, g0, args.n_groups, v); break;
              case 1: store_group_sums<16>(ep, lg, g0, args.n_groups, v); break;
              case 2: store_group_sums<8>(ep, lg, g0, args.n_groups, v); break;
              case 3: store_group_sums<4>(ep, lg, g0, args.n_groups, v); break;
              case 4: store_group_sums<2>(ep, lg, g0, args.n_groups, v); break;
              default: store_group_sums<1>(ep, lg, g0, args.n_groups, v); break;
            }
          }
        }
      } else {
        static_assert(EPI == kEpiSwiGLU || EPI == kEpiSwiGLUInf || BN % 32 == 0, "chunking");
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          float acc[32];
          if (have_acc) {
            tmem_ld32(t_acc + c, acc);
            tmem_ld_wait();
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) acc[j] = 0.f;
          }
          const int n0 = t.nb * BN + c;
          if (!row_ok) continue;
          if constexpr (EPI == kEpiPartialF32) {
            float* pp = args.part + (int64_t)t.ks * args.part_plane + (int64_t)m * args.N + n0;
#pragma unroll
            for (int v = 0; v < 8; ++v)
              if (n0 + v * 4 + 4 <= args.N)
                *reinterpret_cast<float4*>(pp + v * 4) =
                    make_float4(acc[v * 4], acc[v * 4 + 1], acc[v * 4 + 2], acc[v * 4 + 3]);
          } else if constexpr (EPI == kEpiLeakySq) {
            __nv_bfloat16* pp = static_cast<__nv_bfloat16*>(args.out0) + (int64_t)m * args.ld_out + n0;
            __nv_bfloat16* gp = static_cast<__nv_bfloat16*>(const_cast<void*>(args.aux0)) +
                                (int64_t)m * args.ld_aux + n0;
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              if (n0 + v * 8 + 8 <= args.N) {
                float post[8], ag[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                  const float pre = acc[v * 8 + e];
                  const float lk = pre > 0.f ? pre : 0.5f * pre;
                  post[e] = lk * lk;
                  ag[e] = pre > 0.f ? 2.f * pre : 0.5f * pre;
                }
                store_bf16x8(pp + v * 8, post);
                store_bf16x8(gp + v * 8, ag);
              }
            }
          } else if constexpr (EPI == kEpiStore) {
            __nv_bfloat16* op =
                m < args.row_split
                    ? static_cast<__nv_bfloat16*>(args.out0) + (int64_t)m * args.ld_out + n0
                    : static_cast<__nv_bfloat16*>(args.out1) +
                          (int64_t)(m - args.row_split) * args.ld_out + n0;
#pragma unroll
            for (int v = 0; v < 4; ++v)
              if (n0 + v * 8 + 8 <= args.N) store_bf16x8(op + v * 8, acc + v * 8);
          } else if constexpr (EPI == kEpiDGate) {
            const __nv_bfloat16* ap =
                static_cast<const __nv_bfloat16*>(args.aux0) + (int64_t)m * args.ld_aux + n0;
            const __nv_bfloat16* bp =
                static_cast<const __nv_bfloat16*>(args.aux1) + (int64_t)m * args.ld_aux + n0;
            __nv_bfloat16* gp = static_cast<__nv_bfloat16*>(args.out0) + (int64_t)m * args.ld_out + n0;
            __nv_bfloat16* up = gp + args.d_ff;
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              if (n0 + v * 8 + 8 <= args.N) {
                const uint4 av = *reinterpret_cast<const uint4*>(ap + v * 8);
                const uint4 bv = *reinterpret_cast<const uint4*>(bp + v * 8);
                const uint32_t aw[4] = {av.x, av.y, av.z, av.w};
                const uint32_t bw[4] = {bv.x, bv.y, bv.z, bv.w};
                uint32_t gw[4], uw[4];
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                  const float d0 = acc[v * 8 + p * 2], d1 = acc[v * 8 + p * 2 + 1];
                  gw[p] = pack_bf16x2(d0 * bf16_lo(aw[p]), d1 * bf16_hi(aw[p]));
                  uw[p] = pack_bf16x2(d0 * bf16_lo(bw[p]), d1 * bf16_hi(bw[p]));
                }
                st_v4(gp + v * 8, gw[0], gw[1], gw[2], gw[3]);
                st_v4(up + v * 8, uw[0], uw[1], uw[2], uw[3]);
              } else if (n0 + v * 8 < args.pad_cols) {
                st_v4(gp + v * 8, 0u, 0u, 0u, 0u);
                st_v4(up + v * 8, 0u, 0u, 0u, 0u);
              }
            }
          } else if constexpr (EPI == kEpiGroupDWgu) {
            const int G = args.group_size;
            __nv_bfloat16* op = nullptr;
            if (m < G)
              op = static_cast<__nv_bfloat16*>(args.out0) + (int64_t)(t.grp * G + m) * args.ld_out + n0;
            else if (m >= 64 && m < 64 + G)
              op = static_cast<__nv_bfloat16*>(args.out1) +
                   (int64_t)(t.grp * G + m - 64) * args.ld_out + n0;
            if (op) {
#pragma unroll
              for (int v = 0; v < 4; ++v)
                if (n0 + v * 8 + 8 <= args.N) store_bf16x8(op + v * 8, acc + v * 8);
            }
          } else if constexpr (EPI == kEpiGroupDWd) {
            const int G = args.group_size;
            __nv_bfloat16* op = static_cast<__nv_bfloat16*>(args.out0) + (int64_t)m * args.ld_out +
                                t.grp * G + n0;
#pragma unroll
            for (int v = 0; v < 4; ++v)
              if (n0 + v * 8 + 8 <= G) store_bf16x8(op + v * 8, acc + v * 8);
          }
        }
      }
      tc_fence_before();
      if (PAIR && rank != 0) mbar_arrive_remote(tempty_lead + buf * 8);  // TMEM read: own SM
      else mbar_arrive(&tempty[buf]);
      if constexpr (EPI == kEpiEnergyTopK) {
        // this thread wrote its token's whole energy row (all N-blocks of the unit): select
        if (row_ok && t.nb == args.num_n_blk - 1)
          topk_row(reinterpret_cast<const float*>(smem + L::kEpiOffset) + row, kTileM,
                   args.n_groups, args.bias,
                   args.out0 ? static_cast<float*>(args.out0) + (int64_t)m * args.ld_out : nullptr,
                   args.ld_grp ? args.ld_grp : 1, args.sel_k, args.sel_idx + (int64_t)m * args.sel_k);
      }
    }
  }

  __syncthreads();
  if constexpr (PAIR) cluster_sync();  // the pair's MMAs and TMEM reads are all done
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    if constexpr (PAIR) tmem_dealloc_pair(tmem_base, kTmemCols);
    else tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace swf
