// Group-sparse SwiGLU FFN (eugen_sparse README, "What it does", "Parameters and how to choose
// them", "Pitfalls and limitations"): subsample index, grouped top-k selection, group
// bucketing, sparse forward and backward.
//
// Layout of the group-major ("padded") row space shared by the sparse kernels: the
// (token, group) pairs are bucketed by group, ascending token within a group; group g owns the
// rows [seg_start[g], seg_start[g] + seg_rows[g]) where seg_rows[g] is its pair count rounded
// up to 128, so that every 128-row tile belongs to one group (tile_group[tile], -1 when the
// tile is past the last group).  row_token[r] is the token of padded row r (-1: padding);
// padding rows of every group-major buffer are zero, so they add nothing to any sum.
#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include "swf_launch.cuh"
#include "swf_sparse.h"

namespace swf {

namespace {

constexpr int kBucketSmemBytes = 98304;
constexpr int kBucketRowsSmemBytes = 32768;  // the place kernel stages its group_idx tile up to this
// The plain-store TMA epilogue's staging boxes: 32 rows x kStoreBoxCols columns, swizzled by
// the width in bytes (the tensor maps of its outputs must match them).
constexpr int kStoreBoxCols = tma_epi_cols<kEpiStore>();
constexpr int kStoreBoxSwizzle = kStoreBoxCols * 2;
static_assert(kStoreBoxSwizzle == 64 || kStoreBoxSwizzle == 128, "box row = swizzle span");

struct SparseDims {
  int64_t M, d, f;
  int G, K, ng;
  int64_t pairs;
  int64_t rmax;   // rows of the padded space (upper bound)
  int mblk;       // 128-row tiles of the padded space
  int words;      // 32-token words per bucketing block
  int tok_blk;    // tokens per bucketing block
  int nblk;       // bucketing blocks
};

SparseDims dims_of(int64_t M, int64_t d, int64_t f, int32_t G, int32_t K) {
  SparseDims s{};
  s.M = M, s.d = d, s.f = f, s.G = G, s.K = K;
  s.ng = (int)(f / G);
  s.pairs = M * K;
  s.rmax = (int64_t)round_up((size_t)(s.pairs + (int64_t)s.ng * 127), 128);
  s.mblk = (int)(s.rmax / 128);
  // the place kernel's shared memory: bitmaps and prefixes (8 ng words bytes) and per-group bases
  // (8 ng bytes), within kBucketSmemBytes where possible
  const int words_smem = std::max(1, std::min(32, (kBucketSmemBytes - 8 * s.ng) / (8 * std::max(1, s.ng))));
  const int64_t words_fill = (M + 32 * 296 - 1) / (32 * 296);  // about two blocks per SM
  s.words = (int)std::max<int64_t>(1, std::min<int64_t>(words_smem, words_fill));
  s.tok_blk = 32 * s.words;
  s.nblk = (int)((M + s.tok_blk - 1) / s.tok_blk);
  return s;
}

// Carves consecutive 256-byte aligned pieces out of one buffer.
struct Carver {
  char* base;
  size_t off = 0;
  template <class T>
  T* take(size_t count) {
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off = round_up(off + count * sizeof(T), 256);
    return p;
  }
};

struct SavedView {
  int32_t *offs, *tokens, *seg_start, *seg_rows, *tile_group, *row_token, *pair_row;
  __nv_bfloat16 *h, *a, *b;
};

SavedView saved_view(void* base, const SparseDims& s, size_t* bytes) {
  Carver c{static_cast<char*>(base)};
  SavedView v;
  v.offs = c.take<int32_t>(s.ng + 1);
  v.tokens = c.take<int32_t>(s.pairs);
  v.seg_start = c.take<int32_t>(s.ng + 1);
  v.seg_rows = c.take<int32_t>(s.ng);
  v.tile_group = c.take<int32_t>(s.mblk);
  v.row_token = c.take<int32_t>(s.rmax);
  v.pair_row = c.take<int32_t>(s.pairs);
  v.h = c.take<__nv_bfloat16>(s.rmax * s.G);
  v.a = c.take<__nv_bfloat16>(s.rmax * s.G);
  v.b = c.take<__nv_bfloat16>(s.rmax * s.G);
  if (bytes) *bytes = c.off;
  return v;
}

struct FwdWs {
  int32_t* counts;
  __nv_bfloat16* yc;  // per-pair contributions to y, group-major rows
};
FwdWs fwd_ws(void* base, const SparseDims& s, size_t* bytes) {
  Carver c{static_cast<char*>(base)};
  FwdWs w;
  w.counts = c.take<int32_t>((size_t)s.nblk * s.ng);
  w.yc = c.take<__nv_bfloat16>(s.rmax * s.d);
  if (bytes) *bytes = c.off;
  return w;
}

struct BwdWs {
  __nv_bfloat16* dgu;
  __nv_bfloat16* dxc;  // per-pair contributions to dx, group-major rows
};
BwdWs bwd_ws(void* base, const SparseDims& s, size_t* bytes) {
  Carver c{static_cast<char*>(base)};
  BwdWs w;
  w.dgu = c.take<__nv_bfloat16>(s.rmax * 128);
  w.dxc = c.take<__nv_bfloat16>(s.rmax * s.d);
  if (bytes) *bytes = c.off;
  return w;
}

int pow2_at_least(int v) {
  int p = 1;
  while (p < v) p <<= 1;
  return p;
}

struct SelWs {
  __nv_bfloat16* wsub;
  float* energies;
};
SelWs sel_ws(void* base, int64_t M, int64_t d, int ng, int P, bool need_wsub, bool need_e,
             size_t* bytes) {
  Carver c{static_cast<char*>(base)};
  SelWs w{nullptr, nullptr};
  if (need_wsub) w.wsub = c.take<__nv_bfloat16>((size_t)ng * P * d);
  if (need_e) w.energies = c.take<float>((size_t)M * ng);
  if (bytes) *bytes = c.off;
  return w;
}

// ------------------------------------------------------------------ device kernels

// Slot k of a group_idx row counts only if its group is in range and not repeated earlier in
// the row (duplicates and out-of-range values are outside the contract; they are dropped so
// that no kernel reads or writes out of bounds).
__device__ __forceinline__ bool valid_slot(const int32_t* row, int k, int ng) {
  const int c = row[k];
  if (c < 0 || c >= ng) return false;
  for (int j = 0; j < k; ++j)
    if (row[j] == c) return false;
  return true;
}

__global__ void bucket_count_kernel(const int32_t* __restrict__ idx, int64_t M, int K, int ng,
                                    int tok_blk, int32_t* __restrict__ counts,
                                    int32_t* __restrict__ row_token, int64_t rmax) {
  extern __shared__ int32_t hist[];
  for (int c = threadIdx.x; c < ng; c += blockDim.x) hist[c] = 0;
  // the row -> token table starts as all padding (-1); the place kernel fills the rows in use
  if (row_token) {
    for (int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; r < rmax; r += (int64_t)gridDim.x * blockDim.x)
      row_token[r] = -1;
  }
  __syncthreads();
  const int64_t t0 = (int64_t)blockIdx.x * tok_blk;
  for (int i = threadIdx.x; i < tok_blk * K; i += blockDim.x) {
    const int64_t t = t0 + i / K;
    if (t >= M) break;
    const int32_t* row = idx + t * K;
    const int k = i % K;
    if (valid_slot(row, k, ng)) atomicAdd(&hist[row[k]], 1);
  }
  __syncthreads();
  for (int c = threadIdx.x; c < ng; c += blockDim.x) counts[(int64_t)c * gridDim.x + blockIdx.x] = hist[c];
}

// One block: turns the per-block counts (group-major, [ng][nblk]) into exclusive per-block
// bases with one warp-wide scan per group, writes the CSR offsets and, when seg_start is given,
// the padded segments and the tile -> group table.
__global__ void bucket_scan_kernel(int32_t* __restrict__ counts, int nblk, int ng,
                                   int32_t* __restrict__ offs, int32_t* __restrict__ seg_start,
                                   int32_t* __restrict__ seg_rows, int32_t* __restrict__ tile_group,
                                   int mblk) {
  extern __shared__ int32_t sh[];
  int32_t* tot = sh;            // [ng]
  int32_t* sstart = sh + ng;    // [ng + 1]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
  constexpr int kBatch = 8;  // 32-block chunks whose counts are loaded together (one latency)
  for (int c = warp; c < ng; c += nwarps) {
    int32_t* row = counts + (int64_t)c * nblk;
    int32_t run = 0;
    for (int b0 = 0; b0 < nblk; b0 += 32 * kBatch) {
      int32_t v[kBatch];
#pragma unroll
      for (int j = 0; j < kBatch; ++j) {
        const int b = b0 + j * 32 + lane;
        v[j] = b < nblk ? row[b] : 0;
      }
#pragma unroll
      for (int j = 0; j < kBatch; ++j) {
        const int b = b0 + j * 32 + lane;
        int32_t incl = v[j];
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const int32_t n = __shfl_up_sync(0xffffffffu, incl, off);
          if (lane >= off) incl += n;
        }
        if (b < nblk) row[b] = run + incl - v[j];
        run += __shfl_sync(0xffffffffu, incl, 31);
      }
    }
    if (lane == 0) tot[c] = run;
  }
  __syncthreads();
  if (warp == 0) {
    int32_t o = 0, p = 0;
    for (int c0 = 0; c0 < ng; c0 += 32) {
      const int c = c0 + lane;
      const int32_t t = c < ng ? tot[c] : 0;
      const int32_t pt = (t + 127) / 128 * 128;
      int32_t it = t, ip = pt;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int32_t n1 = __shfl_up_sync(0xffffffffu, it, off);
        const int32_t n2 = __shfl_up_sync(0xffffffffu, ip, off);
        if (lane >= off) {
          it += n1;
          ip += n2;
        }
      }
      if (c < ng) {
        offs[c] = o + it - t;
        sstart[c] = p + ip - pt;
      }
      o += __shfl_sync(0xffffffffu, it, 31);
      p += __shfl_sync(0xffffffffu, ip, 31);
    }
    if (lane == 0) {
      offs[ng] = o;
      sstart[ng] = p;
    }
  }
  __syncthreads();
  if (seg_start == nullptr) return;
  for (int c = threadIdx.x; c <= ng; c += blockDim.x) {
    seg_start[c] = sstart[c];
    if (c < ng) seg_rows[c] = sstart[c + 1] - sstart[c];
  }
  for (int mb = threadIdx.x; mb < mblk; mb += blockDim.x) {
    const int r = mb * 128;
    int g = -1;
    if (r < sstart[ng]) {
      int lo = 0, hi = ng - 1;  // last group with sstart[g] <= r
      while (lo < hi) {
        const int mid = (lo + hi + 1) / 2;
        if (sstart[mid] <= r) lo = mid;
        else hi = mid - 1;
      }
      g = lo;
    }
    tile_group[mb] = g;
  }
}

// Places every valid (token, group) pair: rank among the block's tokens of the same group from
// a per-group bitmap of the block's tokens, so the order within a group is ascending token id.
// The block's group_idx rows and, per group, its base (CSR offset + the block's scanned count)
// and padded segment start are staged in shared memory first, so the placement itself makes no
// dependent global loads.
__global__ void bucket_place_kernel(const int32_t* __restrict__ idx, int64_t M, int K, int ng,
                                    int words, const int32_t* __restrict__ counts,
                                    const int32_t* __restrict__ offs, int32_t* __restrict__ tokens,
                                    const int32_t* __restrict__ seg_start,
                                    int32_t* __restrict__ row_token,
                                    int32_t* __restrict__ pair_row, int stage_rows) {
  extern __shared__ uint32_t smem_bits[];
  const int tok_blk = 32 * words;
  uint32_t* bits = smem_bits;                                           // [ng][words]
  int32_t* pre = reinterpret_cast<int32_t*>(smem_bits + (size_t)ng * words);  // [ng][words]
  int32_t* base_tok = pre + (size_t)ng * words;                         // [ng]
  int32_t* base_row = base_tok + ng;                                    // [ng]
  int32_t* rows_smem = base_row + ng;                                   // [tok_blk * K] if staged
  const int64_t t0 = (int64_t)blockIdx.x * tok_blk;
  const int64_t left = M - t0;
  const int nslots = (int)(left < tok_blk ? left : (int64_t)tok_blk) * K;
  for (int i = threadIdx.x; i < ng * words; i += blockDim.x) bits[i] = 0;
  if (stage_rows)
    for (int i = threadIdx.x; i < nslots; i += blockDim.x) rows_smem[i] = idx[t0 * K + i];
  const int32_t* rows = stage_rows ? rows_smem : idx + t0 * K;
  for (int c = threadIdx.x; c < ng; c += blockDim.x) {
    const int32_t cb = counts[(int64_t)c * gridDim.x + blockIdx.x];
    base_tok[c] = offs[c] + cb;
    base_row[c] = seg_start ? seg_start[c] + cb : 0;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < nslots; i += blockDim.x) {
    const int tl = i / K, k = i % K;
    const int32_t* row = rows + tl * K;
    if (valid_slot(row, k, ng)) atomicOr(&bits[row[k] * words + (tl >> 5)], 1u << (tl & 31));
  }
  __syncthreads();
  for (int c = threadIdx.x; c < ng; c += blockDim.x) {
    int32_t run = 0;
    for (int w = 0; w < words; ++w) {
      pre[c * words + w] = run;
      run += __popc(bits[c * words + w]);
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < nslots; i += blockDim.x) {
    const int tl = i / K, k = i % K;
    const int64_t t = t0 + tl;
    const int32_t* row = rows + tl * K;
    if (!valid_slot(row, k, ng)) {
      if (pair_row) pair_row[t * K + k] = -1;
      continue;
    }
    const int c = row[k];
    const int w = tl >> 5;
    const int rank = pre[c * words + w] + __popc(bits[c * words + w] & ((1u << (tl & 31)) - 1u));
    tokens[base_tok[c] + rank] = (int32_t)t;
    if (row_token) row_token[base_row[c] + rank] = (int32_t)t;
    if (pair_row) pair_row[t * K + k] = base_row[c] + rank;
  }
}

// Drops a 128-byte line from L2 without writing it back (its contents become undefined).
__device__ __forceinline__ void discard_l2_line(const void* p) {
  asm volatile("discard.global.L2 [%0], 128;" ::"l"(p) : "memory");
}

// out[t, :] = sum over t's valid slots k (in slot order) of rows[pair_row[t*K + k], :], fp32
// accumulation, bf16 result: the deterministic reduction of the per-pair contributions.  One
// warp per token; each lane issues the (up to 8) row loads of a slot chunk before summing them.
// With discard set (rows whose length is a multiple of 128 bytes), the lines a warp has read are
// dropped from L2 afterwards: each belongs to one (token, group) pair and is read only here.
__global__ void pair_sum_kernel(const uint4* __restrict__ rows, const int32_t* __restrict__ pair_row,
                                int64_t M, int K, int64_t row_vecs, uint4* __restrict__ out, int discard) {
  constexpr int kChunk = 8;
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < M; t += warps) {
    const int32_t* pr = pair_row + t * K;
    for (int64_t v = lane; v < row_vecs; v += 32) {
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      for (int k0 = 0; k0 < K; k0 += kChunk) {
        uint4 q[kChunk];
#pragma unroll
        for (int j = 0; j < kChunk; ++j) {
          const int32_t r = (k0 + j < K) ? pr[k0 + j] : -1;
          q[j] = r >= 0 ? rows[(int64_t)r * row_vecs + v] : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int j = 0; j < kChunk; ++j) {
          const uint32_t w[4] = {q[j].x, q[j].y, q[j].z, q[j].w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            acc[2 * i] += bf16_lo(w[i]);
            acc[2 * i + 1] += bf16_hi(w[i]);
          }
        }
      }
      out[t * row_vecs + v] = make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                                         pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
      if (discard) {
        // The 8 lanes of each 128-byte line read it in this iteration (row_vecs is a multiple of
        // 8); the lanes still in the loop are the first min(32, row_vecs - (v - lane)).
        const int64_t left = row_vecs - (v - lane);
        __syncwarp(left >= 32 ? 0xffffffffu : ((1u << left) - 1u));
        if ((v & 7) == 0)
          for (int k = 0; k < K; ++k) {
            const int32_t r = pr[k];
            if (r >= 0) discard_l2_line(rows + (int64_t)r * row_vecs + v);
          }
      }
    }
  }
}

// Wsub[c*P + i, :] = w_gate[sub[c*spg + i], :] for i < spg, zero rows for spg <= i < P (zero rows
// add |SiLU(0)| = 0 to the energy).  Row ids outside group c are treated as zero rows.
__global__ void select_gather_kernel(const uint4* __restrict__ w, const int32_t* __restrict__ sub,
                                     int ng, int G, int spg, int P, int64_t row_vecs,
                                     uint4* __restrict__ dst) {
  const int lane = threadIdx.x & 31;
  const int64_t rows = (int64_t)ng * P;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps) {
    const int c = (int)(r / P), i = (int)(r % P);
    int src = -1;
    if (i < spg) {
      src = sub[(int64_t)c * spg + i];
      if (src < c * G || src >= (c + 1) * G) src = -1;
    }
    uint4* d = dst + r * row_vecs;
    if (src < 0) {
      for (int64_t v = lane; v < row_vecs; v += 32) d[v] = make_uint4(0u, 0u, 0u, 0u);
    } else {
      const uint4* s = w + (int64_t)src * row_vecs;
      for (int64_t v = lane; v < row_vecs; v += 32) d[v] = s[v];
    }
  }
}

// One warp per token: the bias (if any) added to the group scores and written back, then K rounds
// of a warp-wide argmax over them (larger score first, lower group index among equal scores), then
// the chosen groups written in ascending order.
template <int VPL>
__global__ void topk_kernel(float* __restrict__ E, const float* __restrict__ bias, int64_t M,
                            int ng, int K, int32_t* __restrict__ idx) {
  const int lane = threadIdx.x & 31;
  const int64_t m = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (m >= M) return;  // uniform per warp
  float* row = E + m * ng;
  float v[VPL];
#pragma unroll
  for (int j = 0; j < VPL; ++j) {
    const int c = lane + 32 * j;
    v[j] = c < ng ? row[c] : -INFINITY;
    if (bias && c < ng) {
      v[j] += bias[c];
      row[c] = v[j];
    }
  }
  uint64_t taken = 0;
  int chosen = 0;
  for (int r = 0; r < K; ++r) {
    float bv = -INFINITY;
    int bc = INT32_MAX;
#pragma unroll
    for (int j = 0; j < VPL; ++j) {
      const int c = lane + 32 * j;
      if (c < ng && !((taken >> j) & 1ull) && (v[j] > bv || (v[j] == bv && c < bc))) {
        bv = v[j];
        bc = c;
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
      const int oc = __shfl_xor_sync(0xffffffffu, bc, off);
      if (ov > bv || (ov == bv && oc < bc)) {
        bv = ov;
        bc = oc;
      }
    }
    if (bc >= ng) break;  // nothing left that compares (only NaN scores remain)
    if ((bc & 31) == lane) taken |= 1ull << (bc >> 5);
    ++chosen;
  }
  int base = 0;
#pragma unroll
  for (int j = 0; j < VPL; ++j) {
    const bool bit = (taken >> j) & 1ull;
    const unsigned mask = __ballot_sync(0xffffffffu, bit);
    if (bit) idx[m * K + base + __popc(mask & ((1u << lane) - 1u))] = lane + 32 * j;
    base += __popc(mask);
  }
  for (int p = chosen + lane; p < K; p += 32) idx[m * K + p] = -1;
}

// ------------------------------------------------------------------ host helpers

inline int grid_for(int64_t work, int per_block) {
  return (int)std::max<int64_t>(1, std::min<int64_t>((work + per_block - 1) / per_block, 148 * 16));
}

swf_status launched() { return cudaGetLastError() == cudaSuccess ? SWF_OK : SWF_ERR_LAUNCH; }

swf_status run_buckets(const int32_t* idx, const SparseDims& s, int32_t* counts, int32_t* offs,
                       int32_t* tokens, int32_t* seg_start, int32_t* seg_rows,
                       int32_t* tile_group, int32_t* row_token, int32_t* pair_row, cudaStream_t st) {
  {
    ProfScope prof(SWF_K_BUCKETS, st);
    bucket_count_kernel<<<s.nblk, 256, s.ng * sizeof(int32_t), st>>>(idx, s.M, s.K, s.ng, s.tok_blk, counts,
                                                                    row_token, s.rmax);
    if (launched() != SWF_OK) return SWF_ERR_LAUNCH;
  }
  const size_t scan_smem = (2 * (size_t)s.ng + 1) * sizeof(int32_t);
  if (scan_smem > 48 * 1024 &&
      cudaFuncSetAttribute(bucket_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)scan_smem) != cudaSuccess)
    return SWF_ERR_LAUNCH;
  {
    ProfScope prof(SWF_K_BUCKETS, st);
    bucket_scan_kernel<<<1, 1024, scan_smem, st>>>(counts, s.nblk, s.ng, offs, seg_start, seg_rows,
                                                   tile_group, s.mblk);
    if (launched() != SWF_OK) return SWF_ERR_LAUNCH;
  }
  const size_t rows_bytes = (size_t)4 * s.tok_blk * s.K;
  const int stage_rows = rows_bytes <= (size_t)kBucketRowsSmemBytes ? 1 : 0;
  const size_t place_smem = (size_t)8 * s.ng * s.words + (size_t)8 * s.ng + (stage_rows ? rows_bytes : 0);
  if (cudaFuncSetAttribute(bucket_place_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)place_smem) != cudaSuccess)
    return SWF_ERR_LAUNCH;
  ProfScope prof(SWF_K_BUCKETS, st);
  bucket_place_kernel<<<s.nblk, 256, place_smem, st>>>(idx, s.M, s.K, s.ng, s.words, counts, offs,
                                                       tokens, seg_start, row_token, pair_row, stage_rows);
  return launched();
}

// The per-token sums.  Each per-pair row is read once, so when rows are whole 128-byte lines the
// lines are dropped from L2 after they are read instead of being written back to DRAM.
swf_status run_pair_sum(const void* rows, const int32_t* pair_row, const SparseDims& s, void* out,
                        cudaStream_t st) {
  ProfScope prof(SWF_K_PAIR_SUM, st);
  // a line may be dropped only when no other row shares it
  const int discard = ((s.d * 2) % 128 == 0 && (reinterpret_cast<uintptr_t>(rows) & 127) == 0) ? 1 : 0;
  pair_sum_kernel<<<grid_for(s.M, 8), 256, 0, st>>>(static_cast<const uint4*>(rows), pair_row, s.M, s.K,
                                                   s.d / 8, static_cast<uint4*>(out), discard);
  return launched();
}

// The gathered operand of a sparse GEMM: padded row r is row row_token[r] of src [tokens, d].
void set_gather(TcGemmArgs& a, const int32_t* row_token, const void* src, int64_t d) {
  a.gather_token = row_token;
  a.gather_src = src;
  a.gather_ld = d;
  a.gather_cols = (int)d;
}

template <int VPL>
swf_status launch_topk(float* E, const float* bias, int64_t M, int ng, int K, int32_t* idx,
                       cudaStream_t st) {
  ProfScope prof(SWF_K_SELECT_TOPK, st);
  topk_kernel<VPL><<<(unsigned)((M + 7) / 8), 256, 0, st>>>(E, bias, M, ng, K, idx);
  return launched();
}

constexpr int kMaxSelectGroups = 2048;

}  // namespace

// ------------------------------------------------------------------ sizes and plans

size_t select_workspace_bytes(int64_t M, int64_t d, int64_t f, int32_t G, int32_t K) {
  (void)K;
  const int ng = (int)(f / G);
  size_t bytes = 0;
  // worst case: subsample given (P = G) and energies not supplied by the caller
  sel_ws(nullptr, M, d, ng, G, true, true, &bytes);
  return bytes;
}

size_t sparse_fwd_workspace_bytes(int64_t M, int64_t d, int64_t f, int32_t G, int32_t K) {
  size_t bytes = 0;
  fwd_ws(nullptr, dims_of(M, d, f, G, K), &bytes);
  return bytes;
}

size_t sparse_bwd_workspace_bytes(int64_t M, int64_t d, int64_t f, int32_t G, int32_t K) {
  size_t bytes = 0;
  bwd_ws(nullptr, dims_of(M, d, f, G, K), &bytes);
  return bytes;
}

size_t buckets_workspace_bytes(int64_t M, int32_t K, int32_t ng) {
  const SparseDims s = dims_of(M, 16, (int64_t)ng * 16, 16, K);
  return round_up((size_t)s.nblk * s.ng * sizeof(int32_t), 256);
}

size_t sparse_saved_bytes(int64_t M, int64_t d, int64_t f, int32_t G, int32_t K) {
  size_t bytes = 0;
  saved_view(nullptr, dims_of(M, d, f, G, K), &bytes);
  return bytes;
}

void sparse_plan(int op, int64_t M, int64_t d, int64_t f, int32_t G, int32_t K, int32_t spg,
                 swf_plan_info* p) {
  const SparseDims s = dims_of(M, d, f, G, K);
  p->deterministic = 1;
  p->saved_bytes = (op == SWF_OP_SPARSE_FWD || op == SWF_OP_SPARSE_BWD) ? sparse_saved_bytes(M, d, f, G, K) : 0;
  const int P = spg > 0 ? pow2_at_least(spg) : G;
  switch (op) {
    case SWF_OP_SELECT:
      p->num_kernels = spg > 0 ? 3 : 2;
      p->flops = 2 * M * d * (int64_t)s.ng * (spg > 0 ? spg : G);
      p->gemm_tiles = (int64_t)cdiv(M, 128) * cdiv((int64_t)s.ng * P, 256);
      break;
    case SWF_OP_SPARSE_FWD:
      p->num_kernels = 6;  // bucketing (count with the row -> token fill, scan, place), gate|up, down, pair sum
      p->flops = 6 * M * d * (int64_t)K * G;
      p->gemm_tiles = (int64_t)s.mblk * (1 + cdiv(d, 256));
      p->tile_n = 2 * G;
      break;
    case SWF_OP_SPARSE_BWD:
      p->num_kernels = 5;  // dgate, dW_down, dW_gate|dW_up, dx, pair sum
      p->flops = 12 * M * d * (int64_t)K * G;
      p->gemm_tiles = (int64_t)s.mblk * (1 + cdiv(d, 256)) + (int64_t)s.ng * (cdiv(d, 256) + cdiv(d, 128));
      break;
    case SWF_OP_BUCKETS:
      p->num_kernels = 3;
      p->flops = 0;
      p->gemm_tiles = 0;
      break;
    default:
      break;
  }
}

}  // namespace swf

using namespace swf;

// ------------------------------------------------------------------ subsample (host)

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
      std::swap(perm[i], perm[j]);
    }
    std::sort(perm.begin(), perm.begin() + spg);
    for (int32_t i = 0; i < spg; ++i) out[c * spg + i] = (int32_t)(c * G + perm[i]);
  }
  return SWF_OK;
}

// ------------------------------------------------------------------ selection

extern "C" swf_status grouped_topk_select(const void* x, const void* w_gate,
                                          const int32_t* subsample_idx, int32_t spg,
                                          const float* bias, int32_t G, int32_t K,
                                          int32_t* group_idx, float* energies, void* workspace,
                                          size_t ws_bytes, int64_t M, int64_t d, int64_t f,
                                          swf_dtype dt, void* stream) {
  if (!x || !w_gate || !group_idx) return SWF_ERR_INVALID_ARG;
  swf_status s = check_sparse_shape(M, d, f, G, K, dt);
  if (s != SWF_OK) return s;
  const int ng = (int)(f / G);
  if (ng > kMaxSelectGroups) return SWF_ERR_UNSUPPORTED;
  if (subsample_idx && (spg < 1 || spg > G)) return SWF_ERR_UNSUPPORTED;
  for (const void* p : {x, w_gate, (const void*)group_idx})
    if (!aligned16(p)) return SWF_ERR_ALIGNMENT;
  if ((energies && !aligned16(energies)) || (subsample_idx && !aligned16(subsample_idx)) ||
      (bias && !aligned16(bias)) || (workspace && !aligned16(workspace)))
    return SWF_ERR_ALIGNMENT;
  const int P = subsample_idx ? pow2_at_least(spg) : G;
  size_t need = 0;
  SelWs w = sel_ws(workspace, M, d, ng, P, subsample_idx != nullptr, energies == nullptr, &need);
  if (need > 0 && (!workspace || ws_bytes < need)) return SWF_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float* E = energies ? energies : w.energies;

  const void* wrows = w_gate;
  if (subsample_idx) {
    ProfScope prof(SWF_K_SELECT_GATHER, st);
    select_gather_kernel<<<grid_for((int64_t)ng * P, 8), 256, 0, st>>>(
        static_cast<const uint4*>(w_gate), subsample_idx, ng, G, spg, P, d / 8,
        reinterpret_cast<uint4*>(w.wsub));
    if (launched() != SWF_OK) return SWF_ERR_LAUNCH;
    wrows = w.wsub;
  }
  // scoring GEMM: E[m, c] = sum over the group's P columns of |SiLU(x . w_row)|, then + bias[c]
  // in the top-k step
  CUtensorMap tx, tw;
  const int64_t ncols = (int64_t)ng * P;
  if (!encode_tmap_bf16(&tx, x, d, M, d, 64, 128) || !encode_tmap_bf16(&tw, wrows, d, ncols, d, 64, 256))
    return SWF_ERR_LAUNCH;
  TcGemmArgs a = base_args(M, ncols, 256, d);
  a.out0 = E;
  a.ld_out = ng;
  a.energy_p = P;
  a.n_groups = ng;
  a.bias = bias;
  if (ng <= kTopKMaxGroups) {
    // one CTA scores all groups of its 128 tokens (energies held in shared memory), then each
    // epilogue thread selects its token's groups
    a.raster = 1;
    a.unit = a.num_n_blk;
    a.sel_idx = group_idx;
    a.sel_k = K;
    a.out0 = energies;  // [M][ng] with the bias, only if asked for
    a.ld_grp = 1;
    return launch_tc<256, false, false, false, kEpiEnergyTopK>(SWF_K_SELECT_SCORE, tx, tw, tw, a, st);
  }
  s = launch_tc<256, false, false, false, kEpiEnergy>(SWF_K_SELECT_SCORE, tx, tw, tw, a, st);
  if (s != SWF_OK) return s;
  if (ng <= 32) return launch_topk<1>(E, bias, M, ng, K, group_idx, st);
  if (ng <= 64) return launch_topk<2>(E, bias, M, ng, K, group_idx, st);
  if (ng <= 128) return launch_topk<4>(E, bias, M, ng, K, group_idx, st);
  if (ng <= 256) return launch_topk<8>(E, bias, M, ng, K, group_idx, st);
  if (ng <= 512) return launch_topk<16>(E, bias, M, ng, K, group_idx, st);
  if (ng <= 1024) return launch_topk<32>(E, bias, M, ng, K, group_idx, st);
  return launch_topk<64>(E, bias, M, ng, K, group_idx, st);
}

// ------------------------------------------------------------------ group_idx validation

// Count of invalid group_idx slots found by the last validation on this device.
static __device__ unsigned long long g_swf_bad_slots;

namespace swf {
namespace {

// One warp per row: a slot is invalid if its group is out of [0, ng) or repeats an earlier
// slot of the same row (exactly the slots the bucketing drops).  Adds the count of invalid
// slots to *bad.
__global__ void validate_idx_kernel(const int32_t* __restrict__ idx, int64_t M, int K, int ng,
                                    unsigned long long* __restrict__ bad) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  unsigned long long n = 0;
  for (int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < M; t += warps) {
    const int32_t* row = idx + t * K;
    for (int k = lane; k < K; k += 32) n += valid_slot(row, k, ng) ? 0ull : 1ull;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) n += __shfl_xor_sync(0xffffffffu, n, off);
  if (lane == 0 && n) atomicAdd(bad, n);
}

std::mutex g_debug_mu;
int g_debug = -1;  // -1: not yet read from the environment

bool debug_on() {
  std::lock_guard<std::mutex> lock(g_debug_mu);
  if (g_debug < 0) {
    const char* e = std::getenv("SWF_DEBUG");
    g_debug = (e && *e && std::strcmp(e, "0") != 0) ? 1 : 0;
  }
  return g_debug == 1;
}

std::mutex g_validate_mu;
unsigned long long* g_bad_ptr[64] = {};

// Runs the validation of group_idx on `st` and waits for it.  SWF_ERR_INVALID_ARG if any slot
// is invalid (its count in *bad_out when given).
swf_status validate_idx(const int32_t* idx, int64_t M, int32_t K, int32_t ng, int64_t* bad_out,
                        cudaStream_t st) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return SWF_ERR_LAUNCH;
  std::lock_guard<std::mutex> lock(g_validate_mu);
  if (!g_bad_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_swf_bad_slots) != cudaSuccess || !p) return SWF_ERR_LAUNCH;
    g_bad_ptr[dev] = static_cast<unsigned long long*>(p);
  }
  unsigned long long* bad = g_bad_ptr[dev];
  if (cudaMemsetAsync(bad, 0, sizeof(*bad), st) != cudaSuccess) return SWF_ERR_LAUNCH;
  {
    ProfScope prof(SWF_K_ELEMENTWISE, st);
    validate_idx_kernel<<<grid_for(M, 8), 256, 0, st>>>(idx, M, K, ng, bad);
    if (launched() != SWF_OK) return SWF_ERR_LAUNCH;
  }
  unsigned long long host = 0;
  if (cudaMemcpyAsync(&host, bad, sizeof(host), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return SWF_ERR_LAUNCH;
  if (bad_out) *bad_out = (int64_t)host;
  return host ? SWF_ERR_INVALID_ARG : SWF_OK;
}

// In debug mode: the validation, before an entry point that reads group_idx launches anything.
swf_status debug_check_idx(const int32_t* idx, int64_t M, int32_t K, int32_t ng, cudaStream_t st) {
  return debug_on() ? validate_idx(idx, M, K, ng, nullptr, st) : SWF_OK;
}

}  // namespace
}  // namespace swf

extern "C" swf_status swf_set_debug(int32_t enable) {
  if (enable != 0 && enable != 1) return SWF_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(swf::g_debug_mu);
  swf::g_debug = enable;
  return SWF_OK;
}

extern "C" int32_t swf_get_debug(void) { return swf::debug_on() ? 1 : 0; }

extern "C" swf_status swf_validate_group_idx(const int32_t* group_idx, int64_t M,
                                             int32_t num_active_groups, int32_t num_groups,
                                             int64_t* bad_slots, void* stream) {
  if (!group_idx || M <= 0 || num_active_groups <= 0 || num_groups <= 0) return SWF_ERR_INVALID_ARG;
  if (!aligned16(group_idx)) return SWF_ERR_ALIGNMENT;
  if (M * (int64_t)num_active_groups >= (int64_t(1) << 31)) return SWF_ERR_UNSUPPORTED;
  return validate_idx(group_idx, M, num_active_groups, num_groups, bad_slots,
                      static_cast<cudaStream_t>(stream));
}

// ------------------------------------------------------------------ bucketing

extern "C" swf_status swf_group_buckets(const int32_t* group_idx, int64_t M, int32_t K, int32_t ng,
                                        int32_t* offsets, int32_t* tokens, void* workspace,
                                        size_t ws_bytes, void* stream) {
  if (!group_idx || !offsets || !tokens || !workspace) return SWF_ERR_INVALID_ARG;
  swf_status s = swf_supported(SWF_OP_BUCKETS, M, 0, 0, ng, K, 0, SWF_BF16);
  if (s != SWF_OK) return s;
  if (ng > 12288) return SWF_ERR_UNSUPPORTED;
  if (!aligned16(workspace)) return SWF_ERR_ALIGNMENT;
  if (ws_bytes < buckets_workspace_bytes(M, K, ng)) return SWF_ERR_WORKSPACE;
  if ((s = debug_check_idx(group_idx, M, K, ng, static_cast<cudaStream_t>(stream))) != SWF_OK) return s;
  const SparseDims d = dims_of(M, 16, (int64_t)ng * 16, 16, K);
  return run_buckets(group_idx, d, static_cast<int32_t*>(workspace), offsets, tokens, nullptr,
                     nullptr, nullptr, nullptr, nullptr, static_cast<cudaStream_t>(stream));
}

// ------------------------------------------------------------------ load balancing

namespace swf {
namespace {

// One block: integer counts of the valid slots per group (shared atomics; integers, so the
// result does not depend on their order), then freq[c] = count[c] / M.
__global__ void group_frequency_kernel(const int32_t* __restrict__ idx, int64_t M, int K, int ng,
                                       float* __restrict__ freq) {
  extern __shared__ int32_t cnt[];
  for (int c = threadIdx.x; c < ng; c += blockDim.x) cnt[c] = 0;
  __syncthreads();
  for (int64_t i = threadIdx.x; i < M * K; i += blockDim.x) {
    const int32_t* row = idx + (i / K) * K;
    const int k = (int)(i % K);
    if (valid_slot(row, k, ng)) atomicAdd(&cnt[row[k]], 1);
  }
  __syncthreads();
  for (int c = threadIdx.x; c < ng; c += blockDim.x) freq[c] = (float)cnt[c] / (float)M;
}

__global__ void balance_update_kernel(float* __restrict__ bias, float* __restrict__ ema,
                                      const float* __restrict__ cur, float target, float gamma,
                                      float bias_max, float momentum, int ng) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= ng) return;
  const float e = momentum * ema[c] + (1.0f - momentum) * cur[c];
  ema[c] = e;
  const float sgn = (target > e) ? 1.0f : ((target < e) ? -1.0f : 0.0f);
  bias[c] = fminf(fmaxf(bias[c] + gamma * sgn, -bias_max), bias_max);
}

}  // namespace
}  // namespace swf

extern "C" swf_status swf_group_frequency(const int32_t* group_idx, int64_t M, int32_t K,
                                          int32_t ng, float* freq, void* stream) {
  if (!group_idx || !freq) return SWF_ERR_INVALID_ARG;
  swf_status s = swf_supported(SWF_OP_BUCKETS, M, 0, 0, ng, K, 0, SWF_BF16);
  if (s != SWF_OK) return s;
  if (ng > 12288) return SWF_ERR_UNSUPPORTED;
  if (!aligned16(group_idx) || !aligned16(freq)) return SWF_ERR_ALIGNMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((s = debug_check_idx(group_idx, M, K, ng, st)) != SWF_OK) return s;
  ProfScope prof(SWF_K_BALANCE, st);
  group_frequency_kernel<<<1, 1024, ng * sizeof(int32_t), st>>>(group_idx, M, K, ng, freq);
  return launched();
}

extern "C" swf_status update_load_balance_bias(float* bias, float* freq_ema, const float* cur,
                                               float target, float gamma, float bias_max,
                                               float momentum, int32_t ng, void* stream) {
  if (!bias || !freq_ema || !cur) return SWF_ERR_INVALID_ARG;
  if (ng <= 0 || !(bias_max >= 0.f) || !(momentum >= 0.f && momentum <= 1.f)) return SWF_ERR_INVALID_ARG;
  if (!aligned16(bias) || !aligned16(freq_ema) || !aligned16(cur)) return SWF_ERR_ALIGNMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  ProfScope prof(SWF_K_BALANCE, st);
  balance_update_kernel<<<(ng + 255) / 256, 256, 0, st>>>(bias, freq_ema, cur, target, gamma,
                                                          bias_max, momentum, ng);
  return launched();
}

// ------------------------------------------------------------------ sparse forward

namespace {
swf_status check_sparse_ptrs(std::initializer_list<const void*> ps) {
  for (const void* p : ps)
    if (!p) return SWF_ERR_INVALID_ARG;
  for (const void* p : ps)
    if (!aligned16(p)) return SWF_ERR_ALIGNMENT;
  return SWF_OK;
}
}  // namespace

extern "C" swf_status sparse_swiglu_ffn_fwd(const void* x, const void* w_gate, const void* w_up,
                                            const void* w_down, const int32_t* group_idx,
                                            int32_t G, int32_t K, void* y, void* saved,
                                            size_t saved_bytes, void* workspace, size_t ws_bytes,
                                            int64_t M, int64_t d, int64_t f, swf_dtype dt,
                                            void* stream) {
  swf_status s = check_sparse_ptrs({x, w_gate, w_up, w_down, group_idx, y, saved, workspace});
  if (s != SWF_OK) return s;
  if ((s = check_sparse_shape(M, d, f, G, K, dt)) != SWF_OK) return s;
  if ((int64_t)(f / G) > 12288) return SWF_ERR_UNSUPPORTED;
  const SparseDims sd = dims_of(M, d, f, G, K);
  size_t need_saved = 0, need_ws = 0;
  const SavedView v = saved_view(saved, sd, &need_saved);
  const FwdWs w = fwd_ws(workspace, sd, &need_ws);
  if (saved_bytes < need_saved || ws_bytes < need_ws) return SWF_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((s = debug_check_idx(group_idx, M, K, sd.ng, st)) != SWF_OK) return s;

  if ((s = run_buckets(group_idx, sd, w.counts, v.offs, v.tokens, v.seg_start, v.seg_rows,
                       v.tile_group, v.row_token, v.pair_row, st)) != SWF_OK)
    return s;
  {  // gate|up per group: [h|a|b] rows = SiLU/gating of X rows [W_g[g] | W_u[g]]^T, the X rows
     // of each tile gathered from x by the kernel (from L2)
    CUtensorMap twg, twu;
    if (!encode_tmap_bf16(&twg, w_gate, d, f, d, 64, G) || !encode_tmap_bf16(&twu, w_up, d, f, d, 64, G))
      return SWF_ERR_LAUNCH;
    TcGemmArgs a = base_args(sd.rmax, G, 2 * G, d);
    a.num_n_blk = 1;
    a.tile_group = v.tile_group;
    a.grp_b_n = G;
    a.out0 = v.h;
    a.ld_out = G;
    a.aux0 = v.a;
    a.aux1 = v.b;
    a.ld_aux = G;
    set_gather(a, v.row_token, x, d);
    // G >= 32: h, a, b leave through 32-row x 32-column staging boxes and TMA stores (whole
    // 64-byte row pieces) instead of each thread's 16-byte stores into 32 different rows
    EpiMaps em{};
    if (G >= 32 && (!encode_tmap_bf16(&em.o[0], v.h, G, sd.rmax, G, 32, 32, 64) ||
                    !encode_tmap_bf16(&em.o[1], v.a, G, sd.rmax, G, 32, 32, 64) ||
                    !encode_tmap_bf16(&em.o[2], v.b, G, sd.rmax, G, 32, 32, 64)))
      return SWF_ERR_LAUNCH;
    if (G == 16)
      s = launch_tc<32, false, false, true, kEpiSwiGLU, kModeRowGrouped, false, kGatherA>(SWF_K_SPARSE_UP, twg, twg, twu, a, st);
    else if (G == 32)
      s = launch_tc<64, false, false, true, kEpiSwiGLU, kModeRowGrouped, true, kGatherA>(SWF_K_SPARSE_UP, twg, twg, twu, a, st, em);
    else
      s = launch_tc<128, false, false, true, kEpiSwiGLU, kModeRowGrouped, true, kGatherA>(SWF_K_SPARSE_UP, twg, twg, twu, a, st, em);
    if (s != SWF_OK) return s;
  }
  {  // down per group: yc[r] = h_row W_d[:, g*G .. g*G+G]^T
    CUtensorMap th, twd;
    if (!encode_tmap_bf16(&th, v.h, G, sd.rmax, G, 64, 128) || !encode_tmap_bf16(&twd, w_down, f, d, f, 64, 256))
      return SWF_ERR_LAUNCH;
    EpiMaps em{};
    if (!encode_tmap_bf16(&em.o[0], w.yc, d, sd.rmax, d, kStoreBoxCols, 32, kStoreBoxSwizzle)) return SWF_ERR_LAUNCH;
    TcGemmArgs a = base_args(sd.rmax, d, 256, G);
    a.tile_group = v.tile_group;
    a.grp_b_k = G;
    s = launch_tc<256, false, false, false, kEpiStore, kModeRowGrouped, true>(SWF_K_SPARSE_DOWN, th, twd, twd, a, st, em);
    if (s != SWF_OK) return s;
  }
  return run_pair_sum(w.yc, v.pair_row, sd, y, st);
}

// ------------------------------------------------------------------ sparse backward

extern "C" swf_status sparse_swiglu_ffn_bwd(const void* dy, const void* x, const void* w_gate,
                                            const void* w_up, const void* w_down,
                                            const int32_t* group_idx, const void* saved,
                                            size_t saved_bytes, void* dx, void* dw_gate,
                                            void* dw_up, void* dw_down, void* workspace,
                                            size_t ws_bytes, int64_t M, int64_t d, int64_t f,
                                            int32_t G, int32_t K, swf_dtype dt, void* stream) {
  swf_status s = check_sparse_ptrs({dy, x, w_gate, w_up, w_down, group_idx, saved, dx, dw_gate,
                                    dw_up, dw_down, workspace});
  if (s != SWF_OK) return s;
  if ((s = check_sparse_shape(M, d, f, G, K, dt)) != SWF_OK) return s;
  if ((int64_t)(f / G) > 12288) return SWF_ERR_UNSUPPORTED;
  const SparseDims sd = dims_of(M, d, f, G, K);
  size_t need_saved = 0, need_ws = 0;
  const SavedView v = saved_view(const_cast<void*>(saved), sd, &need_saved);
  const BwdWs w = bwd_ws(workspace, sd, &need_ws);
  if (saved_bytes < need_saved || ws_bytes < need_ws) return SWF_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((s = debug_check_idx(group_idx, M, K, sd.ng, st)) != SWF_OK) return s;

  // the token rows of x and dY are gathered by the GEMMs that read them (from L2)
  {  // dH = dY rows W_d[:, g]; dG = dH * a, dU = dH * b -> dgu [R, 128] (halves padded to 64)
    CUtensorMap twd;
    if (!encode_tmap_bf16(&twd, w_down, f, d, f, 64, 64)) return SWF_ERR_LAUNCH;
    TcGemmArgs a = base_args(sd.rmax, G, 64, d);
    a.num_n_blk = 1;
    a.tile_group = v.tile_group;
    a.grp_b_n = G;
    a.out0 = w.dgu;
    a.ld_out = 128;
    a.d_ff = 64;
    a.pad_cols = 64;
    a.aux0 = v.a;
    a.aux1 = v.b;
    a.ld_aux = G;
    set_gather(a, v.row_token, dy, d);
    // the factors a, b come in and dG, dU leave as 32-row x 64-column boxes by TMA, dG and dU
    // computed in place in the factor boxes (columns G .. 64 read as zero and are stored as zero)
    EpiMaps em{};
    if (!encode_tmap_bf16(&em.o[0], w.dgu, 64, sd.rmax, 128, 64, 32, 128) ||
        !encode_tmap_bf16(&em.o[1], w.dgu + 64, 64, sd.rmax, 128, 64, 32, 128) ||
        !encode_tmap_bf16(&em.o[2], v.a, G, sd.rmax, G, 64, 32, 128) ||
        !encode_tmap_bf16(&em.o[3], v.b, G, sd.rmax, G, 64, 32, 128))
      return SWF_ERR_LAUNCH;
    s = launch_tc<64, false, true, false, kEpiDGate, kModeRowGrouped, true, kGatherA>(SWF_K_SPARSE_DGATE, twd, twd, twd, a,
                                                                                        st, em);
    if (s != SWF_OK) return s;
  }
  // dW_down right after dgate: both gather the same dY rows, which are then still in L2
  {  // per group: dW_d[:, g] = (dY rows of the segment)ᵀ h_seg, the dY rows gathered from dy
    CUtensorMap th;
    if (!encode_tmap_bf16(&th, v.h, G, sd.rmax, G, 64, 64)) return SWF_ERR_LAUNCH;
    TcGemmArgs a = base_args(d, G, 64, 0);
    a.n_groups = sd.ng;
    a.seg_start = v.seg_start;
    a.seg_rows = v.seg_rows;
    a.kb_seg0 = 1 << 30;
    a.group_size = G;
    a.out0 = dw_down;
    a.ld_out = f;
    set_gather(a, v.row_token, dy, d);
    s = launch_tc<64, true, true, false, kEpiGroupDWd, kModeKGrouped, false, kGatherA>(SWF_K_SPARSE_DW, th, th, th, a, st);
  }
  if (s != SWF_OK) return s;
  {  // per group: [dW_g[g] ; dW_u[g]] = dgu_segᵀ X rows of the segment (gathered from x)
    CUtensorMap tdgu;
    if (!encode_tmap_bf16(&tdgu, w.dgu, 128, sd.rmax, 128, 64, 64)) return SWF_ERR_LAUNCH;
    TcGemmArgs a = base_args(128, d, 256, 0);
    a.n_groups = sd.ng;
    a.seg_start = v.seg_start;
    a.seg_rows = v.seg_rows;
    a.kb_seg0 = 1 << 30;
    a.group_size = G;
    a.out0 = dw_gate;
    a.out1 = dw_up;
    a.ld_out = d;
    set_gather(a, v.row_token, x, d);
    s = launch_tc<256, true, true, false, kEpiGroupDWgu, kModeKGrouped, false, kGatherB>(SWF_K_SPARSE_DW, tdgu, tdgu, tdgu, a, st);
    if (s != SWF_OK) return s;
  }
  {  // dxc[r] = dG_row W_g[g] + dU_row W_u[g]
    CUtensorMap tdgu, twg, twu;
    if (!encode_tmap_bf16(&tdgu, w.dgu, 128, sd.rmax, 128, 64, 128) ||
        !encode_tmap_bf16(&twg, w_gate, d, f, d, 64, 64) || !encode_tmap_bf16(&twu, w_up, d, f, d, 64, 64))
      return SWF_ERR_LAUNCH;
    TcGemmArgs a = base_args(sd.rmax, d, 256, 128);
    a.kb_seg0 = 1;
    a.kb_total = 2;
    a.a_koff1 = 64;
    a.tile_group = v.tile_group;
    a.grp_b_k = G;
    EpiMaps em{};
    if (!encode_tmap_bf16(&em.o[0], w.dxc, d, sd.rmax, d, kStoreBoxCols, 32, kStoreBoxSwizzle)) return SWF_ERR_LAUNCH;
    s = launch_tc<256, false, true, false, kEpiStore, kModeRowGrouped, true>(SWF_K_SPARSE_DX, tdgu, twg, twu, a, st, em);
    if (s != SWF_OK) return s;
  }
  if ((s = run_pair_sum(w.dxc, v.pair_row, sd, dx, st)) != SWF_OK) return s;
  return s;
}
