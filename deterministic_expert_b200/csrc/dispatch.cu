// Dispatch: expert offsets and a counting-sort permute that is stable by token
// index (the dispatch step of DeepSeek V4 infra notes §6.1, dispatch ->
// compute -> combine).  Dropless: no capacity, so no token's routing or rows
// depend on the rest of the batch (the linux.do post on MoE variants,
// "MoE是如何影响输出确定性的", names token dropping as a source of batch
// dependence).  Integer-only; the result is unique.
//
//   dispatch  block b (128 tokens) reads the per-block expert counts the router
//             wrote, forms the exclusive prefix over experts (offsets) and over
//             the blocks before it, then ranks each of its (token, slot) pairs
//             among the block's earlier tokens that chose the same expert (a
//             token bitmask per expert + popcount): grouped row
//             p = offsets[e] + (pairs of e in earlier tokens).  Block 0 also
//             writes the counts, the offsets and the two expert-GEMM tile lists.
//   gather    xp[p] = xn[src_token[p]]  (the routed GEMM's A operand)
#include "common.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

__global__ void __launch_bounds__(kDispatchRows) k_dispatch(const DispatchArgs a) {
  constexpr int kWords = kDispatchRows / 32;
  __shared__ int base[256];    // offsets[e] + pairs of e in blocks before this one
  __shared__ int total[256];
  __shared__ int offs[257];
  __shared__ uint32_t mask[256][kWords];
  griddep_wait();
  griddep_launch();
  const int nb = (a.T + kDispatchRows - 1) / kDispatchRows;
  const int b = blockIdx.x;
  for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
    int before = 0, all = 0;
    for (int q = 0; q < nb; ++q) {
      const int c = a.block_counts[q * a.E + e];
      if (q < b) before += c;
      all += c;
    }
    base[e] = before;
    total[e] = all;
  }
  for (int i = threadIdx.x; i < a.E * kWords; i += blockDim.x) mask[i / kWords][i % kWords] = 0;
  __syncthreads();
  if (threadIdx.x == 0) {
    int run = 0;
    for (int q = 0; q < a.E; ++q) { offs[q] = run; run += total[q]; }
    offs[a.E] = run;
  }
  const int tl = threadIdx.x;
  const int t = b * kDispatchRows + tl;
  if (t < a.T)
    for (int j = 0; j < a.k; ++j) atomicOr(&mask[a.idx[t * a.k + j]][tl >> 5], 1u << (tl & 31));
  __syncthreads();
  if (t < a.T) {
    for (int j = 0; j < a.k; ++j) {
      const int e = a.idx[t * a.k + j];
      int rank = __popc(mask[e][tl >> 5] & ((1u << (tl & 31)) - 1u));
      for (int w = 0; w < (tl >> 5); ++w) rank += __popc(mask[e][w]);
      const int p = offs[e] + base[e] + rank;
      a.dest_row[p] = t * a.k + j;
      a.src_token[p] = t;
    }
  }
  if (b == 0) {
    for (int q = threadIdx.x; q <= a.E; q += blockDim.x) a.offsets[q] = offs[q];
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
      a.counts[e] = total[e];
      if (a.user_counts) a.user_counts[e] = total[e];
    }
    if (threadIdx.x == 0) {
      // Tile lists: routed groups first (experts in index order), then shared.
      const int mt_shared = (a.T + a.tile_m - 1) / a.tile_m;
      int gu = 0, dn = 0;
      for (int q = 0; q < a.E; ++q) {
        a.tiles_gu[q] = gu;
        a.tiles_dn[q] = dn;
        const int mt = (total[q] + a.tile_m - 1) / a.tile_m;
        gu += mt * a.gu_ntiles_routed;
        dn += mt * a.dn_ntiles;
      }
      for (int s = 0; s < a.S; ++s) {
        a.tiles_gu[a.E + s] = gu;
        a.tiles_dn[a.E + s] = dn;
        gu += mt_shared * a.gu_ntiles_shared;
        dn += mt_shared * a.dn_ntiles;
      }
      a.tiles_gu[a.E + a.S] = gu;
      a.tiles_dn[a.E + a.S] = dn;
    }
  }
}

// dst[p] = src[src_row[p]], one warp per row, 16-byte vectors.
__global__ void k_gather_rows(const uint16_t* __restrict__ src, const int32_t* __restrict__ src_row,
                              int rows, int D, uint16_t* __restrict__ dst) {
  griddep_wait();
  griddep_launch();
  const int p = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (p >= rows) return;
  const uint4* s = reinterpret_cast<const uint4*>(src + static_cast<size_t>(src_row[p]) * D);
  uint4* d = reinterpret_cast<uint4*>(dst + static_cast<size_t>(p) * D);
  for (int c = lane; c < D / 8; c += 32) d[c] = s[c];
}

}  // namespace

cudaError_t launch_dispatch(const DispatchArgs& a, cudaStream_t s) {
  const int nb = (a.T + kDispatchRows - 1) / kDispatchRows;
  return launch_k(k_dispatch, dim3(nb), dim3(kDispatchRows), 0, s, false, a);
}

cudaError_t launch_gather_rows(const uint16_t* src, const int32_t* src_row, int rows, int D,
                               uint16_t* dst, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  const int warps_per_block = 8;
  return launch_k(k_gather_rows, dim3((rows + warps_per_block - 1) / warps_per_block),
                  dim3(32 * warps_per_block), 0, s, false, src, src_row, rows, D, dst);
}

}  // namespace moe
