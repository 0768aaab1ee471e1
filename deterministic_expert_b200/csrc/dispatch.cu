// Dispatch: expert histogram, scan, and a counting-sort permute that is
// stable by token index (the dispatch step of DeepSeek V4 infra notes §6.1,
// dispatch -> compute -> combine).  Dropless: no capacity, so no token's
// routing or rows depend on the rest of the batch (the linux.do post on MoE
// variants, "MoE是如何影响输出确定性的", names token dropping as a source of
// batch dependence).  Integer-only; the result is unique.
//
//   count    block b (256 tokens) counts its (token, slot) pairs per expert
//   scan     one CTA: per-expert exclusive prefix over blocks in block order,
//            expert offsets, and the tile lists of the two expert GEMMs
//   scatter  block b ranks each pair among the block's earlier tokens that
//            chose the same expert (a token-bitmask per expert + popcount),
//            so grouped row p = offsets[e] + (pairs of e in earlier tokens)
//   gather   xp[p] = xn[src_token[p]]  (the routed GEMM's A operand)
#include "common.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

__global__ void __launch_bounds__(kDispatchRows) k_dispatch_count(const DispatchArgs a) {
  __shared__ int hist[256];
  for (int e = threadIdx.x; e < a.E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const int t = blockIdx.x * kDispatchRows + threadIdx.x;
  if (t < a.T)
    for (int j = 0; j < a.k; ++j) atomicAdd(&hist[a.idx[t * a.k + j]], 1);
  __syncthreads();
  for (int e = threadIdx.x; e < a.E; e += blockDim.x) a.block_counts[blockIdx.x * a.E + e] = hist[e];
}

__global__ void __launch_bounds__(256) k_dispatch_scan(const DispatchArgs a) {
  __shared__ int total[256];
  __shared__ int offs[257];
  const int nb = (a.T + kDispatchRows - 1) / kDispatchRows;
  const int e = threadIdx.x;
  if (e < a.E) {
    int run = 0;
    for (int b = 0; b < nb; ++b) {
      const int c = a.block_counts[b * a.E + e];
      a.block_base[b * a.E + e] = run;
      run += c;
    }
    total[e] = run;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int run = 0;
    for (int q = 0; q < a.E; ++q) { offs[q] = run; run += total[q]; }
    offs[a.E] = run;
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
  __syncthreads();
  for (int q = threadIdx.x; q <= a.E; q += blockDim.x) a.offsets[q] = offs[q];
  if (e < a.E) {
    a.counts[e] = total[e];
    if (a.user_counts) a.user_counts[e] = total[e];
    for (int b = 0; b < nb; ++b) a.block_base[b * a.E + e] += offs[e];
  }
}

__global__ void __launch_bounds__(kDispatchRows) k_dispatch_scatter(const DispatchArgs a) {
  constexpr int kWords = kDispatchRows / 32;
  __shared__ uint32_t mask[256][kWords];
  for (int i = threadIdx.x; i < a.E * kWords; i += blockDim.x) mask[i / kWords][i % kWords] = 0;
  __syncthreads();
  const int tl = threadIdx.x;
  const int t = blockIdx.x * kDispatchRows + tl;
  if (t < a.T)
    for (int j = 0; j < a.k; ++j) atomicOr(&mask[a.idx[t * a.k + j]][tl >> 5], 1u << (tl & 31));
  __syncthreads();
  if (t < a.T) {
    for (int j = 0; j < a.k; ++j) {
      const int e = a.idx[t * a.k + j];
      int rank = __popc(mask[e][tl >> 5] & ((1u << (tl & 31)) - 1u));
      for (int w = 0; w < (tl >> 5); ++w) rank += __popc(mask[e][w]);
      const int p = a.block_base[blockIdx.x * a.E + e] + rank;
      a.dest_row[p] = t * a.k + j;
      a.src_token[p] = t;
    }
  }
}

// dst[p] = src[src_row[p]], one warp per row, 16-byte vectors.
__global__ void k_gather_rows(const uint16_t* __restrict__ src, const int32_t* __restrict__ src_row,
                              int rows, int D, uint16_t* __restrict__ dst) {
  const int p = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (p >= rows) return;
  const uint4* s = reinterpret_cast<const uint4*>(src + static_cast<size_t>(src_row[p]) * D);
  uint4* d = reinterpret_cast<uint4*>(dst + static_cast<size_t>(p) * D);
  for (int c = lane; c < D / 8; c += 32) d[c] = s[c];
}

}  // namespace

cudaError_t launch_dispatch_count(const DispatchArgs& a, cudaStream_t s) {
  const int nb = (a.T + kDispatchRows - 1) / kDispatchRows;
  k_dispatch_count<<<nb, kDispatchRows, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_dispatch_scan(const DispatchArgs& a, cudaStream_t s) {
  k_dispatch_scan<<<1, 256, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_dispatch_scatter(const DispatchArgs& a, cudaStream_t s) {
  const int nb = (a.T + kDispatchRows - 1) / kDispatchRows;
  k_dispatch_scatter<<<nb, kDispatchRows, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_gather_rows(const uint16_t* src, const int32_t* src_row, int rows, int D,
                               uint16_t* dst, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  const int warps_per_block = 8;
  k_gather_rows<<<(rows + warps_per_block - 1) / warps_per_block, 32 * warps_per_block, 0, s>>>(
      src, src_row, rows, D, dst);
  return cudaGetLastError();
}

}  // namespace moe
