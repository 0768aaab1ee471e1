// Dispatch: expert offsets and a counting-sort permute that is stable by token
// index (the dispatch step of DeepSeek V4 infra notes §6.1, dispatch ->
// compute -> combine).  Dropless: no capacity, so no token's routing or rows
// depend on the rest of the batch (the linux.do post on MoE variants,
// "MoE是如何影响输出确定性的", names token dropping as a source of batch
// dependence).  Integer-only; the result is unique.
//
//   dispatch  block b (128 tokens) reads the per-block expert counts the router
//             wrote (all blocks' rows at once, 16-byte loads), forms the exclusive
//             prefix over experts (offsets, a block scan) and over the blocks
//             before it, then ranks each of its (token, slot) pairs
//             among the block's earlier tokens that chose the same expert (a
//             token bitmask per expert + popcount): grouped row
//             p = offsets[e] + (pairs of e in earlier tokens).  Block 0 also
//             writes the counts, the offsets and the two expert-GEMM tile lists.
//   gather    xp[p] = xn[src_token[p]]  (the routed GEMM's A operand; bf16
//             rows, or E4M3 rows and their exponents)
#include "common.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

// Exclusive prefix sum of in[0..n) into out[0..n], out[n] = total, by the
// kDispatchRows threads of the block (n <= kDispatchRows * kScanPer): thread i
// scans a run of consecutive items, a warp scan and the warp totals (left to
// right) give the run's base.  Integer only, so the order is immaterial.
constexpr int kScanPer = 3;
__device__ __forceinline__ void block_exclusive_scan(const int* in, int* out, int n, int* warp_tot) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = (n + kDispatchRows - 1) / kDispatchRows;
  const int i0 = tid * per;
  int v[kScanPer];
  int run = 0;
#pragma unroll
  for (int u = 0; u < kScanPer; ++u) {
    v[u] = (u < per && i0 + u < n) ? in[i0 + u] : 0;
    run += v[u];
  }
  int incl = run;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  int base = incl - run;
  int all = 0;
#pragma unroll
  for (int w = 0; w < kDispatchRows / 32; ++w) {
    if (w < warp) base += warp_tot[w];
    all += warp_tot[w];
  }
#pragma unroll
  for (int u = 0; u < kScanPer; ++u)
    if (u < per && i0 + u < n) { out[i0 + u] = base; base += v[u]; }
  if (tid == 0) out[n] = all;
  __syncthreads();
}

__global__ void __launch_bounds__(kDispatchRows) k_dispatch(const DispatchArgs a) {
  constexpr int kWords = kDispatchRows / 32;
  constexpr int kMaxG = 256 + 8;
  __shared__ int before[256];  // pairs of e in the blocks before this one
  __shared__ int total[256];
  __shared__ int offs[257];
  __shared__ int cnt[kMaxG], tstart[kMaxG + 1];
  __shared__ int warp_tot[kDispatchRows / 32];
  __shared__ uint32_t mask[256][kWords];
  const int tid = threadIdx.x;
  const int b = blockIdx.x;
  const int nb = (a.T + kDispatchRows - 1) / kDispatchRows;
  for (int e = tid; e < a.E; e += kDispatchRows) { before[e] = 0; total[e] = 0; }
  for (int i = tid; i < a.E * kWords; i += kDispatchRows) mask[i / kWords][i % kWords] = 0;
  griddep_wait();
  griddep_launch();
  __syncthreads();
  // Column sums of the [nb, E4] block counts, 16-byte loads eight at a time.
  {
    const int row4 = a.E4 / 4;
    const int n4 = nb * row4;
    const int4* bc4 = reinterpret_cast<const int4*>(a.block_counts);
    for (int f0 = tid; f0 < n4; f0 += 8 * kDispatchRows) {
      int4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int f = f0 + u * kDispatchRows;
        v[u] = f < n4 ? bc4[f] : make_int4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int f = f0 + u * kDispatchRows;
        if (f >= n4) continue;
        const int q = f / row4, e = (f - q * row4) * 4;
        const int c[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
        for (int z = 0; z < 4; ++z) {
          if (c[z] == 0 || e + z >= a.E) continue;
          atomicAdd(&total[e + z], c[z]);
          if (q < b) atomicAdd(&before[e + z], c[z]);
        }
      }
    }
  }
  __syncthreads();
  block_exclusive_scan(total, offs, a.E, warp_tot);

  const int t = b * kDispatchRows + tid;
  if (t < a.T)
    for (int j = 0; j < a.k; ++j) {
      const int e = a.idx[t * a.k + j];
      if (MOE_INDEX_OK(e >= 0 && e < a.E, a.err)) atomicOr(&mask[e][tid >> 5], 1u << (tid & 31));
    }
  __syncthreads();
  if (t < a.T) {
    for (int j = 0; j < a.k; ++j) {
      const int e = a.idx[t * a.k + j];
      if (!MOE_INDEX_OK(e >= 0 && e < a.E, a.err)) continue;
      int rank = __popc(mask[e][tid >> 5] & ((1u << (tid & 31)) - 1u));
      for (int w = 0; w < (tid >> 5); ++w) rank += __popc(mask[e][w]);
      const int p = offs[e] + before[e] + rank;
      if (!MOE_INDEX_OK(p >= 0 && p < a.T * a.k, a.err)) continue;
      a.dest_row[p] = t * a.k + j;
      a.src_token[p] = t;
    }
  }
  if (b == 0) {
    for (int q = tid; q <= a.E; q += kDispatchRows) a.offsets[q] = offs[q];
    for (int e = tid; e < a.E; e += kDispatchRows) {
      a.counts[e] = total[e];
      if (a.user_counts) a.user_counts[e] = total[e];
    }
    // Tile lists: routed groups first (experts in index order), then shared.
    const int G = a.E + a.S;
    const int mt_shared = (a.T + a.tile_m - 1) / a.tile_m;
    for (int g = tid; g < G; g += kDispatchRows)
      cnt[g] = (g < a.E ? (total[g] + a.tile_m - 1) / a.tile_m * a.gu_ntiles_routed
                        : mt_shared * a.gu_ntiles_shared);
    __syncthreads();
    block_exclusive_scan(cnt, tstart, G, warp_tot);
    for (int g = tid; g <= G; g += kDispatchRows) a.tiles_gu[g] = tstart[g];
    __syncthreads();
    for (int g = tid; g < G; g += kDispatchRows)
      cnt[g] = g < a.E ? (total[g] + a.tile_m - 1) / a.tile_m * a.dn_ntiles : mt_shared * a.dn_ntiles_shared;
    __syncthreads();
    block_exclusive_scan(cnt, tstart, G, warp_tot);
    for (int g = tid; g <= G; g += kDispatchRows) a.tiles_dn[g] = tstart[g];
  }
}

// dst[p] = src[src_row[p]], one warp per row, 16-byte vectors.
// Row p of dst = row src_row[p] of src (row_bytes each, a multiple of 16: bf16
// rows or E4M3 rows), and with E4M3 rows also their exponents.
__global__ void k_gather_rows(const uint8_t* __restrict__ src, int src_rows, const int32_t* __restrict__ src_row,
                              int rows, int row_bytes, uint8_t* __restrict__ dst,
                              const int8_t* __restrict__ src_exp, int8_t* __restrict__ dst_exp, int* err) {
  griddep_wait();
  griddep_launch();
  const int p = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (p >= rows) return;
  const int from = src_row[p];
  if (!MOE_INDEX_OK(from >= 0 && from < src_rows, err)) return;
  const uint4* s = reinterpret_cast<const uint4*>(src + static_cast<size_t>(from) * row_bytes);
  uint4* d = reinterpret_cast<uint4*>(dst + static_cast<size_t>(p) * row_bytes);
  // Four 16-byte loads in flight per lane before their stores.
  const int n = row_bytes / 16;
  int c = lane;
  for (; c + 96 < n; c += 128) {
    const uint4 v0 = s[c], v1 = s[c + 32], v2 = s[c + 64], v3 = s[c + 96];
    d[c] = v0; d[c + 32] = v1; d[c + 64] = v2; d[c + 96] = v3;
  }
  for (; c < n; c += 32) d[c] = s[c];
  if (dst_exp != nullptr && lane == 0) dst_exp[p] = src_exp[from];
}

}  // namespace

cudaError_t launch_dispatch(const DispatchArgs& a, cudaStream_t s) {
  const int nb = (a.T + kDispatchRows - 1) / kDispatchRows;
  return launch_k(k_dispatch, dim3(nb), dim3(kDispatchRows), 0, s, false, a);
}

cudaError_t launch_gather_rows(const void* src, int src_rows, const int32_t* src_row, int rows, int row_bytes,
                               void* dst, const int8_t* src_exp, int8_t* dst_exp, int* err, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  const int warps_per_block = 8;
  return launch_k(k_gather_rows, dim3((rows + warps_per_block - 1) / warps_per_block),
                  dim3(32 * warps_per_block), 0, s, false, static_cast<const uint8_t*>(src), src_rows, src_row,
                  rows, row_bytes, static_cast<uint8_t*>(dst), src_exp, dst_exp, err);
}

}  // namespace moe
