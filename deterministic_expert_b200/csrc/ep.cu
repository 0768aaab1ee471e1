// Expert parallelism: the two kernels that move rows between ranks and plan
// the owner's GEMMs (DeepSeek V4 infra notes, §6.1: dispatch -> compute ->
// combine across ranks; the Fireworks parity post, Trap 3: the k results of a
// token are summed on its own rank, in slot order, in fp32).
//
//   ep_send  every (token, slot) row of this rank, already grouped by expert in
//            token order, is stored at its expert's owner: row
//              base(e) + sum of the earlier ranks' counts of e + its index in
//              this rank's group of e,
//            base(e) = the rows of the owner's earlier experts over all ranks;
//            its return address (rank, token * k + slot) goes beside it.  The
//            layout depends only on the counts, so it is the same whatever the
//            timing of the ranks.
//   ep_plan  the owner's per-expert row offsets and the tile lists of its two
//            expert GEMMs (its E / world routed groups, then its shared groups
//            over its own tokens).
//
// Waves (the wave scheduling of §6.1 there: each wave covers a few experts, and
// the rows of wave w + 1 travel while the GEMMs of wave w run): both kernels can
// be limited to local experts [wave_lo, wave_hi) of every owner.  A wave's send
// writes exactly the rows, addresses and bytes that the whole send writes for
// those experts, and the wave's plan lists only their tiles (plus the shared
// experts' in the wave that carries them), so the waves together do the same
// arithmetic on the same rows as one pass.
// Stores to other ranks are plain 16-byte stores to peer-mapped memory.
#include "common.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kEpMaxE = 256;

__global__ void __launch_bounds__(256) k_ep_send(const EpSendArgs a) {
  __shared__ int offs[kEpMaxE + 1];
  __shared__ int dst[kEpMaxE];
  __shared__ int tot[kEpMaxE];
  __shared__ int seg_start[9], seg_pre[9];
  griddep_wait();
  griddep_launch();
  const int tid = threadIdx.x;
  for (int e = tid; e < a.E; e += blockDim.x) {
    int t = 0, pre = 0;
    for (int r = 0; r < a.world; ++r) {
      const int c = a.boards[r][e];
      t += c;
      if (r < a.rank) pre += c;
    }
    tot[e] = t;
    dst[e] = pre;
  }
  for (int e = tid; e <= a.E; e += blockDim.x) offs[e] = a.offsets[e];
  __syncthreads();
  // base(e): rows of the owner's experts before e (all source ranks).
  for (int e = tid; e < a.E; e += blockDim.x) {
    int base = 0;
    for (int f = (e / a.E_loc) * a.E_loc; f < e; ++f) base += tot[f];
    dst[e] += base;
  }
  // This wave's rows: for each owner o, the grouped rows of its experts
  // o * E_loc + [wave_lo, wave_hi), contiguous in this rank's grouping.
  if (tid == 0) {
    int pre = 0;
    for (int o = 0; o < a.world; ++o) {
      seg_start[o] = offs[o * a.E_loc + a.wave_lo];
      seg_pre[o] = pre;
      pre += offs[o * a.E_loc + a.wave_hi] - seg_start[o];
    }
    seg_pre[a.world] = pre;
  }
  __syncthreads();
  const int n = seg_pre[a.world];
  const int warp = tid >> 5, lane = tid & 31;
  const int nw = blockDim.x >> 5;
  for (int q = blockIdx.x * nw + warp; q < n; q += gridDim.x * nw) {
    int o = 0;
    while (o + 1 < a.world && seg_pre[o + 1] <= q) ++o;
    const int p = seg_start[o] + (q - seg_pre[o]);
    if (!MOE_INDEX_OK(p >= 0 && p < a.rows, a.err)) continue;
    // Expert of grouped row p: the largest e with offs[e] <= p.
    int lo = 0, hi = a.E;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (offs[mid] <= p) lo = mid; else hi = mid;
    }
    const int e = lo, owner = e / a.E_loc;
    const int row = dst[e] + (p - offs[e]);
    const int tok = a.src_token[p];
    if (!MOE_INDEX_OK(owner < a.world && row >= 0 && row < a.cap && tok >= 0, a.err)) continue;
    const uint4* s = reinterpret_cast<const uint4*>(a.src_rows + static_cast<size_t>(tok) * a.row_bytes);
    uint4* d = reinterpret_cast<uint4*>(a.recv[owner] + static_cast<size_t>(row) * a.row_bytes);
    for (int c = lane; c < a.row_bytes / 16; c += 32) d[c] = s[c];
    if (lane == 0) {
      a.meta[owner][row] = (a.rank << 24) | a.dest_row[p];
      if (a.src_exp != nullptr) a.recv_exp[owner][row] = a.src_exp[tok];
    }
  }
}

__global__ void __launch_bounds__(256) k_ep_plan(const EpPlanArgs a) {
  __shared__ int cnt[kEpMaxE + 8];
  griddep_wait();
  griddep_launch();
  const int tid = threadIdx.x;
  const int G = a.E_loc + a.S;
  for (int e = tid; e < a.E_loc; e += blockDim.x) {
    int t = 0;
    for (int r = 0; r < a.world; ++r) t += a.boards[r][a.rank * a.E_loc + e];
    cnt[e] = t;
  }
  __syncthreads();
  if (tid == 0) {
    // At most 264 groups: plain serial scans.
    int o = 0;
    for (int e = 0; e < a.E_loc; ++e) {
      a.offsets[e] = o;
      if (e == a.wave_lo) a.rows_received[1] = o;
      if (e == a.wave_hi) a.rows_received[0] = o;
      o += cnt[e];
    }
    a.offsets[a.E_loc] = o;
    if (a.wave_hi == a.E_loc) a.rows_received[0] = o;
    const int mt_shared = (a.T_self + a.tile_m - 1) / a.tile_m;
    int tg = 0, td = 0;
    for (int g = 0; g < G; ++g) {
      a.tiles_gu[g] = tg;
      a.tiles_dn[g] = td;
      if (g < a.E_loc) {
        if (g < a.wave_lo || g >= a.wave_hi) continue;
        const int mt = (cnt[g] + a.tile_m - 1) / a.tile_m;
        tg += mt * a.gu_ntiles_routed;
        td += mt * a.dn_ntiles;
      } else if (a.with_shared) {
        tg += mt_shared * a.gu_ntiles_shared;
        td += mt_shared * a.dn_ntiles_shared;
      }
    }
    a.tiles_gu[G] = tg;
    a.tiles_dn[G] = td;
  }
}

}  // namespace

cudaError_t launch_ep_send(const EpSendArgs& a, int grid, cudaStream_t s) {
  if (a.rows <= 0) return cudaSuccess;
  return launch_k(k_ep_send, dim3(grid), dim3(256), 0, s, false, a);
}

cudaError_t launch_ep_plan(const EpPlanArgs& a, cudaStream_t s) {
  return launch_k(k_ep_plan, dim3(1), dim3(256), 0, s, false, a);
}

}  // namespace moe
