// Router scores and top-k, one warp per token.
//
//   softmax  keys = l (+ logit bias b), p = exp(l + b - max) / sum over all E
//            (nxmr.cn "V4" article, §2.2: Linear -> logits -> softmax -> top-k)
//   sigmoid  s = 1 / (1 + exp(-l)), keys = s + b, the bias only selects
//            (DeepSeek V4 infra notes §6.3: upper layers use sigmoid + balancing;
//            linux.do post, "QuantileBalancing": expert e enters when s + b > tau)
//   hash     e_0 = ((id * mult) mod 2^32) mod E, e_j = (e_0 + j) mod E, w = 1/k
//            (DeepSeek V4 infra notes §6.3 "Hash Routing", no router parameters)
//
// Selection is deterministic: k rounds of a warp arg-max under the total
// order (key descending, expert index ascending), so equal keys go to the
// lower index and slot j holds the j-th best expert.  Each token also adds its
// k experts to the histogram of its 128-token block (integer atomics into a
// buffer the input RMSNorm zeroed; the counts do not depend on the order).  Lane l always owns
// experts l, l + 32, ... and every sum runs in a fixed order (per lane in
// index order, then a 5-step butterfly), so a token's routing does not
// depend on T.  Keys that are NaN rank below every number.  Softmax selects on
// the logits themselves (the softmax is monotone), weights use the
// probabilities; renormalised weights divide by their sum in slot order.
#include <cfloat>

#include "common.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kMaxPerLane = 8;  // E <= 256

__device__ __forceinline__ bool better(float k1, int e1, float k2, int e2) {
  return k1 > k2 || (k1 == k2 && e1 < e2);
}

// Route token t (one warp; lr = its logits row, anywhere in memory; hist = the
// histogram its experts are counted into).  Shared by the per-token kernel and
// the single-block decode kernel, so both take the same arithmetic.
__device__ __forceinline__ void route_token(const RouterArgs& a, int t, int lane, const float* lr,
                                            int32_t* hist) {
  const int k = a.k, E = a.E;

  if (a.router == MOE_ROUTER_HASH) {
    if (lane < k) {
      const uint32_t h = static_cast<uint32_t>(a.token_ids[t]) * a.hash_mult;  // mod 2^32
      const int e0 = static_cast<int>(h % static_cast<uint32_t>(E));
      const int e = (e0 + lane) % E;
      const float w = a.routed_scale / static_cast<float>(k);
      a.idx[t * k + lane] = e;
      a.w[t * k + lane] = w;
      if (a.user_idx) a.user_idx[t * k + lane] = e;
      if (a.user_w) a.user_w[t * k + lane] = w;
      atomicAdd(hist + e, 1);
    }
    return;
  }

  float key[kMaxPerLane], val[kMaxPerLane];
  float zmax = -FLT_MAX;
#pragma unroll
  for (int i = 0; i < kMaxPerLane; ++i) {
    const int e = lane + 32 * i;
    key[i] = -INFINITY;
    val[i] = 0.f;
    if (e < E) {
      const float l = lr[e];
      const float b = a.bias ? a.bias[e] : 0.f;
      if (a.router == MOE_ROUTER_SOFTMAX) {
        key[i] = l + b;
        zmax = fmaxf(zmax, key[i]);
      } else {
        val[i] = 1.0f / (1.0f + expf(-l));
        key[i] = val[i] + b;
      }
      if (isnan(key[i])) key[i] = -INFINITY;
    }
  }
  float denom = 1.f;
  if (a.router == MOE_ROUTER_SOFTMAX) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) zmax = fmaxf(zmax, __shfl_xor_sync(0xffffffffu, zmax, o));
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < kMaxPerLane; ++i) {
      const int e = lane + 32 * i;
      if (e < E) {
        val[i] = expf(key[i] - zmax);
        s += val[i];
      }
    }
    s += __shfl_xor_sync(0xffffffffu, s, 16);
    s += __shfl_xor_sync(0xffffffffu, s, 8);
    s += __shfl_xor_sync(0xffffffffu, s, 4);
    s += __shfl_xor_sync(0xffffffffu, s, 2);
    s += __shfl_xor_sync(0xffffffffu, s, 1);
    denom = s;
  }

  // k rounds of a warp arg-max; the loops run to the compile-time bound 16 so
  // the chosen values stay in registers.
  uint32_t taken = 0;
  float chosen_v[16];
  int chosen_e[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    chosen_v[j] = 0.f;
    chosen_e[j] = 0;
    if (j < k) {
      float bk = -INFINITY;
      int be = 0x7fffffff, bi = -1;
#pragma unroll
      for (int i = 0; i < kMaxPerLane; ++i) {
        const int e = lane + 32 * i;
        if (e < E && !(taken & (1u << i)) && better(key[i], e, bk, be)) { bk = key[i]; be = e; bi = i; }
      }
      float bv = 0.f;
#pragma unroll
      for (int i = 0; i < kMaxPerLane; ++i)
        if (i == bi) bv = val[i];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ok = __shfl_xor_sync(0xffffffffu, bk, o);
        const int oe = __shfl_xor_sync(0xffffffffu, be, o);
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        if (better(ok, oe, bk, be)) { bk = ok; be = oe; bv = ov; }
      }
      if ((be & 31) == lane) taken |= 1u << (be >> 5);
      chosen_e[j] = be;
      chosen_v[j] = bv;
    }
  }

  float norm = denom;
  if (a.renormalize) {
    norm = 0.f;
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (j < k) norm += chosen_v[j];
  }
  // Lane j < k writes slot j.
  float w = 0.f;
  int e = 0;
#pragma unroll
  for (int q = 0; q < 16; ++q)
    if (q == lane) { w = chosen_v[q]; e = chosen_e[q]; }
  if (lane < k) {
    const float wn = ((a.router == MOE_ROUTER_SOFTMAX || a.renormalize) ? w / norm : w) * a.routed_scale;
    a.idx[t * k + lane] = e;
    a.w[t * k + lane] = wn;
    if (a.user_idx) a.user_idx[t * k + lane] = e;
    if (a.user_w) a.user_w[t * k + lane] = wn;
    atomicAdd(hist + e, 1);
  }
}

__global__ void __launch_bounds__(256) k_router_topk(const RouterArgs a) {
  griddep_wait();
  griddep_launch();
  const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (t >= a.T) return;
  route_token(a, t, lane, a.logits + static_cast<size_t>(t) * a.E_pad,
              a.block_counts + static_cast<size_t>(t / kDispatchRows) * a.E4);
}

}  // namespace

cudaError_t launch_router_topk(const RouterArgs& a, cudaStream_t s) {
  if (a.T <= 0) return cudaSuccess;
  const int warps_per_block = 8;
  return launch_k(k_router_topk, dim3((a.T + warps_per_block - 1) / warps_per_block),
                  dim3(32 * warps_per_block), 0, s, false, a);
}

}  // namespace moe
