// Row kernels with a fixed thread layout: one CTA of 256 threads per token
// row, thread i always owning the chunks i, i + 256, i + 512, ... of the row
// (8 elements per chunk for the input norm and the partial reduce, whose
// operands are bf16 and load as 16 bytes; 4 for the combine, whose fp32 slot
// rows load as 16 bytes).  The sum of squares for RMSNorm goes through the fixed tree of
// block_sum_fixed (per-thread sum in element order, a 5-step butterfly with
// masks 16..1, warp partials added left to right), the layout the Fireworks
// parity post (Chinese translation), Trap 2, says must not change with the
// launch shape.  Nothing here depends on T.
//
//   rmsnorm_rows     (also zeroes the routing histogram) xn = bf16(g x / sqrt(mean(x^2) + eps))
//                    (linux.do post on MoE variants, "RMSNorm before up-projection"),
//                    evaluated in fp64 (sum of squares over the same fixed tree, scale
//                    and products) and rounded once to bf16, so the bf16 code of xn,
//                    which decides the routing, is that of the exact value except
//                    within ~2^-52 of a rounding midpoint
//                    (with FP8 expert weights also an E4M3 copy of xn with one
//                    power-of-two scale per row; quant_rows does the same for h)
//   combine_norm     acc = sum_j w_j y_j (slot order) + sum_s y_s; r = acc + residual;
//                    out_residual = bf16(r); out_norm = bf16(RMSNorm(r) * g)
//                    (Fireworks post, Trap 3 unfused chain and case-study "standard path":
//                    fp32 weighted sum, one cast; no atomics)
//   reduce_partials  r = ((p0 + p1) + ... + p_{P-1}) + residual in fp32, every element,
//                    then the same norm (Fireworks post, Trap 1: the r0..r7 order)
#include "common.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kMaxChunks = 16;  // D <= 4 * 256 * 16 = 16384

// Chunks per thread for a row of D elements in chunks of W elements: the
// smallest of 1, 2, 4, 8, 16 with W * 256 * NC >= D.  It depends on D only, so
// thread i owns the same chunks i, i + 256, ... whatever T is; the template
// bound only trims registers (kernels for small D keep fewer live values).
inline int chunks_for(int D, int W = 4) {
  int nc = 1;
  while (nc < kMaxChunks && W * kRowThreads * nc < D) nc *= 2;
  return nc;
}

struct f8 {
  float v[8];
};

__device__ __forceinline__ f8 ld_bf16x8(const uint16_t* p) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  f8 r;
  r.v[0] = bf16_lo(u.x); r.v[1] = bf16_hi(u.x); r.v[2] = bf16_lo(u.y); r.v[3] = bf16_hi(u.y);
  r.v[4] = bf16_lo(u.z); r.v[5] = bf16_hi(u.z); r.v[6] = bf16_lo(u.w); r.v[7] = bf16_hi(u.w);
  return r;
}

__device__ __forceinline__ void st_bf16x8(uint16_t* p, const float (&v)[8]) {
  *reinterpret_cast<uint4*>(p) = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                                            pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
}

__device__ __forceinline__ float4 ld_bf16x4(const uint16_t* p) {
  const uint2 v = *reinterpret_cast<const uint2*>(p);
  return make_float4(bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y));
}

__device__ __forceinline__ void st_bf16x4(uint16_t* p, float a, float b, float c, float d) {
  *reinterpret_cast<uint2*>(p) = make_uint2(pack_bf16x2(a, b), pack_bf16x2(c, d));
}

__device__ __forceinline__ float sumsq4(float s, float4 v) {
  s = fmaf(v.x, v.x, s);
  s = fmaf(v.y, v.y, s);
  s = fmaf(v.z, v.z, s);
  s = fmaf(v.w, v.w, s);
  return s;
}

__device__ __forceinline__ float inv_rms(float ss, int D, float eps) {
  return 1.0f / sqrtf(ss / static_cast<float>(D) + eps);
}

// bf16 code of an fp64 value, round to nearest, ties to even, in one step
// (rounding to fp32 first could land a value exactly on a bf16 midpoint and
// round it a second time).  Normal range: keep the top 7 of the 52 fraction
// bits with the usual add-half-minus-one-plus-lsb carry, then move the
// exponent bias from 1023 to 127; overflow gives infinity.  Below 2^-126 the
// bf16 spacing is 2^-133, so the code is the magnitude in units of 2^-133
// rounded to an integer (an exact scaling, then rint, which rounds half to even).
__device__ __forceinline__ uint32_t f64_to_bf16_rne(double v) {
  const unsigned long long b = static_cast<unsigned long long>(__double_as_longlong(v));
  const uint32_t sign = static_cast<uint32_t>(b >> 48) & 0x8000u;
  const unsigned long long mag = b & 0x7FFFFFFFFFFFFFFFull;
  if (mag > 0x7FF0000000000000ull) return 0x7FC0u;          // NaN
  if ((mag >> 52) >= 897ull) {                                // |v| >= 2^-126
    const unsigned long long r = (mag + 0xFFFFFFFFFFFull + ((mag >> 45) & 1ull)) >> 45;
    const unsigned long long code = r - (896ull << 7);
    return sign | static_cast<uint32_t>(code >= 0x7F80ull ? 0x7F80ull : code);
  }
  return sign | static_cast<uint32_t>(rint(fabs(v) * 0x1p133));
}

// Largest value of amax over the block (max is exact, so any order gives the
// same result); every thread receives it.
__device__ __forceinline__ float block_max(float amax, float* redf) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0) redf[threadIdx.x >> 5] = amax;
  __syncthreads();
  float m = redf[0];
#pragma unroll
  for (int w = 1; w < kRowThreads / 32; ++w) m = fmaxf(m, redf[w]);
  return m;
}

// Eight E4M3 codes of v * 2^-e (exact scaling) packed into 8 bytes, element 0
// in the lowest byte.
__device__ __forceinline__ uint2 e4m3x8(const float (&v)[8], float inv_scale) {
  uint32_t lo = 0, hi = 0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    lo |= e4m3_rn(__fmul_rn(v[q], inv_scale)) << (8 * q);
    hi |= e4m3_rn(__fmul_rn(v[q + 4], inv_scale)) << (8 * q);
  }
  return make_uint2(lo, hi);
}

template <int NC>
__global__ void __launch_bounds__(kRowThreads, NC <= 4 ? 6 : 1) k_rmsnorm_rows(const uint16_t* __restrict__ x,
                                                              const uint16_t* __restrict__ g,
                                                              uint16_t* __restrict__ y, int D,
                                                              float eps, int* err, int32_t* zero,
                                                              int zero_words, uint8_t* __restrict__ yq,
                                                              int8_t* __restrict__ yq_exp) {
  __shared__ double red[kRowThreads / 32 + 1];
  __shared__ float redf[kRowThreads / 32];
  griddep_wait();
  griddep_launch();
  if (err != nullptr && blockIdx.x == 0 && threadIdx.x == 0) *err = kDevOk;
  for (int i = blockIdx.x * kRowThreads + threadIdx.x; i < zero_words; i += gridDim.x * kRowThreads)
    zero[i] = 0;
  const size_t row = blockIdx.x;
  const int nch = D / 8;
  const uint16_t* xr = x + row * D;
  // The row stays in registers as packed bf16 (4 words per 8-element chunk),
  // half the registers of unpacked floats, so more rows fit on an SM.
  uint4 v[NC];
  double ss = 0.0;
#pragma unroll
  for (int i = 0; i < NC; ++i) {
    const int c = threadIdx.x + i * kRowThreads;
    if (c < nch) v[i] = *reinterpret_cast<const uint4*>(xr + 8 * c);
  }
#pragma unroll
  for (int i = 0; i < NC; ++i) {
    const int c = threadIdx.x + i * kRowThreads;
    if (c < nch) {
      const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const double e = static_cast<double>(q & 1 ? bf16_hi(w[q >> 1]) : bf16_lo(w[q >> 1]));
        ss = fma(e, e, ss);
      }
    }
  }
  // The squares of bf16 values are exact in fp64 and their fp64 sum is exact
  // to ~2^-52 relative; the scale and both products are fp64 too, and the
  // result is rounded once to bf16.
  const double ms = block_sum_fixed_f64(ss, red) / static_cast<double>(D);
  const double inv = 1.0 / sqrt(ms + static_cast<double>(eps));
  uint16_t* yr = y + row * D;
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < NC; ++i) {
    const int c = threadIdx.x + i * kRowThreads;
    if (c < nch) {
      const f8 gg = ld_bf16x8(g + 8 * c);
      const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
      uint32_t o[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float xv = q & 1 ? bf16_hi(w[q >> 1]) : bf16_lo(w[q >> 1]);
        o[q] = f64_to_bf16_rne(__dmul_rn(__dmul_rn(static_cast<double>(xv), inv), static_cast<double>(gg.v[q])));
      }
      v[i] = make_uint4(o[0] | (o[1] << 16), o[2] | (o[3] << 16), o[4] | (o[5] << 16), o[6] | (o[7] << 16));
      *reinterpret_cast<uint4*>(yr + 8 * c) = v[i];
      if (yq != nullptr) {
        // The E4M3 copy below reads these bf16 values (what the expert GEMMs read).
#pragma unroll
        for (int q = 0; q < 8; ++q) amax = fmaxf(amax, fabsf(bf16_lo(o[q])));
      }
    }
  }
  if (yq == nullptr) return;
  // E4M3 copy of the row with its power-of-two scale (MOE_WEIGHTS_FP8).
  const int e = act_row_exp(block_max(amax, redf));
  const float inv_scale = exp2_int(-e);
  uint8_t* qr = yq + row * D;
#pragma unroll
  for (int i = 0; i < NC; ++i) {
    const int c = threadIdx.x + i * kRowThreads;
    if (c < nch) {
      float o[8];
      o[0] = bf16_lo(v[i].x); o[1] = bf16_hi(v[i].x); o[2] = bf16_lo(v[i].y); o[3] = bf16_hi(v[i].y);
      o[4] = bf16_lo(v[i].z); o[5] = bf16_hi(v[i].z); o[6] = bf16_lo(v[i].w); o[7] = bf16_hi(v[i].w);
      *reinterpret_cast<uint2*>(qr + 8 * c) = e4m3x8(o, inv_scale);
    }
  }
  if (threadIdx.x == 0) yq_exp[row] = static_cast<int8_t>(e);
}

// Rows of h (bf16) -> E4M3 rows + per-row exponent (MOE_WEIGHTS_FP8, the down
// GEMM's input).  One warp per row, two passes over the row (the second from
// L2): the row's largest magnitude, then the codes.  Two segments in one
// launch: the routed rows (rows0 x w0) and the shared experts' rows (rows1 x w1).
__global__ void __launch_bounds__(256) k_quant_rows(const uint16_t* __restrict__ a0, int rows0, int w0,
                                                    uint8_t* __restrict__ q0, int8_t* __restrict__ e0,
                                                    const uint16_t* __restrict__ a1, int rows1, int w1,
                                                    uint8_t* __restrict__ q1, int8_t* __restrict__ e1,
                                                    const int32_t* __restrict__ rows0_dev) {
  griddep_wait();
  griddep_launch();
  const int r0 = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  const bool first = r0 < rows0;
  if (!first && r0 >= rows0 + rows1) return;
  if (first && rows0_dev != nullptr && (r0 >= rows0_dev[0] || r0 < rows0_dev[1])) return;
  const int r = first ? r0 : r0 - rows0;
  const int w = first ? w0 : w1;
  const uint16_t* ar = (first ? a0 : a1) + static_cast<size_t>(r) * w;
  uint8_t* qr = (first ? q0 : q1) + static_cast<size_t>(r) * w;
  float amax = 0.f;
  for (int c = lane; c < w / 8; c += 32) {
    const f8 v = ld_bf16x8(ar + 8 * c);
#pragma unroll
    for (int q = 0; q < 8; ++q) amax = fmaxf(amax, fabsf(v.v[q]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const int e = act_row_exp(amax);
  const float inv_scale = exp2_int(-e);
  for (int c = lane; c < w / 8; c += 32) {
    const f8 v = ld_bf16x8(ar + 8 * c);
    *reinterpret_cast<uint2*>(qr + 8 * c) = e4m3x8(v.v, inv_scale);
  }
  if (lane == 0) (first ? e0 : e1)[r] = static_cast<int8_t>(e);
}

// Shared tail of the two epilogues: r (kept in registers) -> out_residual,
// out_norm.
template <int NC>
__device__ __forceinline__ void norm_store(const float4 (&r)[NC], float ss, float* red,
                                           const uint16_t* __restrict__ g, uint16_t* on,
                                           int D, float eps) {
  const int nch = D / 4;
  const float inv = inv_rms(block_sum_fixed(ss, red), D, eps);
#pragma unroll
  for (int i = 0; i < NC; ++i) {
    const int c = threadIdx.x + i * kRowThreads;
    if (c < nch) {
      const float4 gg = ld_bf16x4(g + 4 * c);
      st_bf16x4(on + 4 * c, r[i].x * inv * gg.x, r[i].y * inv * gg.y, r[i].z * inv * gg.z,
                r[i].w * inv * gg.w);
    }
  }
}

template <int NC>
__global__ void __launch_bounds__(kRowThreads) k_combine_norm(
    const float* __restrict__ y_slot, const float* __restrict__ topk_w,
    const float* __restrict__ y_shared, int k, int S, const uint16_t* __restrict__ residual,
    const uint16_t* __restrict__ g, uint16_t* __restrict__ out_norm,
    uint16_t* __restrict__ out_residual, int T, int D, float eps) {
  __shared__ float red[kRowThreads / 32 + 1];
  __shared__ float w_s[16];
  griddep_wait();
  griddep_launch();
  const size_t t = blockIdx.x;
  if (threadIdx.x < k) w_s[threadIdx.x] = topk_w != nullptr ? topk_w[t * k + threadIdx.x] : 1.0f;
  __syncthreads();
  const int nch = D / 4;
  float4 r[NC];
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < NC; ++i) {
    const int c = threadIdx.x + i * kRowThreads;
    if (c < nch) {
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int j = 0; j < k; ++j) {  // routed, slot order
        const float4 y = *reinterpret_cast<const float4*>(y_slot + (t * k + j) * D + 4 * c);
        const float w = w_s[j];
        acc.x = fmaf(w, y.x, acc.x); acc.y = fmaf(w, y.y, acc.y);
        acc.z = fmaf(w, y.z, acc.z); acc.w = fmaf(w, y.w, acc.w);
      }
      for (int s = 0; s < S; ++s) {  // shared, index order
        const float4 y = *reinterpret_cast<const float4*>(y_shared + (s * static_cast<size_t>(T) + t) * D + 4 * c);
        acc.x += y.x; acc.y += y.y; acc.z += y.z; acc.w += y.w;
      }
      const float4 res = ld_bf16x4(residual + t * D + 4 * c);
      r[i] = make_float4(acc.x + res.x, acc.y + res.y, acc.z + res.z, acc.w + res.w);
      st_bf16x4(out_residual + t * D + 4 * c, r[i].x, r[i].y, r[i].z, r[i].w);
      ss = sumsq4(ss, r[i]);
    }
  }
  norm_store(r, ss, red, g, out_norm + t * D, D, eps);
}

// Latent MoE: a[t] = bf16(sum_j w_j y[t, j]) over the routed experts' latent
// outputs, in slot order, fp32, one cast (the linux.do post on MoE variants,
// "潜在MoE": the experts' weighted sum before the up-projection).  Thread i owns
// the 4-element chunks i, i + 256, ... of the latent row.
template <int NC>
__global__ void __launch_bounds__(kRowThreads) k_combine_latent(const float* __restrict__ y_slot,
                                                                const float* __restrict__ topk_w, int k,
                                                                int L, uint16_t* __restrict__ agg) {
  __shared__ float w_s[16];
  griddep_wait();
  griddep_launch();
  const size_t t = blockIdx.x;
  if (threadIdx.x < k) w_s[threadIdx.x] = topk_w[t * k + threadIdx.x];
  __syncthreads();
  const int nch = L / 4;
#pragma unroll
  for (int i = 0; i < NC; ++i) {
    const int c = threadIdx.x + i * kRowThreads;
    if (c < nch) {
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int j = 0; j < k; ++j) {
        const float4 y = *reinterpret_cast<const float4*>(y_slot + (t * k + j) * L + 4 * c);
        const float w = w_s[j];
        acc.x = fmaf(w, y.x, acc.x); acc.y = fmaf(w, y.y, acc.y);
        acc.z = fmaf(w, y.z, acc.z); acc.w = fmaf(w, y.w, acc.w);
      }
      st_bf16x4(agg + t * L + 4 * c, acc.x, acc.y, acc.z, acc.w);
    }
  }
}

template <int NC>
__global__ void __launch_bounds__(kRowThreads) k_reduce_partials(
    const PartialPtrs parts, int P, const uint16_t* __restrict__ residual,
    const uint16_t* __restrict__ g, const OutPtrs outs, int n_out, int row0, int D, float eps) {
  __shared__ float red[kRowThreads / 32 + 1];
  griddep_wait();
  griddep_launch();
  const size_t t = static_cast<size_t>(row0) + blockIdx.x;
  const int nch = D / 8;
  f8 r[NC];
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < NC; ++i) {
    const int c = threadIdx.x + i * kRowThreads;
    if (c < nch) {
      const size_t off = t * D + 8 * c;
      // Issue every partial's load before the first add.
      uint4 raw[8];
#pragma unroll
      for (int p = 0; p < 8; ++p)
        if (p < P) raw[p] = *reinterpret_cast<const uint4*>(parts.p[p] + off);
      const f8 res = ld_bf16x8(residual + off);
      const uint32_t* w0 = reinterpret_cast<const uint32_t*>(&raw[0]);
      float acc[8];
#pragma unroll
      for (int q = 0; q < 4; ++q) { acc[2 * q] = bf16_lo(w0[q]); acc[2 * q + 1] = bf16_hi(w0[q]); }
#pragma unroll
      for (int p = 1; p < 8; ++p) {  // r0 + r1 + ... + r_{P-1}, left to right
        if (p < P) {
          const uint32_t* wp = reinterpret_cast<const uint32_t*>(&raw[p]);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            acc[2 * q] = __fadd_rn(acc[2 * q], bf16_lo(wp[q]));
            acc[2 * q + 1] = __fadd_rn(acc[2 * q + 1], bf16_hi(wp[q]));
          }
        }
      }
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        r[i].v[q] = __fadd_rn(acc[q], res.v[q]);
        ss = fmaf(r[i].v[q], r[i].v[q], ss);
      }
#pragma unroll
      for (int d = 0; d < 8; ++d)
        if (d < n_out) st_bf16x8(outs.res[d] + off, r[i].v);
    }
  }
  const float inv = inv_rms(block_sum_fixed(ss, red), D, eps);
#pragma unroll
  for (int i = 0; i < NC; ++i) {
    const int c = threadIdx.x + i * kRowThreads;
    if (c < nch) {
      const f8 gg = ld_bf16x8(g + 8 * c);
      float o[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) o[q] = r[i].v[q] * inv * gg.v[q];
#pragma unroll
      for (int d = 0; d < 8; ++d)
        if (d < n_out) st_bf16x8(outs.norm[d] + t * D + 8 * c, o);
    }
  }
}

// Count bf16 elements of a whose bits differ from the matching row of b
// (b row = b_row_of_a[row], or row itself when NULL).
__global__ void k_bitcompare(const uint16_t* __restrict__ a, const uint16_t* __restrict__ b,
                             const int32_t* __restrict__ b_row_of_a, int rows, int D,
                             unsigned long long* count) {
  griddep_wait();
  griddep_launch();
  const int per_row = D / 8;
  const size_t n = static_cast<size_t>(rows) * per_row;
  unsigned long long mism = 0;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t row = i / per_row, col = (i % per_row) * 8;
    const size_t brow = b_row_of_a ? static_cast<size_t>(b_row_of_a[row]) : row;
    const uint4 va = *reinterpret_cast<const uint4*>(a + row * D + col);
    const uint4 vb = *reinterpret_cast<const uint4*>(b + brow * D + col);
    const uint32_t xa[4] = {va.x, va.y, va.z, va.w}, xb[4] = {vb.x, vb.y, vb.z, vb.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t d = xa[q] ^ xb[q];
      mism += ((d & 0xFFFFu) != 0) + ((d >> 16) != 0);
    }
  }
  for (int o = 16; o > 0; o >>= 1) mism += __shfl_xor_sync(0xffffffffu, mism, o);
  if ((threadIdx.x & 31) == 0 && mism) atomicAdd(count, mism);
}

// xo[i] = x[perm[i]], ro[i] = res[perm[i]], io[i] = ids[perm[i]]: one warp per row.
__global__ void k_permute_inputs(const uint16_t* __restrict__ x, const uint16_t* __restrict__ res,
                                 const int32_t* __restrict__ ids, const int32_t* __restrict__ perm,
                                 int T, int D, uint16_t* __restrict__ xo, uint16_t* __restrict__ ro,
                                 int32_t* __restrict__ io) {
  griddep_wait();
  griddep_launch();
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= T) return;
  const size_t src = perm[warp];
  const uint4* xs = reinterpret_cast<const uint4*>(x + src * D);
  const uint4* rs = reinterpret_cast<const uint4*>(res + src * D);
  uint4* xd = reinterpret_cast<uint4*>(xo + static_cast<size_t>(warp) * D);
  uint4* rd = reinterpret_cast<uint4*>(ro + static_cast<size_t>(warp) * D);
  for (int c = lane; c < D / 8; c += 32) { xd[c] = xs[c]; rd[c] = rs[c]; }
  if (lane == 0 && ids != nullptr) io[warp] = ids[src];
}

// One thread waits on a flag nothing sets, bounded by limit_ns.
__global__ void k_wait_selftest(volatile int* flag, int* err, unsigned long long limit_ns) {
  const uint64_t t0 = globaltimer_ns();
  while (*flag == 0) {
    if (globaltimer_ns() - t0 > limit_ns) {
      atomicExch(err, kDevTimeout);
      return;
    }
    __nanosleep(1000);
  }
}

}  // namespace

cudaError_t launch_rmsnorm_rows(const uint16_t* x, const uint16_t* g, uint16_t* y, int T, int D,
                                float eps, int* err_to_clear, int32_t* zero, int zero_words,
                                uint8_t* yq, int8_t* yq_exp, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  auto go = [&](auto kernel) {
    return launch_k(kernel, dim3(T), dim3(kRowThreads), 0, s, false, x, g, y, D, eps, err_to_clear,
                    zero, zero_words, yq, yq_exp);
  };
  switch (chunks_for(D, 8)) {
    case 1: return go(k_rmsnorm_rows<1>);
    case 2: return go(k_rmsnorm_rows<2>);
    case 4: return go(k_rmsnorm_rows<4>);
    case 8: return go(k_rmsnorm_rows<8>);
    default: return go(k_rmsnorm_rows<16>);
  }
}

cudaError_t launch_quant_rows(const uint16_t* a0, int rows0, int w0, uint8_t* q0, int8_t* e0,
                              const uint16_t* a1, int rows1, int w1, uint8_t* q1, int8_t* e1,
                              const int32_t* rows0_dev, cudaStream_t s) {
  const int rows = rows0 + rows1;
  if (rows <= 0) return cudaSuccess;
  return launch_k(k_quant_rows, dim3((rows + 7) / 8), dim3(256), 0, s, false, a0, rows0, w0, q0, e0, a1,
                  rows1, w1, q1, e1, rows0_dev);
}

cudaError_t launch_combine_norm(const float* y_slot, const float* topk_w, const float* y_shared,
                                int k, int S, const uint16_t* residual, const uint16_t* g,
                                uint16_t* out_norm, uint16_t* out_residual, int T, int D,
                                float eps, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  auto go = [&](auto kernel) {
    return launch_k(kernel, dim3(T), dim3(kRowThreads), 0, s, false, y_slot, topk_w, y_shared, k, S,
                    residual, g, out_norm, out_residual, T, D, eps);
  };
  switch (chunks_for(D)) {
    case 1: return go(k_combine_norm<1>);
    case 2: return go(k_combine_norm<2>);
    case 4: return go(k_combine_norm<4>);
    case 8: return go(k_combine_norm<8>);
    default: return go(k_combine_norm<16>);
  }
}

cudaError_t launch_combine_latent(const float* y_slot, const float* topk_w, int k, int L, uint16_t* agg,
                                  int T, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  auto go = [&](auto kernel) {
    return launch_k(kernel, dim3(T), dim3(kRowThreads), 0, s, false, y_slot, topk_w, k, L, agg);
  };
  switch (chunks_for(L)) {
    case 1: return go(k_combine_latent<1>);
    case 2: return go(k_combine_latent<2>);
    case 4: return go(k_combine_latent<4>);
    case 8: return go(k_combine_latent<8>);
    default: return go(k_combine_latent<16>);
  }
}

cudaError_t launch_reduce_partials(const PartialPtrs& parts, int P, const uint16_t* residual,
                                   const uint16_t* g, const OutPtrs& outs, int n_out, int row0, int rows,
                                   int D, float eps, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  auto go = [&](auto kernel) {
    return launch_k(kernel, dim3(rows), dim3(kRowThreads), 0, s, false, parts, P, residual, g, outs, n_out,
                    row0, D, eps);
  };
  switch (chunks_for(D, 8)) {
    case 1: return go(k_reduce_partials<1>);
    case 2: return go(k_reduce_partials<2>);
    case 4: return go(k_reduce_partials<4>);
    case 8: return go(k_reduce_partials<8>);
    default: return go(k_reduce_partials<16>);
  }
}

cudaError_t launch_bitcompare(const uint16_t* a, const uint16_t* b, const int32_t* b_row_of_a,
                              int rows, int D, unsigned long long* count, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  const size_t n = static_cast<size_t>(rows) * (D / 8);
  int grid = static_cast<int>((n + 255) / 256);
  if (grid > 148 * 8) grid = 148 * 8;
  return launch_k(k_bitcompare, dim3(grid), dim3(256), 0, s, false, a, b, b_row_of_a, rows, D, count);
}

cudaError_t launch_permute_inputs(const uint16_t* x, const uint16_t* res, const int32_t* ids,
                                  const int32_t* perm, int T, int D, uint16_t* xo, uint16_t* ro,
                                  int32_t* io, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  const int warps_per_block = 8;
  return launch_k(k_permute_inputs, dim3((T + warps_per_block - 1) / warps_per_block),
                  dim3(32 * warps_per_block), 0, s, false, x, res, ids, perm, T, D, xo, ro, io);
}

cudaError_t launch_wait_selftest(int* flag, int* err, unsigned long long limit_ns, cudaStream_t s) {
  k_wait_selftest<<<1, 1, 0, s>>>(flag, err, limit_ns);
  return cudaGetLastError();
}

}  // namespace moe
