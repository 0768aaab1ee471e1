// FP4 expert weights (DeepSeek V4 infra notes, §6.2 FP4 QAT: master weights are
// quantised to FP4 (E2M1) with one scale factor per block; FP4 -> FP8 is
// lossless because every E2M1 value times the block's scale is an FP8 value).
// The storage form (packed codes + exponents) and the scale atoms the
// block-scaled expert GEMMs read are built here too.
// One thread per block of 32 consecutive elements along a row (the GEMM's
// contraction axis): the block's power-of-two scale, each element's nearest
// E2M1 value, and the E4M3 code of their product, which the expert GEMMs read.
#include "common.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kFp4Block = 32;

// Smallest integer s with amax <= 6 * 2^s, clamped to [-8, 6] (-8 for amax = 0).
// amax = m 2^E with m in [0.5, 1): 6 * 2^(E-3) = 0.75 * 2^E, so s = E - 3 when
// m <= 0.75, else E - 2.  Within [-8, 6] every E2M1 value times 2^s is an E4M3
// value (0.5 * 2^-8 = 2^-9 is E4M3's smallest subnormal, 6 * 2^6 = 384 <= 448).
__device__ __forceinline__ int fp4_block_exp(float amax) {
  if (!(amax > 0.f)) return -8;
  int E = 0;
  const float m = frexpf(amax, &E);
  const int s = m <= 0.75f ? E - 3 : E - 2;
  return min(max(s, -8), 6);
}

// Nearest E2M1 magnitude to x >= 0 (x is exact: a bf16 value times a power of
// two).  The grid is 0, 0.5, 1, 1.5, 2, 3, 4, 6; a value halfway between two
// neighbours goes to the one with the even code (0, 1, 2, 4), and anything past
// 5 goes to 6.
__device__ __forceinline__ float e2m1_rn(float x) {
  if (x <= 0.25f) return 0.f;
  if (x < 0.75f) return 0.5f;
  if (x <= 1.25f) return 1.f;
  if (x < 1.75f) return 1.5f;
  if (x <= 2.5f) return 2.f;
  if (x < 3.5f) return 3.f;
  if (x <= 5.f) return 4.f;
  return 6.f;
}

__global__ void __launch_bounds__(256) k_quant_weights_fp4(const uint16_t* __restrict__ w,
                                                           uint8_t* __restrict__ w8,
                                                           int8_t* __restrict__ block_exp,
                                                           long long nblocks) {
  const long long b = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (b >= nblocks) return;
  const uint4* src = reinterpret_cast<const uint4*>(w + b * kFp4Block);
  float v[kFp4Block];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 u = src[i];
    const uint32_t word[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      v[8 * i + 2 * j] = bf16_lo(word[j]);
      v[8 * i + 2 * j + 1] = bf16_hi(word[j]);
    }
  }
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < kFp4Block; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const int s = fp4_block_exp(amax);
  const float down = exp2_int(-s), up = exp2_int(s);
  uint32_t out[kFp4Block / 4];
#pragma unroll
  for (int i = 0; i < kFp4Block / 4; ++i) {
    uint32_t word = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float x = v[4 * i + j];
      const float q = e2m1_rn(__fmul_rn(fabsf(x), down));
      const float val = __fmul_rn(q, up);
      word |= e4m3_rn(copysignf(val, x)) << (8 * j);   // -0 and small negatives: code 0x80
    }
    out[i] = word;
  }
  uint4* dst = reinterpret_cast<uint4*>(w8 + b * kFp4Block);
  dst[0] = make_uint4(out[0], out[1], out[2], out[3]);
  dst[1] = make_uint4(out[4], out[5], out[6], out[7]);
  if (block_exp != nullptr) block_exp[b] = static_cast<int8_t>(s);
}

// Index of the nearest E2M1 magnitude to x >= 0 in 0, 0.5, 1, 1.5, 2, 3, 4, 6
// (the same thresholds and ties as e2m1_rn).
__device__ __forceinline__ uint32_t e2m1_index_rn(float x) {
  if (x <= 0.25f) return 0;
  if (x < 0.75f) return 1;
  if (x <= 1.25f) return 2;
  if (x < 1.75f) return 3;
  if (x <= 2.5f) return 4;
  if (x < 3.5f) return 5;
  if (x <= 5.f) return 6;
  return 7;
}

// The storage form: one thread per 32-element block writes its 16 bytes of
// packed E2M1 codes and its exponent byte (word [c, row] of exps, byte kb % 4).
__global__ void __launch_bounds__(256) k_quant_weights_fp4_packed(const uint16_t* __restrict__ w,
                                                                  uint8_t* __restrict__ packed,
                                                                  uint8_t* __restrict__ exps_bytes,
                                                                  long long nblocks, int kblocks,
                                                                  long long rows) {
  const long long b = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (b >= nblocks) return;
  const uint4* src = reinterpret_cast<const uint4*>(w + b * kFp4Block);
  float v[kFp4Block];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 u = src[i];
    const uint32_t word[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      v[8 * i + 2 * j] = bf16_lo(word[j]);
      v[8 * i + 2 * j + 1] = bf16_hi(word[j]);
    }
  }
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < kFp4Block; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const int s = fp4_block_exp(amax);
  const float down = exp2_int(-s);
  uint32_t out[kFp4Block / 8];
#pragma unroll
  for (int i = 0; i < kFp4Block / 8; ++i) {
    uint32_t word = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float x = v[8 * i + j];
      const uint32_t code = e2m1_index_rn(__fmul_rn(fabsf(x), down)) | (signbit(x) ? 8u : 0u);
      word |= code << (4 * j);
    }
    out[i] = word;
  }
  *reinterpret_cast<uint4*>(packed + b * (kFp4Block / 2)) = make_uint4(out[0], out[1], out[2], out[3]);
  const long long row = b / kblocks, kb = b - row * kblocks;
  exps_bytes[((kb >> 2) * rows + row) * 4 + (kb & 3)] = static_cast<uint8_t>(static_cast<int8_t>(s));
}

// Scale atoms for the block-scaled expert GEMMs: thread (atom, word i) writes
// word i = 4 l + w of atom (h, kc), the UE8M0 bytes (exponent + 127, per byte)
// of one weight row's four 32-element blocks of stage kc.  Gate/up halves
// (second != NULL): w = 0, 1 -> first (gate) rows 64 h + 32 w + l, w = 2, 3 ->
// second (up) rows 64 h + 32 (w - 2) + l; down halves: rows 128 h + 32 w + l.
__global__ void __launch_bounds__(256) k_fp4_scale_atoms(const uint32_t* __restrict__ first,
                                                         const uint32_t* __restrict__ second, long long rows,
                                                         int KC, uint32_t* __restrict__ atoms, long long words) {
  const long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= words) return;
  const int i = static_cast<int>(t & 127);
  const long long atom = t >> 7;
  const long long h = atom / KC;
  const int kc = static_cast<int>(atom - h * KC);
  const int l = i >> 2, w = i & 3;
  const uint32_t* src = first;
  long long row;
  if (second != nullptr) {
    if (w >= 2) src = second;
    row = 64 * h + 32 * (w & 1) + l;
  } else {
    row = 128 * h + 32 * w + l;
  }
  atoms[t] = __vadd4(src[static_cast<long long>(kc) * rows + row], 0x7F7F7F7Fu);
}

}  // namespace

cudaError_t launch_fp4_scale_atoms(const uint32_t* first, const uint32_t* second, long long rows, int KC,
                                   uint32_t* atoms, cudaStream_t s) {
  const long long words = rows / (second ? 64 : 128) * KC * 128;
  if (words <= 0) return cudaSuccess;
  const long long grid = (words + 255) / 256;
  if (grid > 0x7FFFFFFFll) return cudaErrorInvalidValue;
  k_fp4_scale_atoms<<<static_cast<unsigned>(grid), 256, 0, s>>>(first, second, rows, KC, atoms, words);
  return cudaGetLastError();
}

cudaError_t launch_quant_weights_fp4_packed(const uint16_t* w, uint8_t* packed, uint32_t* exps, long long rows,
                                            int K, cudaStream_t s) {
  const long long nblocks = rows * (K / kFp4Block);
  if (nblocks <= 0) return cudaSuccess;
  const long long grid = (nblocks + 255) / 256;
  if (grid > 0x7FFFFFFFll) return cudaErrorInvalidValue;
  k_quant_weights_fp4_packed<<<static_cast<unsigned>(grid), 256, 0, s>>>(
      w, packed, reinterpret_cast<uint8_t*>(exps), nblocks, K / kFp4Block, rows);
  return cudaGetLastError();
}

cudaError_t launch_quant_weights_fp4(const uint16_t* w, uint8_t* w8, int8_t* block_exp, long long nblocks,
                                     cudaStream_t s) {
  if (nblocks <= 0) return cudaSuccess;
  const long long grid = (nblocks + 255) / 256;
  if (grid > 0x7FFFFFFFll) return cudaErrorInvalidValue;
  k_quant_weights_fp4<<<static_cast<unsigned>(grid), 256, 0, s>>>(w, w8, block_exp, nblocks);
  return cudaGetLastError();
}

}  // namespace moe
