// Seeded synthetic inputs, device side.
//
// The GPU twin of gen_host.c, written separately from the same definition
// (SplitMix64 output function, Irwin-Hall n = 12 normal, one fp32 multiply,
// round-to-nearest-even to bf16); see gen_host.c for the full statement.  It
// holds none of the MoE layer's arithmetic and is not part of the layer
// library: tests and the benchmark use it to fill large weight tensors in
// place, and regenerate any slice on the host to feed the oracle.
#include <cstdint>
#include <cuda_runtime.h>

namespace {

constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ULL;

__device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

__device__ __forceinline__ uint64_t draw(uint64_t key, uint64_t i) {
  return mix64(key + (i + 1) * kGamma);
}

__device__ __forceinline__ float unit_normal(uint64_t key, uint64_t i) {
  int32_t s = 0;
#pragma unroll
  for (int j = 0; j < 3; ++j) {
    const uint64_t d = draw(key, 3 * i + (uint64_t)j);
    s += (int32_t)(d & 0xFFFF) + (int32_t)((d >> 16) & 0xFFFF) +
         (int32_t)((d >> 32) & 0xFFFF) + (int32_t)(d >> 48);
  }
  // Both conversions are exact: |s - 393210| < 2^20 and the scale is 2^-16.
  return __fmul_rn((float)(s - 393210), 1.0f / 65536.0f);
}

__device__ __forceinline__ uint16_t bf16_rne(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return 0x7FC0;
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

__global__ void k_normal_bf16(uint64_t key, uint64_t start, uint64_t count, float sigma,
                              uint16_t* __restrict__ out) {
  for (uint64_t j = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; j < count;
       j += (uint64_t)gridDim.x * blockDim.x)
    out[j] = bf16_rne(__fmul_rn(unit_normal(key, start + j), sigma));
}

__global__ void k_normal_f32(uint64_t key, uint64_t start, uint64_t count, float sigma,
                             float* __restrict__ out) {
  for (uint64_t j = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; j < count;
       j += (uint64_t)gridDim.x * blockDim.x)
    out[j] = __fmul_rn(unit_normal(key, start + j), sigma);
}

__global__ void k_uniform_int(uint64_t key, uint64_t start, uint64_t count, uint32_t n,
                              int32_t* __restrict__ out) {
  for (uint64_t j = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; j < count;
       j += (uint64_t)gridDim.x * blockDim.x)
    out[j] = (int32_t)(((draw(key, start + j) >> 32) * (uint64_t)n) >> 32);
}

int grid_for(uint64_t count) {
  uint64_t g = (count + 255) / 256;
  if (g > 148ull * 32) g = 148ull * 32;
  return g ? (int)g : 1;
}

}  // namespace

extern "C" {

// Each call enqueues one kernel on `stream` and returns the cudaError_t of
// the launch.  `out` is a device pointer to `count` elements.
int syn_dev_normal_bf16(uint64_t key, uint64_t start, uint64_t count, float sigma,
                        void* out, void* stream) {
  if (count == 0) return 0;
  k_normal_bf16<<<grid_for(count), 256, 0, (cudaStream_t)stream>>>(key, start, count, sigma,
                                                                   (uint16_t*)out);
  return (int)cudaGetLastError();
}

int syn_dev_normal_f32(uint64_t key, uint64_t start, uint64_t count, float sigma, void* out,
                       void* stream) {
  if (count == 0) return 0;
  k_normal_f32<<<grid_for(count), 256, 0, (cudaStream_t)stream>>>(key, start, count, sigma,
                                                                  (float*)out);
  return (int)cudaGetLastError();
}

int syn_dev_uniform_int(uint64_t key, uint64_t start, uint64_t count, uint32_t n, void* out,
                        void* stream) {
  if (count == 0) return 0;
  k_uniform_int<<<grid_for(count), 256, 0, (cudaStream_t)stream>>>(key, start, count, n,
                                                                   (int32_t*)out);
  return (int)cudaGetLastError();
}

}  // extern "C"
