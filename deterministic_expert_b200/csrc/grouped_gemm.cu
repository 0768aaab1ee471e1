// Grouped GEMM on the 5th-generation tensor cores (tcgen05 + TMEM), fed by TMA.
//
// Used three ways by the layer:
//   router : logits[T, E_pad] = xn W_r^T                     one group of T rows
//   gate/up: h = bf16(SiLU(min(g, c_g)) * clamp(u, +-c_u)),  g = A W_g^T, u = A W_u^T,
//            per routed expert (A = its grouped rows of xn) and per shared expert (A = xn)
//   down   : y = h W_d^T in fp32, routed rows scattered to their (token, slot) row
//
// Batch invariance (the Meituan LongCat parity article, "为什么会不一致": keep
// the whole K of a dot product in one accumulation instead of summing split
// partial results).  Every output element is one TMEM accumulator that walks
// all of K in 64-wide steps, 16 per MMA, in the same order for every tile;
// the tile shape (128 x BN) is fixed per layer shape and never chosen from T;
// rows of a tile never mix (a row's result depends only on its own A row), so
// padding rows and rows of a neighbouring group are computed and discarded.
//
// Structure (one CTA per SM, persistent over a device-built tile list):
//   warp 0   one thread issues TMA loads of A and B tiles into a 4-stage ring
//   warp 1   allocates 512 TMEM columns; one thread issues tcgen05.mma and
//            commits stage releases / accumulator-ready signals to mbarriers
//   warps 2-9 epilogue: tcgen05.ld the accumulator (one TMEM lane = one row per
//            thread; two warps per lane quarter split the columns), apply SwiGLU
//            or scatter, store to global memory
// Two accumulator buffers let the epilogue of tile i overlap the MMAs of i+1.
// Every mbarrier wait is bounded in time; on time-out the CTA records an error
// word, drains its own TMA copies and MMAs (bounded), frees TMEM and exits.
#include "common.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr uint32_t kTmemCols = 512;
constexpr unsigned long long kDrainNs = 200ull * 1000 * 1000;  // 200 ms

struct Tile {
  int kind;   // 0 routed, 1 shared
  int idx;    // expert index within its kind
  int rows;   // rows of the group
  int a_row0; // first A row of the group
  int m, n;   // tile coordinates within the group
};

__device__ __forceinline__ void decode_tile(const GemmArgs& a, int t, Tile& ti) {
  if (a.tile_start == nullptr) {
    ti.kind = 0; ti.idx = 0; ti.rows = a.T; ti.a_row0 = 0; ti.m = t; ti.n = 0;
    return;
  }
  // Largest g with tile_start[g] <= t; tile_start[0] = 0 <= t < tile_start[G].
  int lo = 0, hi = a.G;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (a.tile_start[mid] <= t) lo = mid; else hi = mid;
  }
  const int local = t - a.tile_start[lo];
  if (lo < a.E) {
    const int o0 = a.offsets[lo];
    ti.kind = 0; ti.idx = lo; ti.rows = a.offsets[lo + 1] - o0; ti.a_row0 = o0;
  } else {
    ti.kind = 1; ti.idx = lo - a.E; ti.rows = a.T; ti.a_row0 = ti.idx * a.shared_a_stride;
  }
  const int mt = (ti.rows + kBM - 1) / kBM;
  ti.n = local / mt;
  ti.m = local - ti.n * mt;
}

// SiLU(min(g, c_g)) * clamp(u, -c_u, c_u) in fp32 with the fast exponential
// and division (deterministic; about 2 ulp, far below the bf16 rounding of h).
__device__ __forceinline__ float silu_clamped_product(float g, float u, float cg, float cu) {
  g = fminf(g, cg);
  u = fminf(fmaxf(u, -cu), cu);
  return __fdividef(g, 1.0f + __expf(-g)) * u;
}

template <int MODE>
__global__ void __launch_bounds__(kGemmThreads, 1) k_grouped_gemm(const __grid_constant__ GemmArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + kStages * kSmemA;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + kStages * kSmemBMax);
  uint64_t* full = bars;
  uint64_t* empty = bars + kStages;
  uint64_t* tfull = bars + 2 * kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* tdone = tempty + 2;
  uint8_t* epi = reinterpret_cast<uint8_t*>(bars) + 256;  // kEpiWarps x kEpiBytes
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(&tfull[b], 1); mbar_init(&tempty[b], kEpiWarps); }
    mbar_init(tdone, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(&tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_slot;
  volatile int* abort = &abort_flag;

  const int total = (a.tile_start == nullptr) ? a.router_tiles : a.tile_start[a.G];
  const int BN = a.BN;
  const uint32_t bytesB = static_cast<uint32_t>(BN) * kBK * 2;
  constexpr int kNB = (MODE == kGateUp) ? 2 : 1;
  const uint32_t stage_bytes = kSmemA + bytesB * kNB;
  const uint32_t acc_stride = static_cast<uint32_t>(BN * kNB);  // TMEM columns per buffer

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int issued[kStages];
      for (int s = 0; s < kStages; ++s) issued[s] = -1;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < total; t += gridDim.x) {
        Tile ti;
        decode_tile(a, t, ti);
        const int nkb = a.k_kind[ti.kind] / kBK;
        const int a_y = ti.a_row0 + ti.m * kBM;
        const int b_y = ti.idx * a.n_kind[ti.kind] + ti.n * BN;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort, a.err, a.timeout_ns)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[stage], stage_bytes);
          tma_load_2d(sA + stage * kSmemA, &a.mapA[ti.kind], kb * kBK, a_y, &full[stage]);
          uint8_t* b0 = sB + stage * kSmemBMax;
          tma_load_2d(b0, &a.mapB[ti.kind * 2], kb * kBK, b_y, &full[stage]);
          if (MODE == kGateUp)
            tma_load_2d(b0 + bytesB, &a.mapB[ti.kind * 2 + 1], kb * kBK, b_y, &full[stage]);
          issued[stage] = static_cast<int>(phase);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        // Let the copies already in flight land before the CTA goes away.
        for (int s = 0; s < kStages; ++s)
          if (issued[s] >= 0) mbar_wait_drain(&full[s], static_cast<uint32_t>(issued[s]), kDrainNs);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer
    if (lane == 0) {
      // Gate/up: the gate tile (BN rows) and the up tile (BN rows) sit back to
      // back in shared memory, so one N = 2*BN MMA reads A once and writes the
      // gate accumulator to columns [0, BN) and the up accumulator to [BN, 2*BN).
      const uint32_t idesc = idesc_bf16_f32(kBM, MODE == kGateUp ? 2 * BN : BN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < total; t += gridDim.x) {
        Tile ti;
        decode_tile(a, t, ti);
        const int nkb = a.k_kind[ti.kind] / kBK;
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, abort, a.err, a.timeout_ns)) break;
        tc_fence_after();
        const uint32_t d0 = tmem_base + static_cast<uint32_t>(acc) * acc_stride;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort, a.err, a.timeout_ns)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * kSmemA);
          const uint32_t b_addr = smem_u32(sB + stage * kSmemBMax);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint64_t ad = sw128_kmajor_desc(a_addr + kk * 32);
            const uint32_t accum = (kb | kk) != 0 ? 1u : 0u;
            umma_bf16(d0, ad, sw128_kmajor_desc(b_addr + kk * 32), idesc, accum);
          }
          umma_commit(&empty[stage]);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      // Every MMA issued above has finished before TMEM is released.
      umma_commit(tdone);
      mbar_wait_drain(tdone, 0, kDrainNs);
    }
  } else {
    // --------------------------------------------------------- epilogue
    // Two warps per TMEM lane quarter (32 accumulator rows each) split the
    // tile's columns: half 0 takes blocks 0, 2, 4, ..., half 1 blocks 1, 3, ...
    // (64 columns per block for gate/up, 32 otherwise).  Each block is read with
    // tcgen05.ld (lane i = row i), staged in the warp's own 4 KB buffer, and
    // stored back so that every store instruction writes whole 128-byte row
    // segments (8 lanes per row, 4 rows at a time).  The buffer holds 32 rows
    // of 128 bytes; 16-byte chunk m of row r sits at chunk m ^ (r & 7), so both
    // the row-wise writes and the column-wise reads are free of bank conflicts.
    const int q = warp & 3;                  // TMEM lane quarter this warp may access
    const int half = (warp - 2) >> 2;        // which column blocks
    uint8_t* stage_w = epi + (warp - 2) * kEpiBytes;
    const int sr = lane >> 3, sc = lane & 7; // store phase: row offset 0..3, 16-byte chunk 0..7
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x) {
      Tile ti;
      decode_tile(a, t, ti);
      bool ok = mbar_wait(&tfull[acc], acc_phase, abort, a.err, a.timeout_ns);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                          static_cast<uint32_t>(acc) * acc_stride;
      const int grow0 = ti.m * kBM + q * 32;   // first group row of this warp's block
      const int nvalid = max(0, min(32, ti.rows - grow0));
      if (MODE == kGateUp) {
        const int orow0 = (ti.kind == 0 ? ti.a_row0 : ti.idx * a.shared_out_stride) + grow0;
        uint8_t* out0 = reinterpret_cast<uint8_t*>(static_cast<uint16_t*>(a.out[ti.kind]) + ti.n * BN);
        const size_t ld_bytes = static_cast<size_t>(a.ld_out[ti.kind]) * 2;
        for (int c = 64 * half; c < BN; c += 128) {
#pragma unroll
          for (int hb = 0; hb < 2; ++hb) {
            uint32_t g[32], u[32];
            tmem_ld32(tb + c + 32 * hb, g);
            tmem_ld32(tb + BN + c + 32 * hb, u);
            tmem_ld_wait();
            uint32_t p[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              p[i] = pack_bf16x2(
                  silu_clamped_product(__uint_as_float(g[2 * i]), __uint_as_float(u[2 * i]),
                                       a.gate_clamp, a.up_clamp),
                  silu_clamped_product(__uint_as_float(g[2 * i + 1]), __uint_as_float(u[2 * i + 1]),
                                       a.gate_clamp, a.up_clamp));
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int m = 4 * hb + i;
              *reinterpret_cast<uint4*>(stage_w + lane * 128 + ((m ^ (lane & 7)) << 4)) =
                  make_uint4(p[4 * i], p[4 * i + 1], p[4 * i + 2], p[4 * i + 3]);
            }
          }
          __syncwarp();
#pragma unroll
          for (int s8 = 0; s8 < 8; ++s8) {
            const int r = 4 * s8 + sr;
            if (r < nvalid) {
              const uint4 v = *reinterpret_cast<const uint4*>(stage_w + r * 128 + ((sc ^ (r & 7)) << 4));
              *reinterpret_cast<uint4*>(out0 + static_cast<size_t>(orow0 + r) * ld_bytes + c * 2 + 16 * sc) = v;
            }
          }
          __syncwarp();
        }
      } else {
        // fp32 output, 32 columns (128 bytes) per block.
        const bool scatter = (MODE == kDown && ti.kind == 0);
        const int my_dest = (scatter && lane < nvalid) ? a.dest_row[ti.a_row0 + grow0 + lane] : 0;
        const int orow0 = (ti.kind == 0 ? ti.a_row0 : ti.idx * a.shared_out_stride) + grow0;
        float* out0 = static_cast<float*>(a.out[ti.kind]) + ti.n * BN;
        const size_t ld = static_cast<size_t>(a.ld_out[ti.kind]);
        for (int c = 32 * half; c < BN; c += 64) {
          uint32_t v[32];
          tmem_ld32(tb + c, v);
          tmem_ld_wait();
          if (BN - c >= 32) {
#pragma unroll
            for (int m = 0; m < 8; ++m)
              *reinterpret_cast<uint4*>(stage_w + lane * 128 + ((m ^ (lane & 7)) << 4)) =
                  make_uint4(v[4 * m], v[4 * m + 1], v[4 * m + 2], v[4 * m + 3]);
            __syncwarp();
#pragma unroll
            for (int s8 = 0; s8 < 8; ++s8) {
              const int r = 4 * s8 + sr;
              const int drow = __shfl_sync(0xffffffffu, my_dest, r);
              if (r < nvalid) {
                const uint4 val = *reinterpret_cast<const uint4*>(stage_w + r * 128 + ((sc ^ (r & 7)) << 4));
                const size_t orow = scatter ? static_cast<size_t>(drow) : static_cast<size_t>(orow0 + r);
                *reinterpret_cast<uint4*>(out0 + orow * ld + c + 4 * sc) = val;
              }
            }
            __syncwarp();
          } else if (lane < nvalid) {
            // Narrow tail (router with fewer than 32 columns left): direct stores.
            const size_t orow = scatter ? static_cast<size_t>(my_dest) : static_cast<size_t>(orow0 + lane);
            float4* dst = reinterpret_cast<float4*>(out0 + orow * ld + c);
            const int nq = (BN - c) / 4;
#pragma unroll
            for (int i = 0; i < 8; ++i)
              if (i < nq)
                dst[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                     __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace

void gemm_prepare() {
  static int done_dev = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (done_dev == dev) return;
  cudaFuncSetAttribute(k_grouped_gemm<kGateUp>, cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmem);
  cudaFuncSetAttribute(k_grouped_gemm<kDown>, cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmem);
  cudaFuncSetAttribute(k_grouped_gemm<kRouter>, cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmem);
  done_dev = dev;
}

cudaError_t launch_grouped_gemm(int mode, const GemmArgs& a, int grid, cudaStream_t s) {
  if (grid <= 0) return cudaSuccess;
  switch (mode) {
    case kGateUp: k_grouped_gemm<kGateUp><<<grid, kGemmThreads, kGemmSmem, s>>>(a); break;
    case kDown: k_grouped_gemm<kDown><<<grid, kGemmThreads, kGemmSmem, s>>>(a); break;
    default: k_grouped_gemm<kRouter><<<grid, kGemmThreads, kGemmSmem, s>>>(a); break;
  }
  return cudaGetLastError();
}

}  // namespace moe
