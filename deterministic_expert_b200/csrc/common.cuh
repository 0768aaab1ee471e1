// Device helpers shared by the layer's kernels: bf16 conversion, the
// fixed-layout row reduction, and thin PTX wrappers for mbarrier, TMA and the
// 5th-generation tensor core (tcgen05 / TMEM) on sm_100a.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

namespace moe {

// ------------------------------------------------------------------ errors
// Device error word values (first word of every forward's workspace).
enum : int { kDevOk = 0, kDevTimeout = 1, kDevBadIndex = 3 };

// Index checks of a build with -DMOE_CHECK_BOUNDS: every index a kernel
// computes from device data (expert ids, grouped rows, tile coordinates,
// scatter destinations, rows sent to other ranks) is tested against the
// extent of the buffer it addresses; a failing index skips its access and
// records kDevBadIndex in the device error word.  Without the flag the checks
// compile to nothing.
__device__ __forceinline__ bool index_fail(int* err) {
  if (err != nullptr) atomicExch(err, kDevBadIndex);
  return false;
}
#ifdef MOE_CHECK_BOUNDS
#define MOE_INDEX_OK(cond, err) ((cond) ? true : ::moe::index_fail(err))
#else
#define MOE_INDEX_OK(cond, err) true
#endif

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ------------------------------------------------- programmatic launch
// Every kernel of the layer is launched with programmatic stream
// serialisation and calls griddep_wait() before its first global-memory
// access, so it still sees all of the previous kernel's writes (the wait
// returns once that grid has completed and flushed); what overlaps is only
// the launch and the prologue.  griddep_launch() lets the next kernel of the
// stream start launching.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch() { asm volatile("griddepcontrol.launch_dependents;" :::); }

// ------------------------------------------------------------------- bf16
__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);  // round to nearest even
  return *reinterpret_cast<uint32_t*>(&p);
}

// ------------------------------------------------- fixed-layout reduction
// Sum of one value per thread over a block of kRowThreads threads.  The
// tree is fixed: a 5-step butterfly inside each warp (__shfl_xor_sync with
// masks 16, 8, 4, 2, 1), then the warp partials added left to right by one
// thread.  Every lane of a butterfly pair forms the same sum (a + b == b + a
// in IEEE arithmetic), so all lanes end with identical bits.  The result
// depends only on the values and the block size, never on T or on which
// CTA processes the row.  Every thread receives the sum.
constexpr int kRowThreads = 256;

__device__ __forceinline__ float block_sum_fixed(float v, float* smem_warps /*[kRowThreads/32 + 1]*/) {
  v += __shfl_xor_sync(0xffffffffu, v, 16);
  v += __shfl_xor_sync(0xffffffffu, v, 8);
  v += __shfl_xor_sync(0xffffffffu, v, 4);
  v += __shfl_xor_sync(0xffffffffu, v, 2);
  v += __shfl_xor_sync(0xffffffffu, v, 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) smem_warps[warp] = v;
  __syncthreads();
  if (threadIdx.x == 0) {
    float s = smem_warps[0];
#pragma unroll
    for (int w = 1; w < kRowThreads / 32; ++w) s += smem_warps[w];
    smem_warps[kRowThreads / 32] = s;
  }
  __syncthreads();
  return smem_warps[kRowThreads / 32];
}

// The same fixed tree in fp64 (used for the input RMSNorm's sum of squares,
// whose bf16 output feeds the router: an fp64 sum of the exact squares of bf16
// values is itself exact to ~2^-52, so the bf16 code of every element of xn
// follows the exact value of the definition).
__device__ __forceinline__ double block_sum_fixed_f64(double v, double* smem_warps) {
  v += __shfl_xor_sync(0xffffffffu, v, 16);
  v += __shfl_xor_sync(0xffffffffu, v, 8);
  v += __shfl_xor_sync(0xffffffffu, v, 4);
  v += __shfl_xor_sync(0xffffffffu, v, 2);
  v += __shfl_xor_sync(0xffffffffu, v, 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) smem_warps[warp] = v;
  __syncthreads();
  if (threadIdx.x == 0) {
    double s = smem_warps[0];
#pragma unroll
    for (int w = 1; w < kRowThreads / 32; ++w) s += smem_warps[w];
    smem_warps[kRowThreads / 32] = s;
  }
  __syncthreads();
  return smem_warps[kRowThreads / 32];
}

// --------------------------------------------------------------- mbarrier
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for the phase with the given parity to complete, for at most
// limit_ns nanoseconds.  On time-out it raises *abort (shared by the CTA's
// roles) and the device error word, and returns false; it also returns
// false at once when another role has already aborted.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          int* err, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0) {
      if (*abort) return false;
      if (globaltimer_ns() - t0 > limit_ns) {
        *abort = 1;
        atomicExch(err, kDevTimeout);
        return false;
      }
    }
  }
}

// Bounded wait used while tearing down after an abort: records nothing,
// returns whether the phase completed within limit_ns.
__device__ __forceinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer_ns() - t0 > limit_ns) return false;
  return true;
}

// -------------------------------------------------------------------- TMA
// 2D tiled bulk tensor load (no multicast) into CTA shared memory; completes
// `bar`'s transaction count by the box size.  x is the innermost (K)
// coordinate in elements, y the row.
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const void* tmap, int x, int y,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// --------------------------------------------------------------- clusters
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// All threads of every CTA in the cluster.
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Shared::cluster address of the same shared-memory offset in CTA `rank`.
__device__ __forceinline__ uint32_t mapa_shared(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}

__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// Make this thread's generic-proxy shared-memory writes visible to the async
// proxy (tensor-core operand reads, tcgen05.cp).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 2D tiled load into this CTA's shared memory whose completion is counted on
// the mbarrier at `bar_cluster` (which may be the pair leader's), for a CTA
// pair feeding one cta_group::2 MMA.  No multicast.
__device__ __forceinline__ void tma_load_2d_pair(void* smem_dst, const void* tmap, int x, int y,
                                                 uint32_t bar_cluster) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(bar_cluster)
      : "memory");
}

// ------------------------------------------------------------ tcgen05/TMEM
__device__ __forceinline__ void tmem_alloc(uint32_t* smem_slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(smem_slot)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// The same for a CTA pair (both CTAs' TMEM, same column range).  Issued by
// one warp in each CTA of the pair.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* smem_slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(smem_slot)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

// Shared-memory matrix descriptor for a K-major operand tile written by TMA
// with 128-byte swizzling: rows of 64 bf16 (128 B), 8-row swizzle atoms
// 1024 B apart (stride byte offset), tile base 1024-byte aligned.  Fields:
// start address >> 4 [0,14), leading byte offset >> 4 [16,30) (unused for
// swizzled K-major), stride byte offset >> 4 [32,46), version 1 [46,48),
// base offset 0 [49,52), layout SWIZZLE_128B = 2 [61,64).
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(1u) << 16;
  d |= static_cast<uint64_t>(1024u >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(2u) << 61;
  return d;
}

// Instruction descriptor, kind::f16: fp32 accumulator (bits 4-5 = 1), A and
// B bf16 (bits 7-9 = 1, 10-12 = 1), both K-major (bits 15, 16 = 0),
// N >> 3 at bits 17-22, M >> 4 at bits 24-28.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// Instruction descriptor, kind::f8f6f4: fp32 accumulator (bits 4-5 = 1), A and
// B E4M3 (type code 0 at bits 7-9 and 10-12), both K-major, N >> 3 at bits
// 17-22, M >> 4 at bits 24-28.  One MMA then walks 32 K elements (32 bytes of a
// 128-byte swizzled row, as the bf16 form's 16).
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N) {
  return (1u << 4) | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// Block scales (kind::mxf8f6f4.block_scale, one UE8M0 scale per 32 K elements
// of every row of A and of B).  The scales of a 128-row operand for one 128-wide
// K stage form a 512-byte atom in shared memory: 16-byte row l holds the 4-byte
// words of rows l, l + 32, l + 64, l + 96, byte j of a word being the scale of
// K block j.  tcgen05.cp .32x128b.warpx4 puts the atom in 4 TMEM columns (the
// 32 rows into every lane quarter); an MMA over K block j names byte j through
// the scale ids of its instruction descriptor.  For a CTA pair, the even CTA's
// copy moves each CTA's own atom (same shared-memory offset) into its own TMEM.
// Source descriptor: no swizzle, K-major, 8-row x 16-byte core matrices 128
// bytes apart (stride byte offset 128), version 1.
__device__ __forceinline__ uint64_t sf_atom_desc(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(128u >> 4) << 16;
  d |= static_cast<uint64_t>(128u >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  return d;
}

__device__ __forceinline__ void tmem_cp_sf_pair(uint32_t taddr, uint64_t src_desc) {
  asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(src_desc) : "memory");
}

// Instruction descriptor, kind::mxf8f6f4 with block scales: A E2M1 (type 5 at
// bits 7-9: the FP4 weights), B E4M3 (type 0 at bits 10-12: the tokens), both
// K-major, N >> 3 at bits 17-22, UE8M0 scales (bit 23), M >> 4 at bits 24-28,
// scale ids of B at bits 4-5 and of A at bits 29-30 (the K block within the
// scale words); the accumulator is fp32.
__host__ __device__ constexpr uint32_t idesc_e2m1_e4m3_bs(int M, int N, int sf_id) {
  return (static_cast<uint32_t>(sf_id) << 4) | (5u << 7) | (static_cast<uint32_t>(N >> 3) << 17) | (1u << 23) |
         (static_cast<uint32_t>(M >> 4) << 24) | (static_cast<uint32_t>(sf_id) << 29);
}

// The block-scaled pair MMA: one M x N x 32 step, scales read from TMEM at
// sfa (A's rows) and sfb (B's rows).
__device__ __forceinline__ void umma_bs_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                             uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %6, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%4], [%5], p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(sfa_tmem), "r"(sfb_tmem), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, one M x N x 16 step, issued by one thread.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// The E4M3 form: one M x N x 32 step.
__device__ __forceinline__ void umma_e4m3(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on `bar` when every tcgen05 operation this thread issued so far
// has completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// D[tmem] (+)= A * B^T for a CTA pair (M = 256: rows 0-127 from the even CTA's
// shared memory and TMEM, rows 128-255 from the odd CTA's; B split by N
// between the two), issued by one thread of the even CTA.
__device__ __forceinline__ void umma_bf16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                               uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// The E4M3 form of the pair MMA: one M x N x 32 step.
__device__ __forceinline__ void umma_e4m3_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                               uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 2^e as an fp32 value for -126 <= e <= 127 (exact: a normal power of two).
__device__ __forceinline__ float exp2_int(int e) { return __int_as_float((e + 127) << 23); }

// ------------------------------------------------------------ E4M3 rows
// Per-row scale of E4M3 activations: the smallest integer e with
// amax <= 448 * 2^e, clamped to [-126, 126]; 0 for amax = 0.  With
// amax = m 2^E (m in [0.5, 1)) and 448 = 0.875 * 2^9, e = E - 9 when
// m <= 0.875, else E - 8 (exact: frexpf only splits the bits).
__device__ __forceinline__ int act_row_exp(float amax) {
  if (!(amax > 0.f)) return 0;
  int E = 0;
  const float m = frexpf(amax, &E);
  const int e = m <= 0.875f ? E - 9 : E - 8;
  return min(max(e, -126), 126);
}

// E4M3 code of v, round to nearest even, saturating at +-448.
__device__ __forceinline__ uint32_t e4m3_rn(float v) {
  return static_cast<uint32_t>(__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3));
}

// Arrive once on `bar` (same offset) in each CTA of cta_mask when the pair's
// MMAs issued so far by this thread have completed.
__device__ __forceinline__ void umma_commit_pair_mc(uint64_t* bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 "
      "[%0], %1;" ::"r"(smem_u32(bar)),
      "h"(cta_mask)
      : "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane (32x32b shape: lane
// i of the warp reads TMEM lane base + i).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

}  // namespace moe
