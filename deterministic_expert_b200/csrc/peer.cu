// Device-side barrier of the ranks of one node for the tensor-parallel
// epilogue (the Fireworks parity post, Trap 1: every rank must run the same
// fixed-order reduction, so each rank reads all ranks' partials of its rows
// and writes the reduced rows back to every rank; the barrier orders those
// peer reads and writes between steps).  Flags live in memory exported by
// each rank (moe_peer_alloc) and mapped by the others (moe_peer_open).
#include "common.cuh"
#include "moe_internal.h"

namespace moe {

__device__ __forceinline__ void st_release_sys(uint32_t* p, uint32_t v) {
  asm volatile("st.release.sys.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t ld_acquire_sys(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// One warp; lane t < world signals rank t, then waits for rank t's signal.
// Every wait is bounded by limit_ns of global time: on expiry the lane stores
// kDevTimeout to *err and stops waiting, so the kernel always ends.
__global__ void __launch_bounds__(32) k_peer_barrier(PeerFlags f, int world, int rank, uint32_t epoch,
                                                     int* err, unsigned long long limit_ns) {
  const int t = threadIdx.x;
  if (t < world) {
    // Writes of the stream's earlier kernels (the partials, the reduced rows
    // stored to peers) become visible at system scope before the signal.
    __threadfence_system();
    st_release_sys(f.p[t] + rank, epoch);
    const uint32_t* mine = f.p[rank] + t;
    if (static_cast<int32_t>(ld_acquire_sys(mine) - epoch) < 0) {
      const uint64_t t0 = globaltimer_ns();
      while (static_cast<int32_t>(ld_acquire_sys(mine) - epoch) < 0) {
        if (globaltimer_ns() - t0 > limit_ns) {
          atomicExch(err, kDevTimeout);
          break;
        }
        __nanosleep(128);
      }
    }
  }
  __syncwarp();
}

cudaError_t launch_peer_barrier(const PeerFlags& f, int world, int rank, uint32_t epoch, int* err,
                                unsigned long long limit_ns, cudaStream_t s) {
  // A plain launch (no programmatic serialisation): the barrier starts after
  // the previous kernel of the stream has completed, and the next kernel,
  // which waits on griddepcontrol, after the barrier has completed.
  k_peer_barrier<<<1, 32, 0, s>>>(f, world, rank, epoch, err, limit_ns);
  return cudaGetLastError();
}

}  // namespace moe
