// Grouped GEMM on the 5th-generation tensor cores (tcgen05 + TMEM), fed by TMA.
//
// Used three ways by the layer:
//   router : logits[T, E_pad] = xn W_r^T                     one group of T rows
//   gate/up: h = bf16(SiLU(min(g, c_g)) * clamp(u, +-c_u)),  g = A W_g^T, u = A W_u^T,
//            (or the SiTU-GLU unit [b_g tanh(g/b_g) sigmoid(g)] * [b_u tanh(u/b_u)])
//            per routed expert (A = its grouped rows of xn) and per shared expert (A = xn)
//   down   : y = h W_d^T in fp32, routed rows scattered to their (token, slot) row
//   dense  : one group of T rows with N-tiles through the down path (the latent
//            projections; bf16 or fp32 output)
//
// Batch invariance (the Meituan LongCat parity article, "为什么会不一致": keep
// the whole K of a dot product in one accumulation instead of summing split
// partial results).  Every output element is one TMEM accumulator that walks
// all of K in 64-wide steps, 16 per MMA, in the same order for every tile;
// rows of a tile never mix (a row's result depends only on its own A row), so
// padding rows and rows of a neighbouring group are computed and discarded.
// The MMA accumulates an element over K in the same order whatever the tile's
// M, N or operand roles (checked bit for bit on B200), so the tile shapes
// below, which do depend on a group's row count, never change a result.
//
// Two variants, persistent over a device-built tile list:
//   CG = 1  one CTA per 128-row tile (the router GEMM).
//   CG = 2  a CTA pair (cluster of 2) per 256-row tile with cta_group::2 MMAs
//           (the expert GEMMs): each CTA loads its own 128 A rows and half of
//           the B tile (one half of the output columns: gate/up as [gate | up]
//           rows for those columns, down as those rows of W_d), so each SM's
//           shared memory receives and feeds half the B bytes of a 1-CTA tile.
//           The even CTA issues the MMAs; its commits reach both CTAs.  A
//           group's last r < 256 rows run operand-swapped: the CTA's 128 weight
//           rows are the M = 256 MMA's A operand and its r/2 token rows the B
//           operand (N = r rounded up to 16), so a group's padding is under 16
//           rows.  (Shapes whose tiles are not 128 gate/up or 256 down columns
//           use a 128-row pair tile, M = 128, for the last <= 128 rows.)
// Roles in each CTA:
//   warp 0    one thread issues the TMA loads of its CTA into a stage ring
//   warp 1    allocates 512 TMEM columns; in the (even) issuing CTA one thread
//             issues tcgen05.mma and commits stage releases / accumulator-ready
//   warps 2-9 epilogue: tcgen05.ld the accumulator (one TMEM lane = one row per
//             thread; two warps per lane quarter split the columns), apply
//             SwiGLU or scatter, store to global memory
// Two accumulator buffers let the epilogue of tile i overlap the MMAs of i+1.
// FP4 weights (packed E2M1 codes with one power-of-two scale per 32 K
// elements; DeepSeek V4 infra notes, §6.2 FP4 QAT) go to the tensor core as
// they are: TMA spreads each 8 bytes of codes over a 16-byte chunk (the operand
// form kind::mxf8f6f4 reads), the block scales travel as UE8M0 atoms with each
// stage and are copied into TMEM, and every tile is an operand-swapped
// block-scaled pair MMA (weights the M = 256 operand with their scales, the
// E4M3 tokens the N <= 240 operand with scale 1).
// Every mbarrier wait is bounded in time; on time-out the CTA records an error
// word, drains its own TMA copies and MMAs (bounded), frees TMEM and exits.
#include <algorithm>

#include "common.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr uint32_t kTmemCols = 512;
constexpr int kMaxGroups = 256 + 8;   // routed experts + shared experts (checked by moe_init)
constexpr int kRingBytes = kStages * (kSmemA + kSmemBMax);  // shared memory of the stage ring
constexpr int kRingMax = 12;                                // most stages any variant uses
constexpr int kBarBytes = kGemmBarBytes;                    // mbarrier region after the ring
constexpr unsigned long long kDrainNs = 200ull * 1000 * 1000;  // 200 ms

template <int CG>
struct Cfg {
  static constexpr int kTileM = 128 * CG;                                 // rows per tile (pair)
  static constexpr int kSmemB = CG == 1 ? 256 * kBK * 2 : 128 * kBK * 2;  // B bytes per CTA stage
};

struct Tile {
  int kind;   // 0 routed, 1 shared
  int idx;    // expert index within its kind
  int rows;   // rows of the group
  int a_row0; // first A row of the group
  int m, n;   // tile coordinates within the group
  bool small; // pair tile with 128 rows (M = 128): the group's last <= 128 rows
  bool swap;  // operand-swapped pair tile: weights are the M = 256 operand, the
              // group's last r < 256 rows the N = nt operand (nt = r rounded up to 16)
  int nt;
};

// tile_start lives in shared memory (copied once per CTA), so the search costs
// a few shared-memory reads instead of a chain of dependent global loads at
// every tile boundary.
template <int CG>
__device__ __forceinline__ void decode_tile(const GemmArgs& a, const int* tile_start, int t, Tile& ti) {
  int local = t;
  if (a.tile_start == nullptr && a.shared_only_tiles > 0) {
    // The shared groups alone (each T rows, the same tiles per group).
    ti.kind = 1; ti.idx = t / a.shared_only_tiles; ti.rows = a.T; ti.a_row0 = ti.idx * a.shared_a_stride;
    local = t - ti.idx * a.shared_only_tiles;
  } else if (a.tile_start == nullptr) {
    // One dense group of T rows (router, latent projections) of kind dense_kind.
    ti.kind = a.dense_kind; ti.idx = 0; ti.rows = a.T; ti.a_row0 = 0;
  } else {
  // Largest g with tile_start[g] <= t; tile_start[0] = 0 <= t < tile_start[G].
  int lo = 0, hi = a.G;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (tile_start[mid] <= t) lo = mid; else hi = mid;
  }
  local = t - tile_start[lo];
  if (lo < a.E) {
    const int o0 = a.offsets[lo];
    ti.kind = 0; ti.idx = lo; ti.rows = a.offsets[lo + 1] - o0; ti.a_row0 = o0;
  } else {
    ti.kind = 1; ti.idx = lo - a.E; ti.rows = a.T; ti.a_row0 = ti.idx * a.shared_a_stride;
  }
  }
  // Tiles of a group are numbered M-major: (m, n) = (local / nt, local % nt).
  // Pairs take tiles t, t + n_clusters, ...; numbered N-major instead, a group
  // with two M-tiles would put its full tiles on even and its small last tiles
  // on odd tile indices, so with an even number of pairs every full tile
  // would land on the even pairs.  M-major keeps the tiles that share A rows
  // (one M-tile, all N-tiles) and the tiles that share weights (one N-tile,
  // the group's M-tiles) within a few tiles of each other, so both still
  // meet in L2.  (Measured on the V3-shaped layer: N-major with an odd pair
  // count read 10 % more DRAM in gate/up.)
  const int nt = a.n_kind[ti.kind] / a.BN;
  ti.m = local / nt;
  ti.n = local - ti.m * nt;
  // FP4: tiles of kF4TileTokens token rows, every one swapped.
  const int tm = a.fp4 ? kF4TileTokens : Cfg<CG>::kTileM;
  const int r = ti.rows - ti.m * tm;
  ti.swap = CG == 2 && (a.fp4 || (a.swap_ok && r < 256));
  ti.nt = ti.swap ? (min(r, tm) + 15) & ~15 : 0;
  ti.small = CG == 2 && !ti.swap && r <= 128;
}

// SiLU(min(g, c_g)) * clamp(u, -c_u, c_u) in fp32 with the fast exponential
// and division (deterministic; about 2 ulp, far below the bf16 rounding of h).
__device__ __forceinline__ float silu_clamped_product(float g, float u, float cg, float cu) {
  g = fminf(g, cg);
  u = fminf(fmaxf(u, -cu), cu);
  return __fdividef(g, 1.0f + __expf(-g)) * u;
}

// SiTU-GLU: [bg tanh(g / bg) * sigmoid(g)] * [bu tanh(u / bu)] (the linux.do
// post on MoE variants, "SiTU-GLU": soft caps on both branches), written with
// tanh(z) = sign(z) (1 - e^{-2|z|}) / (1 + e^{-2|z|}) and sigmoid(g) =
// 1 / (1 + e^{-g}) over one common denominator:
//   h = sign(g u) bg bu (1 - e1)(1 - e3) / ((1 + e1)(1 + e2)(1 + e3)),
//   e1 = e^{-2|g|/bg}, e2 = e^{-g}, e3 = e^{-2|u|/bu}
// (three exponentials, one division).  A very negative g makes e2 infinite
// and h 0, as the closed gate should.  Every step is an explicitly rounded
// fp32 operation or an intrinsic, which the compiler may not fuse or reorder,
// so the result is the same bits wherever the function is inlined; the error
// is a few ulp of fp32, far below the bf16 rounding of h.  ibg = 1 / bg,
// ibu = 1 / bu are rounded once on the host.
__device__ __forceinline__ float situ_glu_product(float g, float u, float bg, float bu, float ibg,
                                                  float ibu) {
  const float e1 = __expf(__fmul_rn(__fmul_rn(-2.0f, fabsf(g)), ibg));
  const float e2 = __expf(-g);
  const float e3 = __expf(__fmul_rn(__fmul_rn(-2.0f, fabsf(u)), ibu));
  const float num = __fmul_rn(__fsub_rn(1.0f, e1), __fsub_rn(1.0f, e3));
  const float den = __fmul_rn(__fmul_rn(__fadd_rn(1.0f, e1), __fadd_rn(1.0f, e2)), __fadd_rn(1.0f, e3));
  const float mag = __fmul_rn(__fmul_rn(bg, bu), __fdividef(num, den));
  return (g < 0.f) != (u < 0.f) ? -mag : mag;
}

// The experts' gated unit (the same function in every tile shape).
template <int ACT>
__device__ __forceinline__ float glu_unit(float g, float u, const GemmArgs& a) {
  if (ACT == MOE_ACT_SITU_GLU) return situ_glu_product(g, u, a.beta_g, a.beta_u, a.inv_beta_g, a.inv_beta_u);
  return silu_clamped_product(g, u, a.gate_clamp, a.up_clamp);
}

// TMEM columns (FP4): the accumulators take [0, 240) and [256, 496); two
// rotating scale buffers of the weights (4 columns each) follow, then the
// tokens' constant scales (8 columns: N > 128 reads a second atom).
constexpr uint32_t kSfCol = 496;
constexpr uint32_t kSfOneCol = 504;
constexpr int kSfAtomBytes = 512;

template <int MODE, int CG, int ACT, int F8, int F4 = 0>
__global__ void __launch_bounds__(kGemmThreads, 1)
    k_grouped_gemm(const __grid_constant__ GemmArgs a) {
  using C = Cfg<CG>;
  static_assert(!F4 || (F8 && MODE != kRouter && CG == 2), "FP4 weights: the expert GEMMs' E4M3 pair kernels");
  // K elements per 128-byte operand row of a stage: 64 bf16 or 128 E4M3.  Every
  // byte count below (stage slots, TMA boxes, descriptor steps) is the same for
  // both; an E4M3 MMA walks 32 elements where a bf16 one walks 16.
  constexpr int KE = F8 ? 2 * kBK : kBK;
  // Stage ring.  The expert GEMMs use as many stages of kSmemA + C::kSmemB bytes
  // as fit (6); the router, whose B tile is only E_pad rows, packs as many
  // stages of kSmemA + E_pad * 128 bytes as fit (up to 8), so one CTA walking
  // the whole K keeps more loads in flight.
  // Batches of at most 256 tokens make every expert tile a swapped tile whose
  // token operand is at most a_stage_bytes / 128 rows per CTA: the A slot of a
  // stage then shrinks to that and the ring holds more stages (more weight
  // bytes in flight per SM).  No stage layout changes a result.
  const int sa_bytes = (MODE != kRouter && a.a_stage_bytes > 0) ? a.a_stage_bytes : kSmemA;
  const int sb_bytes = MODE == kRouter ? a.BN * kBK * 2 : C::kSmemB;
  // FP4: each stage also carries its scale atom, and the ring ends with the
  // tokens' constant atom.
  const int sf_bytes = F4 ? kSfAtomBytes : 0;
  const int S = MODE == kRouter ? min(8, kRingBytes / (kSmemA + sb_bytes))
                                : min(kRingMax, (kRingBytes - sf_bytes) / (sa_bytes + sb_bytes + sf_bytes));
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;                              // S x sa_bytes
  uint8_t* sB = smem + S * sa_bytes;               // S x sb_bytes
  uint8_t* sSF = sB + S * sb_bytes;                // FP4: S x 512-byte scale atoms
  uint32_t* s_sf_one = reinterpret_cast<uint32_t*>(sSF + S * sf_bytes);  // FP4: atom of ones (UE8M0 127)
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kRingBytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + kRingMax;
  uint64_t* tfull = bars + 2 * kRingMax;
  uint64_t* tempty = tfull + 2;
  uint64_t* tdone = tempty + 2;
  // Swapped gate/up tiles: per warp pair, up values staged for the gate warp
  // (xfull / xempty) and gate values staged for the up warp (gfull / gempty).
  uint64_t* xfull = tdone + 1;   // [4]
  uint64_t* xempty = xfull + 4;  // [4]
  uint64_t* gfull = xempty + 4;  // [4]
  uint64_t* gempty = gfull + 4;  // [4]

  uint8_t* epi = reinterpret_cast<uint8_t*>(bars) + kBarBytes;  // kEpiWarps x kEpiBytes
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  __shared__ int s_tile_start[kMaxGroups + 1];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = CG == 2 ? cluster_ctarank() : 0;   // 0 = the MMA-issuing CTA
  const bool leader = rank == 0;
  if (F4) {
    for (int i = threadIdx.x; i < 128; i += blockDim.x) s_sf_one[i] = 0x7F7F7F7Fu;
    fence_proxy_async_smem();   // read by tcgen05.cp (async proxy) after the cluster barrier below
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) { mbar_init(&tfull[b], 1); mbar_init(&tempty[b], CG * kEpiWarps); }
    mbar_init(tdone, 1);
    for (int p = 0; p < 4; ++p) {
      mbar_init(&xfull[p], 1); mbar_init(&xempty[p], 1);
      mbar_init(&gfull[p], 1); mbar_init(&gempty[p], 1);
    }
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    if (CG == 2) tmem_alloc_pair(&tmem_slot, kTmemCols);
    else tmem_alloc(&tmem_slot, kTmemCols);
  }
  tc_fence_before();
  if (CG == 2) cluster_sync(); else __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_slot;
  volatile int* abort = &abort_flag;
  // The prologue above touches no global memory; wait for the previous kernel
  // of the stream before reading the tile list or any operand.
  griddep_wait();
  griddep_launch();
  if (a.tile_start != nullptr)
    for (int i = threadIdx.x; i <= a.G; i += blockDim.x) s_tile_start[i] = a.tile_start[i];
  __syncthreads();

  const int cluster_id = blockIdx.x / CG, n_clusters = gridDim.x / CG;
  const int total = (a.tile_start == nullptr) ? a.router_tiles : s_tile_start[a.G];
  const int BN = a.BN;                                    // output columns per tile (per matrix)
  const int n_mma = MODE == kGateUp ? 2 * BN : BN;        // N of one MMA
  // B rows each CTA loads per stage, per matrix (gate and up each for gate/up).
  const uint32_t b_rows = static_cast<uint32_t>(BN / CG);
  const uint32_t stage_bytes = kSmemA + b_rows * kBK * 2 * (MODE == kGateUp ? 2 : 1);
  const uint32_t acc_stride = static_cast<uint32_t>(n_mma);  // TMEM columns per buffer
  // Barriers the pair shares live in the even CTA.
  const uint32_t full0 = CG == 2 ? mapa_shared(full, 0) : 0;
  const uint32_t tempty0 = CG == 2 ? mapa_shared(tempty, 0) : 0;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int issued[kRingMax];
      for (int s = 0; s < S; ++s) issued[s] = -1;
      bool ok = true;
      for (int t = cluster_id; ok && t < total; t += n_clusters) {
        Tile ti;
        decode_tile<CG>(a, s_tile_start, t, ti);
        const int nkb = a.k_kind[ti.kind] / KE;
        // A: this CTA's rows of the tile (128, or 64 in a 128-row pair tile,
        // loaded with the 64-row box so no unused rows cross into shared memory).
        // Swapped tile: this CTA's nt / 2 token rows (the B operand's half).
        const int a_rows = ti.swap ? ti.nt / 2 : (ti.small ? 64 : 128);
        const int a_y = ti.a_row0 + ti.m * (F4 ? kF4TileTokens : C::kTileM) + static_cast<int>(rank) * a_rows;
        // Rows of A the MMA uses: a_rows (pairs), or the router tile's valid rows.
        const int need = CG == 2 ? a_rows : min(128, ti.rows - ti.m * 128);
        const int box = need <= 16 ? 16 : (need <= 32 ? 32 : (need <= 64 ? 64 : 128));
        const CUtensorMap* amap = box == 16   ? &a.mapA16[ti.kind]
                                  : box == 32 ? &a.mapA32[ti.kind]
                                  : box == 64 ? &a.mapA64[ti.kind]
                                              : &a.mapA[ti.kind];
        const uint32_t tx = stage_bytes - kSmemA + static_cast<uint32_t>(box) * kBK * 2;
        int b_y = ti.idx * a.n_kind[ti.kind] + ti.n * BN;
        const CUtensorMap* bmap = &a.mapB[ti.kind * 2];
        // Pair B halves: gate/up - the CTA of rank r loads gate rows and up rows
        // [r*BN/2, (r+1)*BN/2) of the tile (interleaved [gate | up] per half, so
        // each accumulator lane holds matching gate and up columns); down - rows
        // [r*BN/2, (r+1)*BN/2) of the tile's output columns.
        if (CG == 2) b_y += static_cast<int>(rank) * (BN / 2);
        // The host sizes the A slot for the largest token box a tile can need;
        // a box that would overrun it is reported and nothing is loaded.
        if (MODE != kRouter && box * kBK * 2 > sa_bytes) {
          atomicExch(a.err, kDevBadIndex);
          *abort = 1;
          ok = false;
          break;
        }
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort, a.err, a.timeout_ns)) { ok = false; break; }
          uint8_t* b0 = sB + stage * sb_bytes;
          if (F4) {
            // This CTA's token rows, its 128 weight rows as E2M1 codes (gate/up:
            // the 64 gate rows, then the 64 up rows; down: 128 rows) and their
            // scale atom (half h = b_y / (BN / 2) of the kind, stage kb), all
            // counted on the even CTA's full.  A 4-bit load counts the bytes it
            // reads (64 a row), not the 128 it fills in shared memory.
            const uint32_t txf = static_cast<uint32_t>(box) * kBK * 2 + 128 * 64 + kSfAtomBytes;
            if (leader) mbar_arrive_expect_tx(&full[stage], 2 * txf);
            const uint32_t fb = full0 + 8 * stage;
            tma_load_2d_pair(sA + stage * sa_bytes, amap, kb * KE, a_y, fb);
            tma_load_2d_pair(b0, &a.mapBp[ti.kind * 2], kb * KE, b_y, fb);
            if (MODE == kGateUp) tma_load_2d_pair(b0 + 64 * 128, &a.mapBp[ti.kind * 2 + 1], kb * KE, b_y, fb);
            tma_load_2d_pair(sSF + stage * kSfAtomBytes, &a.mapSF[ti.kind], 0, (b_y / (BN / 2)) * nkb + kb, fb);
          } else if (CG == 1) {
            mbar_arrive_expect_tx(&full[stage], tx);
            tma_load_2d(sA + stage * sa_bytes, amap, kb * KE, a_y, &full[stage]);
            tma_load_2d(b0, bmap, kb * KE, b_y, &full[stage]);
            if (MODE == kGateUp)
              tma_load_2d(b0 + b_rows * kBK * 2, bmap + 1, kb * KE, b_y, &full[stage]);
          } else {
            // The even CTA expects the bytes of both CTAs on its barrier.
            if (leader) mbar_arrive_expect_tx(&full[stage], 2 * tx);
            tma_load_2d_pair(sA + stage * sa_bytes, amap, kb * KE, a_y, full0 + 8 * stage);
            tma_load_2d_pair(b0, bmap, kb * KE, b_y, full0 + 8 * stage);
            if (MODE == kGateUp)
              tma_load_2d_pair(b0 + (BN / 2) * kBK * 2, bmap + 1, kb * KE, b_y, full0 + 8 * stage);
          }
          issued[stage] = static_cast<int>(phase);
          if (++stage == S) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok && (CG == 1 || leader)) {
        // Let the copies already in flight land before the CTA goes away
        // (bounded like every other wait).
        for (int s = 0; s < S; ++s)
          if (issued[s] >= 0) mbar_wait_drain(&full[s], static_cast<uint32_t>(issued[s]), kDrainNs);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer
    if (lane == 0 && leader) {
      // Gate/up: the gate tile and the up tile sit back to back in shared
      // memory (CG = 1) or in the two CTAs of the pair (CG = 2), so one
      // N = 2*BN MMA reads A once and writes the gate accumulator to columns
      // [0, BN) and the up accumulator to [BN, 2*BN).
      auto idesc_of = [](int M, int N) { return F8 ? idesc_e4m3_f32(M, N) : idesc_bf16_f32(M, N); };
      const uint32_t idesc_full = idesc_of(C::kTileM, n_mma);
      const uint32_t idesc_small = idesc_of(128, n_mma);  // pair tile of 128 rows
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      // FP4: the tokens' scales (all 1, two atoms for up to 256 tokens) once, and
      // two rotating TMEM column groups for the weights' per-stage atoms
      // (tcgen05 operations of this thread run in issue order, so a copy never
      // overtakes an earlier MMA).
      uint32_t sf_buf = 0;
      if (F4) {
        tmem_cp_sf_pair(tmem_base + kSfOneCol, sf_atom_desc(smem_u32(s_sf_one)));
        tmem_cp_sf_pair(tmem_base + kSfOneCol + 4, sf_atom_desc(smem_u32(s_sf_one)));
      }
      for (int t = cluster_id; ok && t < total; t += n_clusters) {
        Tile ti;
        decode_tile<CG>(a, s_tile_start, t, ti);
        const int nkb = a.k_kind[ti.kind] / KE;
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, abort, a.err, a.timeout_ns)) break;
        tc_fence_after();
        const uint32_t d0 = tmem_base + static_cast<uint32_t>(acc) * acc_stride;
        // Swapped tiles are one M = 256 pair MMA per step: 128 weight rows per CTA
        // (gate/up: the 64 gate rows then the 64 up rows of its output columns).
        const uint32_t idesc = ti.swap ? idesc_of(256, ti.nt) : (ti.small ? idesc_small : idesc_full);
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort, a.err, a.timeout_ns)) { ok = false; break; }
          tc_fence_after();
          // A swapped tile reads the weight rows as its A operand and the token
          // rows as its B operand (the same K order, so the same bits per element).
          const uint32_t tok_addr = smem_u32(sA + stage * sa_bytes);
          const uint32_t w_addr = smem_u32(sB + stage * sb_bytes);
          const uint32_t a_addr = ti.swap ? w_addr : tok_addr;
          const uint32_t b_addr = ti.swap ? tok_addr : w_addr;
          if (F4) {
            // Block-scaled: K block kk of the stage takes byte kk of the scale words.
            const uint32_t sfa = tmem_base + kSfCol + 4 * sf_buf;
            tmem_cp_sf_pair(sfa, sf_atom_desc(smem_u32(sSF + stage * kSfAtomBytes)));
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk)
              umma_bs_pair(d0, sw128_kmajor_desc(a_addr + kk * 32), sw128_kmajor_desc(b_addr + kk * 32),
                           idesc_e2m1_e4m3_bs(256, ti.nt, kk), sfa, tmem_base + kSfOneCol,
                           (kb | kk) != 0 ? 1u : 0u);
            sf_buf ^= 1u;
          }
#pragma unroll
          for (int kk = 0; kk < (F4 ? 0 : kBK / 16); ++kk) {
            const uint64_t ad = sw128_kmajor_desc(a_addr + kk * 32);
            const uint64_t bd = sw128_kmajor_desc(b_addr + kk * 32);
            const uint32_t accum = (kb | kk) != 0 ? 1u : 0u;
            if (F8) {
              if (CG == 2) umma_e4m3_pair(d0, ad, bd, idesc, accum);
              else umma_e4m3(d0, ad, bd, idesc, accum);
            } else {
              if (CG == 2) umma_bf16_pair(d0, ad, bd, idesc, accum);
              else umma_bf16(d0, ad, bd, idesc, accum);
            }
          }
          if (CG == 2) umma_commit_pair_mc(&empty[stage], 0x3);
          else umma_commit(&empty[stage]);
          if (++stage == S) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        if (CG == 2) umma_commit_pair_mc(&tfull[acc], 0x3);
        else umma_commit(&tfull[acc]);
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      // Every MMA issued above has finished before TMEM is released.
      if (CG == 2) umma_commit_pair_mc(tdone, 0x1);
      else umma_commit(tdone);
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
    uint32_t xph = 0;  // phase of this warp's exchange channel (swapped gate/up tiles)
    for (int t = cluster_id; t < total; t += n_clusters) {
      Tile ti;
      decode_tile<CG>(a, s_tile_start, t, ti);
      bool ok = mbar_wait(&tfull[acc], acc_phase, abort, a.err, a.timeout_ns);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                          static_cast<uint32_t>(acc) * acc_stride;
      // Index check (MOE_CHECK_BOUNDS builds): the group's rows lie in its A tensor.
      const bool tile_ok = a.a_rows[ti.kind] == 0 ||
                           MOE_INDEX_OK(ti.rows >= 0 && ti.a_row0 >= 0 && ti.a_row0 + ti.rows <= a.a_rows[ti.kind],
                                        a.err);
      if (!tile_ok) {
        // out-of-range group: nothing is stored
      } else if (CG == 2 && ti.swap) {
        // Operand-swapped tile: TMEM lanes are output columns, TMEM columns are
        // the tile's tokens (rows m * 256 + j of the group, j < r valid).
        const int tm = F4 ? kF4TileTokens : C::kTileM;
        const int r = min(tm, ti.rows - ti.m * tm);
        const int trow0 = ti.m * tm;
        if (MODE == kGateUp) {
          // Lanes 0-63 hold the gate rows and lanes 64-127 the up rows of the CTA's
          // 64 output columns; TMEM columns are tokens.  A gate warp (lane quarter
          // 0 or 1) and the up warp of the same columns (quarter 2 or 3) split
          // each 32-token block: the gate warp computes tokens 0-15 and the up
          // warp tokens 16-31, each receiving the other branch's values for its
          // half through shared memory (word j of lane l at j * 32 + l: lane l
          // of both warps is the same column, so both sides are conflict-free),
          // every hand-over under bounded mbarrier waits.  Both warps' SMSPs do
          // half of the unit's arithmetic.
          const bool gate_warp = q < 2;
          const int pch = (q & 1) + 2 * half;  // exchange channel of this warp pair
          uint32_t* sendb = reinterpret_cast<uint32_t*>(stage_w);   // this warp's buffer
          uint32_t* recvb = reinterpret_cast<uint32_t*>(gate_warp ? stage_w - 2 * kEpiBytes
                                                                  : stage_w + 2 * kEpiBytes);
          uint64_t* my_full = gate_warp ? &gfull[pch] : &xfull[pch];
          uint64_t* my_empty = gate_warp ? &gempty[pch] : &xempty[pch];
          uint64_t* their_full = gate_warp ? &xfull[pch] : &gfull[pch];
          uint64_t* their_empty = gate_warp ? &xempty[pch] : &gempty[pch];
          const int base = gate_warp ? 0 : 16;  // first token of this warp's half
          const int col = ti.n * BN + static_cast<int>(rank) * (BN / 2) + 32 * (q & 1) + lane;
          uint16_t* outb = static_cast<uint16_t*>(a.out[ti.kind]);
          const size_t ld = static_cast<size_t>(a.ld_out[ti.kind]);
          const int orow0 = (ti.kind == 0 ? ti.a_row0 : ti.idx * a.shared_out_stride) + trow0;
          for (int c = 32 * half; c < ti.nt && ok; c += 64) {
            uint32_t v[32];
            tmem_ld32(tb + c, v);
            tmem_ld_wait();
            ok = mbar_wait(my_empty, xph ^ 1u, abort, a.err, a.timeout_ns);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            // Hand over the partner's half: the gate warp sends tokens 16-31,
            // the up warp tokens 0-15.
            if (gate_warp) {
#pragma unroll
              for (int jj = 0; jj < 16; ++jj) sendb[jj * 32 + lane] = v[16 + jj];
            } else {
#pragma unroll
              for (int jj = 0; jj < 16; ++jj) sendb[jj * 32 + lane] = v[jj];
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(my_full);
            ok = mbar_wait(their_full, xph, abort, a.err, a.timeout_ns);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            uint32_t o[16];
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) o[jj] = recvb[jj * 32 + lane];
            __syncwarp();
            if (lane == 0) mbar_arrive(their_empty);
            // fp8: token c + lane's row scale, handed to every lane per token.
            float my_sc = 1.f;
            if (F8 && c + lane < r) my_sc = exp2_int(a.a_exp[ti.kind][ti.a_row0 + trow0 + c + lane]);
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) {
              const int j = base + jj;
              const float sc = F8 ? __shfl_sync(0xffffffffu, my_sc, j) : 1.f;
              // Gate warp: own gate values v[jj], received up values o[jj];
              // up warp: received gate values o[jj], own up values v[16 + jj].
              float gv = __uint_as_float(gate_warp ? v[jj] : o[jj]);
              float uv = __uint_as_float(gate_warp ? o[jj] : v[16 + jj]);
              if (c + j < r) {
                if (F8) { gv = __fmul_rn(gv, sc); uv = __fmul_rn(uv, sc); }
                const float hv = glu_unit<ACT>(gv, uv, a);
                outb[static_cast<size_t>(orow0 + c + j) * ld + col] =
                    static_cast<uint16_t>(pack_bf16x2(hv, 0.f) & 0xFFFFu);
              }
            }
            xph ^= 1u;
          }
          // Each warp's buffer is its own staging area in row tiles: do not
          // leave the tile before the partner has read the last block from it.
          if (ok) {
            ok = mbar_wait(my_empty, xph ^ 1u, abort, a.err, a.timeout_ns);
            ok = __all_sync(0xffffffffu, ok);
          }
        } else {
          // One M = 256 pair MMA: lane i = output column n * BN + 128 * rank + i.
          const bool scatter = (MODE == kDown && ti.kind == 0);
          const int col = ti.n * BN + static_cast<int>(rank) * (BN / 2) + 32 * q + lane;
          float* outb = static_cast<float*>(a.out[ti.kind]);
          uint16_t* outh = static_cast<uint16_t*>(a.out[ti.kind]);  // out_bf16
          const size_t ld = static_cast<size_t>(a.ld_out[ti.kind]);
          const int orow0 = (ti.kind == 0 ? ti.a_row0 : ti.idx * a.shared_out_stride) + trow0;
          for (int c = 32 * half; c < ti.nt; c += 64) {
            uint32_t v[32];
            tmem_ld32(tb + c, v);
            tmem_ld_wait();
            // Lane j resolves the output row of token c + j once (its scattered
            // slot row, in its source rank's buffer under expert parallelism);
            // the stores below take it by shuffle.
            const int my_tok = c + lane;
            int my_row = 0;
            float* my_ptr = outb;
            float my_sc = 1.f;
            if (my_tok < r) {
              my_row = scatter ? a.dest_row[ti.a_row0 + trow0 + my_tok] : orow0 + my_tok;
              if (scatter && a.ep) my_ptr = a.out_rank[my_row >> 24] + static_cast<size_t>(my_row & 0xFFFFFF) * ld;
              else my_ptr = outb + static_cast<size_t>(my_row) * ld;
              if (F8) my_sc = exp2_int(a.a_exp[ti.kind][ti.a_row0 + trow0 + my_tok]);
#ifdef MOE_CHECK_BOUNDS
              const bool in_range = (scatter && a.ep)
                                        ? ((my_row >> 24) < a.ep_world && (my_row & 0xFFFFFF) < a.out_rows[0])
                                        : (my_row >= 0 && my_row < a.out_rows[ti.kind]);
              if (!MOE_INDEX_OK(in_range, a.err)) my_ptr = nullptr;
#endif
            }
            if (a.out_bf16) {
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                const int orow = __shfl_sync(0xffffffffu, my_row, j);
                const float sc = F8 ? __shfl_sync(0xffffffffu, my_sc, j) : 1.f;
                if (c + j < r) {
                  const float val = F8 ? __fmul_rn(__uint_as_float(v[j]), sc) : __uint_as_float(v[j]);
                  outh[static_cast<size_t>(orow) * ld + col] =
                      static_cast<uint16_t>(pack_bf16x2(val, 0.f) & 0xFFFFu);
                }
              }
            } else {
              const unsigned long long my_addr = reinterpret_cast<unsigned long long>(my_ptr);
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                float* rowp = reinterpret_cast<float*>(__shfl_sync(0xffffffffu, my_addr, j));
                const float sc = F8 ? __shfl_sync(0xffffffffu, my_sc, j) : 1.f;
#ifdef MOE_CHECK_BOUNDS
                if (rowp == nullptr) continue;
#endif
                if (c + j < r) rowp[col] = F8 ? __fmul_rn(__uint_as_float(v[j]), sc) : __uint_as_float(v[j]);
              }
            }
          }
        }
      } else {
      // Rows and columns this warp owns.  A 256-row pair tile (and every CG = 1
      // tile) keeps row i of the CTA's 128 in TMEM lane i with all n_mma
      // columns.  A 128-row pair tile keeps the CTA's 64 rows twice: lanes 0-63
      // hold output columns [0, n_mma/2) and lanes 64-127 hold [n_mma/2, n_mma),
      // both in TMEM columns [0, n_mma/2).
      const bool small = ti.small;
      const int row_in_cta = small ? (q & 1) * 32 : q * 32;
      const int colhalf = small ? (q >> 1) : 0;           // which half of the columns (small)
      const int grow0 = ti.m * C::kTileM + static_cast<int>(rank) * (small ? 64 : 128) + row_in_cta;
      const int nvalid = max(0, min(32, ti.rows - grow0));
      // fp8: this thread's row scale (row grow0 + lane of the group's A rows).
      float rsc = 1.f;
      if (F8 && lane < nvalid) rsc = exp2_int(a.a_exp[ti.kind][ti.a_row0 + grow0 + lane]);
      if (MODE == kGateUp) {
        // Output block b covers columns [b*G, b*G + G) with its gate values in
        // TMEM columns [2bG, 2bG + G) and up values in [2bG + G, 2bG + 2G), G = BN/2.
        const int G = BN / 2;
        const int orow0 = (ti.kind == 0 ? ti.a_row0 : ti.idx * a.shared_out_stride) + grow0;
        uint8_t* out0 = reinterpret_cast<uint8_t*>(static_cast<uint16_t*>(a.out[ti.kind]) + ti.n * BN);
        const size_t ld_bytes = static_cast<size_t>(a.ld_out[ti.kind]) * 2;
        const int nchunk = G / 8;                  // 16-byte chunks per staged row (4 or 8)
        const int rows_per_st = 32 / nchunk;
        // 256-row tiles: half h takes block h; 128-row tiles: block colhalf, half 0 only.
        const int blk = small ? colhalf : half;
        if (!small || half == 0) {
          const int tcol = small ? 0 : blk * 2 * G;
          for (int c = 0; c < G; c += 32) {
            uint32_t g[32], u[32];
            tmem_ld32(tb + tcol + c, g);
            tmem_ld32(tb + tcol + G + c, u);
            tmem_ld_wait();
            if (F8) {
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                g[i] = __float_as_uint(__fmul_rn(__uint_as_float(g[i]), rsc));
                u[i] = __float_as_uint(__fmul_rn(__uint_as_float(u[i]), rsc));
              }
            }
            uint32_t p[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              p[i] = pack_bf16x2(glu_unit<ACT>(__uint_as_float(g[2 * i]), __uint_as_float(u[2 * i]), a),
                                 glu_unit<ACT>(__uint_as_float(g[2 * i + 1]), __uint_as_float(u[2 * i + 1]), a));
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int m = c / 8 + i;
              *reinterpret_cast<uint4*>(stage_w + lane * 128 + ((m ^ (lane & 7)) << 4)) =
                  make_uint4(p[4 * i], p[4 * i + 1], p[4 * i + 2], p[4 * i + 3]);
            }
          }
          __syncwarp();
          for (int s8 = 0; s8 < nchunk; ++s8) {
            const int r = s8 * rows_per_st + lane / nchunk, cc = lane % nchunk;
            if (r < nvalid) {
              const uint4 v = *reinterpret_cast<const uint4*>(stage_w + r * 128 + ((cc ^ (r & 7)) << 4));
              *reinterpret_cast<uint4*>(out0 + static_cast<size_t>(orow0 + r) * ld_bytes + blk * G * 2 + 16 * cc) = v;
            }
          }
          __syncwarp();
        }
      } else {
        // fp32 output, 32 columns (128 bytes) per block.
        const bool scatter = (MODE == kDown && ti.kind == 0);
        const int my_dest = (scatter && lane < nvalid) ? a.dest_row[ti.a_row0 + grow0 + lane] : 0;
        const int orow0 = (ti.kind == 0 ? ti.a_row0 : ti.idx * a.shared_out_stride) + grow0;
        float* out0 = static_cast<float*>(a.out[ti.kind]) + ti.n * BN + colhalf * (BN / 2);
        const size_t ld = static_cast<size_t>(a.ld_out[ti.kind]);
        const int ncols = small ? BN / 2 : BN;
        for (int c = 32 * half; c < ncols; c += 64) {
          uint32_t v[32];
          tmem_ld32(tb + c, v);
          tmem_ld_wait();
          if (F8) {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__fmul_rn(__uint_as_float(v[i]), rsc));
          }
          if (ncols - c >= 32 && a.out_bf16) {
            // bf16 output (latent down-projection): 64 bytes per row, four
            // 16-byte chunks, staged so each store covers whole row segments.
            uint16_t* oh = static_cast<uint16_t*>(a.out[ti.kind]) + ti.n * BN + colhalf * (BN / 2);
#pragma unroll
            for (int m = 0; m < 4; ++m)
              *reinterpret_cast<uint4*>(stage_w + lane * 128 + ((m ^ (lane & 7)) << 4)) =
                  make_uint4(pack_bf16x2(__uint_as_float(v[8 * m]), __uint_as_float(v[8 * m + 1])),
                             pack_bf16x2(__uint_as_float(v[8 * m + 2]), __uint_as_float(v[8 * m + 3])),
                             pack_bf16x2(__uint_as_float(v[8 * m + 4]), __uint_as_float(v[8 * m + 5])),
                             pack_bf16x2(__uint_as_float(v[8 * m + 6]), __uint_as_float(v[8 * m + 7])));
            __syncwarp();
#pragma unroll
            for (int s4 = 0; s4 < 4; ++s4) {
              const int r = 8 * s4 + (lane >> 2), ch = lane & 3;
              const int drow = __shfl_sync(0xffffffffu, my_dest, r);
              if (r < nvalid) {
                const uint4 val = *reinterpret_cast<const uint4*>(stage_w + r * 128 + ((ch ^ (r & 7)) << 4));
                const size_t orow = scatter ? static_cast<size_t>(drow) : static_cast<size_t>(orow0 + r);
                *reinterpret_cast<uint4*>(oh + orow * ld + c + 8 * ch) = val;
              }
            }
            __syncwarp();
          } else if (ncols - c >= 32) {
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
                float* ob = out0;
                size_t orow = scatter ? static_cast<size_t>(drow) : static_cast<size_t>(orow0 + r);
                if (scatter && a.ep) {
                  // Expert parallelism: the row lives in its source rank's buffer.
                  ob = a.out_rank[drow >> 24] + ti.n * BN + colhalf * (BN / 2);
                  orow = static_cast<size_t>(drow & 0xFFFFFF);
                }
#ifdef MOE_CHECK_BOUNDS
                {
                  const bool in_range = (scatter && a.ep)
                                            ? ((drow >> 24) < a.ep_world && orow < static_cast<size_t>(a.out_rows[0]))
                                            : (orow < static_cast<size_t>(a.out_rows[ti.kind]));
                  if (a.out_rows[ti.kind] != 0 && !MOE_INDEX_OK(in_range, a.err)) continue;
                }
#endif
                *reinterpret_cast<uint4*>(ob + orow * ld + c + 4 * sc) = val;
              }
            }
            __syncwarp();
          } else if (lane < nvalid) {
            // Narrow tail (router with fewer than 32 columns left): direct stores.
            float* ob = out0;
            size_t orow = scatter ? static_cast<size_t>(my_dest) : static_cast<size_t>(orow0 + lane);
            if (scatter && a.ep) {
              ob = a.out_rank[my_dest >> 24] + ti.n * BN + colhalf * (BN / 2);
              orow = static_cast<size_t>(my_dest & 0xFFFFFF);
            }
            float4* dst = reinterpret_cast<float4*>(ob + orow * ld + c);
            const int nq = (ncols - c) / 4;
#pragma unroll
            for (int i = 0; i < 8; ++i)
              if (i < nq)
                dst[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                     __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
          }
        }
      }
      }  // not swapped
      if (!ok) break;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (CG == 2) mbar_arrive_cluster(tempty0 + 8 * acc);   // the even CTA's barrier
        else mbar_arrive(&tempty[acc]);
      }
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
  }

  // Neither CTA of a pair leaves while the other may still signal it.
  tc_fence_before();
  if (CG == 2) cluster_sync(); else __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    if (CG == 2) tmem_dealloc_pair(tmem_base, kTmemCols);
    else tmem_dealloc(tmem_base, kTmemCols);
  }
}

cudaLaunchConfig_t pair_config(int grid, cudaStream_t s, cudaLaunchAttribute* attr) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(kGemmThreads, 1, 1);
  cfg.dynamicSmemBytes = kGemmSmem;
  cfg.stream = s;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cfg;
}

template <int MODE, int CG, int ACT = MOE_ACT_SWIGLU, int F8 = 0, int F4 = 0>
cudaError_t launch_one(const GemmArgs& a, int grid, cudaStream_t s) {
  return launch_k(k_grouped_gemm<MODE, CG, ACT, F8, F4>, dim3(grid), dim3(kGemmThreads),
                  kGemmSmem, s, CG == 2, a);
}

int g_pair_clusters[64] = {0};

}  // namespace

void gemm_prepare() {
  static int done_dev = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (done_dev == dev) return;
  const cudaFuncAttribute smem_attr = cudaFuncAttributeMaxDynamicSharedMemorySize;
  cudaFuncSetAttribute(k_grouped_gemm<kGateUp, 2, MOE_ACT_SWIGLU, 0>, smem_attr, kGemmSmem);
  cudaFuncSetAttribute(k_grouped_gemm<kGateUp, 2, MOE_ACT_SITU_GLU, 0>, smem_attr, kGemmSmem);
  cudaFuncSetAttribute(k_grouped_gemm<kGateUp, 2, MOE_ACT_SWIGLU, 1>, smem_attr, kGemmSmem);
  cudaFuncSetAttribute(k_grouped_gemm<kGateUp, 2, MOE_ACT_SITU_GLU, 1>, smem_attr, kGemmSmem);
  cudaFuncSetAttribute(k_grouped_gemm<kDown, 2, 0, 0>, smem_attr, kGemmSmem);
  cudaFuncSetAttribute(k_grouped_gemm<kDown, 2, 0, 1>, smem_attr, kGemmSmem);
  cudaFuncSetAttribute(k_grouped_gemm<kRouter, 1, 0, 0>, smem_attr, kGemmSmem);
  cudaFuncSetAttribute(k_grouped_gemm<kGateUp, 2, MOE_ACT_SWIGLU, 1, 1>, smem_attr, kGemmSmem);
  cudaFuncSetAttribute(k_grouped_gemm<kGateUp, 2, MOE_ACT_SITU_GLU, 1, 1>, smem_attr, kGemmSmem);
  cudaFuncSetAttribute(k_grouped_gemm<kDown, 2, 0, 1, 1>, smem_attr, kGemmSmem);
  // How many CTA pairs fit on the device at once: the persistent pair grid is
  // never larger, so no pair waits for another to finish before it starts.
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = pair_config(2, nullptr, attr);
  int n = 1 << 30;
  auto occ = [&](const void* fn) {
    int c = 0;
    if (cudaOccupancyMaxActiveClusters(&c, fn, &cfg) != cudaSuccess) c = 0;
    n = std::min(n, c);
  };
  occ(reinterpret_cast<const void*>(k_grouped_gemm<kGateUp, 2, 0, 0>));
  occ(reinterpret_cast<const void*>(k_grouped_gemm<kGateUp, 2, 1, 0>));
  occ(reinterpret_cast<const void*>(k_grouped_gemm<kGateUp, 2, 0, 1>));
  occ(reinterpret_cast<const void*>(k_grouped_gemm<kGateUp, 2, 1, 1>));
  occ(reinterpret_cast<const void*>(k_grouped_gemm<kDown, 2, 0, 0>));
  occ(reinterpret_cast<const void*>(k_grouped_gemm<kDown, 2, 0, 1>));
  occ(reinterpret_cast<const void*>(k_grouped_gemm<kGateUp, 2, 0, 1, 1>));
  occ(reinterpret_cast<const void*>(k_grouped_gemm<kGateUp, 2, 1, 1, 1>));
  occ(reinterpret_cast<const void*>(k_grouped_gemm<kDown, 2, 0, 1, 1>));
  cudaGetLastError();
  if (dev >= 0 && dev < 64) g_pair_clusters[dev] = n;
  done_dev = dev;
}

int gemm_max_pairs() {
  int dev = 0;
  cudaGetDevice(&dev);
  return (dev >= 0 && dev < 64) ? g_pair_clusters[dev] : 0;
}

cudaError_t launch_grouped_gemm(int mode, const GemmArgs& a, int grid, cudaStream_t s) {
  if (grid <= 0) return cudaSuccess;
  const bool f8 = a.fp8 != 0;
  if (a.fp4 != 0) {
    switch (mode) {
      case kGateUp:
        return a.act == MOE_ACT_SITU_GLU ? launch_one<kGateUp, 2, MOE_ACT_SITU_GLU, 1, 1>(a, grid, s)
                                         : launch_one<kGateUp, 2, MOE_ACT_SWIGLU, 1, 1>(a, grid, s);
      case kDown: return launch_one<kDown, 2, 0, 1, 1>(a, grid, s);
      default: return cudaErrorInvalidValue;   // the router GEMM stays bf16
    }
  }
  switch (mode) {
    case kGateUp:
      if (a.act == MOE_ACT_SITU_GLU)
        return f8 ? launch_one<kGateUp, 2, MOE_ACT_SITU_GLU, 1>(a, grid, s)
                  : launch_one<kGateUp, 2, MOE_ACT_SITU_GLU, 0>(a, grid, s);
      return f8 ? launch_one<kGateUp, 2, MOE_ACT_SWIGLU, 1>(a, grid, s)
                : launch_one<kGateUp, 2, MOE_ACT_SWIGLU, 0>(a, grid, s);
    case kDown: return f8 ? launch_one<kDown, 2, 0, 1>(a, grid, s) : launch_one<kDown, 2, 0, 0>(a, grid, s);
    default: return launch_one<kRouter, 1>(a, grid, s);
  }
}

}  // namespace moe
