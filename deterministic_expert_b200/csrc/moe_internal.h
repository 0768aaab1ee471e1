// Internal declarations shared by the library's translation units.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/moe.h"

namespace moe {

// Launch `kernel` on `s` with programmatic stream serialisation (and a cluster
// of 2 CTAs when pair is true).  See griddep_wait() in common.cuh.
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                     bool pair, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  int n = 1;
  if (pair) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 2;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    n = 2;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// ------------------------------------------------------------ grouped GEMM
// One persistent, warp-specialised tcgen05 GEMM serves the router (one group
// of T rows), gate/up + SwiGLU (E routed groups + S shared groups) and down
// (same groups).  Tiles are BM = 128 rows x BN columns with the whole K
// reduced in one TMEM accumulator (no split-K), K walked in 64-wide steps in
// the same order for every tile.
constexpr int kBM = 128;        // rows per CTA of a tile
constexpr int kPairTileM = 256; // rows per tile of the expert GEMMs (a CTA pair)
constexpr int kBK = 64;
constexpr int kStages = 4;
constexpr int kEpiWarps = 8;       // two per TMEM lane quarter, splitting the columns
constexpr int kGemmThreads = 64 + 32 * kEpiWarps;  // warp 0: TMA, warp 1: MMA, warps 2-9: epilogue
// FP4 expert weights: every tile is operand-swapped with at most this many
// token rows (the weights are the M = 256 operand, the tokens N <= 240), so
// the two accumulators (columns [0, 240) and [256, 496)) leave 16 TMEM columns
// for the block scales.
constexpr int kF4TileTokens = 240;
constexpr int kSmemA = kBM * kBK * 2;
constexpr int kSmemBMax = 256 * kBK * 2;
constexpr int kEpiBytes = 32 * 128;  // per epilogue warp: 32 rows x 128 B, XOR-swizzled
constexpr int kGemmBarBytes = 512;  // the GEMM's mbarriers, after its stage ring
constexpr int kGemmSmem = 1024 + kStages * (kSmemA + kSmemBMax) + kGemmBarBytes + kEpiWarps * kEpiBytes;

enum GemmMode : int { kGateUp = 0, kDown = 1, kRouter = 2 };

struct GemmArgs {
  CUtensorMap mapA[2];    // A operand per group kind: 0 routed, 1 shared
  CUtensorMap mapA64[2];  // the same A operands with a 64-row box (128-row pair tiles)
  CUtensorMap mapA16[2];  // ... and a 16-row box (swapped tiles of up to 32 tokens)
  CUtensorMap mapA32[2];  // ... and a 32-row box (swapped tiles of up to 64 tokens)
  CUtensorMap mapB[4];    // B operands: [kind * 2 + 0] first (gate / down / router),
                          //             [kind * 2 + 1] second (up; gate/up only)
  CUtensorMap mapBp[4];   // fp4: the same weight operands as packed E2M1 codes, loaded as
                          //      16U4_ALIGN16B (16 codes per 16-byte chunk) with 128-byte
                          //      swizzling: 128 codes x 64 rows (gate/up) or 128 rows (down)
  CUtensorMap mapSF[2];   // fp4, per kind: the weights' block scales as UE8M0 scale atoms
                          //      (512 bytes each: a CTA's 128 weight rows x one 128-wide
                          //      K stage), atom (h, kc) at row h * K/128 + kc, one per box
  const int* offsets;     // [E + 1] grouped-row offsets of the routed groups
  const int* tile_start;  // [G + 1] first tile of each group; NULL: one group of T rows
  int G, E, T;
  int n_kind[2];          // B rows per expert (N extent) per kind
  int k_kind[2];          // K extent per kind
  int BN;
  int a_stage_bytes;      // expert GEMMs: A bytes per stage (0 = 16 KB); set when every tile is
                          // swapped with at most a_stage_bytes / 128 token rows per CTA
  int swap_ok;            // expert GEMMs: a group's last partial tile may run operand-swapped
                          // (needs 128 weight rows per CTA: gate/up BN = 128, down BN = 256)
  int shared_a_stride;    // A rows between consecutive shared experts (0: all read row 0..T)
  int router_tiles;       // tile count when tile_start is NULL (M-tiles x N-tiles)
  int dense_kind;         // kind of the single group when tile_start is NULL
  int shared_only_tiles;  // > 0 with tile_start NULL: only the shared groups (each of T rows),
                          // this many tiles per group, group s at tiles [s * n, (s + 1) * n)
  int out_bf16;           // down-mode output as bf16 instead of fp32 (latent projection)
  int fp8;                // expert GEMMs: A and B are E4M3 codes (kind::f8f6f4)
  int fp4;                // fp8 with the weights stored as packed E2M1 + block scales:
                          // block-scaled MMAs (kind::mxf8f6f4), every tile swapped
  int ep;                 // down, routed: dest_row = rank << 24 | row, stored at out_rank[rank]
  int ep_world;           // ep: ranks
  int a_rows[2];          // rows of each kind's A tensor (index checks; 0 = unchecked)
  int out_rows[2];        // rows of each kind's output (per rank under ep)
  float* out_rank[8];     // ep: each rank's slot-row output base (addresses on this rank)
  const int8_t* a_exp[2]; // fp8: per kind, power-of-two exponent of each A row; the
                          // accumulator of row r is multiplied by 2^a_exp[kind][r]
  void* out[2];           // output base per kind
  int ld_out[2];          // output row pitch (elements) per kind
  int shared_out_stride;  // output rows between consecutive shared experts
  const int* dest_row;    // down, routed: grouped row -> output row
  float gate_clamp, up_clamp;
  int act;                // moe_activation
  float beta_g, beta_u;   // SiTU-GLU caps
  float inv_beta_g, inv_beta_u;  // their reciprocals (rounded once)
  int* err;               // device error word
  unsigned long long timeout_ns;
};

void gemm_prepare();    // shared memory limit + pair occupancy, once per device
int gemm_max_pairs();   // CTA pairs of the expert GEMMs resident at once (0 = unknown)
cudaError_t launch_grouped_gemm(int mode, const GemmArgs& a, int grid, cudaStream_t s);

// --------------------------------------------------------------- row ops
// Also clears the device error word and zeroes `zero_words` int32 at `zero`.
// yq != NULL: also the E4M3 copy of y with one power-of-two exponent per row.
cudaError_t launch_rmsnorm_rows(const uint16_t* x, const uint16_t* g, uint16_t* y, int T, int D,
                                float eps, int* err_to_clear, int32_t* zero, int zero_words,
                                uint8_t* yq, int8_t* yq_exp, cudaStream_t s);
// bf16 rows -> E4M3 rows + per-row exponents, two segments.
// rows0_dev != NULL: only rows [rows0_dev[1], rows0_dev[0]) of the rows0 rows
// of segment 0 are quantised (the rest are skipped).
cudaError_t launch_quant_rows(const uint16_t* a0, int rows0, int w0, uint8_t* q0, int8_t* e0,
                              const uint16_t* a1, int rows1, int w1, uint8_t* q1, int8_t* e1,
                              const int32_t* rows0_dev, cudaStream_t s);
// FP4 (E2M1, power-of-two scale per 32-element block) -> E4M3 weights.
cudaError_t launch_quant_weights_fp4(const uint16_t* w, uint8_t* w8, int8_t* block_exp, long long nblocks,
                                     cudaStream_t s);
// The same quantisation in storage form: packed E2M1 codes [rows, K/2] and the
// block exponents as uint32 [K/128, rows] (four int8 per word).
// FP4 block scales in the order the expert GEMMs read them: for every half h
// (a CTA's weight rows of a tile) and 128-wide K stage kc, a 512-byte atom whose
// 16-byte lane row l holds the UE8M0 words (exponent + 127 per 32-element block)
// of rows l, l + 32, l + 64, l + 96 of the half.  Gate/up halves are 64 rows of
// `first` (gate) then 64 rows of `second` (up); down halves (second = NULL) are
// 128 rows of `first`.  exps: uint32 [KC, rows] as moe_quantize_weights_fp4_packed
// writes them; atoms: [rows_total / half_rows][KC][128] words.
cudaError_t launch_fp4_scale_atoms(const uint32_t* first, const uint32_t* second, long long rows, int KC,
                                   uint32_t* atoms, cudaStream_t s);
cudaError_t launch_quant_weights_fp4_packed(const uint16_t* w, uint8_t* packed, uint32_t* exps, long long rows,
                                            int K, cudaStream_t s);
// topk_w == NULL: every slot weighs 1.
cudaError_t launch_combine_norm(const float* y_slot, const float* topk_w, const float* y_shared,
                                int k, int S, const uint16_t* residual, const uint16_t* g,
                                uint16_t* out_norm, uint16_t* out_residual, int T, int D,
                                float eps, cudaStream_t s);
// agg[t] = bf16(sum_j topk_w[t, j] * y_slot[t, j, :]) over L latent columns.
cudaError_t launch_combine_latent(const float* y_slot, const float* topk_w, int k, int L, uint16_t* agg,
                                  int T, cudaStream_t s);
struct PartialPtrs {
  const uint16_t* p[8];
};
// Destinations of the reduced rows (n_out pairs; local or peer memory).
struct OutPtrs {
  uint16_t* norm[8];
  uint16_t* res[8];
};
// Rows [row0, row0 + rows) of the P partial buffers (each [T, D], local or peer
// memory) reduced in the fixed order p = 0 .. P-1, + residual, RMSNorm; written
// to the same rows of every destination pair.
cudaError_t launch_reduce_partials(const PartialPtrs& parts, int P, const uint16_t* residual,
                                   const uint16_t* g, const OutPtrs& outs, int n_out, int row0, int rows,
                                   int D, float eps, cudaStream_t s);
cudaError_t launch_bitcompare(const uint16_t* a, const uint16_t* b, const int32_t* b_row_of_a,
                              int rows, int D, unsigned long long* count, cudaStream_t s);
cudaError_t launch_permute_inputs(const uint16_t* x, const uint16_t* res, const int32_t* ids,
                                  const int32_t* perm, int T, int D, uint16_t* xo, uint16_t* ro,
                                  int32_t* io, cudaStream_t s);

// ------------------------------------------------------------- routing
struct RouterArgs {
  const float* logits;      // [T, E_pad]
  int E_pad;
  const float* bias;        // [E] or NULL
  const int32_t* token_ids; // hash routing
  int router, E, k, renormalize;
  float routed_scale;
  uint32_t hash_mult;
  int32_t* idx;             // [T, k]
  float* w;                 // [T, k]
  int32_t* block_counts;    // [ceil(T / 128), E4], zeroed beforehand
  int E4;                   // row stride of block_counts: E rounded up to 4
  int32_t* user_idx;        // [T, k] copy of idx for the caller, or NULL
  float* user_w;            // [T, k] copy of w for the caller, or NULL
  int T;
};
cudaError_t launch_router_topk(const RouterArgs& a, cudaStream_t s);

// ------------------------------------------------------------ dispatch
constexpr int kDispatchRows = 128;  // tokens per dispatch block (= one router GEMM tile)
struct DispatchArgs {
  const int32_t* idx;   // [T, k]
  int T, k, E, S;
  const int32_t* block_counts;  // [nb, E4] expert counts of each 128-token block
  int E4;                       // row stride of block_counts (E rounded up to 4)
  int32_t* counts;        // [E]
  int32_t* offsets;       // [E + 1]
  int32_t* user_counts;   // [E] or NULL
  int32_t* tiles_gu;      // [E + S + 1]
  int32_t* tiles_dn;      // [E + S + 1]
  int gu_ntiles_routed, gu_ntiles_shared, dn_ntiles, dn_ntiles_shared;
  int tile_m;             // rows per expert-GEMM tile (256: a CTA pair)
  int32_t* dest_row;      // [T * k]
  int32_t* src_token;     // [T * k]
  int* err;               // device error word (index checks)
};
cudaError_t launch_dispatch(const DispatchArgs& a, cudaStream_t s);
cudaError_t launch_gather_rows(const void* src, int src_rows, const int32_t* src_row, int rows, int row_bytes,
                               void* dst, const int8_t* src_exp, int8_t* dst_exp, int* err, cudaStream_t s);

// ------------------------------------------------------- expert parallelism
struct EpSendArgs {
  const int32_t* boards[8];  // per rank: its [E] expert counts (addresses on this rank)
  uint8_t* recv[8];          // per rank: received input rows
  int8_t* recv_exp[8];       // per rank: their E4M3 exponents (E4M3 rows only)
  int32_t* meta[8];          // per rank: return address (source rank << 24 | token * k + slot)
  const uint8_t* src_rows;   // this rank's input rows (xn bf16 or xq E4M3)
  const int8_t* src_exp;     // their exponents, or NULL for bf16 rows
  const int32_t* offsets;    // [E + 1] this rank's grouped rows per expert
  const int32_t* src_token;  // [rows] grouped row -> token
  const int32_t* dest_row;   // [rows] grouped row -> token * k + slot
  int rows, row_bytes, E, E_loc, world, rank;
  long long cap;             // rows of each rank's receive buffers
  int wave_lo, wave_hi;      // rows of every owner's local experts [wave_lo, wave_hi) only
  int* err;                  // device error word (index checks)
};
cudaError_t launch_ep_send(const EpSendArgs& a, int grid, cudaStream_t s);

struct EpPlanArgs {
  const int32_t* boards[8];
  int world, rank, E_loc, S, T_self;
  int32_t* offsets;          // [E_loc + 1] received rows per local expert
  int32_t* tiles_gu;         // [E_loc + S + 1]
  int32_t* tiles_dn;         // [E_loc + S + 1]
  int32_t* rows_received;    // [2]: end and start of the wave's received rows
  int gu_ntiles_routed, gu_ntiles_shared, dn_ntiles, dn_ntiles_shared, tile_m;
  int wave_lo, wave_hi;      // tiles of local experts [wave_lo, wave_hi) only
  int with_shared;           // and of the shared experts
};
cudaError_t launch_ep_plan(const EpPlanArgs& a, cudaStream_t s);

// ------------------------------------------------------------ self test
cudaError_t launch_wait_selftest(int* flag, int* err, unsigned long long limit_ns,
                                 cudaStream_t s);

// Flag arrays of the ranks of a peer barrier (addresses in this process).
struct PeerFlags {
  uint32_t* p[8];
};
cudaError_t launch_peer_barrier(const PeerFlags& f, int world, int rank, uint32_t epoch, int* err,
                                unsigned long long limit_ns, cudaStream_t s);

}  // namespace moe
