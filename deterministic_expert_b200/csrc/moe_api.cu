// The C ABI of libmoe.so (declared in include/moe.h): argument checks, the
// workspace layout, TMA descriptor encoding and the launch sequence of one
// layer forward.  Everything here runs on the host; every step of the layer
// runs in the kernels of the other translation units.
#include <cudaTypedefs.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <cstring>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "moe_internal.h"

using namespace moe;

struct moe_handle {
  moe_config cfg;
  moe_weights w;
  int S = 0, G = 0, E_pad = 0, bn_gu = 0, bn_dn = 0, num_sms = 0, device = 0, max_pairs = 0;
  int L = 0;                          // width the router and routed experts read (latent or D)
  bool fp8 = false;                   // MOE_WEIGHTS_FP8 or _FP4: E4M3 expert GEMMs
  bool fp4 = false;                   // MOE_WEIGHTS_FP4: packed E2M1 weights, block-scaled MMAs
  int ep_world = 1, ep_rank = 0;      // expert parallelism (1: none)
  int E_loc = 0;                      // routed experts held here (E / ep_world)
  long long cap = 0;                  // rows a rank can receive: ep_world * T_max * k
  int bn_pd = 0, bn_pu = 0;           // N tiles of the latent down / up projections
  uint16_t* w_router_pad = nullptr;  // [E_pad, L], rows >= E zero
  CUtensorMap map_router, map_wg, map_wu, map_wd, map_wsg, map_wsu, map_wsd, map_pd, map_pu;
  // MOE_WEIGHTS_FP4: the expert matrices as packed codes and their exponent words.
  CUtensorMap pmap_wg, pmap_wu, pmap_wd, pmap_wsg, pmap_wsu, pmap_wsd;
  // FP4: the block scales as the GEMMs' UE8M0 atoms (built at init, owned here)
  // and their maps: routed gate/up, routed down, shared gate/up, shared down.
  uint32_t* sf_atoms[4] = {nullptr, nullptr, nullptr, nullptr};
  CUtensorMap smap[4];
  unsigned long long timeout_ns = 2000ull * 1000 * 1000;
  // Decode-sized batches run the shared experts (which need no routing) on an
  // auxiliary stream while the routing front end runs on the caller's stream;
  // the mutex keeps concurrent forwards on one handle from interleaving their
  // event records.
  cudaStream_t aux = nullptr;
  cudaEvent_t ev_fork = nullptr, ev_join = nullptr;
  std::mutex fork_mu;
  // Per-stage timing (moe_profile_*).
  int prof_mask = 0;
  int prof_fwd = 0;
  std::vector<cudaEvent_t> ev;  // [kProfFwd][MOE_NUM_STAGES][2]
  int prof_launches[MOE_NUM_STAGES] = {0};
};

namespace {

// Device address of the no-allocation forward's static scratch on the current
// device (defined with that entry point at the end of this file).
void* noalloc_scratch();

constexpr int kProfFwd = 256;

size_t align256(size_t b) { return (b + 255) & ~static_cast<size_t>(255); }

struct Layout {
  size_t err, xn, logits, tidx, tw, bcount, counts, offsets, tiles_gu, tiles_dn, dest, src,
      xp, h, hs, y, ys, z, agg, ylat, xq, xqe, xpe, hq, hqs, he, hse,
      hr, hqr, her, epoff, eptg, eptd, eprows, zq, zqe, total;   // hr..eprows: expert parallelism
};

Layout layout(const moe_handle* h, int T) {
  const moe_config& c = h->cfg;
  const size_t Tz = static_cast<size_t>(T), nb = (Tz + kDispatchRows - 1) / kDispatchRows;
  Layout L;
  size_t off = 0;
  auto take = [&](size_t bytes) { const size_t o = off; off += align256(bytes); return o; };
  L.err = take(256);
  L.xn = take(Tz * c.D * 2);
  L.logits = take(c.router == MOE_ROUTER_HASH ? 0 : Tz * h->E_pad * 4);
  L.tidx = take(Tz * c.k * 4);
  L.tw = take(Tz * c.k * 4);
  L.bcount = take(nb * ((c.E + 3) / 4 * 4) * 4);
  L.counts = take(static_cast<size_t>(c.E) * 4);
  L.offsets = take(static_cast<size_t>(c.E + 1) * 4);
  L.tiles_gu = take(static_cast<size_t>(h->G + 1) * 4);
  L.tiles_dn = take(static_cast<size_t>(h->G + 1) * 4);
  L.dest = take(Tz * c.k * 4);
  L.src = take(Tz * c.k * 4);
  const size_t Lw = static_cast<size_t>(h->L);
  const size_t eb = h->fp8 ? 1 : 2;   // bytes per element of the expert GEMMs' inputs
  const bool ep = h->ep_world > 1;    // routed rows live in the exchange buffers
  const size_t rt = ep ? 0 : 1;
  L.xp = take(rt * Tz * c.k * Lw * eb);
  L.h = take(rt * Tz * c.k * c.I * 2);
  L.hs = take(static_cast<size_t>(h->S) * Tz * c.I_shared * 2);
  L.y = take(rt * Tz * c.k * Lw * 4);
  L.ys = take(static_cast<size_t>(h->S) * Tz * c.D * 4);
  const bool lat = c.latent > 0;
  L.z = take(lat ? Tz * Lw * 2 : 0);
  L.agg = take(lat ? Tz * Lw * 2 : 0);
  L.ylat = take(lat ? Tz * c.D * 4 : 0);
  // E4M3 inputs of the expert GEMMs and their per-row exponents.
  const size_t f = h->fp8 ? 1 : 0;
  L.xq = take(f * Tz * c.D);
  L.xqe = take(f * Tz);
  L.xpe = take(rt * f * Tz * c.k);
  L.hq = take(rt * f * Tz * c.k * c.I);
  L.hqs = take(f * static_cast<size_t>(h->S) * Tz * c.I_shared);
  L.he = take(rt * f * Tz * c.k);
  L.hse = take(f * static_cast<size_t>(h->S) * Tz);
  // Expert parallelism: h of the received rows, the owner's plan.
  const size_t cap = ep ? static_cast<size_t>(h->cap) : 0;
  const size_t gl = static_cast<size_t>(h->E_loc + h->S + 1);
  L.hr = take(cap * c.I * 2);
  L.hqr = take(f * cap * c.I);
  L.her = take(f * cap);
  L.epoff = take(ep ? static_cast<size_t>(h->E_loc + 1) * 4 : 0);
  L.eptg = take(ep ? gl * 4 : 0);
  L.eptd = take(ep ? gl * 4 : 0);
  L.eprows = take(ep ? 8 : 0);
  // E4M3 copy of the latent input z (latent width with E4M3 experts).
  L.zq = take(lat ? f * Tz * Lw : 0);
  L.zqe = take(lat ? f * Tz : 0);
  L.total = off;
  return L;
}

// Expert parallelism: the exchange buffer every rank exposes to the others.
struct XLayout {
  size_t board, recv, recv_exp, meta, y, total;
};

XLayout xlayout(const moe_handle* h) {
  const moe_config& c = h->cfg;
  const size_t cap = static_cast<size_t>(h->cap), rowb = static_cast<size_t>(h->L) * (h->fp8 ? 1 : 2);
  XLayout X;
  size_t off = 0;
  auto take = [&](size_t bytes) { const size_t o = off; off += align256(bytes); return o; };
  X.board = take(static_cast<size_t>(c.E) * 4);
  X.recv = take(cap * rowb);
  X.recv_exp = take(h->fp8 ? cap : 0);
  X.meta = take(cap * 4);
  X.y = take(static_cast<size_t>(c.T_max) * c.k * h->L * 4);
  X.total = off;
  return X;
}

struct InvLayout {
  size_t ref_n, ref_r, tst_n, tst_r, xp, rp, ip, cnt, errs, total;
};
constexpr int kMaxInvRuns = 64;

InvLayout inv_layout(const moe_handle* h, int T, size_t base) {
  const size_t rowb = static_cast<size_t>(T) * h->cfg.D * 2;
  InvLayout L;
  size_t off = base;
  auto take = [&](size_t bytes) { const size_t o = off; off += align256(bytes); return o; };
  L.ref_n = take(rowb); L.ref_r = take(rowb); L.tst_n = take(rowb); L.tst_r = take(rowb);
  L.xp = take(rowb); L.rp = take(rowb); L.ip = take(static_cast<size_t>(T) * 4);
  L.cnt = take(8); L.errs = take(kMaxInvRuns * 4);
  L.total = off;
  return L;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2D tensor map over a row-major [rows, inner] matrix of bf16 (elem_bytes 2)
// or E4M3 bytes (elem_bytes 1); box = 128 bytes of a row (the 128-byte swizzle
// span: 64 bf16 or 128 E4M3) x box_rows rows.  Rows past the end read as
// zeros.  An empty matrix leaves the map zeroed (never loaded).
bool make_map(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t rows, uint32_t box_rows,
              int elem_bytes = 2) {
  std::memset(m, 0, sizeof(*m));
  if (rows == 0 || ptr == nullptr) return true;
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner * static_cast<cuuint64_t>(elem_bytes)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / elem_bytes), box_rows};
  cuuint32_t estr[2] = {1, 1};
  const CUtensorMapDataType dt = elem_bytes == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  return fn(m, dt, 2, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// MOE_WEIGHTS_FP4: a [rows, K] expert matrix stored as packed E2M1 codes
// (uint8 [rows, K/2], two codes a byte, low nibble first), loaded as 4-bit
// elements that TMA spreads 16 to a 16-byte chunk (8 bytes of codes, 8 unused:
// the layout the tensor core reads E2M1 operands in), 128-byte swizzled, boxes
// of 128 codes (one K stage) x box_rows rows.  Needs a 32-byte aligned base,
// K a multiple of 128 and rows K/2 bytes apart (a multiple of 32).
bool make_packed_map(CUtensorMap* m, const void* ptr, uint64_t K, uint64_t rows, uint32_t box_rows) {
  std::memset(m, 0, sizeof(*m));
  if (rows == 0 || ptr == nullptr) return true;
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {K, rows};
  cuuint64_t strides[1] = {K / 2};
  cuuint32_t box[2] = {128, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 2, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// MOE_WEIGHTS_FP4: n 512-byte scale atoms as a [n, 128] uint32 tensor, one
// atom per box.
bool make_sf_map(CUtensorMap* m, const void* ptr, uint64_t n) {
  std::memset(m, 0, sizeof(*m));
  if (n == 0 || ptr == nullptr) return true;
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {128, n};
  cuuint64_t strides[1] = {512};
  cuuint32_t box[2] = {128, 1};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int validate_config(const moe_config* c, const moe_weights* w) {
  if (!c || !w) return MOE_EINVAL;
  if (c->router < 0 || c->router > 2 || c->D <= 0 || c->E <= 0 || c->k <= 0 || c->I <= 0 ||
      c->n_shared < 0 || c->T_max <= 0 || !(c->eps >= 0.f) || !(c->routed_scale == c->routed_scale) ||
      !(c->gate_clamp_max == c->gate_clamp_max) || !(c->up_clamp >= 0.f))
    return MOE_EINVAL;
  if (c->n_shared > 0 && c->I_shared <= 0) return MOE_EINVAL;
  if (c->latent < 0) return MOE_EINVAL;
  if (c->latent > 0 && (c->latent % 64 || c->latent > 16384)) return MOE_EUNSUPPORTED;
  if (c->latent > 0 && (!w->w_proj_down || !w->w_proj_up || !aligned16(w->w_proj_down) ||
                        !aligned16(w->w_proj_up)))
    return MOE_EINVAL;
  if (c->activation != MOE_ACT_SWIGLU && c->activation != MOE_ACT_SITU_GLU) return MOE_EINVAL;
  if (c->activation == MOE_ACT_SITU_GLU &&
      !(c->situ_beta_gate > 0.f && c->situ_beta_gate < 3.0e38f && c->situ_beta_up > 0.f &&
        c->situ_beta_up < 3.0e38f))
    return MOE_EINVAL;
  if (c->D % 64 || c->I % 64 || (c->n_shared > 0 && c->I_shared % 64)) return MOE_EUNSUPPORTED;
  if (c->weight_format != MOE_WEIGHTS_BF16 && c->weight_format != MOE_WEIGHTS_FP8 &&
      c->weight_format != MOE_WEIGHTS_FP4)
    return MOE_EINVAL;
  if (c->ep_world < 0 || c->ep_world > 8 || c->ep_rank < 0 || (c->ep_world > 1 && c->ep_rank >= c->ep_world))
    return MOE_EINVAL;
  if (c->ep_world > 1 && (c->E % c->ep_world || c->latent > 0)) return MOE_EUNSUPPORTED;
  if (c->ep_world > 1 && static_cast<long long>(c->ep_world) * c->T_max * c->k >= (1ll << 24))
    return MOE_EUNSUPPORTED;   // return addresses keep the row in 24 bits
  if (c->weight_format != MOE_WEIGHTS_BF16 &&
      (c->D % 128 || c->I % 128 || (c->n_shared > 0 && c->I_shared % 128) || c->latent % 128))
    return MOE_EUNSUPPORTED;
  // FP4: every CTA of a pair holds 128 weight rows with one scale atom a
  // stage, so gate/up tiles of 128 columns and down tiles of 256.
  if (c->weight_format == MOE_WEIGHTS_FP4 && (c->D % 256 || c->latent % 256)) return MOE_EUNSUPPORTED;
  if (c->weight_format == MOE_WEIGHTS_FP4) {
    if (!w->w_gate_exp || !w->w_up_exp || !w->w_down_exp) return MOE_EINVAL;
    if (c->n_shared > 0 && (!w->ws_gate_exp || !w->ws_up_exp || !w->ws_down_exp)) return MOE_EINVAL;
    const void* ep[] = {w->w_gate_exp, w->w_up_exp, w->w_down_exp, w->ws_gate_exp, w->ws_up_exp, w->ws_down_exp};
    for (const void* p : ep)
      if (p && !aligned16(p)) return MOE_EINVAL;
    // 4-bit TMA loads need 32-byte aligned packed weights.
    const void* pw[] = {w->w_gate, w->w_up, w->w_down, w->ws_gate, w->ws_up, w->ws_down};
    for (const void* p : pw)
      if (p && (reinterpret_cast<uintptr_t>(p) & 31u) != 0) return MOE_EINVAL;
  }
  if (c->D > 16384 || c->E > 256 || c->k > c->E || c->k > 16 || c->n_shared > 8 || c->T_max > (1 << 20))
    return MOE_EUNSUPPORTED;
  const long long rows = static_cast<long long>(c->T_max) * std::max(c->k, c->n_shared);
  if (rows * std::max(c->D, std::max(c->I, c->I_shared)) >= (1ll << 31)) return MOE_EUNSUPPORTED;
  if (!w->w_gate || !w->w_up || !w->w_down || !w->g_in || !w->g_out) return MOE_EINVAL;
  if (c->router != MOE_ROUTER_HASH && !w->w_router) return MOE_EINVAL;
  if (c->n_shared > 0 && (!w->ws_gate || !w->ws_up || !w->ws_down)) return MOE_EINVAL;
  const void* ptrs[] = {w->w_router, w->w_gate, w->w_up, w->w_down, w->ws_gate, w->ws_up,
                        w->ws_down, w->g_in, w->g_out, w->router_bias};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return MOE_EINVAL;
  return MOE_OK;
}

// With T < 256 no group reaches 256 rows, so every expert tile is a swapped
// tile with at most ceil(T rounded up to 16 / 2) token rows per CTA; the GEMM
// then sizes its stages' A slot to the TMA box that covers them (16, 32, 64 or
// 128 rows).  0: the default 16 KB slot.
int small_batch_a_bytes(int T) {
  if (T >= 256) return 0;
  const int rows = ((T + 15) / 16 * 16) / 2;
  return (rows <= 16 ? 16 : (rows <= 32 ? 32 : (rows <= 64 ? 64 : 128))) * kBK * 2;
}

// MOE_WEIGHTS_FP4: the scale-atom maps of an expert GEMM (per kind: routed, shared).
void fp4_exponents(const moe_handle* h, GemmArgs& g, bool gateup) {
  if (!h->fp4) return;
  g.mapSF[0] = h->smap[gateup ? 0 : 1];
  g.mapSF[1] = h->smap[gateup ? 2 : 3];
}

// Rows per M-tile of the expert GEMMs (FP4: swapped tiles of at most 240 tokens).
int tile_rows(const moe_handle* h) { return h->fp4 ? kF4TileTokens : kPairTileM; }

// A bytes per stage of the expert GEMMs: small batches size the slot to their
// TMA box (FP4 tiles, every one swapped, hold at most 120 token rows per CTA,
// within the default slot).
int expert_a_bytes(const moe_handle* h, int T, bool swap_ok) {
  return (swap_ok || h->fp4) ? small_batch_a_bytes(T) : 0;
}

int gemm_grid(const moe_handle* h, int tiles_bound) {
  return std::max(1, std::min(h->num_sms, tiles_bound));
}

// Stage names as moe_profile_read numbers them; each stage's launch is also an
// NVTX range of that name (host-side markers for a timeline tool; a no-op
// when none is attached).
const char* const kStageNames[MOE_NUM_STAGES] = {
    "moe.rmsnorm_in", "moe.router_gemm", "moe.router_topk", "moe.dispatch", "moe.gather_rows",
    "moe.gemm_gateup", "moe.gemm_down", "moe.combine_norm", "moe.latent_down", "moe.latent_combine",
    "moe.latent_up", "moe.quant_h"};

struct Prof {
  moe_handle* h;
  cudaStream_t s;
  int f;
  bool on(int stage) const { return f >= 0 && ((h->prof_mask >> stage) & 1); }
  void begin(int stage) {
    nvtxRangePushA(kStageNames[stage]);
    if (on(stage)) cudaEventRecord(h->ev[(static_cast<size_t>(f) * MOE_NUM_STAGES + stage) * 2], s);
  }
  void end(int stage) {
    nvtxRangePop();
    if (on(stage)) {
      cudaEventRecord(h->ev[(static_cast<size_t>(f) * MOE_NUM_STAGES + stage) * 2 + 1], s);
      h->prof_launches[stage] += 1;
    }
  }
};

#define MOE_TRY(expr)                            \
  do {                                           \
    if ((expr) != cudaSuccess) return MOE_ECUDA; \
  } while (0)

// Upper bound on the tiles of the routed + shared expert GEMMs for T rows:
// sum_e ceil(c_e / 128) <= T*k/128 + (number of non-empty experts).
// sum_e ceil(c_e / 256) <= T*k/256 + (number of non-empty experts), in pair tiles.
int expert_tile_bound(const moe_handle* h, int T, int nt_routed, int nt_shared) {
  const moe_config& c = h->cfg;
  const long long tk = static_cast<long long>(T) * c.k;
  const int tm = tile_rows(h);
  const long long mt = (tk + tm - 1) / tm + std::min<long long>(c.E, tk);
  const long long b = mt * nt_routed + static_cast<long long>(h->S) * ((T + tm - 1) / tm) * nt_shared;
  return static_cast<int>(std::min<long long>(b, 1 << 29));
}

// CTA-pair grid: two CTAs per tile, at most one CTA per SM.
int pair_grid(const moe_handle* h, int tiles_bound) {
  return 2 * std::max(1, std::min(h->max_pairs, tiles_bound));
}

// Shared-expert tiles of the gate/up GEMM for T rows.
int shared_gateup_tiles(const moe_handle* h, int T) {
  return h->S * ((T + tile_rows(h) - 1) / tile_rows(h)) * (h->cfg.I_shared / h->bn_gu);
}

// Whether a forward of T rows runs the shared experts on the auxiliary stream:
// only when their gate/up tiles occupy at most two thirds of the CTA pairs, so
// the routing front end and the routed experts keep SMs to run on.  (At
// prefill sizes the shared tiles would hold every SM and gain nothing.)
bool fork_shared(const moe_handle* h, int T) {
  return h->S > 0 && h->aux != nullptr && h->ep_world == 1 &&
         3 * shared_gateup_tiles(h, T) <= 2 * h->max_pairs;
}

// The layer forward.  front_only (expert parallelism): stop after the grouping
// (stages 0-3), with the per-expert counts written to counts_dst.
int forward_impl(moe_handle* h, int T, const uint16_t* x, const uint16_t* residual,
                 const int32_t* token_ids, uint16_t* out_norm, uint16_t* out_residual,
                 int32_t* out_idx, float* out_w, int32_t* out_counts, uint8_t* ws,
                 cudaStream_t s, bool front_only = false, int32_t* counts_dst = nullptr) {
  const moe_config& c = h->cfg;
  const Layout L = layout(h, T);
  int* err = reinterpret_cast<int*>(ws + L.err);
  uint16_t* xn = reinterpret_cast<uint16_t*>(ws + L.xn);
  float* logits = reinterpret_cast<float*>(ws + L.logits);
  int32_t* tidx = reinterpret_cast<int32_t*>(ws + L.tidx);
  float* tw = reinterpret_cast<float*>(ws + L.tw);
  int32_t* offsets = reinterpret_cast<int32_t*>(ws + L.offsets);
  int32_t* tiles_gu = reinterpret_cast<int32_t*>(ws + L.tiles_gu);
  int32_t* tiles_dn = reinterpret_cast<int32_t*>(ws + L.tiles_dn);
  int32_t* dest = reinterpret_cast<int32_t*>(ws + L.dest);
  int32_t* src = reinterpret_cast<int32_t*>(ws + L.src);
  uint16_t* xp = reinterpret_cast<uint16_t*>(ws + L.xp);
  uint16_t* hb = reinterpret_cast<uint16_t*>(ws + L.h);
  uint16_t* hsb = reinterpret_cast<uint16_t*>(ws + L.hs);
  float* y = reinterpret_cast<float*>(ws + L.y);
  float* ys = reinterpret_cast<float*>(ws + L.ys);
  const int TK = T * c.k;
  const bool lat = c.latent > 0;
  uint16_t* zb = reinterpret_cast<uint16_t*>(ws + L.z);
  uint16_t* aggb = reinterpret_cast<uint16_t*>(ws + L.agg);
  float* ylat = reinterpret_cast<float*>(ws + L.ylat);
  const int LW = h->L;
  const bool f8 = h->fp8;
  const int eb = f8 ? 1 : 2;
  uint8_t* xq = ws + L.xq;
  int8_t* xqe = reinterpret_cast<int8_t*>(ws + L.xqe);
  int8_t* xpe = reinterpret_cast<int8_t*>(ws + L.xpe);
  uint8_t* hq = ws + L.hq;
  uint8_t* hqs = ws + L.hqs;
  int8_t* he = reinterpret_cast<int8_t*>(ws + L.he);
  int8_t* hse = reinterpret_cast<int8_t*>(ws + L.hse);

  // One dense group of T rows through the CTA-pair GEMM (latent projections):
  // out[T, N] = A[T, K] B[N, K]^T, bf16 or fp32 out.
  auto dense_gemm = [&](const uint16_t* A, int K, const CUtensorMap& B, int N, int BN, void* out,
                        int out_bf16) -> int {
    GemmArgs g;
    std::memset(&g, 0, sizeof(g));
    if (!make_map(&g.mapA[1], A, K, T, kBM) || !make_map(&g.mapA64[1], A, K, T, kBM / 2) ||
        (!make_map(&g.mapA16[1], A, K, T, 16) || !make_map(&g.mapA32[1], A, K, T, 32)))
      return MOE_ECUDA;
    g.mapB[2] = B;
    g.T = T; g.G = 1; g.E = 0;
    g.n_kind[1] = N; g.k_kind[1] = K;
    g.BN = BN;
    g.swap_ok = BN == 256;
    g.dense_kind = 1;
    g.router_tiles = (T + kPairTileM - 1) / kPairTileM * (N / BN);
    g.out[1] = out; g.ld_out[1] = N; g.out_bf16 = out_bf16;
    g.err = err; g.timeout_ns = h->timeout_ns;
    return launch_grouped_gemm(kDown, g, pair_grid(h, g.router_tiles), s) == cudaSuccess ? MOE_OK : MOE_ECUDA;
  };

  Prof prof{h, s, -1};
  if (h->prof_mask && h->prof_fwd < kProfFwd) prof.f = h->prof_fwd++;

  // 0. input RMSNorm (also clears the device error word and the histogram)
  int32_t* bcount = reinterpret_cast<int32_t*>(ws + L.bcount);
  const int nblk = (T + kDispatchRows - 1) / kDispatchRows;
  const int E4 = (c.E + 3) / 4 * 4;
  prof.begin(0);
  MOE_TRY(launch_rmsnorm_rows(x, h->w.g_in, xn, T, c.D, c.eps, err, bcount, nblk * E4, f8 ? xq : nullptr,
                              f8 ? xqe : nullptr, s));
  prof.end(0);

  // 5-6. gate/up + SwiGLU(+clamp) (routed groups read xp, shared groups read
  // xn), the E4M3 quantisation of h, and down (routed rows scatter to their
  // (token, slot) row of y).  `part` selects the groups: all of them, the
  // routed ones, or the shared ones (each group's tiles are the same in every
  // case, so the bits are too).
  enum Part { kAllGroups, kRoutedGroups, kSharedGroups };
  auto expert_gemms = [&](Part part, cudaStream_t st) -> int {
    const bool routed = part != kSharedGroups, shared = part != kRoutedGroups && h->S > 0;
    const bool timed = st == s;   // stage timing covers the caller's stream only
    const int mt_shared = (T + tile_rows(h) - 1) / tile_rows(h);
    // Which groups a launch walks: the device tile list (all groups, or its
    // routed prefix), or the shared groups alone.
    auto select = [&](GemmArgs& g, int32_t* tiles, int nt_routed, int nt_shared) {
      if (part == kSharedGroups) {
        g.tile_start = nullptr;
        g.shared_only_tiles = mt_shared * nt_shared;
        g.router_tiles = h->S * g.shared_only_tiles;
        return g.router_tiles;
      }
      g.tile_start = tiles;
      g.G = part == kAllGroups ? h->G : c.E;
      return expert_tile_bound(h, T, nt_routed, part == kAllGroups ? nt_shared : 0);
    };
    {
      GemmArgs g;
      std::memset(&g, 0, sizeof(g));
      // E4M3: the routed rows are the gathered E4M3 rows, the shared rows xq.
      const void* xs = f8 ? static_cast<const void*>(xq) : static_cast<const void*>(xn);
      if (!make_map(&g.mapA[0], xp, LW, TK, kBM, eb)) return MOE_ECUDA;
      if (!make_map(&g.mapA64[0], xp, LW, TK, kBM / 2, eb)) return MOE_ECUDA;
      if (!make_map(&g.mapA16[0], xp, LW, TK, 16, eb) || !make_map(&g.mapA32[0], xp, LW, TK, 32, eb))
        return MOE_ECUDA;
      if (h->S > 0 && !make_map(&g.mapA[1], xs, c.D, T, kBM, eb)) return MOE_ECUDA;
      if (h->S > 0 && !make_map(&g.mapA64[1], xs, c.D, T, kBM / 2, eb)) return MOE_ECUDA;
      if (h->S > 0 && (!make_map(&g.mapA16[1], xs, c.D, T, 16, eb) || !make_map(&g.mapA32[1], xs, c.D, T, 32, eb)))
        return MOE_ECUDA;
      g.fp8 = f8;
      g.a_exp[0] = xpe; g.a_exp[1] = xqe;
      g.a_rows[0] = TK; g.a_rows[1] = T;
      g.out_rows[0] = TK; g.out_rows[1] = h->S * T;
      g.mapB[0] = h->map_wg; g.mapB[1] = h->map_wu; g.mapB[2] = h->map_wsg; g.mapB[3] = h->map_wsu;
      g.fp4 = h->fp4;
      g.mapBp[0] = h->pmap_wg; g.mapBp[1] = h->pmap_wu; g.mapBp[2] = h->pmap_wsg; g.mapBp[3] = h->pmap_wsu;
      fp4_exponents(h, g, true);
      g.offsets = offsets; g.G = h->G; g.E = c.E; g.T = T;
      g.n_kind[0] = c.I; g.n_kind[1] = c.I_shared;
      g.k_kind[0] = LW; g.k_kind[1] = c.D;
      g.BN = h->bn_gu;
      g.swap_ok = h->bn_gu == 128;
      g.a_stage_bytes = expert_a_bytes(h, T, g.swap_ok);
      g.shared_a_stride = 0;
      g.out[0] = hb; g.ld_out[0] = c.I;
      g.out[1] = hsb; g.ld_out[1] = c.I_shared;
      g.shared_out_stride = T;
      g.gate_clamp = c.gate_clamp_max; g.up_clamp = c.up_clamp;
      g.act = c.activation; g.beta_g = c.situ_beta_gate; g.beta_u = c.situ_beta_up;
      g.inv_beta_g = 1.0f / c.situ_beta_gate; g.inv_beta_u = 1.0f / c.situ_beta_up;
      g.err = err; g.timeout_ns = h->timeout_ns;
      const int bound = select(g, tiles_gu, c.I / h->bn_gu, h->S > 0 ? c.I_shared / h->bn_gu : 0);
      if (timed) prof.begin(5);
      if (launch_grouped_gemm(kGateUp, g, pair_grid(h, bound), st) != cudaSuccess) return MOE_ECUDA;
      if (timed) prof.end(5);
    }
    // 5b. E4M3: h rows (routed and / or shared) to E4M3 with their row exponents
    if (f8) {
      if (timed) prof.begin(11);
      if (launch_quant_rows(hb, routed ? TK : 0, c.I, hq, he, hsb, shared ? h->S * T : 0, c.I_shared, hqs, hse,
                            nullptr, st) != cudaSuccess)
        return MOE_ECUDA;
      if (timed) prof.end(11);
    }
    {
      GemmArgs g;
      std::memset(&g, 0, sizeof(g));
      const void* ar = f8 ? static_cast<const void*>(hq) : static_cast<const void*>(hb);
      const void* as = f8 ? static_cast<const void*>(hqs) : static_cast<const void*>(hsb);
      const uint64_t srows = static_cast<uint64_t>(h->S) * T;
      if (!make_map(&g.mapA[0], ar, c.I, TK, kBM, eb)) return MOE_ECUDA;
      if (!make_map(&g.mapA64[0], ar, c.I, TK, kBM / 2, eb)) return MOE_ECUDA;
      if (!make_map(&g.mapA16[0], ar, c.I, TK, 16, eb) || !make_map(&g.mapA32[0], ar, c.I, TK, 32, eb))
        return MOE_ECUDA;
      if (h->S > 0 && !make_map(&g.mapA[1], as, c.I_shared, srows, kBM, eb)) return MOE_ECUDA;
      if (h->S > 0 && !make_map(&g.mapA64[1], as, c.I_shared, srows, kBM / 2, eb)) return MOE_ECUDA;
      if (h->S > 0 && (!make_map(&g.mapA16[1], as, c.I_shared, srows, 16, eb) ||
                       !make_map(&g.mapA32[1], as, c.I_shared, srows, 32, eb)))
        return MOE_ECUDA;
      g.fp8 = f8;
      g.a_exp[0] = he; g.a_exp[1] = hse;
      g.a_rows[0] = TK; g.a_rows[1] = h->S * T;
      g.out_rows[0] = TK; g.out_rows[1] = h->S * T;
      g.mapB[0] = h->map_wd; g.mapB[2] = h->map_wsd;
      g.fp4 = h->fp4;
      g.mapBp[0] = h->pmap_wd; g.mapBp[2] = h->pmap_wsd;
      fp4_exponents(h, g, false);
      g.offsets = offsets; g.G = h->G; g.E = c.E; g.T = T;
      g.n_kind[0] = LW; g.n_kind[1] = c.D;
      g.k_kind[0] = c.I; g.k_kind[1] = c.I_shared;
      g.BN = h->bn_dn;
      g.swap_ok = h->bn_dn == 256;
      g.a_stage_bytes = expert_a_bytes(h, T, g.swap_ok);
      g.shared_a_stride = T;
      g.out[0] = y; g.ld_out[0] = LW;
      g.out[1] = ys; g.ld_out[1] = c.D;
      g.shared_out_stride = T;
      g.dest_row = dest;
      g.err = err; g.timeout_ns = h->timeout_ns;
      const int bound = select(g, tiles_dn, LW / h->bn_dn, c.D / h->bn_dn);
      if (timed) prof.begin(6);
      if (launch_grouped_gemm(kDown, g, pair_grid(h, bound), st) != cudaSuccess) return MOE_ECUDA;
      if (timed) prof.end(6);
    }
    return MOE_OK;
  };

  // Decode-sized batches: the shared experts need only xn, so they start now
  // on the auxiliary stream and run beside the routing front end; the caller's
  // stream joins them before the combine.
  const bool fork = !front_only && fork_shared(h, T);
  std::unique_lock<std::mutex> fork_lock(h->fork_mu, std::defer_lock);
  if (fork) {
    fork_lock.lock();
    MOE_TRY(cudaEventRecord(h->ev_fork, s));
    MOE_TRY(cudaStreamWaitEvent(h->aux, h->ev_fork, 0));
    const int r = expert_gemms(kSharedGroups, h->aux);
    if (r != MOE_OK) return r;
    MOE_TRY(cudaEventRecord(h->ev_join, h->aux));
  }

  // Latent MoE: the router and the routed experts read z = bf16(xn W_down^T).
  const uint16_t* xe = xn;
  if (lat) {
    prof.begin(8);
    const int r = dense_gemm(xn, c.D, h->map_pd, LW, h->bn_pd, zb, 1);
    if (r != MOE_OK) return r;
    // E4M3 experts read z as E4M3 rows with their exponents, like xn.
    if (f8)
      MOE_TRY(launch_quant_rows(zb, T, LW, ws + L.zq, reinterpret_cast<int8_t*>(ws + L.zqe), nullptr, 0, 0,
                                nullptr, nullptr, nullptr, s));
    prof.end(8);
    xe = zb;
  }

  // 1. router logits on the tensor cores
  if (c.router != MOE_ROUTER_HASH) {
    GemmArgs g;
    std::memset(&g, 0, sizeof(g));
    if (!make_map(&g.mapA[0], xe, LW, T, kBM)) return MOE_ECUDA;
    if (!make_map(&g.mapA64[0], xe, LW, T, kBM / 2)) return MOE_ECUDA;
    if (!make_map(&g.mapA16[0], xe, LW, T, 16) || !make_map(&g.mapA32[0], xe, LW, T, 32)) return MOE_ECUDA;
    g.mapB[0] = h->map_router;
    g.T = T;
    g.n_kind[0] = h->E_pad;
    g.k_kind[0] = LW;
    g.BN = h->E_pad;
    g.router_tiles = (T + kBM - 1) / kBM;
    g.out[0] = logits;
    g.ld_out[0] = h->E_pad;
    g.err = err;
    g.timeout_ns = h->timeout_ns;
    prof.begin(1);
    MOE_TRY(launch_grouped_gemm(kRouter, g, gemm_grid(h, g.router_tiles), s));
    prof.end(1);
  }

  // 2. scores, top-k, weights, and each 128-token block's expert histogram
  RouterArgs ra;
  ra.logits = logits; ra.E_pad = h->E_pad; ra.bias = h->w.router_bias; ra.token_ids = token_ids;
  ra.router = c.router; ra.E = c.E; ra.k = c.k; ra.renormalize = c.renormalize;
  ra.routed_scale = c.routed_scale; ra.hash_mult = c.hash_mult; ra.idx = tidx; ra.w = tw;
  ra.block_counts = bcount; ra.E4 = E4; ra.user_idx = out_idx; ra.user_w = out_w; ra.T = T;
  prof.begin(2);
  MOE_TRY(launch_router_topk(ra, s));
  prof.end(2);

  // 3. offsets, stable scatter and the expert-GEMM tile lists
  DispatchArgs da;
  da.idx = tidx; da.T = T; da.k = c.k; da.E = c.E; da.S = h->S;
  da.block_counts = bcount; da.E4 = E4;
  da.counts = counts_dst != nullptr ? counts_dst : reinterpret_cast<int32_t*>(ws + L.counts);
  da.offsets = offsets; da.user_counts = out_counts; da.tiles_gu = tiles_gu; da.tiles_dn = tiles_dn;
  da.gu_ntiles_routed = c.I / h->bn_gu;
  da.gu_ntiles_shared = h->S > 0 ? c.I_shared / h->bn_gu : 0;
  da.dn_ntiles = LW / h->bn_dn;
  da.dn_ntiles_shared = c.D / h->bn_dn;
  da.dest_row = dest; da.src_token = src; da.err = err;
  da.tile_m = tile_rows(h);
  prof.begin(3);
  MOE_TRY(launch_dispatch(da, s));
  prof.end(3);
  if (front_only) return MOE_OK;

  // 4. grouped A rows of the routed experts
  prof.begin(4);
  if (f8 && lat)
    MOE_TRY(launch_gather_rows(ws + L.zq, T, src, TK, LW, xp, reinterpret_cast<int8_t*>(ws + L.zqe), xpe, err, s));
  else if (f8) MOE_TRY(launch_gather_rows(xq, T, src, TK, LW, xp, xqe, xpe, err, s));
  else MOE_TRY(launch_gather_rows(xe, T, src, TK, LW * 2, xp, nullptr, nullptr, err, s));
  prof.end(4);

  if (fork) {
    // The shared experts were started on the auxiliary stream after step 0.
    const int r = expert_gemms(kRoutedGroups, s);
    if (r != MOE_OK) return r;
    MOE_TRY(cudaStreamWaitEvent(s, h->ev_join, 0));
  } else {
    const int r = expert_gemms(kAllGroups, s);
    if (r != MOE_OK) return r;
  }

  // 7. fixed-order combine + residual + RMSNorm
  if (lat) {
    // Latent MoE: a = bf16(sum_j w_j y_j) in slot order, then y = a W_up^T, which
    // the epilogue takes as a single slot of weight 1.
    prof.begin(9);
    MOE_TRY(launch_combine_latent(y, tw, c.k, LW, aggb, T, s));
    prof.end(9);
    prof.begin(10);
    const int r = dense_gemm(aggb, LW, h->map_pu, c.D, h->bn_pu, ylat, 0);
    if (r != MOE_OK) return r;
    prof.end(10);
    prof.begin(7);
    MOE_TRY(launch_combine_norm(ylat, nullptr, ys, 1, h->S, residual, h->w.g_out, out_norm, out_residual,
                                T, c.D, c.eps, s));
    prof.end(7);
  } else {
    prof.begin(7);
    MOE_TRY(launch_combine_norm(y, tw, ys, c.k, h->S, residual, h->w.g_out, out_norm, out_residual, T,
                                c.D, c.eps, s));
    prof.end(7);
  }
  return MOE_OK;
}

int check_forward_args(const moe_handle* h, int T, const void* x, const void* residual,
                       const void* token_ids, const void* out_norm, const void* out_residual,
                       const void* workspace, size_t ws_bytes, size_t need) {
  if (!h || T < 0) return MOE_EINVAL;
  if (h->ep_world > 1) return MOE_EINVAL;   // expert-parallel handles run the moe_ep_* phases
  if (T > h->cfg.T_max) return MOE_ETOOBIG;
  if (T == 0) return MOE_OK;
  if (!x || !residual || !out_norm || !out_residual || !workspace) return MOE_EINVAL;
  if (h->cfg.router == MOE_ROUTER_HASH && !token_ids) return MOE_EINVAL;
  if (!aligned16(x) || !aligned16(residual) || !aligned16(out_norm) || !aligned16(out_residual))
    return MOE_EINVAL;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MOE_EINVAL;
  if (ws_bytes < need) return MOE_EWORKSPACE;
  return MOE_OK;
}

}  // namespace

extern "C" {

int moe_init(const moe_config* cfg, const moe_weights* w, moe_handle** out) {
  if (!out) return MOE_EINVAL;
  *out = nullptr;
  const int v = validate_config(cfg, w);
  if (v != MOE_OK) return v;
  moe_handle* h = new (std::nothrow) moe_handle();
  if (!h) return MOE_ECUDA;
  h->cfg = *cfg;
  h->w = *w;
  h->S = cfg->n_shared;
  if (h->S == 0) h->cfg.I_shared = cfg->I;  // unused; keeps the shapes well defined
  h->G = cfg->E + h->S;
  h->E_pad = (cfg->E + 15) / 16 * 16;
  // One GEMM configuration per layer shape, never per T.  The expert GEMMs run
  // on CTA pairs: each CTA loads half of a gate/up tile (bn_gu / 2 gate rows and
  // bn_gu / 2 up rows) or half of a down tile (bn_dn / 2 rows).
  h->L = cfg->latent > 0 ? cfg->latent : cfg->D;
  h->fp8 = cfg->weight_format == MOE_WEIGHTS_FP8 || cfg->weight_format == MOE_WEIGHTS_FP4;
  h->fp4 = cfg->weight_format == MOE_WEIGHTS_FP4;
  h->ep_world = cfg->ep_world > 1 ? cfg->ep_world : 1;
  h->ep_rank = cfg->ep_world > 1 ? cfg->ep_rank : 0;
  h->E_loc = cfg->E / h->ep_world;
  h->cap = h->ep_world > 1 ? static_cast<long long>(h->ep_world) * cfg->T_max * cfg->k : 0;
  h->bn_gu = (cfg->I % 128 == 0 && h->cfg.I_shared % 128 == 0) ? 128 : 64;
  // The down GEMM's routed groups have N = L, its shared groups N = D.
  auto bn_for = [](int n) { return n % 256 == 0 ? 256 : (n % 128 == 0 ? 128 : 64); };
  h->bn_dn = std::min(bn_for(cfg->D), bn_for(h->L));
  h->bn_pd = bn_for(h->L);   // latent down-projection: N = latent
  h->bn_pu = bn_for(cfg->D); // latent up-projection: N = D
  auto fail = [&](int code) { moe_destroy(h); return code; };
  if (cudaGetDevice(&h->device) != cudaSuccess) return fail(MOE_ECUDA);
  if (cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, h->device) != cudaSuccess)
    return fail(MOE_ECUDA);
  gemm_prepare();
  h->max_pairs = gemm_max_pairs();
  if (h->max_pairs <= 0) h->max_pairs = h->num_sms / 2;
  if (h->S > 0 && h->ep_world == 1 &&
      (cudaStreamCreateWithFlags(&h->aux, cudaStreamNonBlocking) != cudaSuccess ||
       cudaEventCreateWithFlags(&h->ev_fork, cudaEventDisableTiming) != cudaSuccess ||
       cudaEventCreateWithFlags(&h->ev_join, cudaEventDisableTiming) != cudaSuccess))
    return fail(MOE_ECUDA);
  const moe_config& c = h->cfg;
  if (c.router != MOE_ROUTER_HASH) {
    const size_t row = static_cast<size_t>(h->L) * 2;
    if (cudaMalloc(&h->w_router_pad, static_cast<size_t>(h->E_pad) * row) != cudaSuccess) return fail(MOE_ECUDA);
    if (cudaMemset(h->w_router_pad, 0, static_cast<size_t>(h->E_pad) * row) != cudaSuccess) return fail(MOE_ECUDA);
    if (cudaMemcpy(h->w_router_pad, w->w_router, static_cast<size_t>(c.E) * row, cudaMemcpyDeviceToDevice) != cudaSuccess)
      return fail(MOE_ECUDA);
  }
  const int eb = h->fp8 ? 1 : 2;   // expert weights: E4M3 or bf16
  bool ok = make_map(&h->map_router, h->w_router_pad, h->L, h->w_router_pad ? h->E_pad : 0, h->E_pad) &&
            make_map(&h->map_wg, w->w_gate, h->L, static_cast<uint64_t>(h->E_loc) * c.I, h->bn_gu / 2, eb) &&
            make_map(&h->map_wu, w->w_up, h->L, static_cast<uint64_t>(h->E_loc) * c.I, h->bn_gu / 2, eb) &&
            make_map(&h->map_wd, w->w_down, c.I, static_cast<uint64_t>(h->E_loc) * h->L, h->bn_dn / 2, eb) &&
            make_map(&h->map_wsg, w->ws_gate, c.D, static_cast<uint64_t>(h->S) * c.I_shared, h->bn_gu / 2, eb) &&
            make_map(&h->map_wsu, w->ws_up, c.D, static_cast<uint64_t>(h->S) * c.I_shared, h->bn_gu / 2, eb) &&
            make_map(&h->map_wsd, w->ws_down, c.I_shared, static_cast<uint64_t>(h->S) * c.D, h->bn_dn / 2, eb) &&
            make_map(&h->map_pd, c.latent > 0 ? w->w_proj_down : nullptr, c.D, c.latent, h->bn_pd / 2) &&
            make_map(&h->map_pu, c.latent > 0 ? w->w_proj_up : nullptr, h->L, c.D, h->bn_pu / 2);
  if (ok && h->fp4) {
    const uint64_t rg = static_cast<uint64_t>(h->E_loc) * c.I, rd = static_cast<uint64_t>(h->E_loc) * h->L;
    const uint64_t rsg = static_cast<uint64_t>(h->S) * c.I_shared, rsd = static_cast<uint64_t>(h->S) * c.D;
    ok = make_packed_map(&h->pmap_wg, w->w_gate, h->L, rg, 64) && make_packed_map(&h->pmap_wu, w->w_up, h->L, rg, 64) &&
         make_packed_map(&h->pmap_wd, w->w_down, c.I, rd, 128) &&
         make_packed_map(&h->pmap_wsg, w->ws_gate, c.D, rsg, 64) &&
         make_packed_map(&h->pmap_wsu, w->ws_up, c.D, rsg, 64) &&
         make_packed_map(&h->pmap_wsd, w->ws_down, c.I_shared, rsd, 128);
    // The scale atoms: gate/up halves of 64 + 64 rows, down halves of 128 rows.
    struct Src { const uint32_t* first; const uint32_t* second; uint64_t rows; int KC; };
    const Src src[4] = {{w->w_gate_exp, w->w_up_exp, rg, h->L / 128},
                        {w->w_down_exp, nullptr, rd, c.I / 128},
                        {w->ws_gate_exp, w->ws_up_exp, rsg, c.D / 128},
                        {w->ws_down_exp, nullptr, rsd, c.I_shared / 128}};
    for (int i = 0; ok && i < 4; ++i) {
      if (src[i].rows == 0) continue;
      const uint64_t atoms = src[i].rows / (src[i].second ? 64 : 128) * static_cast<uint64_t>(src[i].KC);
      ok = cudaMalloc(&h->sf_atoms[i], atoms * 512) == cudaSuccess &&
           launch_fp4_scale_atoms(src[i].first, src[i].second, static_cast<long long>(src[i].rows), src[i].KC,
                                  h->sf_atoms[i], nullptr) == cudaSuccess &&
           make_sf_map(&h->smap[i], h->sf_atoms[i], atoms);
    }
    ok = ok && cudaDeviceSynchronize() == cudaSuccess;
  }
  if (!ok) return fail(MOE_ECUDA);
  *out = h;
  return MOE_OK;
}

size_t moe_workspace_size(const moe_handle* h, int T) {
  if (!h || T <= 0 || T > h->cfg.T_max) return 0;
  return layout(h, T).total;
}

int moe_layer_forward(moe_handle* h, int T, const moe_bf16* x, const moe_bf16* residual,
                      const int32_t* token_ids, moe_bf16* out_norm, moe_bf16* out_residual,
                      int32_t* out_topk_idx, float* out_topk_w, int32_t* out_counts,
                      void* workspace, size_t ws_bytes, void* stream) {
  const size_t need = (h && T > 0 && T <= h->cfg.T_max) ? layout(h, T).total : 0;
  const int v = check_forward_args(h, T, x, residual, token_ids, out_norm, out_residual, workspace,
                                   ws_bytes, need);
  if (v != MOE_OK || T == 0) return v;
  return forward_impl(h, T, x, residual, token_ids, out_norm, out_residual, out_topk_idx, out_topk_w,
                      out_counts, static_cast<uint8_t*>(workspace), static_cast<cudaStream_t>(stream));
}

int moe_get_device_error(moe_handle* h, void* workspace, void* stream) {
  if (!h) return MOE_EINVAL;
  // NULL: the error word of moe_layer_forward_noalloc's static scratch.
  if (!workspace) workspace = noalloc_scratch();
  if (!workspace) return MOE_ECUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int e = 0;
  if (cudaMemcpyAsync(&e, workspace, 4, cudaMemcpyDeviceToHost, s) != cudaSuccess) return MOE_ECUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ECUDA;
  if (cudaMemsetAsync(workspace, 0, 4, s) != cudaSuccess) return MOE_ECUDA;
  switch (e) {
    case kDevOk: return MOE_OK;
    case kDevTimeout: return MOE_ETIMEOUT;
    case kDevBadIndex: return MOE_EINDEX;
    default: return MOE_ECUDA;   // a value no kernel writes: the word itself was overwritten
  }
}

int moe_reduce_partials_rows(int P, const moe_bf16* const* partials, const moe_bf16* residual,
                             const moe_bf16* g, int n_out, moe_bf16* const* out_norm,
                             moe_bf16* const* out_residual, int row0, int rows, int D, float eps,
                             void* stream) {
  if (P < 1 || P > 8 || !partials || n_out < 1 || n_out > 8 || !out_norm || !out_residual || row0 < 0 ||
      rows < 0 || D <= 0 || !(eps >= 0.f))
    return MOE_EINVAL;
  if (D % 64 || D > 16384) return MOE_EUNSUPPORTED;
  if (rows == 0) return MOE_OK;
  if (!residual || !g || !aligned16(residual)) return MOE_EINVAL;
  PartialPtrs pp;
  for (int p = 0; p < 8; ++p) pp.p[p] = nullptr;
  for (int p = 0; p < P; ++p) {
    if (!partials[p] || !aligned16(partials[p])) return MOE_EINVAL;
    pp.p[p] = partials[p];
  }
  OutPtrs op;
  for (int d = 0; d < 8; ++d) op.norm[d] = op.res[d] = nullptr;
  for (int d = 0; d < n_out; ++d) {
    if (!out_norm[d] || !out_residual[d] || !aligned16(out_norm[d]) || !aligned16(out_residual[d]))
      return MOE_EINVAL;
    op.norm[d] = out_norm[d];
    op.res[d] = out_residual[d];
  }
  return launch_reduce_partials(pp, P, residual, g, op, n_out, row0, rows, D, eps,
                                static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? MOE_OK
             : MOE_ECUDA;
}

int moe_reduce_partials(int P, const moe_bf16* const* partials, const moe_bf16* residual,
                        const moe_bf16* g, moe_bf16* out_norm, moe_bf16* out_residual, int T, int D,
                        float eps, void* stream) {
  if (T < 0) return MOE_EINVAL;
  return moe_reduce_partials_rows(P, partials, residual, g, 1, &out_norm, &out_residual, 0, T, D, eps,
                                  stream);
}

size_t moe_invariance_workspace_size(const moe_handle* h, int T) {
  if (!h || T <= 0 || T > h->cfg.T_max) return 0;
  const size_t base = layout(h, T).total;
  return inv_layout(h, T, base).total;
}

int moe_check_invariance(moe_handle* h, int T, const moe_bf16* x, const moe_bf16* residual,
                         const int32_t* token_ids, int n_splits, const int32_t* perm, int repeats,
                         void* workspace, size_t ws_bytes, unsigned long long* out_mismatched_elems,
                         void* stream) {
  if (!h || !out_mismatched_elems || T <= 0 || n_splits < 0 || repeats < 0 || h->ep_world > 1)
    return MOE_EINVAL;
  if (T > h->cfg.T_max) return MOE_ETOOBIG;
  if (n_splits > T || 2 + n_splits + repeats > kMaxInvRuns) return MOE_EINVAL;
  if (!x || !residual || !workspace) return MOE_EINVAL;
  if (h->cfg.router == MOE_ROUTER_HASH && !token_ids) return MOE_EINVAL;
  const size_t base = layout(h, T).total;
  const InvLayout V = inv_layout(h, T, base);
  if (ws_bytes < V.total) return MOE_EWORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MOE_EINVAL;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int D = h->cfg.D;
  auto P16 = [&](size_t off) { return reinterpret_cast<uint16_t*>(ws + off); };
  unsigned long long* cnt = reinterpret_cast<unsigned long long*>(ws + V.cnt);
  int* errs = reinterpret_cast<int*>(ws + V.errs);
  int nrun = 0;
  if (cudaMemsetAsync(cnt, 0, 8, s) != cudaSuccess) return MOE_ECUDA;
  if (cudaMemsetAsync(errs, 0, kMaxInvRuns * 4, s) != cudaSuccess) return MOE_ECUDA;
  auto run = [&](int n, const uint16_t* xx, const uint16_t* rr, const int32_t* ii, uint16_t* on,
                 uint16_t* orr) -> int {
    const int r = forward_impl(h, n, xx, rr, ii, on, orr, nullptr, nullptr, nullptr, ws, s);
    if (r != MOE_OK) return r;
    if (cudaMemcpyAsync(errs + nrun++, ws, 4, cudaMemcpyDeviceToDevice, s) != cudaSuccess) return MOE_ECUDA;
    return MOE_OK;
  };
  auto compare = [&](const int32_t* rowmap) -> int {
    if (launch_bitcompare(P16(V.tst_n), P16(V.ref_n), rowmap, T, D, cnt, s) != cudaSuccess) return MOE_ECUDA;
    if (launch_bitcompare(P16(V.tst_r), P16(V.ref_r), rowmap, T, D, cnt, s) != cudaSuccess) return MOE_ECUDA;
    return MOE_OK;
  };
  int r = run(T, x, residual, token_ids, P16(V.ref_n), P16(V.ref_r));
  if (r != MOE_OK) return r;
  if (n_splits > 0) {
    for (int i = 0; i < n_splits; ++i) {
      const int r0 = static_cast<int>(static_cast<long long>(T) * i / n_splits);
      const int r1 = static_cast<int>(static_cast<long long>(T) * (i + 1) / n_splits);
      if (r1 == r0) continue;
      const size_t o = static_cast<size_t>(r0) * D;
      r = run(r1 - r0, x + o, residual + o, token_ids ? token_ids + r0 : nullptr, P16(V.tst_n) + o,
              P16(V.tst_r) + o);
      if (r != MOE_OK) return r;
    }
    if ((r = compare(nullptr)) != MOE_OK) return r;
  }
  if (perm) {
    int32_t* ip = reinterpret_cast<int32_t*>(ws + V.ip);
    if (launch_permute_inputs(x, residual, token_ids, perm, T, D, P16(V.xp), P16(V.rp),
                              token_ids ? ip : nullptr, s) != cudaSuccess)
      return MOE_ECUDA;
    r = run(T, P16(V.xp), P16(V.rp), token_ids ? ip : nullptr, P16(V.tst_n), P16(V.tst_r));
    if (r != MOE_OK) return r;
    if ((r = compare(perm)) != MOE_OK) return r;
  }
  for (int i = 0; i < repeats; ++i) {
    r = run(T, x, residual, token_ids, P16(V.tst_n), P16(V.tst_r));
    if (r != MOE_OK) return r;
    if ((r = compare(nullptr)) != MOE_OK) return r;
  }
  int herr[kMaxInvRuns];
  if (cudaMemcpyAsync(out_mismatched_elems, cnt, 8, cudaMemcpyDeviceToHost, s) != cudaSuccess) return MOE_ECUDA;
  if (cudaMemcpyAsync(herr, errs, kMaxInvRuns * 4, cudaMemcpyDeviceToHost, s) != cudaSuccess) return MOE_ECUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ECUDA;
  for (int i = 0; i < nrun; ++i)
    if (herr[i] != kDevOk) return MOE_ETIMEOUT;
  return MOE_OK;
}

int moe_workspace_views(const moe_handle* h, int T, void* workspace, moe_views* out) {
  if (!h || !workspace || !out || T <= 0 || T > h->cfg.T_max) return MOE_EINVAL;
  const Layout L = layout(h, T);
  const uint8_t* ws = static_cast<const uint8_t*>(workspace);
  out->xn = reinterpret_cast<const moe_bf16*>(ws + L.xn);
  out->logits = h->cfg.router == MOE_ROUTER_HASH ? nullptr : reinterpret_cast<const float*>(ws + L.logits);
  out->E_pad = h->E_pad;
  out->topk_idx = reinterpret_cast<const int32_t*>(ws + L.tidx);
  out->topk_w = reinterpret_cast<const float*>(ws + L.tw);
  out->counts = reinterpret_cast<const int32_t*>(ws + L.counts);
  out->offsets = reinterpret_cast<const int32_t*>(ws + L.offsets);
  out->src_token = reinterpret_cast<const int32_t*>(ws + L.src);
  out->dest_row = reinterpret_cast<const int32_t*>(ws + L.dest);
  out->h_routed = reinterpret_cast<const moe_bf16*>(ws + L.h);
  out->h_shared = reinterpret_cast<const moe_bf16*>(ws + L.hs);
  out->y_slot = reinterpret_cast<const float*>(ws + L.y);
  out->y_shared = reinterpret_cast<const float*>(ws + L.ys);
  const bool lat = h->cfg.latent > 0;
  out->z = lat ? reinterpret_cast<const moe_bf16*>(ws + L.z) : nullptr;
  out->agg = lat ? reinterpret_cast<const moe_bf16*>(ws + L.agg) : nullptr;
  out->y_latent = lat ? reinterpret_cast<const float*>(ws + L.ylat) : nullptr;
  const bool f8 = h->fp8;
  out->xq = f8 ? ws + L.xq : nullptr;
  out->xq_exp = f8 ? reinterpret_cast<const int8_t*>(ws + L.xqe) : nullptr;
  out->hq_routed = f8 ? ws + L.hq : nullptr;
  out->hq_routed_exp = f8 ? reinterpret_cast<const int8_t*>(ws + L.he) : nullptr;
  out->hq_shared = f8 ? ws + L.hqs : nullptr;
  out->hq_shared_exp = f8 ? reinterpret_cast<const int8_t*>(ws + L.hse) : nullptr;
  return MOE_OK;
}

int moe_profile_enable(moe_handle* h, int stage_mask) {
  if (!h || stage_mask < 0 || stage_mask >= (1 << MOE_NUM_STAGES)) return MOE_EINVAL;
  if (stage_mask && h->ev.empty()) {
    h->ev.resize(static_cast<size_t>(kProfFwd) * MOE_NUM_STAGES * 2);
    for (auto& e : h->ev)
      if (cudaEventCreate(&e) != cudaSuccess) return MOE_ECUDA;
  }
  h->prof_mask = stage_mask;
  h->prof_fwd = 0;
  for (int i = 0; i < MOE_NUM_STAGES; ++i) h->prof_launches[i] = 0;
  return MOE_OK;
}

int moe_profile_read(moe_handle* h, float* ms, int* launches) {
  if (!h || !ms || !launches) return MOE_EINVAL;
  for (int i = 0; i < MOE_NUM_STAGES; ++i) { ms[i] = 0.f; launches[i] = h->prof_launches[i]; }
  for (int f = 0; f < h->prof_fwd; ++f) {
    for (int st = 0; st < MOE_NUM_STAGES; ++st) {
      if (!((h->prof_mask >> st) & 1)) continue;
      cudaEvent_t a = h->ev[(static_cast<size_t>(f) * MOE_NUM_STAGES + st) * 2];
      cudaEvent_t b = h->ev[(static_cast<size_t>(f) * MOE_NUM_STAGES + st) * 2 + 1];
      if (cudaEventQuery(b) == cudaErrorNotReady && cudaEventSynchronize(b) != cudaSuccess) return MOE_ECUDA;
      float t = 0.f;
      if (cudaEventElapsedTime(&t, a, b) == cudaSuccess) ms[st] += t;
      else cudaGetLastError();  // stage not recorded in this forward (e.g. no router GEMM)
    }
  }
  h->prof_fwd = 0;
  for (int i = 0; i < MOE_NUM_STAGES; ++i) h->prof_launches[i] = 0;
  return MOE_OK;
}

int moe_forward_launch_count(const moe_handle* h, int T) {
  if (!h || T < 0) return -1;
  if (T == 0) return 0;
  const bool fork = fork_shared(h, T);
  const int base = 8 + (h->cfg.latent > 0 ? 3 : 0)   // latent: two projections and the latent sum
                   + (fork ? 2 : 0)                   // shared experts' two GEMMs on their own
                   + (h->fp8 ? (fork ? 2 : 1) : 0)    // E4M3: quantisation of h (routed, shared)
                   + (h->fp8 && h->cfg.latent > 0 ? 1 : 0);   // ... and of z
  return h->cfg.router == MOE_ROUTER_HASH ? base - 1 : base;  // hash routing: no router GEMM
}

int moe_selftest_wait_timeout(int limit_us, void* stream) {
  if (limit_us < 1 || limit_us > 1000000) return MOE_EINVAL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* buf = nullptr;
  if (cudaMalloc(&buf, 8) != cudaSuccess) return MOE_ECUDA;
  int res = MOE_ECUDA;
  int host[2] = {0, 0};
  if (cudaMemsetAsync(buf, 0, 8, s) == cudaSuccess &&
      launch_wait_selftest(buf, buf + 1, static_cast<unsigned long long>(limit_us) * 1000ull, s) == cudaSuccess &&
      cudaMemcpyAsync(host, buf, 8, cudaMemcpyDeviceToHost, s) == cudaSuccess &&
      cudaStreamSynchronize(s) == cudaSuccess)
    res = host[1] == kDevTimeout ? MOE_ETIMEOUT : MOE_OK;
  cudaFree(buf);
  return res;
}

// ---------------------------------------------------------------- expert parallelism
namespace {

int ep_check(const moe_handle* h, int T, const void* workspace, size_t ws_bytes) {
  if (!h || h->ep_world <= 1 || T < 0 || !workspace) return MOE_EINVAL;
  if (T > h->cfg.T_max) return MOE_ETOOBIG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MOE_EINVAL;
  if (T > 0 && ws_bytes < layout(h, T).total) return MOE_EWORKSPACE;
  return MOE_OK;
}

int ep_peers_ok(const moe_handle* h, const moe_ep_peers* p) {
  if (!p) return MOE_EINVAL;
  for (int r = 0; r < h->ep_world; ++r)
    if (!p->xbuf[r] || (reinterpret_cast<uintptr_t>(p->xbuf[r]) & 255u) != 0) return MOE_EINVAL;
  return MOE_OK;
}

// Local experts of wave `wave` of `n_waves`: [wave * E_loc / n, (wave + 1) * E_loc / n).
bool ep_wave(const moe_handle* h, int wave, int n_waves, int* lo, int* hi) {
  if (n_waves < 1 || n_waves > h->E_loc || wave < 0 || wave >= n_waves) return false;
  *lo = static_cast<int>(static_cast<long long>(wave) * h->E_loc / n_waves);
  *hi = static_cast<int>(static_cast<long long>(wave + 1) * h->E_loc / n_waves);
  return true;
}

}  // namespace

size_t moe_ep_exchange_size(const moe_handle* h) {
  if (!h || h->ep_world <= 1) return 0;
  return xlayout(h).total;
}

int moe_ep_route(moe_handle* h, int T, const moe_bf16* x, const int32_t* token_ids, void* xbuf_self,
                 void* workspace, size_t ws_bytes, void* stream) {
  const int v = ep_check(h, T, workspace, ws_bytes);
  if (v != MOE_OK) return v;
  if (!xbuf_self || (reinterpret_cast<uintptr_t>(xbuf_self) & 255u) != 0) return MOE_EINVAL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t* board = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(xbuf_self) + xlayout(h).board);
  if (T == 0) {
    // No tokens: publish zero counts and clear the device error word (which the
    // input RMSNorm clears otherwise).
    MOE_TRY(cudaMemsetAsync(board, 0, static_cast<size_t>(h->cfg.E) * 4, s));
    MOE_TRY(cudaMemsetAsync(workspace, 0, 4, s));
    return MOE_OK;
  }
  if (!x || !aligned16(x) || (h->cfg.router == MOE_ROUTER_HASH && !token_ids)) return MOE_EINVAL;
  return forward_impl(h, T, x, nullptr, token_ids, nullptr, nullptr, nullptr, nullptr, nullptr,
                      static_cast<uint8_t*>(workspace), s, true, board);
}

int moe_ep_send(moe_handle* h, int T, const moe_ep_peers* peers, void* workspace, size_t ws_bytes,
                void* stream) {
  return moe_ep_send_wave(h, T, peers, 0, 1, workspace, ws_bytes, stream);
}

int moe_ep_send_wave(moe_handle* h, int T, const moe_ep_peers* peers, int wave, int n_waves, void* workspace,
                     size_t ws_bytes, void* stream) {
  int v = ep_check(h, T, workspace, ws_bytes);
  if (v == MOE_OK) v = ep_peers_ok(h, peers);
  int wlo = 0, whi = 0;
  if (v == MOE_OK && !ep_wave(h, wave, n_waves, &wlo, &whi)) v = MOE_EINVAL;
  if (v != MOE_OK || T == 0) return v;
  const moe_config& c = h->cfg;
  const Layout L = layout(h, T);
  const XLayout X = xlayout(h);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  EpSendArgs a;
  std::memset(&a, 0, sizeof(a));
  for (int r = 0; r < h->ep_world; ++r) {
    uint8_t* xb = static_cast<uint8_t*>(peers->xbuf[r]);
    a.boards[r] = reinterpret_cast<const int32_t*>(xb + X.board);
    a.recv[r] = xb + X.recv;
    a.recv_exp[r] = h->fp8 ? reinterpret_cast<int8_t*>(xb + X.recv_exp) : nullptr;
    a.meta[r] = reinterpret_cast<int32_t*>(xb + X.meta);
  }
  a.src_rows = h->fp8 ? ws + L.xq : ws + L.xn;
  a.src_exp = h->fp8 ? reinterpret_cast<const int8_t*>(ws + L.xqe) : nullptr;
  a.offsets = reinterpret_cast<const int32_t*>(ws + L.offsets);
  a.src_token = reinterpret_cast<const int32_t*>(ws + L.src);
  a.dest_row = reinterpret_cast<const int32_t*>(ws + L.dest);
  a.rows = T * c.k;
  a.row_bytes = h->L * (h->fp8 ? 1 : 2);
  a.E = c.E; a.E_loc = h->E_loc; a.world = h->ep_world; a.rank = h->ep_rank;
  a.cap = h->cap; a.err = reinterpret_cast<int*>(ws + L.err);
  a.wave_lo = wlo; a.wave_hi = whi;
  const int grid = std::max(1, std::min((a.rows + 7) / 8, 4 * h->num_sms));
  return launch_ep_send(a, grid, static_cast<cudaStream_t>(stream)) == cudaSuccess ? MOE_OK : MOE_ECUDA;
}

int moe_ep_experts(moe_handle* h, int T, const moe_ep_peers* peers, void* workspace, size_t ws_bytes,
                   void* stream) {
  return moe_ep_experts_wave(h, T, peers, 0, 1, workspace, ws_bytes, stream);
}

int moe_ep_experts_wave(moe_handle* h, int T, const moe_ep_peers* peers, int wave, int n_waves,
                        void* workspace, size_t ws_bytes, void* stream) {
  int v = ep_check(h, T, workspace, ws_bytes);
  if (v == MOE_OK) v = ep_peers_ok(h, peers);
  int wlo = 0, whi = 0;
  if (v == MOE_OK && !ep_wave(h, wave, n_waves, &wlo, &whi)) v = MOE_EINVAL;
  if (v != MOE_OK) return v;
  const bool with_shared = wave == 0;   // the shared experts run with the first wave
  // T == 0: this rank has no tokens (no shared-expert tiles) but still serves
  // its routed experts for the other ranks.
  const moe_config& c = h->cfg;
  const Layout L = layout(h, std::max(T, 1));
  const XLayout X = xlayout(h);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool f8 = h->fp8;
  const int eb = f8 ? 1 : 2;
  uint8_t* self = static_cast<uint8_t*>(peers->xbuf[h->ep_rank]);
  int* err = reinterpret_cast<int*>(ws + L.err);
  int32_t* off = reinterpret_cast<int32_t*>(ws + L.epoff);
  int32_t* tg = reinterpret_cast<int32_t*>(ws + L.eptg);
  int32_t* td = reinterpret_cast<int32_t*>(ws + L.eptd);
  int32_t* nrows = reinterpret_cast<int32_t*>(ws + L.eprows);
  const int nt_gu = c.I / h->bn_gu, nt_gus = h->S > 0 ? c.I_shared / h->bn_gu : 0;
  const int nt_dn = h->L / h->bn_dn, nt_dns = c.D / h->bn_dn;
  // 1. The owner's plan from every rank's counts.
  EpPlanArgs pa;
  std::memset(&pa, 0, sizeof(pa));
  for (int r = 0; r < h->ep_world; ++r)
    pa.boards[r] = reinterpret_cast<const int32_t*>(static_cast<uint8_t*>(peers->xbuf[r]) + X.board);
  pa.world = h->ep_world; pa.rank = h->ep_rank; pa.E_loc = h->E_loc; pa.S = h->S; pa.T_self = T;
  pa.offsets = off; pa.tiles_gu = tg; pa.tiles_dn = td; pa.rows_received = nrows;
  pa.gu_ntiles_routed = nt_gu; pa.gu_ntiles_shared = nt_gus; pa.dn_ntiles = nt_dn; pa.dn_ntiles_shared = nt_dns;
  pa.tile_m = tile_rows(h);
  pa.wave_lo = wlo; pa.wave_hi = whi; pa.with_shared = with_shared ? 1 : 0;
  MOE_TRY(launch_ep_plan(pa, s));
  const long long cap = h->cap;
  const int G = h->E_loc + h->S;
  // Tiles at most: sum over local experts of ceil(rows / 256) <= cap / 256 + E_loc.
  auto bound = [&](int nt_r, int nt_s) {
    const int tm = tile_rows(h);
    const long long b = (cap / tm + h->E_loc) * nt_r + static_cast<long long>(h->S) * ((T + tm - 1) / tm) * nt_s;
    return static_cast<int>(std::min<long long>(b, 1 << 29));
  };
  const uint8_t* recv = self + X.recv;
  const int8_t* recv_exp = f8 ? reinterpret_cast<const int8_t*>(self + X.recv_exp) : nullptr;
  uint16_t* xn = reinterpret_cast<uint16_t*>(ws + L.xn);
  uint16_t* hr = reinterpret_cast<uint16_t*>(ws + L.hr);
  uint16_t* hsb = reinterpret_cast<uint16_t*>(ws + L.hs);
  float* ys = reinterpret_cast<float*>(ws + L.ys);
  // 2. gate/up: routed groups read the received rows, shared groups this rank's xn.
  {
    GemmArgs g;
    std::memset(&g, 0, sizeof(g));
    const void* xs = f8 ? static_cast<const void*>(ws + L.xq) : static_cast<const void*>(xn);
    if (!make_map(&g.mapA[0], recv, h->L, cap, kBM, eb) || !make_map(&g.mapA64[0], recv, h->L, cap, kBM / 2, eb) ||
        (!make_map(&g.mapA16[0], recv, h->L, cap, 16, eb) || !make_map(&g.mapA32[0], recv, h->L, cap, 32, eb)))
      return MOE_ECUDA;
    if (h->S > 0 && T > 0 &&
        (!make_map(&g.mapA[1], xs, c.D, T, kBM, eb) || !make_map(&g.mapA64[1], xs, c.D, T, kBM / 2, eb) ||
         (!make_map(&g.mapA16[1], xs, c.D, T, 16, eb) || !make_map(&g.mapA32[1], xs, c.D, T, 32, eb))))
      return MOE_ECUDA;
    g.mapB[0] = h->map_wg; g.mapB[1] = h->map_wu; g.mapB[2] = h->map_wsg; g.mapB[3] = h->map_wsu;
    g.fp4 = h->fp4;
    g.mapBp[0] = h->pmap_wg; g.mapBp[1] = h->pmap_wu; g.mapBp[2] = h->pmap_wsg; g.mapBp[3] = h->pmap_wsu;
    fp4_exponents(h, g, true);
    g.offsets = off; g.tile_start = tg; g.G = G; g.E = h->E_loc; g.T = T;
    g.n_kind[0] = c.I; g.n_kind[1] = c.I_shared;
    g.k_kind[0] = h->L; g.k_kind[1] = c.D;
    g.BN = h->bn_gu;
    g.swap_ok = h->bn_gu == 128;
    // The owner's groups hold rows from every rank, so tiles reach their full
    // height whatever this rank's T: the default A slot.
    g.a_stage_bytes = 0;
    g.shared_a_stride = 0;
    g.out[0] = hr; g.ld_out[0] = c.I;
    g.out[1] = hsb; g.ld_out[1] = c.I_shared;
    g.shared_out_stride = T;
    g.gate_clamp = c.gate_clamp_max; g.up_clamp = c.up_clamp;
    g.act = c.activation; g.beta_g = c.situ_beta_gate; g.beta_u = c.situ_beta_up;
    g.inv_beta_g = 1.0f / c.situ_beta_gate; g.inv_beta_u = 1.0f / c.situ_beta_up;
    g.fp8 = f8;
    g.a_exp[0] = recv_exp; g.a_exp[1] = reinterpret_cast<const int8_t*>(ws + L.xqe);
    g.a_rows[0] = static_cast<int>(cap); g.a_rows[1] = T;
    g.out_rows[0] = static_cast<int>(cap); g.out_rows[1] = h->S * T;
    g.err = err; g.timeout_ns = h->timeout_ns;
    MOE_TRY(launch_grouped_gemm(kGateUp, g, pair_grid(h, bound(nt_gu, nt_gus)), s));
  }
  // 3. E4M3: the wave's received rows' h and the shared h.
  uint8_t* hqr = ws + L.hqr;
  int8_t* her = reinterpret_cast<int8_t*>(ws + L.her);
  uint8_t* hqs = ws + L.hqs;
  int8_t* hse = reinterpret_cast<int8_t*>(ws + L.hse);
  if (f8)
    MOE_TRY(launch_quant_rows(hr, static_cast<int>(cap), c.I, hqr, her, hsb, with_shared ? h->S * T : 0,
                              c.I_shared, hqs, hse, nrows, s));
  // 4. down: routed rows go back to their source rank's slot rows, shared rows stay here.
  {
    GemmArgs g;
    std::memset(&g, 0, sizeof(g));
    const void* ar = f8 ? static_cast<const void*>(hqr) : static_cast<const void*>(hr);
    const void* as = f8 ? static_cast<const void*>(hqs) : static_cast<const void*>(hsb);
    const uint64_t srows = static_cast<uint64_t>(h->S) * T;
    if (!make_map(&g.mapA[0], ar, c.I, cap, kBM, eb) || !make_map(&g.mapA64[0], ar, c.I, cap, kBM / 2, eb) ||
        (!make_map(&g.mapA16[0], ar, c.I, cap, 16, eb) || !make_map(&g.mapA32[0], ar, c.I, cap, 32, eb)))
      return MOE_ECUDA;
    if (h->S > 0 && T > 0 &&
        (!make_map(&g.mapA[1], as, c.I_shared, srows, kBM, eb) ||
         !make_map(&g.mapA64[1], as, c.I_shared, srows, kBM / 2, eb) ||
         (!make_map(&g.mapA16[1], as, c.I_shared, srows, 16, eb) || !make_map(&g.mapA32[1], as, c.I_shared, srows, 32, eb))))
      return MOE_ECUDA;
    g.mapB[0] = h->map_wd; g.mapB[2] = h->map_wsd;
    g.fp4 = h->fp4;
    g.mapBp[0] = h->pmap_wd; g.mapBp[2] = h->pmap_wsd;
    fp4_exponents(h, g, false);
    g.offsets = off; g.tile_start = td; g.G = G; g.E = h->E_loc; g.T = T;
    g.n_kind[0] = h->L; g.n_kind[1] = c.D;
    g.k_kind[0] = c.I; g.k_kind[1] = c.I_shared;
    g.BN = h->bn_dn;
    g.swap_ok = h->bn_dn == 256;
    g.a_stage_bytes = 0;
    g.shared_a_stride = T;
    g.out[0] = nullptr; g.ld_out[0] = h->L;
    g.out[1] = ys; g.ld_out[1] = c.D;
    g.shared_out_stride = T;
    g.dest_row = reinterpret_cast<const int32_t*>(self + X.meta);
    g.ep = 1;
    g.ep_world = h->ep_world;
    g.a_rows[0] = static_cast<int>(cap); g.a_rows[1] = h->S * T;
    g.out_rows[0] = c.T_max * c.k; g.out_rows[1] = h->S * T;
    for (int r = 0; r < h->ep_world; ++r)
      g.out_rank[r] = reinterpret_cast<float*>(static_cast<uint8_t*>(peers->xbuf[r]) + X.y);
    g.fp8 = f8;
    g.a_exp[0] = her; g.a_exp[1] = hse;
    g.err = err; g.timeout_ns = h->timeout_ns;
    MOE_TRY(launch_grouped_gemm(kDown, g, pair_grid(h, bound(nt_dn, nt_dns)), s));
  }
  return MOE_OK;
}

int moe_ep_combine(moe_handle* h, int T, const moe_bf16* residual, void* xbuf_self, moe_bf16* out_norm,
                   moe_bf16* out_residual, int32_t* out_topk_idx, float* out_topk_w, void* workspace,
                   size_t ws_bytes, void* stream) {
  const int v = ep_check(h, T, workspace, ws_bytes);
  if (v != MOE_OK || T == 0) return v;
  if (!residual || !out_norm || !out_residual || !xbuf_self || !aligned16(residual) || !aligned16(out_norm) ||
      !aligned16(out_residual))
    return MOE_EINVAL;
  const moe_config& c = h->cfg;
  const Layout L = layout(h, T);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const float* y = reinterpret_cast<const float*>(static_cast<uint8_t*>(xbuf_self) + xlayout(h).y);
  const float* tw = reinterpret_cast<const float*>(ws + L.tw);
  MOE_TRY(launch_combine_norm(y, tw, reinterpret_cast<const float*>(ws + L.ys), c.k, h->S, residual, h->w.g_out,
                              out_norm, out_residual, T, c.D, c.eps, s));
  const size_t tk = static_cast<size_t>(T) * c.k * 4;
  if (out_topk_idx) MOE_TRY(cudaMemcpyAsync(out_topk_idx, ws + L.tidx, tk, cudaMemcpyDeviceToDevice, s));
  if (out_topk_w) MOE_TRY(cudaMemcpyAsync(out_topk_w, ws + L.tw, tk, cudaMemcpyDeviceToDevice, s));
  return MOE_OK;
}

int moe_quantize_weights_fp4(const moe_bf16* w, uint8_t* w8, int8_t* block_exp, long long rows, int K,
                             void* stream) {
  if (!w || !w8 || rows < 0 || K <= 0 || K % 32 || !aligned16(w) || !aligned16(w8)) return MOE_EINVAL;
  return launch_quant_weights_fp4(w, w8, block_exp, rows * (K / 32), static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? MOE_OK
             : MOE_ECUDA;
}

int moe_quantize_weights_fp4_packed(const moe_bf16* w, uint8_t* packed, uint32_t* exps, long long rows, int K,
                                    void* stream) {
  if (!w || !packed || !exps || rows < 0 || K <= 0 || K % 128 || !aligned16(w) || !aligned16(packed) ||
      !aligned16(exps))
    return MOE_EINVAL;
  return launch_quant_weights_fp4_packed(w, packed, exps, rows, K, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? MOE_OK
             : MOE_ECUDA;
}

int moe_peer_alloc(size_t bytes, void** dptr, unsigned char* handle) {
  if (!dptr || !handle || bytes == 0) return MOE_EINVAL;
  *dptr = nullptr;
  static_assert(sizeof(cudaIpcMemHandle_t) == MOE_PEER_HANDLE_BYTES, "IPC handle size");
  void* p = nullptr;
  if (cudaMalloc(&p, bytes) != cudaSuccess) return MOE_ECUDA;
  cudaIpcMemHandle_t ih;
  if (cudaMemset(p, 0, bytes) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess ||
      cudaIpcGetMemHandle(&ih, p) != cudaSuccess) {
    cudaFree(p);
    return MOE_ECUDA;
  }
  std::memcpy(handle, &ih, sizeof ih);
  *dptr = p;
  return MOE_OK;
}

int moe_peer_free(void* dptr) {
  if (!dptr) return MOE_EINVAL;
  return cudaFree(dptr) == cudaSuccess ? MOE_OK : MOE_ECUDA;
}

int moe_peer_open(const unsigned char* handle, void** dptr) {
  if (!handle || !dptr) return MOE_EINVAL;
  *dptr = nullptr;
  cudaIpcMemHandle_t ih;
  std::memcpy(&ih, handle, sizeof ih);
  void* p = nullptr;
  if (cudaIpcOpenMemHandle(&p, ih, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) {
    cudaGetLastError();  // leave no stale error for the next runtime call
    return MOE_ECUDA;
  }
  *dptr = p;
  return MOE_OK;
}

int moe_peer_close(void* dptr) {
  if (!dptr) return MOE_EINVAL;
  return cudaIpcCloseMemHandle(dptr) == cudaSuccess ? MOE_OK : MOE_ECUDA;
}

int moe_peer_barrier(int world, int rank, uint32_t* const* flags, uint32_t epoch, int* err, int limit_us,
                     void* stream) {
  if (world < 1 || world > 8 || rank < 0 || rank >= world || !flags || !err || epoch == 0 || limit_us < 1 ||
      limit_us > 60000000)
    return MOE_EINVAL;
  moe::PeerFlags f;
  for (int r = 0; r < 8; ++r) f.p[r] = nullptr;
  for (int r = 0; r < world; ++r) {
    if (!flags[r] || (reinterpret_cast<uintptr_t>(flags[r]) & 3)) return MOE_EINVAL;
    f.p[r] = flags[r];
  }
  const unsigned long long limit_ns = static_cast<unsigned long long>(limit_us) * 1000ull;
  return moe::launch_peer_barrier(f, world, rank, epoch, err, limit_ns, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? MOE_OK
             : MOE_ECUDA;
}

int moe_destroy(moe_handle* h) {
  if (!h) return MOE_EINVAL;
  for (auto& e : h->ev)
    if (e) cudaEventDestroy(e);
  if (h->ev_fork) cudaEventDestroy(h->ev_fork);
  if (h->ev_join) cudaEventDestroy(h->ev_join);
  if (h->aux) cudaStreamDestroy(h->aux);
  if (h->w_router_pad) cudaFree(h->w_router_pad);
  for (auto* p : h->sf_atoms)
    if (p) cudaFree(p);
  delete h;
  return MOE_OK;
}

const char* moe_status_string(int status) {
  switch (status) {
    case MOE_OK: return "ok";
    case MOE_EINVAL: return "invalid argument";
    case MOE_ETOOBIG: return "T exceeds T_max";
    case MOE_EWORKSPACE: return "workspace too small";
    case MOE_EUNSUPPORTED: return "unsupported shape";
    case MOE_ECUDA: return "CUDA error";
    case MOE_ETIMEOUT: return "device wait timed out";
    case MOE_EINDEX: return "device index out of range (bounds-checked build)";
    default: return "unknown status";
  }
}

}  // extern "C"

// ------------------------------------------------- no-allocation forward
// The workspace of moe_layer_forward_noalloc: one static device array per GPU
// (held by every GPU that loads the library until the process exits).  Host
// code only knows a host-side stand-in for its name, so its device address is
// looked up once per device with cudaGetSymbolAddress and cached.
static __device__ __align__(256) unsigned char g_noalloc_scratch[MOE_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {nullptr};

// Device address of g_noalloc_scratch on the current device (nullptr on failure).
void* noalloc_scratch() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    g_noalloc_ptr[dev] = p;
  }
  return g_noalloc_ptr[dev];
}
}  // namespace

extern "C" int moe_layer_forward_noalloc(moe_handle* h, int T, const moe_bf16* x,
                                         const moe_bf16* residual, const int32_t* token_ids,
                                         moe_bf16* out_norm, moe_bf16* out_residual,
                                         int32_t* out_topk_idx, float* out_topk_w,
                                         int32_t* out_counts, void* stream) {
  if (!h || T < 0) return MOE_EINVAL;
  if (T > h->cfg.T_max) return MOE_ETOOBIG;
  if (T == 0) return MOE_OK;
  const size_t need = layout(h, T).total;
  if (need > MOE_NOALLOC_SCRATCH_BYTES) return MOE_EWORKSPACE;
  void* ws = noalloc_scratch();
  if (!ws) return MOE_ECUDA;
  const int v = check_forward_args(h, T, x, residual, token_ids, out_norm, out_residual, ws,
                                   MOE_NOALLOC_SCRATCH_BYTES, need);
  if (v != MOE_OK) return v;
  return forward_impl(h, T, x, residual, token_ids, out_norm, out_residual, out_topk_idx,
                      out_topk_w, out_counts, static_cast<uint8_t*>(ws),
                      static_cast<cudaStream_t>(stream));
}
