/*
 * moe.h -- C ABI of libmoe.so: a batch-invariant Mixture-of-Experts FFN layer
 * forward for NVIDIA B200 (sm_100a).
 *
 * The layer (one token row t at a time; nothing depends on other rows):
 *   xn    = bf16(RMSNorm(x_t) * g_in)                 RMSNorm, epsilon inside the root
 *   l     = xn W_r^T                                   router Linear, fp32, full K
 *   idx,w = top-k of softmax(l [+ b]) | sigmoid(l) + b | hash(token id)
 *   h     = bf16(SiLU(min(xn W_g^T, c_g)) * clamp(xn W_u^T, -c_u, c_u))   per chosen expert
 *   y     = h W_d^T                                    fp32, full K
 *   acc   = sum_j w_j y_j (slot order) + sum_s y_s (shared, index order), fp32
 *   r     = acc + residual_t;  out_residual = bf16(r);  out_norm = bf16(RMSNorm(r) * g_out)
 * Passages (web pages on MoE numerics, cited by title and section):
 *   RMSNorm ............ linux.do post on MoE variants, "RMSNorm before up-projection"
 *   router ............. nxmr.cn "V4" article, §2.2 (Linear -> softmax -> top-k);
 *                        DeepSeek V4 infra notes §6.3 (sigmoid + balance upper layers,
 *                        hash routing expert = hash(token_id) % n_experts)
 *   selection bias ..... linux.do post, "QuantileBalancing" (s + b > tau)
 *   SwiGLU + clamp ..... DeepSeek V4 infra notes §6.5 "SwiGLU Clamping"
 *   shared experts ..... linux.do post, "共享专家" (always active, added to the routed sum)
 *   combine ............ Fireworks parity post (Chinese translation), Trap 3 and the
 *                        Qwen3.5-MoE case study: all k contributions in fp32, one cast
 *   residual + norm .... same post, Trap 2 (normed, residual = rmsnorm(full_out, residual))
 *   r0..r7 reduction ... same post, Trap 1 (the uniform r0 + r1 + ... + r7 order, fp32)
 *   full-K GEMMs ....... Meituan LongCat parity article, "为什么会不一致" (a full-K
 *                        computation instead of summing split partial results)
 * Variants (moe_config fields):
 *   activation ......... SiTU-GLU units instead of SwiGLU (linux.do post, "SiTU-GLU")
 *   latent ............. router and routed experts at a latent width l, their sum
 *                        projected back (linux.do post, "潜在MoE (Latent MoE)")
 *   weight_format ...... FP4-valued expert weights stored as E4M3, E4M3 x E4M3 expert
 *                        GEMMs (DeepSeek V4 infra notes, §6.2 FP4 QAT)
 *   ep_world, ep_rank .. expert parallelism over ranks, phases moe_ep_* (§6.1 there:
 *                        dispatch -> compute -> combine)
 * Multi-GPU epilogue: moe_reduce_partials_rows over peer memory (moe_peer_*) is the
 * tensor-parallel all-reduce + residual + RMSNorm in the fixed r0..r7 order.
 *
 * Determinism contract.  For every row t, out_norm[t], out_residual[t],
 * out_topk_idx[t] and out_topk_w[t] are bit-identical whatever T is, where
 * the row sits in the batch, what the other rows hold, and how often the
 * call is repeated.  No kernel picks its tiling, split or reduction order
 * from T; there is no split-K and no floating-point atomic.
 *
 * Conventions.
 *  - "bf16" buffers hold raw bfloat16 bit patterns (moe_bf16 = uint16_t).
 *  - All tensor arguments are DEVICE pointers, row-major, densely packed,
 *    16-byte aligned, owned by the caller; the library never frees them.
 *    Weight pointers given to moe_init must stay valid until moe_destroy.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *  - Every call is asynchronous on `stream` unless its comment says it
 *    synchronises.  Nothing throws or aborts across the ABI: every call
 *    returns a moe_status.
 *  - Limits: D % 64 == 0, I % 64 == 0, I_shared % 64 == 0, 1 <= E <= 256,
 *    1 <= k <= min(E, 16), 0 <= n_shared <= 8, 1 <= T_max <= 2^20,
 *    T * max(k, n_shared) * max(D, I) < 2^31.
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t moe_bf16;

typedef enum {
  MOE_OK = 0,
  MOE_EINVAL = -1,        /* bad argument: NULL pointer, negative size, bad enum    */
  MOE_ETOOBIG = -2,       /* T > T_max of the handle                                */
  MOE_EWORKSPACE = -3,    /* workspace smaller than moe_workspace_size()            */
  MOE_EUNSUPPORTED = -4,  /* shape outside the limits above                         */
  MOE_ECUDA = -5,         /* a CUDA runtime call failed (launch, copy, allocation)  */
  MOE_ETIMEOUT = -6,      /* a device-side wait gave up (see moe_get_device_error)  */
  MOE_EINDEX = -7         /* a device-side index check failed (only in a library
                             built with MOE_CHECK_BOUNDS; see moe_get_device_error)  */
} moe_status;

typedef enum {
  MOE_ROUTER_SOFTMAX = 0,       /* keys = logits (+ optional per-expert logit bias);
                                   w_j = softmax prob, / sum over chosen if renormalize */
  MOE_ROUTER_SIGMOID_BIAS = 1,  /* s = sigmoid(logit); keys = s + bias (selection only);
                                   w_j = s_j, / sum over chosen if renormalize          */
  MOE_ROUTER_HASH = 2           /* e_0 = ((id * hash_mult) mod 2^32) mod E,
                                   e_j = (e_0 + j) mod E, w_j = 1/k                     */
} moe_router;

/* The experts' gated unit. */
typedef enum moe_activation {
  MOE_ACT_SWIGLU = 0,    /* SiLU(min(g, gate_clamp_max)) * clamp(u, +-up_clamp)
                            (DeepSeek V4 infra notes §6.5; the clamps may be +INF)  */
  MOE_ACT_SITU_GLU = 1   /* [bg tanh(g / bg) * sigmoid(g)] * [bu tanh(u / bu)],
                            bg = situ_beta_gate, bu = situ_beta_up (linux.do post on
                            MoE variants, "SiTU-GLU": 4 and 25); clamps unused    */
} moe_activation;

/* Format of the expert weights (DeepSeek V4 infra notes, §6.2 FP4 QAT: expert
 * weights are FP4 (E2M1) with one scale per block, dequantised losslessly to
 * FP8, and the experts run FP8 x FP8 GEMMs). */
typedef enum moe_weight_format {
  MOE_WEIGHTS_BF16 = 0,  /* bf16 weights, bf16 x bf16 GEMMs                          */
  MOE_WEIGHTS_FP8 = 1,   /* E4M3 bytes (as moe_quantize_weights_fp4 writes them),
                            E4M3 x E4M3 GEMMs with fp32 accumulation.  Each expert
                            GEMM's input rows are E4M3 with one power-of-two scale
                            per row: e = the smallest integer with max|row| <=
                            448 * 2^e (clamped to [-126, 126]; 0 for a zero row),
                            code = E4M3 round-to-nearest-even of value / 2^e; the
                            row's accumulators are multiplied by 2^e.  The gate/up
                            input is xn (after its bf16 rounding), the down input
                            is h (with a latent width, the routed experts' input
                            is z).  The router GEMM and the latent projections stay
                            bf16.  Needs D, I, I_shared and latent multiples of 128. */
  MOE_WEIGHTS_FP4 = 2    /* FP4 storage: each expert matrix [rows, K] is held as packed
                            E2M1 codes, uint8 [rows, K / 2] (element 2i in the low
                            nibble of byte i, 2i + 1 in the high nibble; bit 3 of a code
                            is the sign, bits 0-2 the index of the magnitude in
                            0, 0.5, 1, 1.5, 2, 3, 4, 6), plus its block exponents
                            (moe_weights.*_exp): one power-of-two scale 2^s per 32
                            consecutive elements of a row, s in [-8, 6].  The expert
                            GEMMs feed the codes to the tensor core's block-scaled
                            E2M1 x E4M3 MMA (kind::mxf8f6f4, one UE8M0 scale 2^s per
                            32 weights, the E4M3 activations with scale 1 and their
                            row scale applied after), every tile operand-swapped with
                            at most 240 tokens; moe_init copies the exponents into the
                            order the GEMMs read them (device memory the handle owns,
                            as many bytes as the exponents).  Each product code * 2^s
                            is an E4M3 value, and on B200 the results are bit for bit
                            those of the E4M3 weights that moe_quantize_weights_fp4
                            writes for the same master weights.  Half a byte per
                            weight (plus 1/32 byte of exponent) instead of one.  Same
                            shape limits as MOE_WEIGHTS_FP8, D and latent multiples of
                            256, and the packed matrices 32-byte aligned.            */
} moe_weight_format;

typedef struct moe_config {
  int D;               /* hidden size                                                  */
  int E;               /* routed experts                                               */
  int k;               /* experts per token                                            */
  int I;               /* routed expert intermediate size                              */
  int n_shared;        /* always-active shared experts (0 allowed)                     */
  int I_shared;        /* shared expert intermediate size                              */
  int T_max;           /* largest T any call will pass                                 */
  int router;          /* moe_router                                                   */
  int renormalize;     /* 1: divide chosen weights by their sum (softmax / sigmoid)    */
  float routed_scale;  /* multiplies every routed weight (1.0 = none)                  */
  float gate_clamp_max;/* SwiGLU gate upper bound (+INF = off); the gate has no lower  */
  float up_clamp;      /* SwiGLU up branch clipped to [-up_clamp, up_clamp] (+INF = off)*/
  float eps;           /* RMSNorm epsilon, inside the square root                      */
  uint32_t hash_mult;  /* multiplicative hash constant for MOE_ROUTER_HASH             */
  int activation;      /* moe_activation of routed and shared experts                  */
  float situ_beta_gate;/* SiTU-GLU gate cap (> 0, finite; read for MOE_ACT_SITU_GLU)    */
  float situ_beta_up;  /* SiTU-GLU up cap (> 0, finite)                                 */
  int latent;          /* latent MoE width l (0 = none; else a multiple of 64, at most
                          16384): the router and the routed experts work on
                          z = bf16(xn W_proj_down^T) of width l, their weighted sum is
                          cast to bf16 once and projected back by W_proj_up; shared
                          experts stay at width D (linux.do post on MoE variants,
                          "潜在MoE (Latent MoE)" and K3's Stable Latent MoE)          */
  int weight_format;   /* moe_weight_format of the routed and shared expert weights     */
  int ep_world;        /* expert parallelism over this many ranks (0 or 1 = none; at most
                          8, dividing E): rank r owns routed experts [r E/ep_world,
                          (r+1) E/ep_world) and its w_gate / w_up / w_down hold only
                          those; router and shared experts are whole on every rank.
                          Such a handle runs the moe_ep_* phases, not moe_layer_forward.
                          Not combined with a latent width (MOE_EUNSUPPORTED), and
                          ep_world * T_max * k must stay below 2^24                   */
  int ep_rank;         /* this rank, 0 <= ep_rank < ep_world                             */
} moe_config;

typedef struct moe_weights {      /* device pointers, caller-owned; L = latent if
                                     latent > 0, else D.  The six expert matrices are
                                     bf16, E4M3 bytes or packed E2M1 codes ([rows, K/2]
                                     bytes), as weight_format says.                   */
  const moe_bf16* w_router;       /* [E, L]      (unused for hash routing)            */
  const float* router_bias;       /* [E] fp32 or NULL: logit bias (softmax) or
                                     selection bias (sigmoid)                         */
  const void* w_gate;             /* [E, I, L]                                        */
  const void* w_up;               /* [E, I, L]                                        */
  const void* w_down;             /* [E, L, I]                                        */
  const void* ws_gate;            /* [S, I_shared, D]  (NULL when n_shared == 0)      */
  const void* ws_up;              /* [S, I_shared, D]                                 */
  const void* ws_down;            /* [S, D, I_shared]                                 */
  const moe_bf16* g_in;           /* [D] input RMSNorm gain                           */
  const moe_bf16* g_out;          /* [D] output RMSNorm gain                          */
  const moe_bf16* w_proj_down;    /* [latent, D] latent down-projection (latent > 0)  */
  const moe_bf16* w_proj_up;      /* [D, latent] latent up-projection (latent > 0)    */
  /* MOE_WEIGHTS_FP4 only (else NULL): the block exponents of the six expert
   * matrices, as moe_quantize_weights_fp4_packed writes them: for a matrix of
   * R rows (all experts stacked: E*I for w_gate / w_up, E*L for w_down, S*I_shared
   * for ws_gate / ws_up, S*D for ws_down) and K columns, uint32 [K / 128, R]:
   * word [c, r] holds the four int8 exponents of row r's 32-element blocks
   * 4c .. 4c + 3, block 4c in the lowest byte. */
  const uint32_t* w_gate_exp;
  const uint32_t* w_up_exp;
  const uint32_t* w_down_exp;
  const uint32_t* ws_gate_exp;
  const uint32_t* ws_up_exp;
  const uint32_t* ws_down_exp;
} moe_weights;

typedef struct moe_handle moe_handle;

/* Kernel stages of one forward, in launch order (one kernel each), as
 * moe_profile_read reports them:
 * 0 rmsnorm_in, 1 router_gemm (not launched for MOE_ROUTER_HASH), 2 router_topk
 * (scores, top-k, weights, per-128-token expert histogram), 3 dispatch (offsets
 * and stable scatter), 4 gather_rows, 5 gemm_gateup_swiglu, 6 gemm_down,
 * 7 combine_norm; with a latent width also 8 latent_down (launched before
 * stage 1), 9 latent_combine and 10 latent_up (both before stage 7); with
 * MOE_WEIGHTS_FP8 also 11 quant_h (h to E4M3 rows, between stages 5 and 6). */
#define MOE_NUM_STAGES 12

/* Validate `cfg`, keep the weight pointers and build the weight TMA
 * descriptors on the current CUDA device.  Allocates handle-owned device
 * memory: the router weights zero-padded to a multiple of 16 rows, and with
 * MOE_WEIGHTS_FP4 the block exponents rearranged as the expert GEMMs read them
 * (as many bytes as the exponents; built by a kernel on the legacy default
 * stream, after which moe_init synchronises the device); the exponent arrays
 * themselves are read only during moe_init.
 * Returns MOE_EINVAL / MOE_EUNSUPPORTED for bad configs (checked before any
 * CUDA call), MOE_ECUDA when a CUDA call fails.  *out is NULL on failure. */
int moe_init(const moe_config* cfg, const moe_weights* w, moe_handle** out);

/* Bytes of device workspace moe_layer_forward needs for T rows (0 < T <= T_max).
 * Returns 0 for a NULL handle or T outside (0, T_max]. */
size_t moe_workspace_size(const moe_handle* h, int T);

/* One layer forward over T rows.
 *   x, residual       [T, D] bf16
 *   token_ids         [T] int32, required for hash routing, else may be NULL
 *   out_norm          [T, D] bf16   bf16(RMSNorm(r) * g_out)
 *   out_residual      [T, D] bf16   bf16(r)
 *   out_topk_idx      [T, k] int32 or NULL: chosen experts, slot order (descending key,
 *                     ties to the lower index)
 *   out_topk_w        [T, k] fp32 or NULL: their weights
 *   out_counts        [E] int32 or NULL: tokens per expert (dropless; no capacity)
 *   workspace         device buffer of >= moe_workspace_size(h, T) bytes, 256-byte
 *                     aligned, not used by any other call in flight
 * T == 0 returns MOE_OK and launches nothing.  Errors: MOE_EINVAL, MOE_ETOOBIG,
 * MOE_EWORKSPACE, MOE_ECUDA (launch failure).  A device-side wait that times
 * out is reported later by moe_get_device_error. */
int moe_layer_forward(moe_handle* h, int T, const moe_bf16* x, const moe_bf16* residual,
                      const int32_t* token_ids, moe_bf16* out_norm, moe_bf16* out_residual,
                      int32_t* out_topk_idx, float* out_topk_w, int32_t* out_counts,
                      void* workspace, size_t ws_bytes, void* stream);

/* Read and clear the device error word the last forward on `workspace` left:
 * MOE_OK; MOE_ETIMEOUT when a bounded device wait gave up; MOE_EINDEX when a
 * device-side index check failed (bounds-checked library only); MOE_ECUDA when
 * the copy failed or the word holds a value no kernel writes.  workspace NULL
 * reads the error word of moe_layer_forward_noalloc's static scratch on the
 * current device.  Synchronises `stream`. */
int moe_get_device_error(moe_handle* h, void* workspace, void* stream);

/* The tensor-parallel epilogue on one GPU (Fireworks parity post, Trap 1 + 2):
 *   r = ((((p_0 + p_1) + p_2) + ...) + p_{P-1}) + residual   every element, fp32,
 *   out_residual = bf16(r), out_norm = bf16(RMSNorm(r) * g).
 * partials: HOST array of P device pointers, each [T, D] bf16; 1 <= P <= 8.
 * residual [T, D] bf16, g [D] bf16, outputs [T, D] bf16.  D % 64 == 0.
 * Needs no handle and no workspace.  Errors: MOE_EINVAL, MOE_EUNSUPPORTED, MOE_ECUDA. */
int moe_reduce_partials(int P, const moe_bf16* const* partials, const moe_bf16* residual,
                        const moe_bf16* g, moe_bf16* out_norm, moe_bf16* out_residual, int T,
                        int D, float eps, void* stream);

/* The same reduction for rows [row0, row0 + rows) only, written to n_out
 * destination pairs (1 <= n_out <= 8): the fused form of the tensor-parallel
 * all-reduce + residual + RMSNorm over NVLink.  With P ranks, rank i passes the
 * P ranks' partial buffers in rank order (its own and its peers', mapped into
 * its address space, e.g. by moe_peer_open), its row slice, and every rank's
 * output buffers: each rank reads all partials of its rows with plain loads,
 * reduces them in the fixed order p = 0 .. P-1, and stores the rows to every
 * rank.  Every rank then holds the same bits as moe_reduce_partials over all T
 * rows on one GPU.  The caller orders the ranks (a barrier after the partials
 * are written, another before they are overwritten); the call itself does not
 * synchronise.  Pointers: [T, D] buffers, 16-byte aligned.  Errors as above. */
int moe_reduce_partials_rows(int P, const moe_bf16* const* partials, const moe_bf16* residual,
                             const moe_bf16* g, int n_out, moe_bf16* const* out_norm,
                             moe_bf16* const* out_residual, int row0, int rows, int D, float eps,
                             void* stream);

/* Bytes of device workspace moe_check_invariance needs for T rows. */
size_t moe_invariance_workspace_size(const moe_handle* h, int T);

/* The bitwise invariance test of the Meituan parity article ("逐 token logprob
 * 一致": compare bit patterns, change one configuration axis at a time):
 * run the forward on all T rows (the reference), then
 *   - on n_splits contiguous chunks (sizes differ by at most one row),
 *   - on the rows in the order perm (perm[i] = source row of row i; NULL = skip),
 *   - `repeats` more times on all T rows,
 * and count output elements (out_norm and out_residual) whose bits differ from
 * the reference.  Synchronises `stream`; writes the count to
 * *out_mismatched_elems.  Returns MOE_ETIMEOUT if any run hit a device timeout. */
int moe_check_invariance(moe_handle* h, int T, const moe_bf16* x, const moe_bf16* residual,
                         const int32_t* token_ids, int n_splits, const int32_t* perm,
                         int repeats, void* workspace, size_t ws_bytes,
                         unsigned long long* out_mismatched_elems, void* stream);

/* Device pointers into a forward's workspace, for stage-by-stage checks.
 * Valid after a forward with the same T and workspace has completed. */
typedef struct moe_views {
  const moe_bf16* xn;          /* [T, D]          normalised input                   */
  const float* logits;         /* [T, E_pad]      router logits (NULL for hash)      */
  int E_pad;                   /* row pitch of logits (E rounded up to 16)           */
  const int32_t* topk_idx;     /* [T, k]          copy used inside the layer         */
  const float* topk_w;         /* [T, k]                                             */
  const int32_t* counts;       /* [E]                                                */
  const int32_t* offsets;      /* [E + 1]         exclusive prefix of counts         */
  const int32_t* src_token;    /* [T * k]         grouped row p -> token             */
  const int32_t* dest_row;     /* [T * k]         grouped row p -> t * k + slot      */
  const moe_bf16* h_routed;    /* [T * k, I]      grouped order                      */
  const moe_bf16* h_shared;    /* [S, T, I_shared]                                   */
  const float* y_slot;         /* [T, k, L]       routed expert outputs, slot order  */
  const float* y_shared;       /* [S, T, D]                                          */
  const moe_bf16* z;           /* [T, latent]     latent input (NULL unless latent)  */
  const moe_bf16* agg;         /* [T, latent]     bf16 routed sum (NULL unless latent)*/
  const float* y_latent;       /* [T, D]          up-projected sum (NULL unless latent)*/
  /* MOE_WEIGHTS_FP8 only (NULL otherwise): E4M3 expert inputs and the power-of-two
   * exponent of each row (row value = code value * 2^exp).                      */
  const uint8_t* xq;           /* [T, D]          xn as E4M3                          */
  const int8_t* xq_exp;        /* [T]                                                 */
  const uint8_t* hq_routed;    /* [T * k, I]      h_routed as E4M3, grouped order     */
  const int8_t* hq_routed_exp; /* [T * k]                                             */
  const uint8_t* hq_shared;    /* [S, T, I_shared]                                    */
  const int8_t* hq_shared_exp; /* [S, T]                                              */
} moe_views;

int moe_workspace_views(const moe_handle* h, int T, void* workspace, moe_views* out);

/* Per-stage device timing.  stage_mask selects stages (bit s = stage s;
 * 0 = off; (1 << MOE_NUM_STAGES) - 1 = all).  While enabled, every forward
 * records a CUDA event pair on its stream around each selected stage's launch.
 * moe_profile_read synchronises, adds each stage's elapsed time over all
 * forwards since the last read into ms[MOE_NUM_STAGES] (milliseconds) and
 * launches[MOE_NUM_STAGES] (kernels launched per stage, selected stages only),
 * then resets.  At most 256 forwards are recorded between reads; later ones
 * are not timed. */
int moe_profile_enable(moe_handle* h, int stage_mask);
int moe_profile_read(moe_handle* h, float* ms, int* launches);

/* Kernels launched by one forward with this T (for launch accounting). */
int moe_forward_launch_count(const moe_handle* h, int T);

/* Fault path check: launch one CTA that waits on a flag nothing sets, with a
 * time limit of `limit_us` microseconds (1..1000000).  Returns MOE_ETIMEOUT
 * when the wait gave up as designed (the CUDA context stays usable), MOE_OK
 * if the flag was seen, MOE_EINVAL / MOE_ECUDA otherwise.  Synchronises `stream`. */
int moe_selftest_wait_timeout(int limit_us, void* stream);

/* Forward without any allocation, for callers that cannot call cudaMalloc:
 * a plugin or custom-op enqueue path that must not allocate, a process whose
 * own allocator already holds all free device memory, or a latency-critical
 * path that cannot afford cudaMalloc's device-wide synchronisation.  (The
 * source pages have no counterpart of this entry point.)
 * Same arguments and results as moe_layer_forward, minus the workspace: the
 * scratch is one static device array of MOE_NOALLOC_SCRATCH_BYTES (32 MiB)
 * that every GPU loading the library holds until the process exits.  T must
 * satisfy moe_workspace_size(h, T) <= MOE_NOALLOC_SCRATCH_BYTES (decode-sized
 * batches: about 280 tokens for D=2048, top-6, I=1408, 2 shared experts);
 * larger T returns MOE_EWORKSPACE and launches nothing.
 * The first call on each device looks up the array's device address with that
 * device current; make that first call before any stream capture.
 * Every call shares the array and it keeps the last call's contents; the
 * only value that must start at zero (the device error word) is cleared by
 * the call's first kernel.  Calls whose kernels overlap on the GPU (other
 * streams, or another thread's call) race on the array: serialise them.
 * A device-side wait time-out (or, in the bounds-checked library, an index
 * fault) is recorded in the array's error word, which the call itself does
 * not read: moe_get_device_error(h, NULL, stream) reads and clears it on the
 * current device. */
#define MOE_NOALLOC_SCRATCH_BYTES (32u << 20)
int moe_layer_forward_noalloc(moe_handle* h, int T, const moe_bf16* x, const moe_bf16* residual,
                              const int32_t* token_ids, moe_bf16* out_norm,
                              moe_bf16* out_residual, int32_t* out_topk_idx, float* out_topk_w,
                              int32_t* out_counts, void* stream);

/* FP4 weight quantisation (DeepSeek V4 infra notes, §6.2 FP4 QAT: master
 * weights -> FP4 (E2M1) with a scale per block -> lossless FP8).  `w` is a
 * row-major [rows, K] bf16 matrix (the master weights), K a multiple of 32,
 * the contraction axis of the GEMM that will read it.  Every block of 32
 * consecutive elements of a row gets the power-of-two scale 2^s with s the
 * smallest integer such that max|block| <= 6 * 2^s, clamped to [-8, 6] (-8 for
 * an all-zero block); each element becomes q = the E2M1 value (0, 0.5, 1, 1.5,
 * 2, 3, 4, 6, signed) nearest to w / 2^s, ties to the even code, and
 * w8[i] = the E4M3 code of q * 2^s, which that range of s keeps exact.
 * block_exp (NULL allowed) receives s, [rows, K / 32] int8.  Pointers are
 * device memory the caller owns; w and w8 16-byte aligned.  Asynchronous on
 * `stream`.  Errors: MOE_EINVAL (NULL, misaligned, rows < 0, K not a positive
 * multiple of 32), MOE_ECUDA (launch). */
int moe_quantize_weights_fp4(const moe_bf16* w, uint8_t* w8, int8_t* block_exp, long long rows, int K,
                             void* stream);

/* The same FP4 quantisation (DeepSeek V4 infra notes, §6.2: FP4 (E2M1) weights
 * with one scale per block) written in its storage form for
 * MOE_WEIGHTS_FP4: `packed` uint8 [rows, K / 2], two E2M1 codes per byte (element
 * 2i in the low nibble; sign in bit 3, magnitude index in bits 0-2; a value that
 * rounds to zero keeps its sign), and `exps` uint32 [K / 128, rows], word [c, r]
 * holding the int8 exponents s of row r's blocks 4c .. 4c + 3 (block 4c in the
 * lowest byte).  Block scale and rounding exactly as moe_quantize_weights_fp4, so
 * code * 2^s is the E4M3 value that function writes.  K must be a multiple of
 * 128; all pointers 16-byte aligned device memory.  Asynchronous on `stream`.
 * Errors: MOE_EINVAL (NULL, misaligned, rows < 0, K not a positive multiple of
 * 128), MOE_ECUDA (launch). */
int moe_quantize_weights_fp4_packed(const moe_bf16* w, uint8_t* packed, uint32_t* exps, long long rows,
                                    int K, void* stream);

/* ------------------------------------------------------------------------
 * Expert parallelism (DeepSeek V4 infra notes, §6.1: dispatch -> compute ->
 * combine, with tokens sent to the rank that holds their expert and results
 * sent back; the Fireworks parity post, Trap 3 and its case study: the k
 * contributions of a token are added in fp32, in slot order, on the token's
 * own rank, never in bf16 or in arrival order).
 *
 * Every rank holds its own T tokens (T may differ between ranks, each at most
 * T_max) and one exchange buffer of moe_ep_exchange_size bytes that the other
 * ranks can address (moe_peer_alloc / moe_peer_open across processes, or plain
 * device memory when several ranks share one device and one process).  A step
 * is four calls on each rank, in this order, with every rank's call of one
 * phase complete before any rank's call of the next phase reads what it wrote
 * (a device barrier such as moe_peer_barrier between phases, or stream order
 * when the ranks share a stream):
 *   moe_ep_route    RMSNorm, router, top-k, the stable grouping of the rank's
 *                   (token, slot) rows by expert; its per-expert counts go to
 *                   its own exchange buffer.
 *   moe_ep_send     from every rank's counts, the row each (token, slot) takes at
 *                   its expert's owner (owner's experts in order; inside an
 *                   expert, source ranks in order; inside a source rank, tokens
 *                   in order, then slots); the input row (bf16, or E4M3 and its
 *                   exponent) and its return address are stored there.
 *   moe_ep_experts  the owner's routed experts over the rows it received and the
 *                   shared experts over its own tokens; each routed output row
 *                   (fp32) is stored into its source rank's exchange buffer at
 *                   that token's slot row.
 *   moe_ep_combine  the fixed slot-order combine + residual + RMSNorm of the
 *                   rank's own tokens (as moe_layer_forward).
 * Each (token, slot) row goes through the same full-K GEMMs as in
 * moe_layer_forward, whose bits do not depend on which rows share a tile, so
 * every rank's outputs are bit for bit those of moe_layer_forward on its
 * tokens with all experts on one device.
 * `peers` lists the exchange buffer of every rank (index = rank) as addresses
 * valid on this rank.  `workspace` is this rank's (moe_workspace_size for its
 * T), kept across the four calls.  Errors: MOE_EINVAL (NULL, wrong rank
 * count, not an EP handle), MOE_ETOOBIG, MOE_EWORKSPACE, MOE_ECUDA.  No call
 * synchronises.
 * ------------------------------------------------------------------------ */
typedef struct moe_ep_peers {
  void* xbuf[8];
} moe_ep_peers;

size_t moe_ep_exchange_size(const moe_handle* h);
int moe_ep_route(moe_handle* h, int T, const moe_bf16* x, const int32_t* token_ids, void* xbuf_self,
                 void* workspace, size_t ws_bytes, void* stream);
int moe_ep_send(moe_handle* h, int T, const moe_ep_peers* peers, void* workspace, size_t ws_bytes,
                void* stream);
int moe_ep_experts(moe_handle* h, int T, const moe_ep_peers* peers, void* workspace, size_t ws_bytes,
                   void* stream);
int moe_ep_combine(moe_handle* h, int T, const moe_bf16* residual, void* xbuf_self, moe_bf16* out_norm,
                   moe_bf16* out_residual, int32_t* out_topk_idx, float* out_topk_w, void* workspace,
                   size_t ws_bytes, void* stream);

/* Waves (DeepSeek V4 infra notes, §6.1 "MegaMoE": the experts are scheduled in
 * waves, each covering a few of them, so that the rows of the next wave travel
 * while the current wave computes).  Wave w of n (1 <= n <= E / ep_world,
 * 0 <= w < n) covers local experts [w * E_loc / n, (w + 1) * E_loc / n) of
 * every owner, E_loc = E / ep_world; the shared experts run in wave 0.
 *   moe_ep_send_wave     the part of moe_ep_send whose rows go to the wave's
 *                        experts: the same rows, return addresses and bytes at
 *                        the same places.
 *   moe_ep_experts_wave  moe_ep_experts over the wave's experts only (their
 *                        received rows, which the wave's send of every rank
 *                        must have completed), plus the shared experts in wave 0.
 * moe_ep_send and moe_ep_experts are wave 0 of 1.  Running every wave's send
 * and experts (in any interleaving that keeps each wave's experts after every
 * rank's send of that wave, and one rank's experts calls in wave order) stores
 * the same bits as the two whole calls, because every (token, slot) row still
 * meets the same weights in the same full-K GEMM and lands in the same slot
 * row.  The point of the split: the send of wave w + 1 may run on another
 * stream while the GEMMs of wave w run.  A rank's workspace holds the plan of
 * one wave at a time, so its experts calls must not overlap one another.
 * Errors: as moe_ep_send / moe_ep_experts, and MOE_EINVAL for a wave outside
 * [0, n) or n outside [1, E_loc]. */
int moe_ep_send_wave(moe_handle* h, int T, const moe_ep_peers* peers, int wave, int n_waves, void* workspace,
                     size_t ws_bytes, void* stream);
int moe_ep_experts_wave(moe_handle* h, int T, const moe_ep_peers* peers, int wave, int n_waves,
                        void* workspace, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Peer memory for the tensor-parallel epilogue (one process per GPU).
 *
 * moe_peer_alloc allocates `bytes` of zeroed device memory on the current
 * device and exports it: `handle` (MOE_PEER_HANDLE_BYTES bytes, host memory the
 * caller owns) is the CUDA IPC handle of the allocation, to be sent to the
 * other ranks of one node by any host channel.  The allocation is 256-byte
 * aligned and owned by the caller: release it with moe_peer_free after every
 * rank has closed its mapping.  Errors: MOE_EINVAL (NULL or bytes == 0),
 * MOE_ECUDA (allocation or export failed; *dptr is NULL).
 *
 * moe_peer_open maps another process's exported allocation into this process
 * (on the current device, with peer access enabled) and writes its address to
 * *dptr; moe_peer_close unmaps it.  Opening a handle of this same process is
 * an error (MOE_ECUDA): use the exporter's own pointer.
 *
 * moe_peer_barrier is a device-side barrier of `world` ranks (1 <= world <= 8)
 * on `stream`: flags[r] is the address (in this process) of rank r's array of
 * `world` uint32 flag words, zero when allocated.  One thread per rank first
 * makes this GPU's earlier writes (the stream's previous kernels, local and
 * peer stores) visible at system scope, then writes `epoch` to slot `rank` of
 * every rank's array, and waits until every slot of its own array holds a
 * value >= epoch (wrap-around compare).  All ranks call it with the same epoch
 * sequence, starting at 1 and growing by one per call.  Each wait gives up
 * after `limit_us` microseconds (1..60000000): it then stores 1 to the device
 * int *err (which the caller zeroes and reads), and returns; the CUDA context
 * stays usable and later kernels run as usual.  Errors: MOE_EINVAL, MOE_ECUDA
 * (launch failure).  The call does not synchronise. */
#define MOE_PEER_HANDLE_BYTES 64
int moe_peer_alloc(size_t bytes, void** dptr, unsigned char* handle);
int moe_peer_free(void* dptr);
int moe_peer_open(const unsigned char* handle, void** dptr);
int moe_peer_close(void* dptr);
int moe_peer_barrier(int world, int rank, uint32_t* const* flags, uint32_t epoch, int* err, int limit_us,
                     void* stream);

int moe_destroy(moe_handle* h);
const char* moe_status_string(int status);

#ifdef __cplusplus
}
#endif
#endif /* MOE_H_ */
