"""Oracle: a plain, slow, fp64 CPU statement of the batch-invariant MoE layer forward.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute this module: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code with the CUDA library and does not import it.

Every step follows a passage of the source pages, cited by page title and
section.  The pages (web articles, quoted here by short name):

* [FW]  "MoE 模型中的訓練與推論一致性：數值漂移發生之處" -- a translation of the
        Fireworks AI post on train/inference parity in MoE models
        (easyvibecoding.app/curated/746).
* [LC]  "美团把训练和推理的概率做到逐位相同:分歧藏在一个加法顺序里"
        (bbs.huaweicloud.com/blogs/524918).
* [DS]  "6 基建与训练稳定性优化" -- DeepSeek V4 infrastructure notes
        (liyongzhi.xyz/files/deepseek_v4/sections/06-infra.html).
* [LD]  The linux.do post on MoE FLOPs, parameters and variants
        (feedbbs.com/linuxdo/72580).
* [V4]  The nxmr.cn article on a "V4" MoE model (nxmr.cn/news/146660).

The layer, in order:
  1. input RMSNorm                       [LD] "RMSNorm before up-projection"
  2. router logits  l = xn W_r^T         [DS] §6.3 "普通路由" (scores = W·h);
                                          [V4] §2.2 (a Linear layer, logits per expert)
  3. scores + top-k                      softmax [V4] §2.2; sigmoid + per-expert
                                          bias [DS] §6.3 (upper layers), [LD] "QB"
                                          (s + b > tau); hash [DS] §6.3
  4. expert histogram, no capacity       [LD] "MoE是如何影响输出确定性的" (token
                                          dropping is batch dependent: none here)
  5. stable permute (dispatch)           [DS] §6.1 (dispatch -> compute -> combine)
  6. routed + shared SwiGLU experts      [DS] §6.5, [LD] "SiTU-GLU" (SwiGLU form),
                                          [LD] "共享专家"; or SiTU-GLU experts
                                          ([LD] "SiTU-GLU", beta 4 / 25)
  7. weighted combine in fp32, one cast  [FW] Trap 3 and the case study ("standard
                                          path": all k contributions kept in fp32,
                                          weighted sum, one final cast)
  8. residual add + RMSNorm epilogue     [FW] Trap 2 / Trap 3 (rmsnorm(full_out + residual))
  9. fixed r0..r7 partial reduction      [FW] Trap 1 (Lamport kernel order)
  FP4 expert weights (optional)          [DS] §6.2 "FP4 QAT": weights FP4 (E2M1) with a
                                          scale per block, dequantised losslessly to
                                          FP8, FP8 x FP8 expert GEMMs (activations
                                          E4M3 with a power-of-two scale per row)
  Latent MoE (optional)                  [LD] "潜在MoE (Latent MoE)", K3 flow: the
                                          router and routed experts read
                                          z = bf16(xn W_down^T); their weighted
                                          sum is cast once and projected back by
                                          W_up; shared experts stay at full width

Precision.  Every floating-point step runs in fp64, on the bf16-rounded values
the GPU path reads (x, residual, weights, xn between steps 1 and 2/6, h between
the two expert matmuls).  Rounding to bf16 is done directly from fp64 (round to
nearest, ties to even), never through fp32.  One exception: step 9, whose
precision the pages fix (both all-reduce orders accumulate in FP32, [FW] Trap
1), is emulated in IEEE fp32 left to right.

Forced routing.  ``moe_layer`` can take the top-k indices from the caller
(``force_idx``) instead of choosing them, with the weights still computed from
the oracle's own scores of those experts.  A token whose top-k is decided by a
near tie (or by an xn element that sits on a bf16 rounding boundary) may
legitimately route differently on another implementation; with its indices
forced, the rest of the layer for that token can still be checked.

Readings of points the pages leave open (each is also listed in the design
notes): epsilon inside the square root; gains g_in = g_out = 1 unless given;
ties in top-k go to the lower expert index and slots are ordered by
descending key; the sigmoid bias only selects (weights use the unbiased
score); a softmax logit bias, when given, is added to the logits before the
softmax; hash routing takes e_0 = ((id * mult) mod 2^32) mod E and
e_j = (e_0 + j) mod E with weight 1/k; the clamp bounds the gate from above
only and the up branch on both sides; routed weights are multiplied by
``routed_scale``; the routed sum is taken in slot order, then the shared
experts in index order, then the residual is added.
"""
from __future__ import annotations

import numpy as np

ROUTER_SOFTMAX, ROUTER_SIGMOID_BIAS, ROUTER_HASH = 0, 1, 2

# Multiply-adds performed by expert matmuls since the last reset (FLOP pin).
MAC_COUNTER = [0]


# ----------------------------------------------------------------- bf16 data
def bf16_bits_to_f64(bits) -> np.ndarray:
    """Exact value of bf16 bit patterns."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def round_bf16(a) -> np.ndarray:
    """Round fp64 values to the nearest bf16 value, ties to even (fp64 result).

    bf16 keeps 8 significant bits and fp32's exponent range.  Writing
    a = m * 2^e with 0.5 <= |m| < 1, the rounding quantum is 2^(e-8), but
    never finer than the subnormal spacing 2^-133.  np.rint rounds half to
    even and the power-of-two scalings are exact, so this is one rounding.
    """
    a = np.asarray(a, dtype=np.float64)
    _, e = np.frexp(a)
    q = np.maximum(e.astype(np.int64) - 8, -133)
    r = np.ldexp(np.rint(np.ldexp(a, -q)), q)
    big = np.abs(r) > 3.3895313892515355e38  # (2 - 2^-7) * 2^127, the largest bf16
    return np.where(big, np.copysign(np.inf, a), r)


def f64_to_bf16_bits(a) -> np.ndarray:
    """bf16 bit pattern of values that are already bf16-representable."""
    f = np.asarray(a, dtype=np.float64).astype(np.float32)
    return (f.view(np.uint32) >> 16).astype(np.uint16)


# -------------------------------------------------------------- 1. RMSNorm
def rmsnorm(x, g, eps: float) -> np.ndarray:
    """RMSNorm(x) = g * x / sqrt(mean(x^2) + eps), over the last axis, fp64.

    [LD] "RMSNorm before up-projection": RMS(x) = sqrt((1/d) sum x_i^2 + eps),
    x_hat = x / RMS(x), y = g * x_hat (the epsilon sits inside the root).
    """
    x = np.asarray(x, dtype=np.float64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return np.asarray(g, dtype=np.float64) * (x / np.sqrt(ms + eps))


def xn_bf16(x, g, eps: float) -> np.ndarray:
    """xn = bf16(g * x / sqrt(mean(x^2) + eps)): the input RMSNorm of [LD]
    "RMSNorm before up-projection" in fp64, rounded once to bf16 (the
    activation the router and the expert matmuls read)."""
    return round_bf16(rmsnorm(x, g, eps))


# ------------------------------------------------------- 2-3. router, top-k
def router_logits(xn, w_router) -> np.ndarray:
    """l[t, e] = sum_d xn[t, d] * W_r[e, d]: the router Linear ([V4] §2.2;
    [DS] §6.3 "scores = W·h"), full K accumulated at once."""
    return np.asarray(xn, np.float64) @ np.asarray(w_router, np.float64).T


def topk_desc(keys, k: int) -> np.ndarray:
    """Indices of the k largest keys per row, largest first; equal keys go to
    the lower index; NaN ranks below every number.  (A stable sort of the
    negated keys keeps equal keys in ascending index order.)"""
    keys = np.asarray(keys, np.float64)
    neg = np.where(np.isnan(keys), np.inf, -keys)
    return np.argsort(neg, axis=-1, kind="stable")[..., :k].astype(np.int64)


def softmax(z) -> np.ndarray:
    z = np.asarray(z, np.float64)
    m = np.max(z, axis=-1, keepdims=True)
    p = np.exp(z - m)
    return p / np.sum(p, axis=-1, keepdims=True)


def sigmoid(z) -> np.ndarray:
    return 1.0 / (1.0 + np.exp(-np.asarray(z, np.float64)))


def route_softmax(logits, k: int, renormalize: bool, routed_scale: float, logit_bias=None, idx=None):
    """Softmax router ([V4] §2.2: Linear -> logits -> softmax weights -> top-k).

    Optional logit bias b (a per-expert offset added to the logits, used for
    the skewed workload).  Keys are the probabilities p; weights are p_j,
    divided by the sum over the chosen k when ``renormalize``, times
    ``routed_scale``.  ``idx`` (optional, [T,k]) replaces the top-k choice.
    Returns (idx [T,k], w [T,k], keys [T,E]).
    """
    z = np.asarray(logits, np.float64)
    if logit_bias is not None:
        z = z + np.asarray(logit_bias, np.float64)
    p = softmax(z)
    idx = topk_desc(p, k) if idx is None else np.asarray(idx, np.int64)
    w = np.take_along_axis(p, idx, axis=-1)
    if renormalize:
        w = w / np.sum(w, axis=-1, keepdims=True)
    return idx, w * routed_scale, p


def route_sigmoid_bias(logits, bias, k: int, renormalize: bool, routed_scale: float, idx=None):
    """Sigmoid scores with a per-expert balancing bias ([DS] §6.3: upper layers
    keep "sigmoid + balance"; [LD] "QuantileBalancing": expert e enters token
    t's top-k when s_{t,e} + b_e exceeds the boundary).

    The bias only selects: keys are s + b, weights are the unbiased s_j,
    normalised over the chosen k when ``renormalize``, times ``routed_scale``.
    ``idx`` (optional, [T,k]) replaces the top-k choice.
    """
    s = sigmoid(logits)
    keys = s + (0.0 if bias is None else np.asarray(bias, np.float64))
    idx = topk_desc(keys, k) if idx is None else np.asarray(idx, np.int64)
    w = np.take_along_axis(s, idx, axis=-1)
    if renormalize:
        w = w / np.sum(w, axis=-1, keepdims=True)
    return idx, w * routed_scale, keys


def hash_expert0(token_ids, E: int, mult: int) -> np.ndarray:
    """[DS] §6.3 "Hash Routing": expert_id = hash(token_id) % n_experts, with
    the multiplicative hash h(id) = (id * mult) mod 2^32."""
    ids = np.asarray(token_ids, np.int64).astype(np.uint64)
    h = (ids * np.uint64(mult)) & np.uint64(0xFFFFFFFF)
    return (h % np.uint64(E)).astype(np.int64)


def route_hash(token_ids, E: int, k: int, mult: int, routed_scale: float):
    """Hash routing with k experts: e_j = (e_0 + j) mod E (distinct experts), no
    router parameters, equal weights 1/k times ``routed_scale``."""
    e0 = hash_expert0(token_ids, E, mult)
    idx = (e0[:, None] + np.arange(k)[None, :]) % E
    w = np.full(idx.shape, routed_scale / k, np.float64)
    return idx.astype(np.int64), w, None


def route(cfg, logits, bias, token_ids, force_idx=None):
    """Dispatch on the router variant; returns (idx, w, keys).  ``force_idx``
    ([T,k], optional) replaces the top-k choice; the weights are then those
    the router gives the forced experts."""
    if cfg.router == ROUTER_SOFTMAX:
        return route_softmax(logits, cfg.k, bool(cfg.renormalize), cfg.routed_scale, bias, force_idx)
    if cfg.router == ROUTER_SIGMOID_BIAS:
        return route_sigmoid_bias(logits, bias, cfg.k, bool(cfg.renormalize), cfg.routed_scale, force_idx)
    if cfg.router == ROUTER_HASH:
        idx, w, keys = route_hash(token_ids, cfg.E, cfg.k, cfg.hash_mult, cfg.routed_scale)
        return (idx if force_idx is None else np.asarray(force_idx, np.int64)), w, keys
    raise ValueError(f"unknown router {cfg.router}")


def topk_margin(keys, k: int) -> np.ndarray:
    """key of the k-th chosen expert minus the (k+1)-th largest key: the
    boundary tau_t of [LD] "QuantileBalancing" seen from the chosen side.
    A token whose margin is tiny can flip experts under any perturbation
    ([LD] "MoE是如何影响输出确定性的")."""
    if keys is None:
        return None
    keys = np.asarray(keys, np.float64)
    if k >= keys.shape[-1]:
        return np.full(keys.shape[0], np.inf)
    s = -np.sort(-np.where(np.isnan(keys), -np.inf, keys), axis=-1)
    return s[:, k - 1] - s[:, k]


# --------------------------------------------------- 4-5. histogram, permute
def expert_histogram(idx, E: int) -> np.ndarray:
    """counts[e] = number of (token, slot) pairs routed to e.  Dropless: no
    capacity, so no token depends on the rest of the batch."""
    return np.bincount(np.asarray(idx).ravel(), minlength=E).astype(np.int64)


def stable_permute(idx, E: int):
    """Group (token, slot) pairs by expert; inside expert e's segment the rows
    are in ascending token order (a token picks an expert at most once).

    Returns offsets [E+1] (exclusive prefix of the histogram), perm_token and
    perm_slot [T*k] (row p of the grouped order holds token perm_token[p],
    slot perm_slot[p]) and pos [T, k] (the inverse map).
    """
    idx = np.asarray(idx, np.int64)
    T, k = idx.shape
    counts = expert_histogram(idx, E)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    flat = idx.ravel()                       # flat position f = t*k + j
    order = np.argsort(flat, kind="stable")  # by expert, then by f (i.e. by t)
    perm_token = order // k
    perm_slot = order % k
    pos = np.empty(T * k, np.int64)
    pos[order] = np.arange(T * k)
    return offsets, perm_token, perm_slot, pos.reshape(T, k)


# -------------------------------------------------------------- 6. experts
def swiglu(g, u, gate_clamp_max: float = np.inf, up_clamp: float = np.inf) -> np.ndarray:
    """SwiGLU(x) = SiLU(W_g x) * (W_u x) with Swish(a) = a * sigmoid(a)
    ([LD] "SiTU-GLU", SwiGLU form); with the clamp of [DS] §6.5,
    SiLU(clamp(W_g x, max=c_g)) * clamp(W_u x, -c_u, c_u)."""
    g = np.minimum(np.asarray(g, np.float64), gate_clamp_max)
    u = np.clip(np.asarray(u, np.float64), -up_clamp, up_clamp)
    return g * sigmoid(g) * u


ACT_SWIGLU = 0
ACT_SITU_GLU = 1


def situ_glu(g, u, beta_g: float = 4.0, beta_u: float = 25.0) -> np.ndarray:
    """SiTU-GLU ([LD] "SiTU-GLU", the K3 report's formula as the post quotes
    it): [beta_g tanh(W_g x / beta_g) * Sigmoid(W_g x)] * [beta_u tanh(W_u x /
    beta_u)], a soft cap on both branches (the post gives beta_g = 4 for the
    gate and beta_u = 25 for the up branch), so |h| < beta_g * beta_u."""
    g = np.asarray(g, np.float64)
    u = np.asarray(u, np.float64)
    return (beta_g * np.tanh(g / beta_g) * sigmoid(g)) * (beta_u * np.tanh(u / beta_u))


def glu_unit(g, u, act: int = ACT_SWIGLU, gate_clamp_max: float = np.inf, up_clamp: float = np.inf,
             beta_g: float = 4.0, beta_u: float = 25.0) -> np.ndarray:
    """The expert's gated unit: SwiGLU (with the optional clamp) or SiTU-GLU."""
    if act == ACT_SITU_GLU:
        return situ_glu(g, u, beta_g, beta_u)
    return swiglu(g, u, gate_clamp_max, up_clamp)


def unit_args(cfg) -> dict:
    """glu_unit keyword arguments of a layer configuration (SwiGLU when the
    configuration names no activation)."""
    return dict(act=getattr(cfg, "activation", ACT_SWIGLU), gate_clamp_max=cfg.gate_clamp_max,
                up_clamp=cfg.up_clamp, beta_g=getattr(cfg, "situ_beta_gate", 4.0),
                beta_u=getattr(cfg, "situ_beta_up", 25.0))


def expert_ffn(xn_rows, w_gate, w_up, w_down, gate_clamp_max=np.inf, up_clamp=np.inf,
               act: int = ACT_SWIGLU, beta_g: float = 4.0, beta_u: float = 25.0):
    """One gated expert on a block of rows: g = xn W_g^T, u = xn W_u^T (full
    K = D), h = bf16(unit(g, u)) with the SwiGLU or SiTU-GLU unit, y = h W_d^T
    (full K = I).  Returns (h, y)."""
    x = np.asarray(xn_rows, np.float64)
    Wg = np.asarray(w_gate, np.float64)
    Wu = np.asarray(w_up, np.float64)
    Wd = np.asarray(w_down, np.float64)
    n, D = x.shape
    I = Wg.shape[0]
    MAC_COUNTER[0] += n * (2 * D * I + I * Wd.shape[0])
    h = round_bf16(glu_unit(x @ Wg.T, x @ Wu.T, act, gate_clamp_max, up_clamp, beta_g, beta_u))
    return h, h @ Wd.T


# ------------------------------------------- FP4 expert weights, FP8 compute
# [DS] §6.2 "FP4 QAT": expert weights are quantised from the master weights to
# FP4 (E2M1) with one scale factor per block; FP4 -> FP8 dequantisation is
# lossless (the 16 FP4 values times the block's scale fit FP8 exactly); the
# forward is an FP8 x FP8 GEMM.  Readings where the page is silent: the block
# is 32 consecutive elements along the contraction axis (the last axis of
# every weight here) and its scale is a power of two 2^s; the FP8 format is
# E4M3; activations enter each expert GEMM as E4M3 with one power-of-two
# scale per row (row-local, so batch-invariant); products accumulate exactly
# and the row scale is applied to the sum.  Every quantisation step divides by
# a power of two (exact) and rounds to nearest, ties to even.
# WEIGHTS_FP4 is the storage form of the same FP4 weights ([DS] §6.2: FP4 with
# a scale per block, dequantised losslessly to FP8): its GEMMs read the same FP8
# values, so the oracle computes it exactly as WEIGHTS_FP8.
WEIGHTS_BF16, WEIGHTS_FP8, WEIGHTS_FP4 = 0, 1, 2
E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])   # magnitudes, code order
FP4_BLOCK = 32
FP4_SCALE_MIN, FP4_SCALE_MAX = -8, 6     # 2^s keeps every q * 2^s an E4M3 value
E4M3_MAX = 448.0
ACT_EXP_MIN, ACT_EXP_MAX = -126, 126


def round_e2m1(x) -> np.ndarray:
    """Nearest E2M1 value to each x (ties to the even code, i.e. the grid
    point whose index in E2M1_GRID is even); beyond 6 the nearest is 6."""
    x = np.asarray(x, np.float64)
    mag = np.abs(x)
    d = np.abs(mag[..., None] - E2M1_GRID)                 # distance to every grid point
    best = d.min(axis=-1, keepdims=True)
    cand = d == best                                       # one or two nearest points
    even = cand & (np.arange(8) % 2 == 0)
    pick = np.where(even.any(axis=-1), even.argmax(axis=-1), cand.argmax(axis=-1))
    return np.copysign(E2M1_GRID[pick], x)


def fp4_block_exponent(amax) -> np.ndarray:
    """Smallest integer s with amax <= 6 * 2^s, clamped to [-8, 6] (amax = 0
    gives -8).  Written with frexp: amax = m 2^E, m in [0.5, 1); 6 * 2^(E-3) =
    0.75 * 2^E, so s = E - 3 when m <= 0.75, else E - 2."""
    amax = np.asarray(amax, np.float64)
    m, E = np.frexp(amax)
    s = np.where(m <= 0.75, E - 3, E - 2)
    s = np.where(amax == 0, FP4_SCALE_MIN, s)
    return np.clip(s, FP4_SCALE_MIN, FP4_SCALE_MAX).astype(np.int64)


def quantize_weights_fp4(w, block: int = FP4_BLOCK):
    """Master weights -> FP4: for each block of ``block`` consecutive elements
    of the last axis, s = fp4_block_exponent(max |w|) and q = round_e2m1(w / 2^s).
    Returns (q, s) with s of shape [..., K / block]."""
    w = np.asarray(w, np.float64)
    K = w.shape[-1]
    if K % block:
        raise ValueError("the contraction axis must be a multiple of the block")
    wb = w.reshape(w.shape[:-1] + (K // block, block))
    s = fp4_block_exponent(np.abs(wb).max(axis=-1))
    q = round_e2m1(wb / np.exp2(s)[..., None])
    return q.reshape(w.shape), s


def dequantize_fp4(q, s, block: int = FP4_BLOCK) -> np.ndarray:
    """FP4 -> FP8 values: q * 2^s per block (exact; every result is an E4M3 value)."""
    q = np.asarray(q, np.float64)
    K = q.shape[-1]
    qb = q.reshape(q.shape[:-1] + (K // block, block))
    return (qb * np.exp2(np.asarray(s))[..., None]).reshape(q.shape)


def fp4_weights_as_fp8(w, block: int = FP4_BLOCK) -> np.ndarray:
    """The FP8 operand values the expert GEMMs read for master weights w."""
    return dequantize_fp4(*quantize_weights_fp4(w, block), block)


def e2m1_codes(q) -> np.ndarray:
    """4-bit E2M1 code of FP4 values (sign bit 3, then the index of the
    magnitude in E2M1_GRID: exponent bits 2-1, mantissa bit 0)."""
    q = np.asarray(q, np.float64)
    mag = np.abs(q)
    idx = np.searchsorted(E2M1_GRID, mag)
    if not np.array_equal(E2M1_GRID[np.minimum(idx, 7)], mag):
        raise ValueError("not E2M1 values")
    return (idx | np.where(np.signbit(q), 8, 0)).astype(np.uint8)


def pack_fp4(q, s):
    """Storage form of FP4 weights: two E2M1 codes per byte along the last axis
    (element 2i in the low nibble, 2i + 1 in the high nibble) and the block
    exponents s as int8.  Returns (packed uint8 [..., K / 2], s int8)."""
    c = e2m1_codes(q)
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8), np.asarray(s).astype(np.int8)


def unpack_fp4(packed, s, block: int = FP4_BLOCK) -> np.ndarray:
    """Inverse of pack_fp4 followed by dequantize_fp4: the FP8 values."""
    packed = np.asarray(packed, np.uint8)
    codes = np.empty(packed.shape[:-1] + (2 * packed.shape[-1],), np.uint8)
    codes[..., 0::2] = packed & 0xF
    codes[..., 1::2] = packed >> 4
    q = np.where(codes & 8, -1.0, 1.0) * E2M1_GRID[codes & 7]
    return dequantize_fp4(q, np.asarray(s, np.int64), block)


def round_e4m3(x) -> np.ndarray:
    """Nearest E4M3 value (1 sign, 4 exponent bits with bias 7, 3 mantissa
    bits; subnormals m/8 * 2^-6; largest finite 448), ties to even; magnitudes
    above 448 saturate to 448."""
    x = np.asarray(x, np.float64)
    mag = np.abs(x)
    _, E = np.frexp(mag)                       # mag = m 2^E, m in [0.5, 1): binade 2^(E-1)
    e = np.maximum(E - 1, -6)                  # below 2^-6 the spacing stays 2^-9
    ulp = np.exp2(e - 3)
    r = np.rint(mag / ulp) * ulp               # np.rint: ties to even
    r = np.where(mag == 0, 0.0, np.minimum(r, E4M3_MAX))
    return np.copysign(r, x)


def e4m3_bits(v) -> np.ndarray:
    """uint8 code of E4M3-representable values (sign | exponent | mantissa)."""
    v = np.asarray(v, np.float64)
    if not np.array_equal(round_e4m3(v), v):
        raise ValueError("not E4M3 values")
    mag = np.abs(v)
    _, E = np.frexp(mag)
    sub = mag < 2.0 ** -6
    expo = np.where(sub | (mag == 0), 0, E - 1 + 7)
    mant = np.where(sub | (mag == 0), mag / 2.0 ** -9, (mag / np.exp2(E - 1) - 1.0) * 8)
    code = (expo.astype(np.int64) << 3) | mant.astype(np.int64)
    return (code | np.where(np.signbit(v), 0x80, 0)).astype(np.uint8)


def act_row_exponent(amax) -> np.ndarray:
    """Smallest integer e with amax <= 448 * 2^e, clamped to [-126, 126] (amax =
    0 gives 0).  448 = 0.875 * 2^9, so with amax = m 2^E (m in [0.5, 1)):
    e = E - 9 when m <= 0.875, else E - 8."""
    amax = np.asarray(amax, np.float64)
    m, E = np.frexp(amax)
    e = np.where(m <= 0.875, E - 9, E - 8)
    e = np.where(amax == 0, 0, e)
    return np.clip(e, ACT_EXP_MIN, ACT_EXP_MAX).astype(np.int64)


def quantize_act_rows(a):
    """Per row: e = act_row_exponent(max |a|), q = round_e4m3(a / 2^e).
    Returns (q, e); the row's value is q * 2^e."""
    a = np.asarray(a, np.float64)
    e = act_row_exponent(np.abs(a).max(axis=-1) if a.shape[-1] else np.zeros(a.shape[:-1]))
    return round_e4m3(a / np.exp2(e)[..., None]), e


def expert_ffn_fp8(xn_rows, w8_gate, w8_up, w8_down, gate_clamp_max=np.inf, up_clamp=np.inf,
                   act: int = ACT_SWIGLU, beta_g: float = 4.0, beta_u: float = 25.0):
    """One gated expert with FP8 weights (the values fp4_weights_as_fp8 gives)
    and FP8 activations: xn rows -> (qx, ex); g = (qx W_g^T) 2^ex, u likewise,
    h = bf16(unit(g, u)); h -> (qh, eh); y = (qh W_d^T) 2^eh.  The sums are of
    exact products (E4M3 x E4M3 has at most 8 significant bits) and are taken
    in fp64.  Returns (h, y)."""
    qx, ex = quantize_act_rows(xn_rows)
    Wg = np.asarray(w8_gate, np.float64)
    Wu = np.asarray(w8_up, np.float64)
    Wd = np.asarray(w8_down, np.float64)
    n, D = qx.shape
    I = Wg.shape[0]
    MAC_COUNTER[0] += n * (2 * D * I + I * Wd.shape[0])
    sx = np.exp2(ex)[:, None]
    h = round_bf16(glu_unit((qx @ Wg.T) * sx, (qx @ Wu.T) * sx, act, gate_clamp_max, up_clamp, beta_g, beta_u))
    qh, eh = quantize_act_rows(h)
    return h, (qh @ Wd.T) * np.exp2(eh)[:, None]


def expert_fn(cfg):
    """expert_ffn or expert_ffn_fp8, by the configuration's weight format."""
    fmt = int(getattr(cfg, "weight_format", WEIGHTS_BF16))
    return expert_ffn_fp8 if fmt in (WEIGHTS_FP8, WEIGHTS_FP4) else expert_ffn


# ------------------------------------------------------------ latent MoE
def latent_down(xn, w_proj_down) -> np.ndarray:
    """z = bf16(xn W_down^T): the down-projection W_down of [LD] "潜在MoE (Latent
    MoE)" / "K3 的 Stable Latent MoE" (input -> down-projection -> choose the
    experts -> each expert's GLU in the latent space of width l -> weighted sum
    -> up-projection -> back to the hidden space).  z is an activation between
    two matmuls, so it is a bf16 value like xn and h."""
    return round_bf16(np.asarray(xn, np.float64) @ np.asarray(w_proj_down, np.float64).T)


def latent_up(w, y_slots, w_proj_up):
    """s = sum_j w_j y_j (the routed experts' latent outputs, slot order),
    a = bf16(s) (one cast; [FW] case study's standard path for the weighted
    sum), then y = a W_up^T, the up-projection back to the hidden width ([LD]
    "潜在MoE").  Returns (s, a, y)."""
    s = np.einsum("tj,tjl->tl", np.asarray(w, np.float64), np.asarray(y_slots, np.float64))
    a = round_bf16(s)
    return s, a, a @ np.asarray(w_proj_up, np.float64).T


# --------------------------------------------- 7-8. combine + residual + norm
def combine(w, y_slots, y_shared) -> np.ndarray:
    """acc[t] = sum_j w[t,j] * y[t,j] (slot order) + sum_s y_shared[s,t]
    ([FW] Trap 3, unfused path: moe_finalize, then += shared_expert; the
    case study's standard path keeps all k contributions and sums them in
    one weighted sum before a single cast)."""
    acc = np.einsum("tj,tjd->td", np.asarray(w, np.float64), np.asarray(y_slots, np.float64))
    if y_shared is not None and len(y_shared):
        acc = acc + np.sum(np.asarray(y_shared, np.float64), axis=0)
    return acc


def residual_rmsnorm(acc, residual, g_out, eps: float):
    """r = full_out + residual; returns (bf16(RMSNorm(r)), bf16(r), r)
    ([FW] Trap 2 / Trap 3: normed, residual = rmsnorm(full_out + residual))."""
    r = np.asarray(acc, np.float64) + np.asarray(residual, np.float64)
    return round_bf16(rmsnorm(r, g_out, eps)), round_bf16(r), r


# ------------------------------------------------ 9. partial-sum epilogue
def allreduce_fixed_order_f32(partials) -> np.ndarray:
    """r0 + r1 + ... + r_{P-1}, left to right, every element, IEEE fp32
    ([FW] Trap 1: the Lamport kernel's uniform r0..r7 order, FP32 accumulation)."""
    parts = np.asarray(partials, dtype=np.float32)
    acc = parts[0].copy()
    for p in range(1, parts.shape[0]):
        acc = np.add(acc, parts[p], dtype=np.float32)
    return acc


def allreduce_ring_order_f32(partials) -> np.ndarray:
    """The NCCL ring reduce-scatter order ([FW] Trap 1): the hidden vector is cut
    into P contiguous chunks; chunk c starts from its owner r_c and then adds
    r_{c-1}, r_{c-2}, ... around the ring, in fp32.  Used only to show that a
    different order changes bits."""
    parts = np.asarray(partials, dtype=np.float32)
    P, D = parts.shape[0], parts.shape[-1]
    bounds = [(c * D) // P for c in range(P + 1)]
    out = np.empty(parts.shape[1:], np.float32)
    for c in range(P):
        sl = slice(bounds[c], bounds[c + 1])
        acc = parts[c][..., sl].copy()
        for step in range(1, P):
            acc = np.add(acc, parts[(c - step) % P][..., sl], dtype=np.float32)
        out[..., sl] = acc
    return out


def reduce_partials(partials, residual, g, eps: float):
    """The tensor-parallel epilogue simulated on one GPU: r = (r0 + ... + r7) +
    residual, all in fp32 (the sum in fixed order), then RMSNorm in fp64 on that
    fp32 r.  Returns (bf16(RMSNorm(r)), bf16(r), r as fp32)."""
    s = allreduce_fixed_order_f32(partials)
    r = np.add(s, np.asarray(residual, np.float32), dtype=np.float32)
    out_residual = round_bf16(r.astype(np.float64))
    out_norm = round_bf16(rmsnorm(r.astype(np.float64), g, eps))
    return out_norm, out_residual, r


# ------------------------------------------------------------- the layer
class Weights:
    """In-memory weights (fp64 arrays holding bf16 values).  Any object with the
    same attributes and ``routed(e)`` / ``shared(s)`` methods will do, e.g. one
    that regenerates a single expert on demand."""

    def __init__(self, w_router, router_bias, w_gate, w_up, w_down, ws_gate, ws_up, ws_down,
                 g_in, g_out, w_proj_down=None, w_proj_up=None):
        self.w_proj_down, self.w_proj_up = w_proj_down, w_proj_up  # latent MoE only
        self.w_router = w_router
        self.router_bias = router_bias
        self.w_gate, self.w_up, self.w_down = w_gate, w_up, w_down
        self.ws_gate, self.ws_up, self.ws_down = ws_gate, ws_up, ws_down
        self.g_in, self.g_out = g_in, g_out

    def routed(self, e):
        return self.w_gate[e], self.w_up[e], self.w_down[e]

    def shared(self, s):
        return self.ws_gate[s], self.ws_up[s], self.ws_down[s]


class FP4Weights:
    """The weights of a layer with FP4 experts ([DS] §6.2): the master weights
    ``master`` (any Weights-like object) with every expert matrix replaced, on
    first use, by its FP8 values fp4_weights_as_fp8(w).  Router, gains and
    projections are the master's."""

    def __init__(self, master):
        self._master = master
        self._cache = {}
        for n in ("w_router", "router_bias", "g_in", "g_out", "w_proj_down", "w_proj_up"):
            setattr(self, n, getattr(master, n, None))

    def _q(self, key, mats):
        if key not in self._cache:
            self._cache[key] = tuple(fp4_weights_as_fp8(m) for m in mats)
        return self._cache[key]

    def routed(self, e):
        return self._q(("r", int(e)), self._master.routed(e))

    def shared(self, s):
        return self._q(("s", int(s)), self._master.shared(s))


def moe_layer(cfg, W, x, residual, token_ids=None, rows=None, force_idx=None) -> dict:
    """The whole layer.  Routing, histogram and permutation are computed for
    every token; the experts, combine and epilogue for ``rows`` (all tokens
    when None).  ``cfg`` carries D, E, k, I, n_shared, I_shared, router,
    renormalize, routed_scale, gate_clamp_max, up_clamp, eps, hash_mult and
    optionally activation, situ_beta_gate, situ_beta_up (SiTU-GLU experts),
    latent (the latent width l; 0 or absent: no latent projection) and
    weight_format (WEIGHTS_FP8: the expert weights in ``W`` are FP8 values, as
    fp4_weights_as_fp8 gives, and the experts run expert_ffn_fp8).

    ``force_idx`` ([T,k] expert indices, optional) replaces the top-k choice
    of every token; the weights are still the router's own for those experts,
    and ``margin`` stays that of the oracle's own choice.

    Latent MoE ([LD] "潜在MoE" and its K3 flow): the router and the routed
    experts read z = latent_down(xn) (width l), the routed experts' weighted sum
    is projected back by latent_up, and the shared experts keep the full width
    (they read xn)."""
    x = np.asarray(x, np.float64)
    T = x.shape[0]
    rows = np.arange(T) if rows is None else np.asarray(rows, np.int64)
    xn = xn_bf16(x, W.g_in, cfg.eps)
    lat = int(getattr(cfg, "latent", 0) or 0)
    xe = latent_down(xn, W.w_proj_down) if lat else xn   # what the router and routed experts read
    logits = None
    if cfg.router != ROUTER_HASH:
        logits = router_logits(xe, W.w_router)
    idx, w, keys = route(cfg, logits, W.router_bias, token_ids, force_idx)
    margin = topk_margin(keys, cfg.k)
    counts = expert_histogram(idx, cfg.E)
    offsets, perm_token, perm_slot, pos = stable_permute(idx, cfg.E)

    # Expert compute for the selected rows, grouped by expert.
    ffn = expert_fn(cfg)
    n, k = len(rows), cfg.k
    y_slots = np.zeros((n, k, lat or cfg.D))
    sel = idx[rows]                                   # [n, k]
    for e in np.unique(sel):
        rr, jj = np.nonzero(sel == e)
        Wg, Wu, Wd = W.routed(int(e))
        _, y = ffn(xe[rows[rr]], Wg, Wu, Wd, **unit_args(cfg))
        y_slots[rr, jj] = y
    y_shared = np.zeros((cfg.n_shared, n, cfg.D))
    for s in range(cfg.n_shared):
        Wg, Wu, Wd = W.shared(s)
        # The clamp is a property of the SwiGLU unit and applies to shared experts too.
        _, y_shared[s] = ffn(xn[rows], Wg, Wu, Wd, **unit_args(cfg))
    agg = lat_sum = None
    if lat:
        lat_sum, agg, y_lat = latent_up(w[rows], y_slots, W.w_proj_up)
        acc = combine(np.ones((n, 1)), y_lat[:, None, :], y_shared)   # projected sum, then shared
    else:
        acc = combine(w[rows], y_slots, y_shared)
    out_norm, out_residual, r = residual_rmsnorm(acc, np.asarray(residual, np.float64)[rows],
                                                 W.g_out, cfg.eps)
    return dict(rows=rows, xn=xn, z=xe if lat else None, lat_sum=lat_sum, agg=agg, logits=logits,
                keys=keys, idx=idx,
                w=w, margin=margin,
                counts=counts, offsets=offsets, perm_token=perm_token, perm_slot=perm_slot,
                pos=pos, y_slots=y_slots, y_shared=y_shared, acc=acc, r=r,
                out_norm=out_norm, out_residual=out_residual)


def moe_layer_dense_masked(cfg, W, x, residual, token_ids=None, force_idx=None) -> dict:
    """Cross-check of the routed path: run every expert on every token, weight
    each output by the token's routing weight for that expert (0 when not
    chosen) and sum over all experts.  Mathematically equal to ``moe_layer``
    (up to the order of the routed sum)."""
    x = np.asarray(x, np.float64)
    T = x.shape[0]
    xn = xn_bf16(x, W.g_in, cfg.eps)
    lat = int(getattr(cfg, "latent", 0) or 0)
    xe = latent_down(xn, W.w_proj_down) if lat else xn
    logits = None if cfg.router == ROUTER_HASH else router_logits(xe, W.w_router)
    idx, w, _ = route(cfg, logits, W.router_bias, token_ids, force_idx)
    mask = np.zeros((T, cfg.E))
    np.put_along_axis(mask, idx, w, axis=-1)
    acc = np.zeros((T, lat or cfg.D))
    ffn = expert_fn(cfg)
    for e in range(cfg.E):
        Wg, Wu, Wd = W.routed(e)
        _, y = ffn(xe, Wg, Wu, Wd, **unit_args(cfg))
        acc += mask[:, e:e + 1] * y
    lat_sum = None
    if lat:
        lat_sum = acc
        acc = round_bf16(acc) @ np.asarray(W.w_proj_up, np.float64).T
    for s in range(cfg.n_shared):
        Wg, Wu, Wd = W.shared(s)
        _, y = ffn(xn, Wg, Wu, Wd, **unit_args(cfg))
        acc += y
    out_norm, out_residual, r = residual_rmsnorm(acc, residual, W.g_out, cfg.eps)
    return dict(acc=acc, r=r, out_norm=out_norm, out_residual=out_residual, idx=idx, w=w, lat_sum=lat_sum)
