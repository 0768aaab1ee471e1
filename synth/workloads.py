"""Layer shapes and the synthetic input recipe for the five workloads.

Shapes, router variants and value distributions follow the workload list of
this project (tiny, fine-grained, DeepSeek-V3-shaped, decode sweep, skewed /
hash routing); every tensor is drawn from the counter-based generator of this
package with seed 0 and its own stream id, so any slice can be regenerated on
the host or filled in place on the device.  Nothing here computes any part of
the MoE layer.
"""
from __future__ import annotations

import dataclasses
import json
import math
import os

import numpy as np

from . import key, normal_bf16, normal_bf16_as_f64, normal_f32, uniform_int, _h  # noqa: F401

SEED = 0

# One stream per tensor.  Partial buffer p of the 8-partial epilogue uses
# stream PARTIAL0 + p.
STREAM = {
    "x": 1, "residual": 2, "w_router": 3, "router_bias": 4,
    "w_gate": 5, "w_up": 6, "w_down": 7,
    "ws_gate": 8, "ws_up": 9, "ws_down": 10,
    "g_in": 11, "g_out": 12, "token_ids": 13, "zipf_rank": 14,
    "decode_subset": 15, "perm": 16, "w_proj_down": 17, "w_proj_up": 18, "PARTIAL0": 32,
}

ROUTER_SOFTMAX, ROUTER_SIGMOID_BIAS, ROUTER_HASH = 0, 1, 2
HASH_MULT = 2654435761
INF = float("inf")


@dataclasses.dataclass(frozen=True)
class MoEConfig:
    name: str
    T: int
    D: int
    E: int
    k: int
    I: int
    n_shared: int
    I_shared: int
    router: int = ROUTER_SOFTMAX
    renormalize: int = 0
    routed_scale: float = 1.0
    gate_clamp_max: float = INF
    up_clamp: float = INF
    eps: float = 1e-6
    hash_mult: int = HASH_MULT
    bias: str = "none"            # "none" | "normal" (sigmoid selection bias) | "zipf" (logit bias)
    bias_sigma: float = 0.0
    weight_sigma: float = 0.02
    x_sigma: float = 1.0
    token_id_range: int = 128000
    activation: int = 0             # 0 SwiGLU (+ clamp), 1 SiTU-GLU
    situ_beta_gate: float = 4.0
    situ_beta_up: float = 25.0
    latent: int = 0                 # latent MoE width (0: none)
    weight_format: int = 0          # 0 bf16 experts, 1 FP4-valued experts stored as E4M3,
                                    # 2 the same experts stored as packed E2M1 + block exponents

    def with_T(self, T: int) -> "MoEConfig":
        return dataclasses.replace(self, T=T)


# Tiny MoE layer.
C1 = MoEConfig("tiny", T=64, D=256, E=8, k=2, I=128, n_shared=1, I_shared=128)
# Fine-grained MoE, softmax renormalised over the chosen 6.
C2 = MoEConfig("fine_grained", T=4096, D=2048, E=64, k=6, I=1408, n_shared=2, I_shared=1408,
               renormalize=1)
# DeepSeek-V3-shaped: sigmoid scores + per-expert selection bias, normalised
# over the chosen 8, routed scale 2.5, SwiGLU clamp.
C3 = MoEConfig("v3_shaped", T=8192, D=7168, E=256, k=8, I=2048, n_shared=1, I_shared=2048,
               router=ROUTER_SIGMOID_BIAS, renormalize=1, routed_scale=2.5,
               gate_clamp_max=10.0, up_clamp=10.0, bias="normal", bias_sigma=0.01)
# Decode sweep on the fine-grained weights; batches are taken from an 8192-row input.
C4_T = (1, 8, 64, 128, 512)
C4_SOURCE_T = 8192
# Skewed routing: softmax over logits plus a Zipf(1.2) expert bias.
C5 = MoEConfig("skew_zipf", T=16384, D=4096, E=128, k=8, I=1024, n_shared=0, I_shared=1024,
               bias="zipf")
# Hash-routing variant of the skewed workload.
C5H = dataclasses.replace(C5, name="skew_hash", router=ROUTER_HASH, bias="none")
# SiTU-GLU experts (the linux.do post on MoE variants, "SiTU-GLU": caps 4 and
# 25) on the fine-grained shapes.
C2S = dataclasses.replace(C2, name="fine_grained_situ", activation=1)
# Latent MoE in the K3 manner (the linux.do post on MoE variants, "潜在MoE" and
# "K3 的 Stable Latent MoE": many small routed experts with 16 active, working
# at a latent width, SiTU-GLU inside the experts, a full-width shared expert).
# The post gives no sizes; these are the fine-grained shapes with l = D / 4.
C6 = MoEConfig("latent_situ", T=4096, D=2048, E=256, k=16, I=512, n_shared=1, I_shared=2048,
               renormalize=1, activation=1, latent=512)
# FP4 expert weights with FP8 x FP8 expert GEMMs (the DeepSeek V4 infra notes,
# §6.2 FP4 QAT) on the tiny and fine-grained shapes; the master weights are the
# bf16 weights of those workloads.
C1F = dataclasses.replace(C1, name="tiny_fp8", weight_format=1)
C2F = dataclasses.replace(C2, name="fine_grained_fp8", weight_format=1)
# The 8-partial fixed-order reduce + residual + RMSNorm epilogue of that workload.
EPILOGUE_P = 8
EPILOGUE_T = 16384
EPILOGUE_D = 4096
EPILOGUE_SIGMA = 1.0 / 8.0

# The latent workload with FP4 expert weights (routed and shared).
C6F = dataclasses.replace(C6, name="latent_situ_fp8", weight_format=1)
# The same FP4 experts in their storage form (packed E2M1 codes, half a byte a
# weight, plus block exponents), read as they are by block-scaled GEMMs.
C1P = dataclasses.replace(C1, name="tiny_fp4", weight_format=2)
C2P = dataclasses.replace(C2, name="fine_grained_fp4", weight_format=2)
C6P = dataclasses.replace(C6, name="latent_situ_fp4", weight_format=2)
# A small case of the V3-shaped kernels for profiler captures (a few GB on the
# device): the same D, I, top-8 and about 256 rows per expert, with 32 experts.
C3P = dataclasses.replace(C3, name="v3_shaped_e32", T=1024, E=32)
CONFIGS = {c.name: c for c in (C1, C2, C3, C5, C5H, C2S, C6, C1F, C2F, C6F, C3P, C1P, C2P, C6P)}

_ZIPF_FILE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "zipf_beta.json")
ZIPF_S = 1.2


def zipf_beta() -> float:
    """The frozen bias scale beta (written by zipf_calibrate.py)."""
    with open(_ZIPF_FILE) as f:
        return float(json.load(f)["beta"])


def k_(name: str, index: int = 0) -> int:
    return key(SEED, STREAM[name] + index)


# ------------------------------------------------------------------ host side
def tensor_shape(cfg: MoEConfig, name: str, T: int | None = None):
    T = cfg.T if T is None else T
    D, E, I, S, Is = cfg.D, cfg.E, cfg.I, cfg.n_shared, cfg.I_shared
    L = cfg.latent or D   # width the router and routed experts read
    return {
        "x": (T, D), "residual": (T, D), "w_router": (E, L), "router_bias": (E,),
        "w_gate": (E, I, L), "w_up": (E, I, L), "w_down": (E, L, I),
        "w_proj_down": (cfg.latent, D), "w_proj_up": (D, cfg.latent),
        "ws_gate": (S, Is, D), "ws_up": (S, Is, D), "ws_down": (S, D, Is),
        "g_in": (D,), "g_out": (D,), "token_ids": (T,),
    }[name]


def host_bf16(cfg: MoEConfig, name: str, start: int = 0, count: int | None = None,
              T: int | None = None) -> np.ndarray:
    """bf16 bit patterns of a bf16 tensor, or of the flat slice [start, start+count)."""
    shape = tensor_shape(cfg, name, T)
    n = int(np.prod(shape))
    if name in ("g_in", "g_out"):
        # RMSNorm gains are ones (the standard initialisation).
        return np.full(n if count is None else count, 0x3F80, np.uint16).reshape(
            shape if count is None else (count,))
    sigma = cfg.x_sigma if name in ("x", "residual") else cfg.weight_sigma
    cnt = n - start if count is None else count
    out = normal_bf16(k_(name), start, cnt, sigma)
    return out.reshape(shape) if (start == 0 and count is None) else out


def host_f64(cfg: MoEConfig, name: str, start: int = 0, count: int | None = None,
             T: int | None = None) -> np.ndarray:
    """The values of host_bf16 widened to float64 (flat)."""
    n = int(np.prod(tensor_shape(cfg, name, T)))
    cnt = n - start if count is None else count
    if name in ("g_in", "g_out"):
        return np.ones(cnt)
    sigma = cfg.x_sigma if name in ("x", "residual") else cfg.weight_sigma
    return normal_bf16_as_f64(k_(name), start, cnt, sigma)


def host_router_bias(cfg: MoEConfig) -> np.ndarray | None:
    if cfg.bias == "none":
        return None
    if cfg.bias == "normal":
        return normal_f32(k_("router_bias"), 0, cfg.E, cfg.bias_sigma)
    if cfg.bias == "zipf":
        return zipf_bias(cfg.E, zipf_beta())
    raise ValueError(cfg.bias)


def zipf_ranks(E: int) -> np.ndarray:
    """A seeded permutation of 1..E: expert e gets popularity rank ranks[e]."""
    draws = np.array([int(_h().syn_draw(k_("zipf_rank"), i)) for i in range(E)], dtype=np.uint64)
    order = np.argsort(draws, kind="stable")
    ranks = np.empty(E, np.int64)
    ranks[order] = np.arange(1, E + 1)
    return ranks


def zipf_bias(E: int, beta: float) -> np.ndarray:
    """Logit bias b_e = -beta * s * ln(rank_e) with s = 1.2 (Zipf exponent)."""
    r = zipf_ranks(E).astype(np.float64)
    return (-beta * ZIPF_S * np.log(r)).astype(np.float32)


def host_token_ids(cfg: MoEConfig, T: int | None = None) -> np.ndarray:
    T = cfg.T if T is None else T
    return uniform_int(k_("token_ids"), 0, T, cfg.token_id_range)


def decode_subset(T: int, source_T: int = C4_SOURCE_T) -> np.ndarray:
    """A seeded random subset of T distinct rows of the decode source batch, sorted."""
    draws = np.array([int(_h().syn_draw(key(SEED, STREAM["decode_subset"] + T), i))
                      for i in range(source_T)], dtype=np.uint64)
    return np.sort(np.argsort(draws, kind="stable")[:T]).astype(np.int64)


def token_permutation(T: int, salt: int = 0) -> np.ndarray:
    """A seeded permutation of 0..T-1."""
    kk = key(SEED, STREAM["perm"] * 1000 + salt)
    draws = np.empty(T, np.uint64)
    lib = _h()
    for i in range(T):
        draws[i] = lib.syn_draw(kk, i)
    return np.argsort(draws, kind="stable").astype(np.int64)


def host_partial(p: int, T: int = EPILOGUE_T, D: int = EPILOGUE_D, start: int = 0,
                 count: int | None = None) -> np.ndarray:
    cnt = T * D - start if count is None else count
    return normal_bf16(k_("PARTIAL0", p), start, cnt, EPILOGUE_SIGMA)


def moe_flops(cfg: MoEConfig, T: int | None = None) -> dict:
    """Algorithmic FLOPs of one layer call: 2 per multiply-add.

    routed = 2*T*k*3*L*I, shared = 2*T*S*3*D*I_s, router = 2*T*E*L (none for
    hash routing), with L the latent width (D without one); a latent layer adds
    its two projections, 2*2*T*D*L.  Gate/up is two thirds of each expert's work.
    """
    T = cfg.T if T is None else T
    L = cfg.latent or cfg.D
    routed = 2 * T * cfg.k * 3 * L * cfg.I
    shared = 2 * T * cfg.n_shared * 3 * cfg.D * cfg.I_shared
    router = 0 if cfg.router == ROUTER_HASH else 2 * T * cfg.E * L
    proj = 2 * 2 * T * cfg.D * cfg.latent
    gateup = 2 * T * (cfg.k * 2 * L * cfg.I + cfg.n_shared * 2 * cfg.D * cfg.I_shared)
    return {"routed": routed, "shared": shared, "router": router, "proj": proj,
            "total": routed + shared + router + proj, "gateup": gateup, "down": routed + shared - gateup}


def weight_bytes(cfg: MoEConfig, n: int) -> int:
    """HBM bytes of n expert weights as the GEMMs read them: bf16 (2), E4M3 (1),
    or packed E2M1 (1/2) plus one 4-byte exponent word per 128 weights (1/32)."""
    return {0: 2 * n, 1: n, 2: n * 17 // 32}[cfg.weight_format]


def expert_bytes(cfg: MoEConfig) -> int:
    return weight_bytes(cfg, 3 * (cfg.latent or cfg.D) * cfg.I)


def layer_bytes(cfg: MoEConfig, T: int, distinct_experts: int) -> int:
    """Algorithmic HBM bytes: the touched routed experts, shared and router
    weights, x and residual in, two bf16 outputs."""
    w = distinct_experts * expert_bytes(cfg) + weight_bytes(cfg, cfg.n_shared * 3 * cfg.D * cfg.I_shared)
    if cfg.router != ROUTER_HASH:
        w += cfg.E * (cfg.latent or cfg.D) * 2
    w += 2 * cfg.D * cfg.latent * 2   # latent projections
    act = 4 * T * cfg.D * 2
    return w + act


def pretty(cfg: MoEConfig) -> str:
    r = {0: "softmax", 1: "sigmoid+bias", 2: "hash"}[cfg.router]
    act = "" if cfg.activation == 0 else f" SiTU-GLU({cfg.situ_beta_gate:g},{cfg.situ_beta_up:g})"
    lat = f" latent={cfg.latent}" if cfg.latent else ""
    if cfg.weight_format == 1:
        act += " FP4 weights as E4M3 bytes (E4M3 x E4M3 GEMMs)"
    elif cfg.weight_format == 2:
        act += " FP4 weights packed (E2M1 + block exponents; block-scaled E2M1 x E4M3 GEMMs)"
    return (f"{cfg.name}: T={cfg.T} D={cfg.D}{lat} E={cfg.E} top-{cfg.k} {r} I={cfg.I} "
            f"shared={cfg.n_shared}x{cfg.I_shared}{act}")


__all__ = ["MoEConfig", "C1", "C1F", "C1P", "C2", "C2F", "C2P", "C2S", "C3", "C4_T", "C5", "C5H", "C6", "C6F", "C6P",
           "CONFIGS", "STREAM", "SEED",
           "host_bf16", "host_router_bias", "host_token_ids", "moe_flops", "math"]
