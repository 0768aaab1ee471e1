"""Workload tensors on the device (filled in place by the GPU twin) and on the
host (regenerated slices for the oracle).  Input generation only: nothing
here computes any part of the MoE layer."""
from __future__ import annotations

import numpy as np

from . import bf16_bits_to_f32, dev_normal_bf16, dev_normal_f32, dev_uniform_int
from . import workloads as W


def _stream_ptr(stream):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream)


def device_bf16(cfg, name, T=None, device="cuda", stream=None):
    import torch
    shape = W.tensor_shape(cfg, name, T)
    t = torch.empty(shape, dtype=torch.bfloat16, device=device)
    n = int(np.prod(shape))
    if n == 0:
        return t
    if name in ("g_in", "g_out"):
        t.fill_(1.0)
        return t
    sigma = cfg.x_sigma if name in ("x", "residual") else cfg.weight_sigma
    dev_normal_bf16(W.k_(name), 0, n, sigma, t.data_ptr(), _stream_ptr(stream))
    return t


def layer_config(cfg, T_max=None):
    """The library's LayerConfig for a workload (every field of the layer)."""
    import deterministic_expert_b200 as moe
    return moe.LayerConfig(D=cfg.D, E=cfg.E, k=cfg.k, I=cfg.I, n_shared=cfg.n_shared,
                           I_shared=cfg.I_shared, T_max=T_max or cfg.T, router=cfg.router,
                           renormalize=cfg.renormalize, routed_scale=cfg.routed_scale,
                           gate_clamp_max=cfg.gate_clamp_max, up_clamp=cfg.up_clamp, eps=cfg.eps,
                           hash_mult=cfg.hash_mult, activation=cfg.activation,
                           situ_beta_gate=cfg.situ_beta_gate, situ_beta_up=cfg.situ_beta_up,
                           latent=cfg.latent, weight_format=cfg.weight_format)


def device_weights(cfg, device="cuda", stream=None) -> dict:
    """moe_weights field name -> device tensor."""
    import torch
    w = {n: device_bf16(cfg, n, device=device, stream=stream)
         for n in ("w_router", "w_gate", "w_up", "w_down", "g_in", "g_out")}
    if cfg.n_shared:
        for n in ("ws_gate", "ws_up", "ws_down"):
            w[n] = device_bf16(cfg, n, device=device, stream=stream)
    if cfg.latent:
        for n in ("w_proj_down", "w_proj_up"):
            w[n] = device_bf16(cfg, n, device=device, stream=stream)
    if cfg.bias == "normal":
        b = torch.empty(cfg.E, dtype=torch.float32, device=device)
        dev_normal_f32(W.k_("router_bias"), 0, cfg.E, cfg.bias_sigma, b.data_ptr(), _stream_ptr(stream))
        w["router_bias"] = b
    elif cfg.bias == "zipf":
        w["router_bias"] = torch.from_numpy(W.host_router_bias(cfg)).to(device)
    return w


def device_inputs(cfg, T=None, device="cuda", stream=None):
    """x, residual [T, D] bf16 and token_ids [T] int32 for the workload."""
    import torch
    T = cfg.T if T is None else T
    x = device_bf16(cfg, "x", T=T, device=device, stream=stream)
    r = device_bf16(cfg, "residual", T=T, device=device, stream=stream)
    ids = torch.empty(T, dtype=torch.int32, device=device)
    if T:
        dev_uniform_int(W.k_("token_ids"), 0, T, cfg.token_id_range, ids.data_ptr(), _stream_ptr(stream))
    return x, r, ids


def device_partials(P=W.EPILOGUE_P, T=W.EPILOGUE_T, D=W.EPILOGUE_D, device="cuda", stream=None):
    import torch
    out = []
    for p in range(P):
        t = torch.empty((T, D), dtype=torch.bfloat16, device=device)
        fill_partial(t, p, stream)
        out.append(t)
    return out


def fill_partial(t, p, stream=None):
    """Write partial buffer p of the epilogue workload into the [T, D] bf16 tensor t."""
    dev_normal_bf16(W.k_("PARTIAL0", p), 0, t.numel(), W.EPILOGUE_SIGMA, t.data_ptr(), _stream_ptr(stream))


# ------------------------------------------------------------------ host side
def f64(bits):
    return bf16_bits_to_f32(bits).astype(np.float64)


class HostWeights:
    """The workload's weights as fp64 arrays of bf16 values, regenerated from
    the host twin one expert at a time (the oracle's weight source).  Any
    expert can be produced without generating the others."""

    def __init__(self, cfg, cache_experts: int = 512):
        self.cfg = cfg
        E, D, I = cfg.E, cfg.D, cfg.I
        L = cfg.latent or D
        self.w_router = f64(W.host_bf16(cfg, "w_router")).reshape(E, L) if cfg.router != W.ROUTER_HASH else None
        self.w_proj_down = f64(W.host_bf16(cfg, "w_proj_down")).reshape(cfg.latent, D) if cfg.latent else None
        self.w_proj_up = f64(W.host_bf16(cfg, "w_proj_up")).reshape(D, cfg.latent) if cfg.latent else None
        b = W.host_router_bias(cfg)
        self.router_bias = None if b is None else b.astype(np.float64)
        self.g_in = f64(W.host_bf16(cfg, "g_in"))
        self.g_out = f64(W.host_bf16(cfg, "g_out"))
        self._cache = {}
        self._cap = cache_experts

    def _slice(self, name, index, rows, cols):
        n = rows * cols
        return W.host_f64(self.cfg, name, start=index * n, count=n).reshape(rows, cols)

    def routed(self, e):
        key = ("r", int(e))
        if key not in self._cache:
            c = self.cfg
            if len(self._cache) >= self._cap:
                self._cache.pop(next(iter(self._cache)))
            L = c.latent or c.D
            self._cache[key] = (self._slice("w_gate", e, c.I, L), self._slice("w_up", e, c.I, L),
                                self._slice("w_down", e, L, c.I))
        return self._cache[key]

    def shared(self, s):
        key = ("s", int(s))
        if key not in self._cache:
            c = self.cfg
            self._cache[key] = (self._slice("ws_gate", s, c.I_shared, c.D),
                                self._slice("ws_up", s, c.I_shared, c.D),
                                self._slice("ws_down", s, c.D, c.I_shared))
        return self._cache[key]


def host_rows(cfg, name, rows, T=None):
    """fp64 values of the given rows of x or residual ([len(rows), D])."""
    D = cfg.D
    rows = np.asarray(rows, np.int64)
    if len(rows) and np.all(np.diff(rows) == 1):
        return W.host_f64(cfg, name, start=int(rows[0]) * D, count=len(rows) * D, T=T).reshape(-1, D)
    return np.stack([W.host_f64(cfg, name, start=int(r) * D, count=D, T=T) for r in rows]) \
        if len(rows) else np.zeros((0, D))
