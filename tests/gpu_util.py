"""Helpers for the GPU tests: run the layer through the C ABI on a workload and
compare with the oracle.  Inputs come from the seeded generator twins; no
oracle input or expected value comes from the CUDA path."""
from __future__ import annotations

import numpy as np

import oracle as O
from synth import device as SD
from synth import workloads as W

TOL_MAX = 2e-2     # max |gpu - oracle| / max(1, |oracle|) per element
TOL_MEAN = 4e-3    # mean of the same
NEAR_TIE = 1e-5    # routing margin below which a token may route differently


def layer_config(cfg, T_max):
    return SD.layer_config(cfg, T_max)


class Run:
    """One configured layer on the device with its inputs and outputs."""

    def __init__(self, cfg, T=None, T_max=None, weights=None, device="cuda"):
        import torch
        import deterministic_expert_b200 as moe
        self.cfg = cfg
        self.T = cfg.T if T is None else T
        self.T_max = T_max or max(self.T, 1)
        if weights is None:
            weights = SD.device_weights(cfg, device=device)
            if cfg.weight_format:
                # FP4 expert weights: the library's own quantiser writes their E4M3 codes.
                weights = moe.quantize_expert_weights(weights)
        self.w = weights
        self.layer = moe.MoELayer(layer_config(cfg, self.T_max), self.w)
        self.device = device

    def inputs(self, T=None):
        return SD.device_inputs(self.cfg, T=self.T if T is None else T, device=self.device)

    def forward(self, x, r, ids, ws=None):
        import torch
        T = int(x.shape[0])
        if ws is None:
            # The workspace starts as 0xFF bytes (NaN for every float view, -1
            # for every int view): no stage may read what it did not write.
            ws = torch.full((max(self.layer.workspace_size(T), 256),), 0xFF, dtype=torch.uint8, device=self.device)
        # Outputs start poisoned (NaN, -1), so an element the layer leaves
        # unwritten fails every comparison instead of passing on stale memory.
        on = torch.full((T, self.cfg.D), float("nan"), dtype=torch.bfloat16, device=self.device)
        orr = torch.full_like(on, float("nan"))
        idx = torch.full((T, self.cfg.k), -1, dtype=torch.int32, device=self.device)
        tw = torch.full((T, self.cfg.k), float("nan"), dtype=torch.float32, device=self.device)
        cnt = torch.full((self.cfg.E,), -1, dtype=torch.int32, device=self.device)
        self.layer.forward(x, r, on, orr, ws, token_ids=ids, out_topk_idx=idx, out_topk_w=tw,
                           out_counts=cnt)
        torch.cuda.synchronize()
        assert self.layer.device_error(ws) == 0, "device wait timed out"
        return dict(out_norm=on, out_residual=orr, idx=idx, w=tw, counts=cnt, ws=ws)


def np64(t):
    import torch
    return t.to(torch.float32).cpu().numpy().astype(np.float64)


def rel_err(gpu, ref):
    return np.abs(gpu - ref) / np.maximum(1.0, np.abs(ref))


def check_outputs(out, ref, rows=None, same_rows=None):
    """Tolerance check of out_norm / out_residual on the rows whose routing
    matches the oracle (``same_rows``: boolean over ``rows``)."""
    rows = np.arange(out["out_norm"].shape[0]) if rows is None else np.asarray(rows)
    stats = {}
    for name in ("out_norm", "out_residual"):
        g = np64(out[name])[rows]
        o = ref[name]
        if same_rows is not None:
            g, o = g[same_rows], o[same_rows]
        e = rel_err(g, o)
        stats[name] = (float(e.max()) if e.size else 0.0, float(e.mean()) if e.size else 0.0)
        assert e.size == 0 or e.max() <= TOL_MAX, (name, stats[name])
        assert e.size == 0 or e.mean() <= TOL_MEAN, (name, stats[name])
    return stats


def routing_consistent(gi, keys, tol=NEAR_TIE):
    """Is ``gi`` (one token's GPU slots) a top-k of ``keys`` (the oracle's fp64
    keys) up to near ties?  Every chosen expert must be within ``tol`` of the
    oracle's k-th key, every expert left out must not beat the chosen ones by
    more than ``tol``, and consecutive slots must descend up to ``tol``."""
    k = len(gi)
    if len(set(gi.tolist())) != k:
        return False
    kth = np.sort(keys)[-k]
    chosen = keys[gi]
    if np.any(chosen < kth - tol):
        return False
    rest = np.delete(keys, gi)
    if rest.size and rest.max() > chosen.min() + tol:
        return False
    return bool(np.all(chosen[:-1] >= chosen[1:] - tol))


def check_routing(out, ref, report=None):
    """Top-k indices must equal the oracle's (set and slot order) except on
    near-tie tokens: where the oracle's keys of the experts that differ lie
    within 1e-5 (at the k-th/(k+1)-th boundary, or between adjacent slots).
    Those tokens must still hold a valid top-k of the oracle's keys up to
    1e-5; they are counted (``report``) and left out of the value comparison.
    Returns the boolean mask of rows that route exactly like the oracle."""
    gi = out["idx"].cpu().numpy()
    same = np.all(gi == ref["idx"], axis=1)
    if ref["keys"] is None:  # hash routing: exact
        assert np.all(same)
        return same
    bad = [t for t in np.nonzero(~same)[0] if not routing_consistent(gi[t], ref["keys"][t])]
    assert not bad, f"routing differs beyond near ties on tokens {bad[:10]}"
    if report is not None:
        report["near_tie_tokens"] = int((~same).sum())
    if (~same).any():
        print(f"near-tie tokens (routing differs within 1e-5 of the oracle's keys): {int((~same).sum())}")
    return same


def cfg_k(ref):
    return ref["idx"].shape[1]


def host_weights(cfg):
    hw = SD.HostWeights(cfg)
    return O.FP4Weights(hw) if cfg.weight_format else hw


def oracle_full(cfg, T=None, rows=None):
    """Oracle on the workload's inputs (all T rows routed; experts for ``rows``)."""
    T = cfg.T if T is None else T
    hw = host_weights(cfg)
    x = SD.host_rows(cfg, "x", range(T), T=T)
    r = SD.host_rows(cfg, "residual", range(T), T=T)
    ids = W.host_token_ids(cfg, T)
    return O.moe_layer(cfg, hw, x, r, ids, rows=rows), hw
