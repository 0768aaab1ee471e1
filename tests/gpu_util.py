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
            if cfg.weight_format == 1:
                # FP4 expert weights: the library's own quantiser writes their E4M3 codes.
                weights = moe.quantize_expert_weights(weights)
            elif cfg.weight_format == 2:
                # ... or their storage form (packed E2M1 codes and exponent words).
                weights = moe.pack_expert_weights_fp4(weights)
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


XN_STEP_FRAC = 1e-4   # xn elements allowed one bf16 step away from the oracle's
W_TOL = 2e-3          # |w_gpu - w_oracle| on tokens routed alike (fp32 vs fp64 scores)


def ws_array(run, out, ptr, shape, dtype):
    """A tensor view of ``shape`` at device address ``ptr`` inside the forward's workspace."""
    import torch
    ws = out["ws"]
    n = int(np.prod(shape))
    nbytes = n * torch.empty(0, dtype=dtype).element_size()
    off = ptr - ws.data_ptr()
    assert 0 <= off and off + nbytes <= ws.numel()
    return ws[off:off + nbytes].view(dtype).reshape(shape)


def bf16_steps_apart(a, b):
    """Elements where a != b, and whether each such pair is one bf16 step apart
    (the spacing at the larger magnitude)."""
    d = a != b
    big = np.maximum(np.abs(a[d]), np.abs(b[d]))
    ulp = np.ldexp(1.0, np.frexp(np.maximum(big, 2.0 ** -126))[1].astype(np.int64) - 8)
    return d, np.abs(a[d] - b[d]) <= ulp * 1.0000001


def check_xn(xg, xo, frac=XN_STEP_FRAC):
    """The GPU's bf16 xn against the oracle's (the fp64 definition rounded once):
    differences, if any, are single bf16 steps on at most ``frac`` of the
    elements (values within ~2^-52 of a rounding midpoint).  Returns their count."""
    d, one = bf16_steps_apart(xg, xo)
    assert np.all(one), "xn differs from the oracle by more than one bf16 step"
    assert d.mean() <= frac, d.mean()
    return int(d.sum())


def classify_routing(cfg, out, ref, hw, xe_gpu, token_ids):
    """Top-k indices must equal the oracle's (set and slot order).  A token that
    routes differently is accepted as
      * a rounding-boundary flip when the oracle's router, run on the GPU's own
        router input for that token (xn, or z with a latent width), chooses
        exactly the GPU's experts -- an input element sat on a bf16 rounding
        boundary and the two sides rounded it to neighbouring values;
      * a near tie when the GPU's choice is a valid top-k of the oracle's keys
        up to 1e-5 (the stated exception);
    and as a failure otherwise.  Returns (mask of tokens routed alike, counts)."""
    gi = out["idx"].cpu().numpy()
    same = np.all(gi == ref["idx"], axis=1)
    rep = {"flip_tokens": 0, "near_tie_tokens": 0}
    if ref["keys"] is None:  # hash routing: exact
        assert np.all(same)
        return same, rep
    diff = np.nonzero(~same)[0]
    bad = []
    if diff.size:
        logits = O.router_logits(xe_gpu[diff], hw.w_router)
        ids = None if token_ids is None else np.asarray(token_ids)[diff]
        idx2, _, keys2 = O.route(cfg, logits, hw.router_bias, ids)
        for j, t in enumerate(diff):
            if np.array_equal(idx2[j], gi[t]):
                rep["flip_tokens"] += 1
            elif routing_consistent(gi[t], ref["keys"][t]) or routing_consistent(gi[t], keys2[j]):
                rep["near_tie_tokens"] += 1
            else:
                bad.append(int(t))
    assert not bad, f"routing differs beyond rounding-boundary flips and near ties on tokens {bad[:10]}"
    return same, rep


def check_values(cfg, out, ref, hw, x, r, ids, rows, same):
    """out_norm / out_residual of every token in ``rows``: tokens routed like
    the oracle against ``ref``; the others against the oracle run with the
    GPU's indices forced (weights from the oracle's own scores).  Returns the
    number of tokens checked on forced routing."""
    check_outputs(out, ref, rows=rows, same_rows=same[rows])
    gi = out["idx"].cpu().numpy()
    w = out["w"].cpu().numpy().astype(np.float64)
    sr = rows[same[rows]]
    if sr.size:
        assert np.abs(w[sr] - ref["w"][sr]).max() < W_TOL
    dr = rows[~same[rows]]
    if dr.size:
        ref2 = O.moe_layer(cfg, hw, x, r, ids, rows=dr, force_idx=gi)
        check_outputs(out, ref2, rows=dr)
        assert np.abs(w[dr] - ref2["w"][dr]).max() < W_TOL
    return int(dr.size)


def verify(run, out, rows=None, ref=None, hw=None, inputs=None, z_frac=1e-2):
    """Whole-layer parity of one forward against the oracle.  The oracle routes
    every token; outputs are compared on ``rows`` (all tokens when None).
    Returns (ref, mask of tokens routed like the oracle, report)."""
    cfg = run.cfg
    T = int(out["idx"].shape[0])
    hw = host_weights(cfg) if hw is None else hw
    if inputs is None:
        inputs = (SD.host_rows(cfg, "x", range(T), T=T), SD.host_rows(cfg, "residual", range(T), T=T),
                  W.host_token_ids(cfg, T))
    x, r, ids = inputs
    rows = np.arange(T) if rows is None else np.asarray(rows, np.int64)
    if ref is None:
        ref = O.moe_layer(cfg, hw, x, r, ids, rows=rows)
    import torch
    v = run.layer.views(T, out["ws"])
    xg = np64(ws_array(run, out, v.xn, (T, cfg.D), torch.bfloat16))
    rep = {"xn_step_elements": check_xn(xg, ref["xn"])}
    xe = xg
    if cfg.latent:
        # z = bf16(xn W_down^T) is rounded from the tensor cores' fp32 sum on the
        # GPU and from fp64 in the oracle: about 0.1 % of z lands one bf16 step
        # apart (or, where the dot product cancels to a tiny z, within the fp32
        # accumulation error of its terms).
        zg = np64(ws_array(run, out, v.z, (T, cfg.latent), torch.bfloat16))
        d, one = bf16_steps_apart(zg, ref["z"])
        tiny = np.abs(zg[d] - ref["z"][d]) <= 2.0 ** -16
        assert np.all(one | tiny)
        assert d.mean() < z_frac, d.mean()
        rep["z_step_elements"] = int(d.sum())
        xe = zg
    same, rr = classify_routing(cfg, out, ref, hw, xe, ids)
    rep.update(rr)
    gi = out["idx"].cpu().numpy()
    assert np.array_equal(out["counts"].cpu().numpy(), O.expert_histogram(gi, cfg.E))
    rep["forced_value_tokens"] = check_values(cfg, out, ref, hw, x, r, ids, rows, same)
    rep["value_checked_tokens"] = int(rows.size)
    print(f"parity {cfg.name} T={T}: {rep}")
    return ref, same, rep


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


def run_and_verify(cfg, **kw):
    """Forward the workload on the GPU and verify it against the oracle."""
    run = Run(cfg)
    out = run.forward(*run.inputs())
    ref, same, rep = verify(run, out, **kw)
    return run, out, ref, same, rep
