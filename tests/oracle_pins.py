"""Pins for the oracle: checks against what the pages and the mathematics fix.

Each ``pin_*`` takes the oracle module ``O`` and raises AssertionError when the
oracle disagrees with its pin.  ``test_oracle_pins.py`` runs them on the real
oracle; ``test_oracle_mutations.py`` runs them on copies with planted mistakes
and requires every mistake to trip at least one pin.

Pins use worked examples printed on the pages (``tests/golden``), closed
forms derived by hand for tiny inputs, brute force, invariants, and library
routines on special cases (torch's fp32 -> bf16 rounding).
"""
from __future__ import annotations

import json
import math
import os
import types

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _cfg(**kw):
    base = dict(D=2, E=2, k=1, I=2, n_shared=0, I_shared=2, router=0, renormalize=0,
                routed_scale=1.0, gate_clamp_max=math.inf, up_clamp=math.inf, eps=1e-6,
                hash_mult=2654435761)
    base.update(kw)
    return types.SimpleNamespace(**base)


def _torch_bf16(v):
    """Library routine: torch's fp32 -> bf16 conversion (round to nearest even)."""
    import torch
    return torch.tensor(np.asarray(v, np.float32)).to(torch.bfloat16).to(torch.float64).numpy()


# ------------------------------------------------------------------ bf16
def pin_round_bf16(O):
    # Ties go to even: 1 + 2^-8 lies halfway between 1 and 1 + 2^-7.
    assert O.round_bf16(1 + 2.0 ** -8) == 1.0
    assert O.round_bf16(1 + 3 * 2.0 ** -8) == 1 + 2.0 ** -6
    assert O.round_bf16(-(1 + 2.0 ** -8)) == -1.0
    # Just above a tie rounds up; rounding through fp32 first would land on
    # the tie and round down (double rounding), so this pins one rounding.
    assert O.round_bf16(1 + 2.0 ** -8 + 2.0 ** -40) == 1 + 2.0 ** -7
    # 3/sqrt(12.5) = 0.84852...: quantum 2^-9 in [0.5, 1), 434.45 -> 434.
    assert O.round_bf16(3 / math.sqrt(12.5)) == 434 * 2.0 ** -9
    # fp32-representable values: agree with torch's RNE conversion.
    rng = np.random.default_rng(5)
    v = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-30, 30, 20000),
                        [0.0, -0.0, 1e-40, -3e-39, 3.3e38]]).astype(np.float32).astype(np.float64)
    assert np.array_equal(O.round_bf16(v), _torch_bf16(v))


# --------------------------------------------------------------- RMSNorm
def pin_rmsnorm_worked_example(O):
    g = golden("rmsnorm_worked_example.json")
    x = np.array([g["x"]])
    y = O.rmsnorm(x, np.ones(2), 1e-6)[0]
    tol = 0.5 * 10.0 ** -g["printed_decimals"] + 1e-6
    rms = math.sqrt((3.0 ** 2 + 4.0 ** 2) / 2)  # the page's RMS, 3.536
    assert abs(rms - g["rms_printed"]) <= tol
    assert np.allclose(y, g["normalized_printed"], atol=tol, rtol=0)
    assert abs(math.sqrt(np.mean(y * y)) - g["rms_of_output_printed"]) <= tol
    # The epsilon sits inside the root: with eps = 1, RMS = sqrt(12.5 + 1).
    y1 = O.rmsnorm(x, np.ones(2), 1.0)[0]
    assert np.allclose(y1, [3 / math.sqrt(13.5), 4 / math.sqrt(13.5)], rtol=1e-15, atol=0)
    # Gains multiply element-wise after the normalisation.
    y2 = O.rmsnorm(x, np.array([2.0, -0.5]), 0.0)[0]
    assert np.allclose(y2, [2 * 3 / math.sqrt(12.5), -0.5 * 4 / math.sqrt(12.5)], rtol=1e-15)


def pin_rmsnorm_scale_invariance(O):
    g = golden("rmsnorm_scale_invariance.json")
    u = np.random.default_rng(1).standard_normal((4, 64))
    a = O.rmsnorm(u, np.ones(64), 0.0)
    b = O.rmsnorm(g["scale"] * u, np.ones(64), 0.0)
    assert np.allclose(a, b, rtol=1e-13, atol=0)
    # Each normalised row has RMS 1 (eps = 0).
    assert np.allclose(np.sqrt(np.mean(a * a, axis=-1)), 1.0, rtol=1e-13)


def pin_xn_bf16_by_hand(O):
    # By hand: [3,4], eps 1e-6: 3/sqrt(12.5) = 0.848528 -> 434 * 2^-9; 4/sqrt(12.5) = 1.131371 -> 145 * 2^-7.
    assert np.array_equal(O.xn_bf16(np.array([[3.0, 4.0]]), np.ones(2), 1e-6)[0],
                          [434 * 2.0 ** -9, 145 * 2.0 ** -7])
    # eps = 1 sits inside the root: 3/sqrt(13.5) = 0.816497 -> 418 * 2^-9; 4/sqrt(13.5) = 1.088662 -> 139 * 2^-7.
    assert np.array_equal(O.xn_bf16(np.array([[3.0, 4.0]]), np.ones(2), 1.0)[0],
                          [418 * 2.0 ** -9, 139 * 2.0 ** -7])
    # Gains after the scale: 2 * 0.848528 = 1.697056 -> 217 * 2^-7; -0.5 * 1.131371 = -0.565685 -> -290 * 2^-9.
    assert np.array_equal(O.xn_bf16(np.array([[3.0, 4.0]]), np.array([2.0, -0.5]), 0.0)[0],
                          [217 * 2.0 ** -7, -290 * 2.0 ** -9])


def _bf16_mag_value(m):
    """Exact value (a Fraction) of the non-negative bf16 whose magnitude bits are m."""
    from fractions import Fraction
    return Fraction(float(np.array([m << 16], np.uint32).view(np.float32)[0]))


def _is_correct_bf16(c, gx, S):
    """Is the bf16 value c the round-to-nearest-even of v = gx / sqrt(S)?
    Decided in exact rational arithmetic: v lies between the midpoints
    m- < v < m+ around c  <=>  (m-)^2 S < gx^2 < (m+)^2 S (signs apart), and a
    value exactly on a midpoint goes to the even code."""
    from fractions import Fraction
    bits = int(np.array([c], np.float32).view(np.uint32)[0] >> 16)
    mag, neg = bits & 0x7FFF, bool(bits & 0x8000)
    if gx == 0:
        return mag == 0
    if (gx < 0) != neg:
        return False
    lo = (_bf16_mag_value(mag - 1) + _bf16_mag_value(mag)) / 2 if mag > 0 else Fraction(0)
    hi = (_bf16_mag_value(mag) + _bf16_mag_value(mag + 1)) / 2
    a2 = gx * gx
    even = mag % 2 == 0
    below = lo * lo * S
    above = hi * hi * S
    ok_lo = a2 > below or (a2 == below and even)
    ok_hi = a2 < above or (a2 == above and even)
    return ok_lo and ok_hi


def pin_xn_bf16_exact_at_rounding_boundaries(O):
    """xn = bf16(g x / sqrt(mean(x^2) + eps)) rounded once from the exact value
    ([LD] "RMSNorm before up-projection").  Rows are screened for elements that
    lie within 2^-16 of a bf16 quantum from a rounding midpoint -- where any
    intermediate rounding to fp32 (of the scale or of a product) can move the
    value across the midpoint -- and every element of those rows is checked in
    exact rational arithmetic."""
    from fractions import Fraction
    rng = np.random.default_rng(2024)
    D, n = 256, 3000
    x = O.round_bf16(rng.standard_normal((n, D)))
    g = O.round_bf16(1 + 0.1 * rng.standard_normal(D))
    eps = 1e-6
    # Screen in fp64: distance from the nearest midpoint in units of the quantum.
    v = g * x / np.sqrt(np.mean(x * x, axis=1, keepdims=True) + eps)
    _, e = np.frexp(v)
    t = np.ldexp(v, -(e.astype(np.int64) - 8))          # v in units of its bf16 quantum
    dist = np.abs(t - np.floor(t) - 0.5)
    rows = np.unique(np.nonzero(dist < 2.0 ** -16)[0])
    assert len(rows) >= 8, len(rows)                     # enough boundary cases to test
    xn = O.xn_bf16(x[rows], g, eps)
    eps_q = Fraction(eps)
    gq = [Fraction(float(gi)) for gi in g]
    for ri, r in enumerate(rows):
        xr = [Fraction(float(xi)) for xi in x[r]]
        S = sum(xi * xi for xi in xr) / D + eps_q
        for d in range(D):
            assert _is_correct_bf16(xn[ri, d], gq[d] * xr[d], S), (int(r), d)


# ------------------------------------------------------------------ SwiGLU
def pin_swish_example(O):
    g = golden("swish_worked_example.json")
    v = float(O.swiglu(g["gate"], g["up"]))
    assert abs(v - g["printed"]) <= 1e-3 * g["printed"]
    # Closed form: Swish(20) * 30 = 600 / (1 + e^-20).
    assert abs(v - 600.0 / (1.0 + math.exp(-20.0))) <= 1e-12 * 600
    # Swish(a) = a * sigmoid(a): Swish(0) = 0 and Swish(-a) = Swish(a) - a.
    assert float(O.swiglu(0.0, 5.0)) == 0.0
    a = 1.7
    assert abs(float(O.swiglu(-a, 1.0)) - (float(O.swiglu(a, 1.0)) - a)) < 1e-15


def pin_swiglu_clamp(O):
    g = golden("swiglu_clamp.json")
    cg, cu = g["gate_clamp_max"], g["up_clamp"]
    silu10 = 10.0 / (1.0 + math.exp(-10.0))
    # Large inputs: SiLU(10) * 10, below 10 * 10.
    assert abs(float(O.swiglu(20.0, 30.0, cg, cu)) - silu10 * 10) < 1e-12
    assert float(O.swiglu(20.0, 30.0, cg, cu)) < 100.0
    assert abs(float(O.swiglu(20.0, -30.0, cg, cu)) + silu10 * 10) < 1e-12
    # The gate has no lower bound: SiLU(-20) * (-10), not SiLU(-10) * (-10).
    want = (-20.0 / (1.0 + math.exp(20.0))) * -10.0
    assert abs(float(O.swiglu(-20.0, -30.0, cg, cu)) - want) < 1e-18
    # Inside the bounds the clamp changes nothing.
    rng = np.random.default_rng(2)
    gg, uu = rng.uniform(-9.9, 9.9, 1000), rng.uniform(-9.9, 9.9, 1000)
    assert np.array_equal(O.swiglu(gg, uu, cg, cu), O.swiglu(gg, uu))
    # Bound over any input: |out| <= SiLU(10) * 10.
    big = rng.standard_normal((2, 10000)) * 50
    assert np.max(np.abs(O.swiglu(big[0], big[1], cg, cu))) <= silu10 * 10 + 1e-12


def pin_situ_glu(O):
    """SiTU-GLU against the limits and bounds the page states, not its formula."""
    g = golden("situ_glu.json")
    b1, b2 = g["beta_gate"], g["beta_up"]

    def situ(gg, uu):
        return np.asarray(O.glu_unit(gg, uu, O.ACT_SITU_GLU, beta_g=b1, beta_u=b2), np.float64)

    # Bounded by beta1 * beta2 (the page's 4 x 25 = 100) on any input, and the
    # page's example (20, 30) is far below SwiGLU's ~600.
    rng = np.random.default_rng(5)
    big = rng.standard_normal((2, 20000)) * 200
    assert np.max(np.abs(situ(big[0], big[1]))) <= g["bound_printed"]
    v = float(situ(g["gate"], g["up"]))
    assert 0.0 < v < g["bound_printed"] < float(O.swiglu(g["gate"], g["up"]))
    # Near the origin the soft caps are the identity to second order, so the
    # unit equals SwiGLU up to a relative O(x^2) term (the page: it keeps
    # SwiGLU's local response).
    for s_ in (1e-2, 1e-3):
        gg, uu = 0.7 * s_, -0.4 * s_
        assert abs(float(situ(gg, uu)) / float(O.swiglu(gg, uu)) - 1.0) < 2 * s_ ** 2
    # Saturation of each branch alone: a large gate passes beta1 * u for a small
    # up value; a large up value passes beta2 * Swish(g) for a small gate.
    u0, g0 = 1e-4, 1e-4
    assert abs(float(situ(60.0, u0)) / (b1 * u0) - 1.0) < 1e-6
    assert abs(float(situ(g0, 1e4)) / (b2 * g0 / (1.0 + math.exp(-g0))) - 1.0) < 1e-6
    # Both large: the product of the caps.
    assert abs(float(situ(1e3, 1e4)) - b1 * b2) < 1e-9 * b1 * b2
    # The Sigmoid of the gate closes the unit for a very negative gate,
    # whatever the up branch.
    assert abs(float(situ(-60.0, 1e4))) < 1e-20
    # The up branch is odd.
    assert float(situ(2.0, -3.0)) == -float(situ(2.0, 3.0))


# ------------------------------------------------------------------ top-k
def _brute_topk(row, k):
    order = sorted(range(len(row)), key=lambda e: (-row[e], e))
    return order[:k]


def pin_topk_bruteforce(O):
    rng = np.random.default_rng(3)
    for E, k in [(8, 2), (64, 6), (256, 8), (5, 5), (7, 1)]:
        keys = np.round(rng.standard_normal((50, E)), 1)  # rounding makes many ties
        got = O.topk_desc(keys, k)
        for t in range(50):
            assert list(got[t]) == _brute_topk(list(keys[t]), k), (E, k, t)
    # All equal: the lowest indices, in order.
    assert list(O.topk_desc(np.zeros((1, 6)), 3)[0]) == [0, 1, 2]


def pin_margin(O):
    keys = np.array([[0.1, 0.5, 0.3, 0.45]])
    assert abs(O.topk_margin(keys, 2)[0] - (0.45 - 0.3)) < 1e-15
    assert abs(O.topk_margin(keys, 1)[0] - (0.5 - 0.45)) < 1e-15
    assert O.topk_margin(keys, 4)[0] == np.inf


# ------------------------------------------------------------------ routers
def pin_softmax_router(O):
    # E = 2, k = 1: the chosen weight is p_max = sigmoid(l_max - l_min).
    logits = np.array([[0.2, 1.1], [3.0, -1.0]])
    idx, w, _ = O.route_softmax(logits, 1, False, 1.0)
    assert list(idx[:, 0]) == [1, 0]
    assert abs(w[0, 0] - 1 / (1 + math.exp(-0.9))) < 1e-15
    assert abs(w[1, 0] - 1 / (1 + math.exp(-4.0))) < 1e-15
    # Renormalised weights sum to routed_scale; plain ones are the probabilities.
    rng = np.random.default_rng(4)
    L = rng.standard_normal((20, 64))
    idx, w, p = O.route_softmax(L, 6, True, 1.0)
    assert np.allclose(w.sum(-1), 1.0, rtol=1e-14)
    idx2, w2, _ = O.route_softmax(L, 6, False, 1.0)
    assert np.array_equal(idx, idx2)
    assert np.allclose(w2.sum(-1), np.sort(p, -1)[:, -6:].sum(-1), rtol=1e-14)
    assert np.all(w2.sum(-1) < 1.0)
    # A logit bias is added before the softmax.
    idx3, w3, _ = O.route_softmax(np.array([[0.0, 0.0]]), 1, False, 1.0, np.array([0.0, math.log(3)]))
    assert idx3[0, 0] == 1 and abs(w3[0, 0] - 0.75) < 1e-15


def pin_sigmoid_router(O):
    # The bias moves selection but not the weights: expert 0 has the larger
    # score, expert 1 wins on score + bias, and its weight uses its own score.
    logits = np.array([[1.0, 0.5, -2.0]])
    bias = np.array([0.0, 0.2, 0.0])
    s = [1 / (1 + math.exp(-v)) for v in logits[0]]
    idx, w, _ = O.route_sigmoid_bias(logits, bias, 1, False, 1.0)
    assert idx[0, 0] == 1 and abs(w[0, 0] - s[1]) < 1e-15
    idx, w, _ = O.route_sigmoid_bias(logits, bias, 2, True, 2.5)
    assert list(idx[0]) == [1, 0]
    assert abs(w[0, 0] - 2.5 * s[1] / (s[0] + s[1])) < 1e-15
    rng = np.random.default_rng(6)
    L = rng.standard_normal((30, 256)) * 1.7
    _, w, _ = O.route_sigmoid_bias(L, rng.standard_normal(256) * 0.01, 8, True, 2.5)
    assert np.allclose(w.sum(-1), 2.5, rtol=1e-14)


def pin_hash(O):
    g = golden("hash_routing.json")
    for c in g["cases"]:
        assert int(O.hash_expert0(np.array([c["id"]]), c["E"], g["mult"])[0]) == c["expert"], c
    idx, w, _ = O.route_hash(np.array([1, 2]), 128, 8, g["mult"], 1.0)
    assert list(idx[0]) == [(49 + j) % 128 for j in range(8)]
    assert list(idx[1]) == [(98 + j) % 128 for j in range(8)]
    assert np.all(w == 1.0 / 8)
    # Wrap-around keeps the k experts distinct.
    idx, _, _ = O.route_hash(np.array([1]), 50, 8, g["mult"], 1.0)  # e0 = 2654435761 % 50 = 11
    assert list(idx[0]) == list(range(11, 19))
    idx, _, _ = O.route_hash(np.array([3]), 8, 8, g["mult"], 1.0)   # e0 = 0xDAA66D13 % 8 = 3
    assert sorted(idx[0]) == list(range(8)) and idx[0, 0] == 3


# -------------------------------------------------------- histogram/permute
def pin_histogram_permute_bruteforce(O):
    rng = np.random.default_rng(7)
    for T, E, k in [(40, 8, 2), (100, 16, 4), (33, 5, 5), (1, 8, 3)]:
        idx = np.stack([rng.permutation(E)[:k] for _ in range(T)])
        counts = O.expert_histogram(idx, E)
        offsets, ptok, pslot, pos = O.stable_permute(idx, E)
        want_counts = [sum(1 for t in range(T) for j in range(k) if idx[t, j] == e) for e in range(E)]
        assert list(counts) == want_counts
        rows = []
        for e in range(E):
            seg = sorted((t, j) for t in range(T) for j in range(k) if idx[t, j] == e)
            assert offsets[e] == len(rows)
            rows += seg
        assert offsets[E] == T * k
        assert list(zip(ptok.tolist(), pslot.tolist())) == rows
        for p, (t, j) in enumerate(rows):
            assert pos[t, j] == p


# ---------------------------------------------------- partial-sum epilogue
def pin_fixed_vs_ring_order(O):
    # Non-associativity (the pages' (a + b) + c != a + (b + c)), by hand in
    # fp32 with three partials and one element per chunk:
    #   fixed, every element: (1 + 2^-24) + 2^-24 = 1 + 2^-24 -> 1 (tie, even), then 1.
    #   ring, chunk 2 (owner r2): (2^-24 + 2^-24) + 1 = 2^-23 + 1, representable.
    r = np.zeros((3, 3), np.float32)
    r[0, :] = 1.0
    r[1, :] = 2.0 ** -24
    r[2, :] = 2.0 ** -24
    assert np.array_equal(O.allreduce_fixed_order_f32(r), np.float32([1, 1, 1]))
    assert np.array_equal(O.allreduce_ring_order_f32(r), np.float32([1, 1, 1 + 2.0 ** -23]))
    # Chunk ownership follows the ring (chunk c: r_c, r_{c-1}, ...).  P = 4,
    # r0 = r1 = 2^-24, r2 = 2, r3 = -2; fp32 ulp is 2^-23 in [1,2), 2^-22 in [2,4):
    #   fixed, every element: ((2^-23) + 2) -> tie -> 2 ; - 2 = 0.
    #   chunk 0: r0 + r3 = -(2 - 2^-24) -> tie -> -2 ; + 2 = 0 ; + 2^-24 = 2^-24.
    #   chunk 1: r1 + r0 = 2^-23 ; - 2 = -(2 - 2^-23), exact ; + 2 = 2^-23.
    #   chunk 2: r2 + r1 -> 2 ; + r0 -> 2 ; - 2 = 0.
    #   chunk 3: r3 + r2 = 0 ; + 2^-24 ; + 2^-24 = 2^-23.
    q = np.zeros((4, 4), np.float32)
    q[0, :] = 2.0 ** -24
    q[1, :] = 2.0 ** -24
    q[2, :] = 2.0
    q[3, :] = -2.0
    assert np.array_equal(O.allreduce_fixed_order_f32(q), np.float32([0, 0, 0, 0]))
    assert np.array_equal(O.allreduce_ring_order_f32(q),
                          np.float32([2.0 ** -24, 2.0 ** -23, 0, 2.0 ** -23]))
    # Random case: both orders stay within the fp32 error bound of the exact sum.
    rng = np.random.default_rng(8)
    parts = (rng.standard_normal((8, 4, 512)) / 8).astype(np.float32)
    exact = parts.astype(np.float64).sum(0)
    bound = 7 * 2.0 ** -24 * np.abs(parts.astype(np.float64)).sum(0) * 1.0001
    for got in (O.allreduce_fixed_order_f32(parts), O.allreduce_ring_order_f32(parts)):
        assert np.all(np.abs(got.astype(np.float64) - exact) <= bound)
    assert not np.array_equal(O.allreduce_fixed_order_f32(parts), O.allreduce_ring_order_f32(parts))


def pin_reduce_partials(O):
    # r = fixed-order sum + residual in fp32; one element by hand:
    # partials 0.5, 0.25, 2^-30 ... sum = 0.75 (2^-30 lost), + residual 1.0 = 1.75.
    parts = np.zeros((3, 1, 2), np.float32)
    parts[:, 0, 0] = [0.5, 0.25, 2.0 ** -30]
    parts[:, 0, 1] = [-1.0, 0.0, 0.0]
    res = np.array([[1.0, 0.0]], np.float32)
    out_norm, out_res, r = O.reduce_partials(parts, res, np.ones(2), 0.0)
    assert r[0, 0] == np.float32(1.75) and r[0, 1] == np.float32(-1.0)
    assert np.array_equal(out_res[0], [1.75, -1.0])
    rms = math.sqrt((1.75 ** 2 + 1.0) / 2)
    assert np.allclose(out_norm[0], _torch_bf16([1.75 / rms, -1.0 / rms]), rtol=0, atol=0)


# --------------------------------------------------------- closed-form layer
def closed_form_case():
    """T=1, D=2, I=2, E=2, top-1 softmax, one shared expert, chosen so every
    step can be done by hand."""
    cfg = _cfg(D=2, E=2, k=1, I=2, n_shared=1, I_shared=2)
    Z = np.zeros((2, 2))
    w_router = np.array([[1.0, 0.0], [0.0, 1.0]])            # logits = xn
    w_gate = np.stack([Z, [[1.0, 0.0], [0.0, 0.0]]])          # g = [xn0, 0]
    w_up = np.stack([Z, [[0.0, 1.0], [1.0, 0.0]]])            # u = [xn1, xn0]
    w_down = np.stack([Z, [[1.0, 0.0], [-1.0, 0.0]]])         # y = [h0, -h0]
    ws_gate = np.array([[[0.0, 1.0], [0.0, 0.0]]])            # gs = [xn1, 0]
    ws_up = np.array([[[1.0, 0.0], [0.0, 0.0]]])              # us = [xn0, 0]
    ws_down = np.array([[[0.0, 0.0], [1.0, 0.0]]])            # ys = [0, hs0]
    W = types.SimpleNamespace(w_router=w_router, router_bias=None, g_in=np.ones(2),
                              g_out=np.ones(2))
    W.routed = lambda e: (w_gate[e], w_up[e], w_down[e])
    W.shared = lambda s: (ws_gate[s], ws_up[s], ws_down[s])
    x = np.array([[3.0, 4.0]])
    residual = np.array([[0.5, -0.25]])
    return cfg, W, x, residual


def pin_closed_form_layer(O):
    cfg, W, x, residual = closed_form_case()
    out = O.moe_layer(cfg, W, x, residual)
    # By hand.  RMS([3,4]) = sqrt(12.5 + 1e-6); xn = bf16(3/RMS, 4/RMS):
    # 0.848528 -> 434 * 2^-9 = 0.84765625 ; 1.131371 -> 145 * 2^-7 = 1.1328125.
    xn0, xn1 = 434 * 2.0 ** -9, 145 * 2.0 ** -7
    assert np.array_equal(out["xn"][0], [xn0, xn1])
    # Router: logits = xn; expert 1 wins; weight = p_1 = 1/(1 + e^-(xn1 - xn0)).
    assert out["idx"][0, 0] == 1
    w = 1.0 / (1.0 + math.exp(-(xn1 - xn0)))
    assert abs(out["w"][0, 0] - w) < 1e-15
    silu = lambda a: a / (1.0 + math.exp(-a))  # noqa: E731
    h0 = float(_torch_bf16(silu(xn0) * xn1))      # gate = xn0, up = xn1
    hs0 = float(_torch_bf16(silu(xn1) * xn0))     # shared: gate = xn1, up = xn0
    r = np.array([w * h0 + 0.5, -w * h0 + hs0 - 0.25])
    assert np.allclose(out["r"][0], r, rtol=1e-15, atol=1e-16)
    rms = math.sqrt((r[0] ** 2 + r[1] ** 2) / 2 + 1e-6)
    assert np.array_equal(out["out_residual"][0], _torch_bf16(r))
    assert np.array_equal(out["out_norm"][0], _torch_bf16(r / rms))
    # Counts / permutation of the single routed row.
    assert list(out["counts"]) == [0, 1] and list(out["offsets"]) == [0, 0, 1]


def pin_forced_routing(O):
    """Forced indices replace the top-k choice; the weights stay the router's
    own scores of the forced experts (worked by hand on the closed-form case)."""
    cfg, W, x, residual = closed_form_case()
    out = O.moe_layer(cfg, W, x, residual, force_idx=np.array([[0]]))
    xn0, xn1 = 434 * 2.0 ** -9, 145 * 2.0 ** -7
    # Expert 0 (all-zero weights) instead of expert 1: its output is 0; its
    # weight is p_0 = 1/(1 + e^(xn1 - xn0)).
    assert out["idx"][0, 0] == 0
    assert abs(out["w"][0, 0] - 1.0 / (1.0 + math.exp(xn1 - xn0))) < 1e-15
    silu = lambda a: a / (1.0 + math.exp(-a))  # noqa: E731
    hs0 = float(_torch_bf16(silu(xn1) * xn0))
    assert np.allclose(out["r"][0], [0.5, hs0 - 0.25], rtol=1e-15, atol=1e-16)
    assert list(out["counts"]) == [1, 0]
    # The margin still describes the oracle's own choice (expert 1 over 0).
    p1 = 1.0 / (1.0 + math.exp(-(xn1 - xn0)))
    assert abs(out["margin"][0] - (p1 - (1 - p1))) < 1e-15
    # Forcing the oracle's own choice changes nothing; forcing the reversed
    # slot order reverses the weights and reorders only the routed sum.
    for router, extra in [(0, {}), (1, {"renormalize": 1, "routed_scale": 2.5}), (2, {})]:
        cfg, W, xr, res, ids = small_random_case(O, router=router, **extra)
        a = O.moe_layer(cfg, W, xr, res, ids)
        b = O.moe_layer(cfg, W, xr, res, ids, force_idx=a["idx"])
        assert np.array_equal(a["out_norm"], b["out_norm"]) and np.array_equal(a["w"], b["w"])
        c = O.moe_layer(cfg, W, xr, res, ids, force_idx=a["idx"][:, ::-1])
        assert np.array_equal(c["idx"], a["idx"][:, ::-1])
        if router != 2:
            assert np.array_equal(c["w"], a["w"][:, ::-1])
        assert np.allclose(c["r"], a["r"], rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------- dense cross-check
def small_random_case(O, router=0, T=24, D=64, E=8, k=2, I=32, S=1, seed=9, **kw):
    rng = np.random.default_rng(seed)
    bf = lambda a: O.round_bf16(a)  # noqa: E731
    cfg = _cfg(D=D, E=E, k=k, I=I, n_shared=S, I_shared=I, router=router, **kw)
    W = O.Weights(
        w_router=bf(rng.standard_normal((E, D)) * 0.3),
        router_bias=(rng.standard_normal(E) * 0.01) if router == 1 else None,
        w_gate=bf(rng.standard_normal((E, I, D)) * 0.1), w_up=bf(rng.standard_normal((E, I, D)) * 0.1),
        w_down=bf(rng.standard_normal((E, D, I)) * 0.1),
        ws_gate=bf(rng.standard_normal((S, I, D)) * 0.1), ws_up=bf(rng.standard_normal((S, I, D)) * 0.1),
        ws_down=bf(rng.standard_normal((S, D, I)) * 0.1),
        g_in=bf(1 + 0.1 * rng.standard_normal(D)), g_out=bf(1 + 0.1 * rng.standard_normal(D)))
    x = bf(rng.standard_normal((T, D)))
    res = bf(rng.standard_normal((T, D)))
    ids = rng.integers(0, 128000, T)
    return cfg, W, x, res, ids


def pin_dense_masked(O):
    for router, extra in [(0, {}), (0, {"renormalize": 1}), (1, {"renormalize": 1, "routed_scale": 2.5,
                                                                     "gate_clamp_max": 0.3, "up_clamp": 0.3}),
                          (2, {})]:
        cfg, W, x, res, ids = small_random_case(O, router=router, **extra)
        a = O.moe_layer(cfg, W, x, res, ids)
        b = O.moe_layer_dense_masked(cfg, W, x, res, ids)
        assert np.allclose(a["r"], b["r"], rtol=1e-12, atol=1e-12), router
        assert np.array_equal(a["idx"], b["idx"])
        # Sampled rows give the same rows as the full run.
        rows = np.array([3, 0, 17])
        c = O.moe_layer(cfg, W, x, res, ids, rows=rows)
        assert np.array_equal(c["out_norm"], a["out_norm"][rows])


def pin_mac_count(O):
    # [LD] "FLOPs与参数量": an MoE with k active experts costs k times one expert;
    # a SwiGLU expert multiplies by three D x I matrices, so the expert matmuls
    # perform T*k*3*D*I + T*S*3*D*I_s multiply-adds.
    for S in (0, 1, 2):
        cfg, W, x, res, ids = small_random_case(O, S=S, T=10, D=64, E=8, k=3, I=32)
        O.MAC_COUNTER[0] = 0
        O.moe_layer(cfg, W, x, res, ids)
        assert O.MAC_COUNTER[0] == 10 * 3 * 3 * 64 * 32 + 10 * S * 3 * 64 * 32


# ------------------------------------------------------------ latent MoE
def pin_latent_closed_form(O):
    """[LD] "潜在MoE": down-project, route and run the experts in the latent
    space, sum, up-project; shared experts at full width.  T=1, D=2, l=1, two
    routed experts (top-1, renormalised), one shared expert, by hand."""
    bf = O.round_bf16
    cfg = _cfg(D=2, E=2, k=1, I=1, n_shared=1, I_shared=1, renormalize=1, latent=1)
    W = O.Weights(w_router=np.array([[1.0], [-1.0]]), router_bias=None,
                  w_gate=np.array([[[2.0]], [[1.0]]]), w_up=np.array([[[1.0]], [[1.0]]]),
                  w_down=np.array([[[0.375]], [[1.0]]]),
                  ws_gate=np.array([[[0.5, 0.5]]]), ws_up=np.array([[[1.0, -0.5]]]),
                  ws_down=np.array([[[1.0], [0.25]]]), g_in=np.ones(2), g_out=np.ones(2),
                  w_proj_down=np.array([[129 / 256, 129 / 512]]), w_proj_up=np.array([[2.0], [-4.0]]))
    assert np.array_equal(bf(W.w_proj_down), W.w_proj_down)
    out = O.moe_layer(cfg, W, np.array([[1.0, 1.0]]), np.zeros((1, 2)))
    # xn = bf16(1 / sqrt(1 + 1e-6)) = 1; z = bf16(387/512), a tie between 193/256
    # and 194/256 that goes to the even 194/256.
    assert np.array_equal(out["xn"][0], [1.0, 1.0])
    z = 194 / 256
    assert out["z"][0, 0] == z
    # Router on z: logits [z, -z], expert 0, weight 1 after renormalising.
    assert out["idx"][0, 0] == 0 and out["w"][0, 0] == 1.0
    # Expert 0 in the latent space: g = 2z, u = z, h = bf16(g sigmoid(g) u).
    g = 2 * z
    hv = g / (1.0 + math.exp(-g)) * z
    assert 240.5 / 256 < hv < 241.5 / 256
    # y0 = h * 0.375 = 723/2048; a = bf16(y0) = 181/512 (723/2048 = 180.75/512).
    assert out["lat_sum"][0, 0] == 723 / 2048
    assert out["agg"][0, 0] == 181 / 512
    # Shared expert on xn at full width: g = 1, u = 0.5, h = bf16(sigmoid(1) / 2) = 187/512.
    hs = 0.5 / (1.0 + math.exp(-1.0))
    assert 186.5 / 512 < hs < 187.5 / 512
    acc = np.array([181 / 256 + 187 / 512, -181 / 128 + 187 / 2048])
    assert np.array_equal(out["acc"][0], acc)
    # out_residual = bf16(acc): 137.25/128 -> 137/128, -169.3125/128 -> -169/128.
    assert np.array_equal(out["out_residual"][0], [137 / 128, -169 / 128])


def _latent_case(O, l=16, router=0, S=1, seed=11, **kw):
    cfg, W, x, res, ids = small_random_case(O, router=router, S=S, seed=seed, **kw)
    rng = np.random.default_rng(seed + 1)
    bf = O.round_bf16
    E, D, I = cfg.E, cfg.D, cfg.I
    cfg.latent = l
    W.w_router = bf(rng.standard_normal((E, l)) * 0.3)
    W.w_gate = bf(rng.standard_normal((E, I, l)) * 0.2)
    W.w_up = bf(rng.standard_normal((E, I, l)) * 0.2)
    W.w_down = bf(rng.standard_normal((E, l, I)) * 0.2)
    W.w_proj_down = bf(rng.standard_normal((l, D)) * 0.15)
    W.w_proj_up = bf(rng.standard_normal((D, l)) * 0.2)
    return cfg, W, x, res, ids


def pin_latent_dense_masked(O):
    # The routed latent sum equals every expert run on every token's z, masked
    # to its routing weights, and sampled rows equal the full run's rows.
    for router, extra in [(0, {"renormalize": 1}), (1, {"renormalize": 1, "routed_scale": 2.5})]:
        cfg, W, x, res, ids = _latent_case(O, router=router, **extra)
        a = O.moe_layer(cfg, W, x, res, ids)
        b = O.moe_layer_dense_masked(cfg, W, x, res, ids)
        assert np.array_equal(a["idx"], b["idx"])
        assert np.allclose(a["lat_sum"], b["lat_sum"], rtol=1e-12, atol=1e-13)
        rows = np.array([5, 1])
        c = O.moe_layer(cfg, W, x, res, ids, rows=rows)
        assert np.array_equal(c["out_norm"], a["out_norm"][rows])


def pin_latent_identity_projection(O):
    # With l = D and identity projections the latent layer is the plain layer
    # with its routed sum cast to bf16 before the shared experts are added.
    cfg, W, x, res, ids = small_random_case(O, router=0, renormalize=1, seed=13)
    plain = O.moe_layer(cfg, W, x, res, ids)
    cfg_l = _cfg(**{**vars(cfg), "latent": cfg.D})
    eye = np.eye(cfg.D)
    W.w_proj_down, W.w_proj_up = eye, eye
    lat = O.moe_layer(cfg_l, W, x, res, ids)
    assert np.array_equal(lat["z"], plain["xn"]) and np.array_equal(lat["idx"], plain["idx"])
    routed = np.einsum("tj,tjd->td", plain["w"], plain["y_slots"])
    want = O.round_bf16(routed) + np.sum(plain["y_shared"], axis=0)
    assert np.allclose(lat["acc"], want, rtol=1e-15, atol=1e-15)


def pin_latent_mac_count(O):
    # [LD] "FLOPs与参数量" with the routed experts at the latent width l: the
    # expert matmuls perform T*k*3*l*I + T*S*3*D*I_s multiply-adds.
    cfg, W, x, res, ids = _latent_case(O, l=16, S=1)
    O.MAC_COUNTER[0] = 0
    O.moe_layer(cfg, W, x, res, ids)
    T = x.shape[0]
    assert O.MAC_COUNTER[0] == T * cfg.k * 3 * 16 * cfg.I + T * 1 * 3 * cfg.D * cfg.I_shared


# ------------------------------------------------ FP4 weights, FP8 compute
def _torch_e4m3(v):
    """torch's own float8_e4m3fn cast (round to nearest even) of fp32 values."""
    import torch
    return torch.from_numpy(np.asarray(v, np.float32)).to(torch.float8_e4m3fn).float().numpy().astype(np.float64)


def pin_e4m3_rounding(O):
    """round_e4m3 / e4m3_bits against torch's float8_e4m3fn conversion (a
    library routine): every finite code round-trips with its own bits, every
    midpoint between neighbours goes to the even one, and random values of
    every binade (normal and subnormal) round the same."""
    import torch
    codes = np.arange(256, dtype=np.uint8)
    vals = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    fin = np.isfinite(vals)
    assert fin.sum() == 254 and vals[fin].max() == O.E4M3_MAX
    assert np.array_equal(O.round_e4m3(vals[fin]), vals[fin])
    assert np.array_equal(O.e4m3_bits(vals[fin]), codes[fin])
    pos = np.unique(vals[fin & (vals >= 0)])
    mids = (pos[1:] + pos[:-1]) / 2
    assert np.array_equal(O.round_e4m3(mids), _torch_e4m3(mids))
    assert np.array_equal(O.round_e4m3(-mids), _torch_e4m3(-mids))
    rng = np.random.default_rng(21)
    r = (rng.standard_normal(50000) * np.exp2(rng.integers(-14, 9, 50000))).astype(np.float32).astype(np.float64)
    r = r[np.abs(r) <= O.E4M3_MAX]
    assert np.array_equal(O.round_e4m3(r), _torch_e4m3(r))
    # Saturation instead of overflow.
    assert float(O.round_e4m3(1e6)) == O.E4M3_MAX and float(O.round_e4m3(-500.0)) == -O.E4M3_MAX


def pin_e2m1_grid(O):
    """The E2M1 grid from the format's definition (1 sign, 2 exponent bits with
    bias 1, 1 mantissa bit; exponent field 0 is subnormal), against the page's
    facts (16 codes, largest magnitude 6), and round_e2m1 against a second,
    binade-based rounding (spacing 0.5 below 2, 1 in [2, 4), 2 in [4, 6])."""
    g = golden("fp4_fp8_quantisation.json")
    vals = []
    for sign in (1.0, -1.0):
        for e in range(4):
            for m in range(2):
                vals.append(sign * ((m / 2.0) if e == 0 else (1.0 + m / 2.0) * 2.0 ** (e - 1)))
    assert len(vals) == g["e2m1_codes"] and max(vals) == g["e2m1_max"]
    assert np.array_equal(np.array(vals[:8]), O.E2M1_GRID)
    x = np.concatenate([np.linspace(-7, 7, 28001), (O.E2M1_GRID[1:] + O.E2M1_GRID[:-1]) / 2])
    mag = np.abs(x)
    spacing = np.where(mag < 2, 0.5, np.where(mag < 4, 1.0, 2.0))
    # Each binade starts at an even multiple of its spacing, so the even
    # multiple (np.rint: ties to even) is the even code; above 6 the nearest is 6.
    alt = np.minimum(np.rint(mag / spacing) * spacing, 6.0)
    assert np.array_equal(np.abs(O.round_e2m1(x)), alt)
    assert np.array_equal(np.signbit(O.round_e2m1(x[x != 0])), np.signbit(x[x != 0]))


def pin_fp4_lossless(O):
    """The page's lossless claim: every FP4 value times a block scale 2^s with
    s in [FP4_SCALE_MIN, FP4_SCALE_MAX] is an E4M3 value (checked with torch's
    cast), and the range is the widest for which that holds."""
    q = np.concatenate([O.E2M1_GRID, -O.E2M1_GRID])
    for s_ in range(O.FP4_SCALE_MIN, O.FP4_SCALE_MAX + 1):
        v = q * 2.0 ** s_
        assert np.array_equal(_torch_e4m3(v), v), s_
    assert not np.array_equal(_torch_e4m3(6.0 * 2.0 ** (O.FP4_SCALE_MAX + 1)), 6.0 * 2.0 ** (O.FP4_SCALE_MAX + 1))
    assert float(_torch_e4m3(0.5 * 2.0 ** (O.FP4_SCALE_MIN - 1))) != 0.5 * 2.0 ** (O.FP4_SCALE_MIN - 1)


def pin_fp4_weight_blocks(O):
    """Hand-derived FP4 quantisation of two blocks (the golden file's
    derivation), blocks along the contraction (last) axis only, and the
    dequantised values lying on E4M3."""
    g = golden("fp4_fp8_quantisation.json")
    w = np.zeros((2, 64))
    w[0, :6] = g["weight_block"]
    w[0, 32:36] = g["weight_block2"]
    w[1, 40:46] = g["weight_block"]
    q, s_ = O.quantize_weights_fp4(w)
    assert s_.shape == (2, 2)
    assert s_.tolist() == [[g["weight_block_scale_exp"], g["weight_block2_scale_exp"]],
                           [O.FP4_SCALE_MIN, g["weight_block_scale_exp"]]]
    w8 = O.dequantize_fp4(q, s_)
    assert w8[0, :6].tolist() == g["weight_block_fp8"]
    assert w8[0, 32:36].tolist() == g["weight_block2_fp8"]
    assert w8[1, 40:46].tolist() == g["weight_block_fp8"]
    assert np.count_nonzero(w8) == np.count_nonzero(w8[0, :6]) + 4 + np.count_nonzero(w8[1, 40:46])
    assert np.array_equal(O.fp4_weights_as_fp8(w), w8)
    # Scales outside the lossless range are clamped: a block of magnitude 1e-4
    # would want s = -15 (6 * 2^-15 = 1.8e-4) and gets -8, so its values
    # (1e-4 / 2^-8 = 0.0256) round to 0; a block of magnitude 1000 would want
    # s = 8 and gets 6, so 1000 / 64 = 15.6 saturates to 6 * 64 = 384.
    wc = np.zeros((1, 64))
    wc[0, 0], wc[0, 32] = 1e-4, -1000.0
    qc, sc = O.quantize_weights_fp4(wc)
    assert sc.tolist() == [[O.FP4_SCALE_MIN, O.FP4_SCALE_MAX]] == [[-8, 6]]
    assert O.dequantize_fp4(qc, sc)[0, [0, 32]].tolist() == [0.0, -384.0]
    # Random weights: every value is q * 2^s with q on the grid, |w - w8| within
    # half a grid step of the block (2^s below 2, more above), and E4M3-exact.
    rng = np.random.default_rng(3)
    wr = rng.standard_normal((4, 128)) * 0.02
    q, s_ = O.quantize_weights_fp4(wr)
    assert np.all(np.isin(np.abs(q), O.E2M1_GRID))
    w8 = O.dequantize_fp4(q, s_)
    assert np.array_equal(O.round_e4m3(w8), w8)
    step = np.repeat(np.exp2(s_), 32, axis=-1)
    assert np.all(np.abs(wr - w8) <= step)   # worst gap on the grid is 2 units (between 4 and 6)


def pin_fp4_packed_storage(O):
    """The packed FP4 form: codes from the E2M1 bit layout (sign in bit 3,
    exponent in bits 2-1 with bias 1, mantissa in bit 0), a hand-packed pair,
    and the round trip master -> (packed, exponents) -> FP8 values."""
    # Codes rebuilt from the bit layout, against the oracle's grid order.
    for code in range(16):
        sign, e, m = code >> 3, (code >> 1) & 3, code & 1
        val = (m / 2.0) if e == 0 else (1.0 + m / 2.0) * 2.0 ** (e - 1)
        val = -val if sign else val
        assert int(O.e2m1_codes(np.array([val]))[0]) == (code if val != 0 or not sign else 8), code
    # [1.5, -6, 0.5, 3]: codes 3, 15, 1, 5 -> bytes 0xF3, 0x51 (low nibble first).
    packed, _ = O.pack_fp4(np.array([[1.5, -6.0, 0.5, 3.0]]), np.array([[0]]))
    assert packed.tolist() == [[0xF3, 0x51]]
    rng = np.random.default_rng(12)
    w = rng.standard_normal((3, 96)) * 0.03
    q, s_ = O.quantize_weights_fp4(w)
    packed, s8 = O.pack_fp4(q, s_)
    assert packed.shape == (3, 48) and s8.dtype == np.int8
    assert np.array_equal(O.unpack_fp4(packed, s8), O.fp4_weights_as_fp8(w))


def pin_fp8_activation_rows(O):
    """Hand-derived per-row activation scales and E4M3 codes, the scale being
    the smallest power of two that brings the row into +-448."""
    g = golden("fp4_fp8_quantisation.json")
    q, e = O.quantize_act_rows(np.array(g["act_rows"]))
    assert e.tolist() == g["act_row_exp"]
    assert q.tolist() == g["act_row_q"]
    rng = np.random.default_rng(4)
    a = rng.standard_normal((64, 96)) * np.exp2(rng.integers(-20, 20, (64, 1)))
    q, e = O.quantize_act_rows(a)
    amax = np.abs(a).max(axis=1)
    assert np.all(amax <= 448.0 * np.exp2(e)) and np.all(amax > 448.0 * np.exp2(e - 1))
    assert np.array_equal(q, _torch_e4m3(a / np.exp2(e)[:, None]))


def pin_fp8_expert_reduces_to_bf16(O):
    """When quantisation is the identity -- weights already FP4 values with
    block scale 1 (every block holds a 6 or -6) and activations E4M3 values
    whose row maximum is 448 -- the FP8 expert equals the plain expert exactly;
    with rows scaled by powers of two, g and u scale exactly."""
    rng = np.random.default_rng(8)
    D, I, n = 64, 32, 5
    grid = np.concatenate([O.E2M1_GRID, -O.E2M1_GRID])
    Wg, Wu, Wd = (rng.choice(grid, size=sh) for sh in ((I, D), (I, D), (D, I)))
    for Wm in (Wg, Wu, Wd):
        Wm[:, ::32] = 6.0
        assert np.array_equal(O.fp4_weights_as_fp8(Wm), Wm)
    x = _torch_e4m3(rng.standard_normal((n, D)) * 30)
    x[:, 3] = 448.0
    h_ref, y_ref = O.expert_ffn(x, Wg, Wu, Wd)
    h8, y8 = O.expert_ffn_fp8(x, Wg, Wu, Wd)
    assert np.array_equal(h8, h_ref)
    qh, eh = O.quantize_act_rows(h_ref)
    assert np.array_equal(y8, (qh @ Wd.T) * np.exp2(eh)[:, None])
    # The down input is quantised: y8 differs from the unquantised down product
    # wherever h is not an E4M3 multiple of its row scale.
    assert not np.array_equal(y8, y_ref)
    # Scaling a row of x by 2^j scales its gate/up sums by exactly 2^j.
    xs = x * 2.0 ** -7
    qx, ex = O.quantize_act_rows(xs)
    assert np.array_equal(qx, x) and np.all(ex == -7)


def _fp8_weights(O, W):
    """The same layer with every expert weight replaced by its FP8 values."""
    q = O.fp4_weights_as_fp8
    return O.Weights(W.w_router, W.router_bias, q(W.w_gate), q(W.w_up), q(W.w_down), q(W.ws_gate),
                     q(W.ws_up), q(W.ws_down), W.g_in, W.g_out)


def pin_fp8_dense_masked(O):
    """The FP8 layer's routed path against the every-expert masked sum, and
    sampled rows against the full run."""
    cfg, W, x, res, ids = small_random_case(O, weight_format=O.WEIGHTS_FP8, renormalize=1)
    W8 = _fp8_weights(O, W)
    a = O.moe_layer(cfg, W8, x, res, ids)
    b = O.moe_layer_dense_masked(cfg, W8, x, res, ids)
    assert np.array_equal(a["idx"], b["idx"])
    assert np.allclose(a["r"], b["r"], rtol=1e-12, atol=1e-12)
    rows = np.array([5, 1, 20])
    c = O.moe_layer(cfg, W8, x, res, ids, rows=rows)
    assert np.array_equal(c["out_norm"], a["out_norm"][rows])
    # The layer's slot outputs are the FP8 expert's (activations quantised per
    # row), not the plain expert's on the FP8 weights.
    for t, j in ((0, 0), (7, 1), (23, 0)):
        e = int(a["idx"][t, j])
        y8 = O.expert_ffn_fp8(a["xn"][[t]], *W8.routed(e))[1][0]
        assert np.array_equal(a["y_slots"][t, j], y8)
        assert not np.array_equal(O.expert_ffn(a["xn"][[t]], *W8.routed(e))[1][0], y8)
    # FP8 experts follow the bf16 layer on the master weights loosely (4-bit
    # weights of Gaussian values with power-of-two block scales are off by about
    # 12% in norm; two of them in series give about 20% here) and never equal it.
    ref = O.moe_layer(types.SimpleNamespace(**{**vars(cfg), "weight_format": O.WEIGHTS_BF16}), W, x, res, ids)
    rel = np.linalg.norm(a["acc"] - ref["acc"]) / np.linalg.norm(ref["acc"])
    assert 1e-2 < rel < 0.5


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
