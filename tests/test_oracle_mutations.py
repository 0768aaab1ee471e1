"""Plant plausible mistakes in copies of the oracle and require a pin to catch each.

The mistakes are planted on the CPU, in a private copy of the oracle's source;
the real oracle is never modified.
"""
import os
import types

import numpy as np
import pytest

import oracle_pins as P

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "oracle", "moe_oracle.py")

MUTATIONS = {
    "eps_outside_sqrt": ("x / np.sqrt(ms + eps)", "x / (np.sqrt(ms) + eps)"),
    "gain_dropped": ("return np.asarray(g, dtype=np.float64) * (x / np.sqrt(ms + eps))",
                     "return (x / np.sqrt(ms + eps))"),
    # xn decided in a GPU kernel's fp32 precision (an fp32 scale and two fp32
    # products before the bf16 rounding) instead of the fp64 definition.
    "xn_kernel_precision": ("    return round_bf16(rmsnorm(x, g, eps))\n",
                            "    x = np.asarray(x, np.float64)\n"
                            "    s = (1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)).astype(np.float32)\n"
                            "    y = np.multiply(x.astype(np.float32), s, dtype=np.float32)\n"
                            "    y = np.multiply(y, np.asarray(g, np.float64).astype(np.float32), dtype=np.float32)\n"
                            "    return round_bf16(y.astype(np.float64))\n"),
    "xn_not_rounded": ("    return round_bf16(rmsnorm(x, g, eps))\n", "    return rmsnorm(x, g, eps)\n"),
    "forced_routing_ignored": ("idx = topk_desc(p, k) if idx is None else np.asarray(idx, np.int64)",
                               "idx = topk_desc(p, k)"),
    "forced_weights_of_natural_choice": ("    idx = topk_desc(p, k) if idx is None else np.asarray(idx, np.int64)\n    w = np.take_along_axis(p, idx, axis=-1)",
                                         "    w = np.take_along_axis(p, topk_desc(p, k), axis=-1)\n    idx = topk_desc(p, k) if idx is None else np.asarray(idx, np.int64)"),
    "double_rounding_via_fp32": ("a = np.asarray(a, dtype=np.float64)\n    _, e",
                                 "a = np.asarray(a, dtype=np.float64).astype(np.float32).astype(np.float64)\n    _, e"),
    "topk_ascending": ("neg = np.where(np.isnan(keys), np.inf, -keys)",
                       "neg = np.where(np.isnan(keys), np.inf, keys)"),
    "topk_ties_to_higher_index": ('return np.argsort(neg, axis=-1, kind="stable")[..., :k].astype(np.int64)',
                                  'return (neg.shape[-1] - 1 - np.argsort(neg[..., ::-1], axis=-1, kind="stable"))[..., :k].astype(np.int64)'),
    "softmax_no_renorm": ("    if renormalize:\n        w = w / np.sum(w, axis=-1, keepdims=True)\n    return idx, w * routed_scale, p",
                          "    return idx, w * routed_scale, p"),
    "sigmoid_weights_use_bias": ("w = np.take_along_axis(s, idx, axis=-1)",
                                 "w = np.take_along_axis(keys, idx, axis=-1)"),
    "hash_without_multiply": ("h = (ids * np.uint64(mult)) & np.uint64(0xFFFFFFFF)",
                              "h = ids & np.uint64(0xFFFFFFFF)"),
    "gate_up_swapped": ("glu_unit(x @ Wg.T, x @ Wu.T,", "glu_unit(x @ Wu.T, x @ Wg.T,"),
    "situ_betas_swapped": ("return (beta_g * np.tanh(g / beta_g) * sigmoid(g)) * (beta_u * np.tanh(u / beta_u))",
                           "return (beta_u * np.tanh(g / beta_u) * sigmoid(g)) * (beta_g * np.tanh(u / beta_g))"),
    "situ_sigmoid_of_up": ("return (beta_g * np.tanh(g / beta_g) * sigmoid(g)) * (beta_u * np.tanh(u / beta_u))",
                           "return (beta_g * np.tanh(g / beta_g) * sigmoid(u)) * (beta_u * np.tanh(u / beta_u))"),
    "situ_caps_unscaled": ("return (beta_g * np.tanh(g / beta_g) * sigmoid(g)) * (beta_u * np.tanh(u / beta_u))",
                           "return (np.tanh(g / beta_g) * sigmoid(g)) * (np.tanh(u / beta_u))"),
    "situ_falls_back_to_swiglu": ("    if act == ACT_SITU_GLU:\n        return situ_glu(g, u, beta_g, beta_u)\n", ""),
    "down_not_transposed": ("return h, h @ Wd.T", "return h, h @ Wd"),
    "silu_sign": ("return g * sigmoid(g) * u", "return g * sigmoid(-g) * u"),
    "gate_clamped_both_sides": ("g = np.minimum(np.asarray(g, np.float64), gate_clamp_max)",
                                "g = np.clip(np.asarray(g, np.float64), -gate_clamp_max, gate_clamp_max)"),
    "shared_dropped": ("        acc = acc + np.sum(np.asarray(y_shared, np.float64), axis=0)",
                       "        acc = acc"),
    "residual_after_norm": ("r = np.asarray(acc, np.float64) + np.asarray(residual, np.float64)\n    return round_bf16(rmsnorm(r, g_out, eps))",
                            "r = np.asarray(acc, np.float64) + np.asarray(residual, np.float64)\n    return round_bf16(rmsnorm(acc, g_out, eps) + residual)"),
    "slot_weights_reversed": ('acc = np.einsum("tj,tjd->td", np.asarray(w, np.float64)',
                              'acc = np.einsum("tj,tjd->td", np.asarray(w, np.float64)[:, ::-1]'),
    "permute_unstable_desc_token": ('order = np.argsort(flat, kind="stable")',
                                    'order = (len(flat) - 1 - np.argsort(flat[::-1], kind="stable"))'),
    "ring_order_used_as_fixed": ("    acc = parts[0].copy()\n    for p in range(1, parts.shape[0]):",
                                 "    return allreduce_ring_order_f32(partials)\n    acc = parts[0].copy()\n    for p in range(1, parts.shape[0]):"),
    "fixed_order_reversed": ("    acc = parts[0].copy()\n    for p in range(1, parts.shape[0]):\n        acc = np.add(acc, parts[p], dtype=np.float32)",
                             "    acc = parts[-1].copy()\n    for p in range(parts.shape[0] - 2, -1, -1):\n        acc = np.add(acc, parts[p], dtype=np.float32)"),
    "partials_residual_in_fp64": ("r = np.add(s, np.asarray(residual, np.float32), dtype=np.float32)",
                                  "r = s.astype(np.float64) + np.asarray(residual, np.float64) + 2.0 ** -30"),
    "latent_z_not_rounded": ("    return round_bf16(np.asarray(xn, np.float64) @ np.asarray(w_proj_down, np.float64).T)",
                             "    return np.asarray(xn, np.float64) @ np.asarray(w_proj_down, np.float64).T"),
    "latent_sum_not_rounded": ("    a = round_bf16(s)\n", "    a = s\n"),
    "latent_router_reads_xn": ("        logits = router_logits(xe, W.w_router)", "        logits = router_logits(xn, W.w_router)"),
    "latent_experts_read_xn": ("_, y = ffn(xe[rows[rr]]", "_, y = ffn(xn[rows[rr]]"),
    "latent_shared_reads_z": ("_, y_shared[s] = ffn(xn[rows]", "_, y_shared[s] = ffn(xe[rows]"),
    "latent_shared_dropped": ("        acc = combine(np.ones((n, 1)), y_lat[:, None, :], y_shared)",
                              "        acc = combine(np.ones((n, 1)), y_lat[:, None, :], None)"),
    "fp4_scale_floor": ("s = np.where(m <= 0.75, E - 3, E - 2)", "s = np.where(m <= 0.75, E - 4, E - 3)"),
    "fp4_ties_to_odd": ("even = cand & (np.arange(8) % 2 == 0)", "even = cand & (np.arange(8) % 2 == 1)"),
    "fp4_block_along_rows": ("    wb = w.reshape(w.shape[:-1] + (K // block, block))\n    s = fp4_block_exponent(np.abs(wb).max(axis=-1))",
                             "    wb = w.reshape(w.shape[:-1] + (K // block, block))\n    s = np.broadcast_to(fp4_block_exponent(np.abs(wb).max(axis=(-1, 0))), wb.shape[:-1])"),
    "fp4_scale_range_unclamped": ("return np.clip(s, FP4_SCALE_MIN, FP4_SCALE_MAX).astype(np.int64)",
                                  "return np.clip(s, FP4_SCALE_MIN - 4, FP4_SCALE_MAX + 4).astype(np.int64)"),
    "e4m3_no_subnormals": ("e = np.maximum(E - 1, -6)", "e = E - 1"),
    "e4m3_ties_away": ("r = np.rint(mag / ulp) * ulp", "r = np.floor(mag / ulp + 0.5) * ulp"),
    "act_scale_off_by_one": ("e = np.where(m <= 0.875, E - 9, E - 8)", "e = np.where(m <= 0.875, E - 8, E - 7)"),
    "act_scale_not_applied": ("h = round_bf16(glu_unit((qx @ Wg.T) * sx, (qx @ Wu.T) * sx,",
                              "h = round_bf16(glu_unit((qx @ Wg.T), (qx @ Wu.T),"),
    "down_input_not_quantised": ("return h, (qh @ Wd.T) * np.exp2(eh)[:, None]", "return h, h @ Wd.T"),
    "fp8_path_ignored": ("return expert_ffn_fp8 if fmt in (WEIGHTS_FP8, WEIGHTS_FP4) else expert_ffn",
                         "return expert_ffn"),
    "fp4_nibbles_swapped": ("return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8), np.asarray(s).astype(np.int8)",
                            "return (c[..., 1::2] | (c[..., 0::2] << 4)).astype(np.uint8), np.asarray(s).astype(np.int8)"),
    "fp4_sign_in_wrong_bit": ("return (idx | np.where(np.signbit(q), 8, 0)).astype(np.uint8)",
                              "return (idx | np.where(np.signbit(q), 4, 0)).astype(np.uint8)"),
    "histogram_off_by_one": ("return np.bincount(np.asarray(idx).ravel(), minlength=E).astype(np.int64)",
                             "return np.bincount(np.asarray(idx).ravel() % max(E - 1, 1), minlength=E).astype(np.int64)"),
}


def mutated_module(name):
    old, new = MUTATIONS[name]
    with open(SRC) as f:
        src = f.read()
    assert src.count(old) == 1, f"mutation {name}: anchor not found once in the oracle"
    mod = types.ModuleType(f"oracle_mutant_{name}")
    exec(compile(src.replace(old, new), f"<mutant {name}>", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name):
    M = mutated_module(name)
    caught = []
    for pin in P.ALL_PINS:
        try:
            with np.errstate(over="ignore", invalid="ignore", divide="ignore"):  # mutants may overflow
                pin(M)
        except Exception as e:  # AssertionError, or a shape error from a wrong operand
            caught.append((pin.__name__, type(e).__name__))
    assert caught, f"no pin caught the planted mistake {name}"
