"""GPU parity of FP4 expert weights with E4M3 x E4M3 expert GEMMs (the
DeepSeek V4 infra notes, §6.2 FP4 QAT) against the oracle.

Integer work is compared bit for bit: the FP4 quantiser's E4M3 codes and block
exponents, and the E4M3 codes and row exponents of the expert inputs (each
decision divides by a power of two and rounds to nearest even, exact on both
sides).  Floating-point stages and outputs use the layer tolerances
(max |gpu - oracle| / max(1, |oracle|) <= 2e-2, mean <= 4e-3).  The GPU sums
E4M3 products in fp32 on the tensor cores and the oracle sums them exactly, so
h may differ by one bf16 step, and then its E4M3 code by one step; the down
GEMM's output is therefore compared on the oracle's own chain.
"""
import dataclasses

import numpy as np
import pytest

import oracle as O
from gpu_util import Run, check_xn, host_weights, np64, rel_err, verify
from synth import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


def _edge_weights(torch):
    """bf16 master weights [rows, 128] mixing Gaussian blocks with the edge
    cases of the quantiser: exact E2M1 midpoints (ties), zeros and negative
    zeros, blocks far below and far above the lossless scale range, bf16
    subnormals, and values just beside the rounding thresholds."""
    g = torch.Generator().manual_seed(17)
    w = torch.randn((64, 128), generator=g) * 0.02
    mids = torch.tensor([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0])
    for r, s in enumerate(range(-8, 7)):
        blk = torch.zeros(32)
        blk[:8] = mids * 2.0 ** s
        blk[8:16] = -mids * 2.0 ** s
        blk[16] = 6.0 * 2.0 ** s     # fixes the block's scale at s
        w[r, :32] = blk
    w[20, 32:64] = 0.0
    w[21, 32:64] = -0.0
    w[22, 32:64] = torch.randn(32, generator=g) * 1e-6    # wants s far below -8
    w[23, 32:64] = torch.randn(32, generator=g) * 1e4     # wants s far above 6
    w[24, 32:64] = torch.tensor(2.0 ** -130) * torch.arange(32)   # bf16 subnormals
    eps = 2.0 ** -9
    w[25, 64:96] = torch.cat([(mids + eps)[:8], (mids - eps)[:8], torch.zeros(15), torch.tensor([6.0])])
    return w.to(torch.bfloat16)


def test_fp4_quantiser_bit_exact(torch_cuda):
    torch = torch_cuda
    import deterministic_expert_b200 as moe
    wh = _edge_weights(torch)
    w = wh.cuda()
    q = torch.empty(w.shape, dtype=torch.uint8, device="cuda")
    s = torch.empty((w.shape[0], w.shape[1] // 32), dtype=torch.int8, device="cuda")
    moe.quantize_weights_fp4(w, q, s)
    torch.cuda.synchronize()
    master = wh.to(torch.float64).numpy()
    oq, os_ = O.quantize_weights_fp4(master)
    want = O.e4m3_bits(O.dequantize_fp4(oq, os_))
    assert np.array_equal(s.cpu().numpy().astype(np.int64), os_)
    got = q.cpu().numpy()
    bad = np.nonzero(got != want)
    assert got.shape == want.shape and bad[0].size == 0, (bad[0][:5], bad[1][:5], got[bad][:5], want[bad][:5])


def test_fp4_quantiser_workload_weights(torch_cuda):
    """The fine-grained workload's first experts, quantised on the GPU, equal
    the oracle's FP4 quantisation of the same master weights code for code."""
    torch = torch_cuda
    import deterministic_expert_b200 as moe
    from synth import device as SD
    cfg = W.C2F
    hw = SD.HostWeights(cfg)
    w = SD.device_weights(cfg)
    q = moe.quantize_expert_weights(w)
    torch.cuda.synchronize()
    for e in (0, 1, cfg.E - 1):
        Wg, Wu, Wd = hw.routed(e)
        for name, mw in (("w_gate", Wg), ("w_up", Wu), ("w_down", Wd)):
            got = q[name].view(cfg.E, *mw.shape)[e].cpu().numpy()
            assert np.array_equal(got, O.e4m3_bits(O.fp4_weights_as_fp8(mw))), (e, name)
    Wg, _, Wd = hw.shared(0)
    assert np.array_equal(q["ws_gate"].view(cfg.n_shared, *Wg.shape)[0].cpu().numpy(),
                          O.e4m3_bits(O.fp4_weights_as_fp8(Wg)))
    assert np.array_equal(q["ws_down"].view(cfg.n_shared, *Wd.shape)[0].cpu().numpy(),
                          O.e4m3_bits(O.fp4_weights_as_fp8(Wd)))


def _ws(ws, ptr, nbytes, torch, dtype):
    off = ptr - ws.data_ptr()
    assert 0 <= off and off + nbytes <= ws.numel()
    return ws[off:off + nbytes].view(dtype)


def _fp8_stage_checks(run, out, ref, hw, torch):
    c, T = run.cfg, run.T
    ws = out["ws"]
    v = run.layer.views(T, ws)
    TK = T * c.k
    xn = np64(_ws(ws, v.xn, T * c.D * 2, torch, torch.bfloat16).reshape(T, c.D))
    check_xn(xn, ref["xn"])   # the quantisation below reads the GPU's own xn
    # E4M3 copy of xn: codes and row exponents exactly the oracle's quantisation.
    xq = _ws(ws, v.xq, T * c.D, torch, torch.uint8).reshape(T, c.D).cpu().numpy()
    xe = _ws(ws, v.xq_exp, T, torch, torch.int8).cpu().numpy().astype(np.int64)
    oq, oe = O.quantize_act_rows(xn)
    assert np.array_equal(xe, oe)
    assert np.array_equal(xq, O.e4m3_bits(oq))
    # h of the routed rows: from the GPU's codes through the oracle's FP8 expert
    # (fp64 sums of the same E4M3 products), within the layer tolerance.
    h = np64(_ws(ws, v.h_routed, TK * c.I * 2, torch, torch.bfloat16).reshape(TK, c.I))
    offs = _ws(ws, v.offsets, (c.E + 1) * 4, torch, torch.int32).cpu().numpy()
    src = _ws(ws, v.src_token, TK * 4, torch, torch.int32).cpu().numpy()
    for e in range(c.E):
        a, b = offs[e], offs[e + 1]
        if a == b:
            continue
        Wg, Wu, Wd = hw.routed(e)
        ho, _ = O.expert_ffn_fp8(xn[src[a:b]], Wg, Wu, Wd, **O.unit_args(c))
        er = rel_err(h[a:b], ho)
        assert er.max() <= 2e-2, (e, er.max())
    # E4M3 copy of h: exactly the quantisation of the GPU's own h.
    hq = _ws(ws, v.hq_routed, TK * c.I, torch, torch.uint8).reshape(TK, c.I).cpu().numpy()
    he = _ws(ws, v.hq_routed_exp, TK, torch, torch.int8).cpu().numpy().astype(np.int64)
    oq, oe = O.quantize_act_rows(h)
    assert np.array_equal(he, oe)
    assert np.array_equal(hq, O.e4m3_bits(oq))
    if c.n_shared:
        S, Is = c.n_shared, c.I_shared
        hs = np64(_ws(ws, v.h_shared, S * T * Is * 2, torch, torch.bfloat16).reshape(S * T, Is))
        hsq = _ws(ws, v.hq_shared, S * T * Is, torch, torch.uint8).reshape(S * T, Is).cpu().numpy()
        hse = _ws(ws, v.hq_shared_exp, S * T, torch, torch.int8).cpu().numpy().astype(np.int64)
        oq, oe = O.quantize_act_rows(hs)
        assert np.array_equal(hse, oe)
        assert np.array_equal(hsq, O.e4m3_bits(oq))
    # y of each slot: the GPU's h codes through the oracle's down product.
    y = np64(_ws(ws, v.y_slot, TK * c.D * 4, torch, torch.float32).reshape(T, c.k, c.D))
    dest = _ws(ws, v.dest_row, TK * 4, torch, torch.int32).cpu().numpy()
    worst = 0.0
    for e in range(c.E):
        a, b = offs[e], offs[e + 1]
        if a == b:
            continue
        _, _, Wd = hw.routed(e)
        qv = O.quantize_act_rows(h[a:b])
        yo = (qv[0] @ Wd.T) * np.exp2(qv[1])[:, None]
        yg = y.reshape(TK, c.D)[dest[a:b]]
        er = rel_err(yg, yo)
        worst = max(worst, float(er.max()))
    # The same E4M3 products, summed in fp32 by the tensor cores and exactly by
    # the oracle: the difference is the accumulation's rounding alone.
    print(f"down GEMM on identical E4M3 inputs: max rel err {worst:.2e}")
    assert worst <= 2e-3, worst


def test_fp8_tiny_parity_with_stages(torch_cuda):
    cfg = W.C1F
    run = Run(cfg)
    out = run.forward(*run.inputs())
    hw = host_weights(cfg)
    ref, _, _ = verify(run, out, hw=hw)
    _fp8_stage_checks(run, out, ref, hw, torch_cuda)


@pytest.mark.parametrize("T", [1, 17, 129, 1000])
def test_fp8_ragged_batches(torch_cuda, T):
    cfg = dataclasses.replace(W.C1F, T=T)
    run = Run(cfg)
    out = run.forward(*run.inputs())
    hw = host_weights(cfg)
    ref, _, _ = verify(run, out, hw=hw)
    _fp8_stage_checks(run, out, ref, hw, torch_cuda)


@pytest.mark.parametrize("T", [512, 4096])
def test_fp8_fine_grained_parity(torch_cuda, T):
    """Fine-grained shapes: at T = 512 every expert tile is operand-swapped, at
    T = 4096 most groups also run full 256-row pair tiles."""
    cfg = dataclasses.replace(W.C2F, T=T)
    run = Run(cfg)
    out = run.forward(*run.inputs())
    hw = host_weights(cfg)
    ref, _, _ = verify(run, out, hw=hw)
    _fp8_stage_checks(run, out, ref, hw, torch_cuda)


def test_fp8_situ_parity(torch_cuda):
    """SiTU-GLU experts with FP4 weights (both variants of the gate/up kernel)."""
    cfg = dataclasses.replace(W.C1F, T=300, activation=1, name="tiny_fp8_situ")
    run = Run(cfg)
    out = run.forward(*run.inputs())
    hw = host_weights(cfg)
    ref, _, _ = verify(run, out, hw=hw)
    _fp8_stage_checks(run, out, ref, hw, torch_cuda)


def test_fp8_latent_situ_parity(torch_cuda):
    """FP4 expert weights with a latent width (the routed experts read z as E4M3
    rows, the shared expert xn) and SiTU-GLU units, on a 512-token batch."""
    from test_gpu_layer import _latent_parity
    cfg = dataclasses.replace(W.C6F, T=512)
    run = Run(cfg)
    _latent_parity(run, cfg, torch_cuda)


@pytest.mark.parametrize("variant", ["hash", "sigmoid_clamp", "no_shared"])
def test_fp8_layer_variants(torch_cuda, variant):
    """E4M3 experts under the other router variants: hash routing, sigmoid
    scores with a selection bias and tight SwiGLU clamps, no shared expert.
    (A V3-shaped case is left out: the oracle's FP4 quantisation of its
    7168 x 2048 expert matrices in fp64 takes tens of minutes.)"""
    base = dataclasses.replace(W.C1F, T=300)
    cfg = {
        "hash": dataclasses.replace(base, router=W.ROUTER_HASH, k=3, name="tiny_fp8_hash"),
        "sigmoid_clamp": dataclasses.replace(base, router=W.ROUTER_SIGMOID_BIAS, renormalize=1, routed_scale=2.5,
                                             gate_clamp_max=0.05, up_clamp=0.05, bias="normal", bias_sigma=0.01,
                                             name="tiny_fp8_sigmoid"),
        "no_shared": dataclasses.replace(base, n_shared=0, name="tiny_fp8_noshared"),
    }[variant]
    run = Run(cfg)
    out = run.forward(*run.inputs())
    hw = host_weights(cfg)
    ref, _, _ = verify(run, out, hw=hw)
    _fp8_stage_checks(run, out, ref, hw, torch_cuda)
