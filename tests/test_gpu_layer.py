"""GPU parity: the CUDA layer through the C ABI against the fp64 oracle.

Inputs are the seeded synthetic workloads (both sides draw them from the same
counter-based generator).  Floating-point outputs must satisfy
max |gpu - oracle| / max(1, |oracle|) <= 2e-2 and a mean of the same <= 4e-3
on every token; xn may differ from the oracle's by one bf16 step on at most
1e-4 of its elements; integer stages (routing, histogram, permutation) must
match exactly except on tokens whose top-k margin is below 1e-5 in the
oracle's key space (near ties) or whose routing the oracle reproduces from the
GPU's own xn (rounding-boundary flips).  Tokens routed differently are
value-checked on the oracle with the GPU's indices forced.
"""
import dataclasses

import numpy as np
import pytest

import oracle as O
from gpu_util import Run, host_weights, np64, rel_err, verify
from synth import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


def _views_np(run, T, ws, torch):
    """Intermediates of the last forward, as tensors sliced out of its workspace."""
    v = run.layer.views(T, ws)
    c = run.cfg
    base = ws.data_ptr()

    def arr(ptr, shape, dtype):
        n = int(np.prod(shape))
        nbytes = n * torch.empty(0, dtype=dtype).element_size()
        off = ptr - base
        assert 0 <= off and off + nbytes <= ws.numel()
        return ws[off:off + nbytes].view(dtype).reshape(shape)

    out = dict(
        xn=arr(v.xn, (T, c.D), torch.bfloat16),
        counts=arr(v.counts, (c.E,), torch.int32),
        offsets=arr(v.offsets, (c.E + 1,), torch.int32),
        src_token=arr(v.src_token, (T * c.k,), torch.int32),
        dest_row=arr(v.dest_row, (T * c.k,), torch.int32),
        h_routed=arr(v.h_routed, (T * c.k, c.I), torch.bfloat16),
        y_slot=arr(v.y_slot, (T, c.k, c.D), torch.float32),
    )
    if v.logits:
        out["logits"] = arr(v.logits, (T, v.E_pad), torch.float32)[:, :c.E]
    if c.n_shared:
        out["y_shared"] = arr(v.y_shared, (c.n_shared, T, c.D), torch.float32)
    return out


def _stage_checks(run, out, ref, hw, torch):
    """Intermediate stages against the oracle's own intermediates (xn itself is
    checked by verify)."""
    c, T = run.cfg, run.T
    v = _views_np(run, T, out["ws"], torch)
    if "logits" in v:
        e = np.abs(np64(v["logits"]) - ref["logits"])
        assert e.max() < 5e-3 * (1 + np.abs(ref["logits"]).max()), e.max()
    same = np.all(out["idx"].cpu().numpy() == ref["idx"], axis=1)
    if np.all(same):
        assert np.array_equal(v["counts"].cpu().numpy(), ref["counts"])
        assert np.array_equal(v["offsets"].cpu().numpy(), ref["offsets"])
        assert np.array_equal(v["src_token"].cpu().numpy(), ref["perm_token"])
        assert np.array_equal(v["dest_row"].cpu().numpy(), ref["perm_token"] * c.k + ref["perm_slot"])
        # h of every grouped row, expert by expert.
        hg = np64(v["h_routed"])
        offs = ref["offsets"]
        for e in range(c.E):
            a, b = offs[e], offs[e + 1]
            if a == b:
                continue
            Wg, Wu, Wd = hw.routed(e)
            h, _ = O.expert_ffn(ref["xn"][ref["perm_token"][a:b]], Wg, Wu, Wd, c.gate_clamp_max, c.up_clamp)
            er = rel_err(hg[a:b], h)
            assert er.max() <= 2e-2, (e, er.max())
    yg = np64(v["y_slot"])
    er = rel_err(yg[same], ref["y_slots"][same])
    assert er.max() <= 2e-2 and er.mean() <= 4e-3, (er.max(), er.mean())
    if c.n_shared:
        er = rel_err(np64(v["y_shared"]), ref["y_shared"])
        assert er.max() <= 2e-2 and er.mean() <= 4e-3, (er.max(), er.mean())


def test_tiny_layer_parity_with_stages(torch_cuda):
    cfg = W.C1
    run = Run(cfg)
    out = run.forward(*run.inputs())
    hw = host_weights(cfg)
    ref, same, _ = verify(run, out, hw=hw)
    _stage_checks(run, out, ref, hw, torch_cuda)


def test_fine_grained_layer_parity(torch_cuda):
    cfg = W.C2
    run = Run(cfg)
    out = run.forward(*run.inputs())
    hw = host_weights(cfg)
    ref, same, rep = verify(run, out, hw=hw)
    w = out["w"].cpu().numpy().astype(np.float64)
    assert np.allclose(w.sum(1), 1.0, atol=1e-5)  # renormalised
    _stage_checks(run, out, ref, hw, torch_cuda)


@pytest.mark.parametrize("T", [1, 5, 127, 129, 1000])
def test_ragged_and_tiny_batches(torch_cuda, T):
    cfg = dataclasses.replace(W.C1, T=T)
    run = Run(cfg)
    verify(run, run.forward(*run.inputs()))


@pytest.mark.parametrize("variant", ["all_experts", "no_shared", "hash_small", "sigmoid_clamp", "k1",
                                     "situ_caps", "situ_tight_caps"])
def test_layer_variants(torch_cuda, variant):
    base = dataclasses.replace(W.C1, T=300)
    cfg = {
        "all_experts": dataclasses.replace(base, k=8, renormalize=1),
        "no_shared": dataclasses.replace(base, n_shared=0),
        "hash_small": dataclasses.replace(base, router=W.ROUTER_HASH, E=8, k=3, name="hash_small"),
        "sigmoid_clamp": dataclasses.replace(base, router=W.ROUTER_SIGMOID_BIAS, renormalize=1,
                                             routed_scale=2.5, gate_clamp_max=0.05, up_clamp=0.05,
                                             bias="normal", bias_sigma=0.01),
        "k1": dataclasses.replace(base, k=1, E=16, n_shared=2, I=192, I_shared=64),
        # SiTU-GLU experts.  Weights N(0, 0.15) drive the gate past its cap of 4
        # on about 1 element in 10 while the layer's outputs stay near the scale
        # the tolerance is stated for (at N(0, 0.5) outputs in the hundreds
        # cancel, and a one-ulp flip of a bf16 h moves them past it); tight
        # caps saturate both branches on the default weights.
        "situ_caps": dataclasses.replace(base, activation=1, weight_sigma=0.15, name="situ_caps"),
        "situ_tight_caps": dataclasses.replace(base, activation=1, situ_beta_gate=0.25,
                                               situ_beta_up=0.5, name="situ_tight"),
    }[variant]
    run = Run(cfg)
    verify(run, run.forward(*run.inputs()))


def test_fine_grained_situ_parity(torch_cuda):
    """SiTU-GLU experts on the fine-grained shapes (a 512-token batch)."""
    cfg = dataclasses.replace(W.C2S, T=512)
    run = Run(cfg)
    verify(run, run.forward(*run.inputs()))


def _latent_parity(run, cfg, torch):
    """Latent layers: z = bf16(xn W_down^T) is rounded from fp32 on the GPU and
    from fp64 in the oracle (verify allows single bf16 steps on under 1 % of
    z); routing differences are classified on the GPU's own z, and every token
    is value-checked."""
    out = run.forward(*run.inputs())
    ref, same, rep = verify(run, out)
    return out, ref


def test_latent_tiny_parity(torch_cuda):
    cfg = dataclasses.replace(W.C1, T=300, latent=64, name="tiny_latent")
    run = Run(cfg)
    _latent_parity(run, cfg, torch_cuda)


def test_latent_situ_parity(torch_cuda):
    """The K3-style latent workload (l = 512, 256 experts top-16, SiTU-GLU, a
    full-width shared expert) at T=512."""
    cfg = dataclasses.replace(W.C6, T=512)
    run = Run(cfg)
    _latent_parity(run, cfg, torch_cuda)


def test_empty_batch_launches_nothing(torch_cuda):
    import deterministic_expert_b200 as moe
    run = Run(W.C1)
    torch = torch_cuda
    x = torch.empty((0, W.C1.D), dtype=torch.bfloat16, device="cuda")
    on = torch.empty_like(x)
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    run.layer.forward(x, x, on, on, ws)
    assert run.layer.launch_count(0) == 0
    with pytest.raises(moe.MoEError) as e:
        x2 = torch.empty((W.C1.T + 1, W.C1.D), dtype=torch.bfloat16, device="cuda")
        run.layer.forward(x2, x2, x2, x2, ws)
    assert e.value.status == moe.MOE_ETOOBIG
    with pytest.raises(moe.MoEError) as e:
        x3 = torch.empty((8, W.C1.D), dtype=torch.bfloat16, device="cuda")
        run.layer.forward(x3, x3, x3, x3, ws)
    assert e.value.status == moe.MOE_EWORKSPACE


def test_device_wait_timeout_is_reported(torch_cuda):
    import deterministic_expert_b200 as moe
    assert moe.selftest_wait_timeout(2000) == moe.MOE_ETIMEOUT
    # The context is still usable afterwards.
    run = Run(dataclasses.replace(W.C1, T=8))
    out = run.forward(*run.inputs())
    assert out["out_norm"].isfinite().all()
