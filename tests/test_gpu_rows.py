"""GPU parity of the fixed-order partial reduction + residual + RMSNorm.

The fixed r0 + r1 + ... + r7 order of the Fireworks parity post (Trap 1) is
emulated in fp32 by the oracle, so out_residual = bf16(r) must match bit for
bit; out_norm follows the tolerance of the layer.  A ring-order emulation
(the NCCL reduce-scatter order of the same passage) must differ in bits
somewhere, which shows the test can see an order change.
"""
import numpy as np
import pytest

import oracle as O
from gpu_util import TOL_MAX, TOL_MEAN, np64, rel_err
from synth import device as SD
from synth import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


def _run(torch, parts, res, g, eps=1e-6):
    import deterministic_expert_b200 as moe
    on = torch.empty_like(res)
    orr = torch.empty_like(res)
    moe.reduce_partials(parts, res, g, on, orr, eps=eps)
    torch.cuda.synchronize()
    return on, orr


@pytest.mark.parametrize("P,T,D", [(8, 37, 256), (8, 300, 4096), (1, 5, 64), (3, 129, 7168), (8, 1, 16384)])
def test_fixed_order_bit_exact(torch_cuda, P, T, D):
    torch = torch_cuda
    gen = torch.Generator().manual_seed(P * 1000 + T)
    parts = [(torch.randn((T, D), generator=gen) / 8).to(torch.bfloat16) for _ in range(P)]
    res = torch.randn((T, D), generator=gen).to(torch.bfloat16)
    g = (1 + 0.1 * torch.randn(D, generator=gen)).to(torch.bfloat16)
    on, orr = _run(torch, [p.cuda() for p in parts], res.cuda(), g.cuda())
    pf = np.stack([p.float().numpy() for p in parts])
    want_n, want_r, r32 = O.reduce_partials(pf, res.float().numpy(), g.float().numpy().astype(np.float64), 1e-6)
    assert np.array_equal(np64(orr), want_r)
    e = rel_err(np64(on), want_n)
    assert e.max() <= TOL_MAX and e.mean() <= TOL_MEAN
    if P == 8 and T * D >= 8 * 8192:
        ring = O.allreduce_ring_order_f32(pf) + res.float().numpy()
        ring_bf = O.round_bf16(ring.astype(np.float64))
        assert not np.array_equal(ring_bf, want_r)


def test_epilogue_full_size_sampled_rows(torch_cuda):
    """The skewed workload's epilogue: 8 buffers of [16384, 4096] N(0,1)/8,
    run in full on the GPU, checked on sampled rows regenerated on the host."""
    torch = torch_cuda
    parts = SD.device_partials()
    cfg = W.C5
    res = SD.device_bf16(cfg, "residual", T=W.EPILOGUE_T)
    g = SD.device_bf16(cfg, "g_out")
    on, orr = _run(torch, parts, res, g)
    rows = np.array([0, 1, 4095, 8191, 12345, 16383])
    D = W.EPILOGUE_D
    pf = np.stack([np.stack([SD.f64(W.host_partial(p, start=int(t) * D, count=D)) for t in rows])
                   for p in range(W.EPILOGUE_P)]).astype(np.float32)
    rr = SD.host_rows(cfg, "residual", rows, T=W.EPILOGUE_T)
    want_n, want_r, _ = O.reduce_partials(pf, rr.astype(np.float32), np.ones(D), cfg.eps)
    assert np.array_equal(np64(orr)[rows], want_r)
    e = rel_err(np64(on)[rows], want_n)
    assert e.max() <= TOL_MAX and e.mean() <= TOL_MEAN
