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


def test_order_change_is_visible(torch_cuda):
    """A case where the two orders differ after bf16 rounding, derived by hand
    in fp32 (P = 8, residual 0, every element r0 = 1, r1 = -1, r2 = 2^-25,
    r3..r7 = 0; the ring cuts D into 8 chunks):
      fixed, every element: (1 - 1) + 2^-25 = 2^-25.
      ring chunk 0: 1 + 0 .. + 2^-25 -> 1 (2^-25 < half an ulp of 1), - 1 = 0.
      ring chunk 1: (-1 + 1) + 0 .. + 2^-25 = 2^-25.
      ring chunks 2..7: 2^-25 - 1 is a tie between -1 and -(1 - 2^-24) and
      rounds to the even -1; + 1 = 0.
    The kernel must give 2^-25 everywhere: the fixed order, not the ring's."""
    torch = torch_cuda
    T, D = 4, 256
    vals = [1.0, -1.0, 2.0 ** -25, 0, 0, 0, 0, 0]
    parts = [torch.full((T, D), v, dtype=torch.bfloat16) for v in vals]
    res = torch.zeros((T, D), dtype=torch.bfloat16)
    g = torch.ones(D, dtype=torch.bfloat16)
    on, orr = _run(torch, [p.cuda() for p in parts], res.cuda(), g.cuda())
    got = np64(orr)
    assert np.all(got == 2.0 ** -25)
    pf = np.stack([p.float().numpy() for p in parts])
    assert np.array_equal(O.allreduce_fixed_order_f32(pf), np.full((T, D), 2.0 ** -25, np.float32))
    ring = O.allreduce_ring_order_f32(pf)
    c = D // 8
    assert np.all(ring[:, :c] == 0) and np.all(ring[:, c:2 * c] == 2.0 ** -25) and np.all(ring[:, 2 * c:] == 0)
    assert not np.array_equal(O.round_bf16(ring.astype(np.float64)), got)



def test_row_slices_to_several_destinations(torch_cuda):
    """moe_reduce_partials_rows over three row slices, each written to two
    destination pairs: both destinations must equal moe_reduce_partials over
    all rows bit for bit (the form the tensor-parallel epilogue launches on
    each rank)."""
    import deterministic_expert_b200 as moe
    torch = torch_cuda
    P, T, D = 8, 301, 2048
    gen = torch.Generator().manual_seed(77)
    parts = [(torch.randn((T, D), generator=gen) / 8).to(torch.bfloat16).cuda() for _ in range(P)]
    res = torch.randn((T, D), generator=gen).to(torch.bfloat16).cuda()
    g = (1 + 0.1 * torch.randn(D, generator=gen)).to(torch.bfloat16).cuda()
    on, orr = _run(torch, parts, res, g)
    outs = [(torch.zeros_like(res), torch.zeros_like(res)) for _ in range(2)]
    for row0, rows in moe.row_slices(T, 3):
        moe.reduce_partials_rows(parts, res, g, [o[0] for o in outs], [o[1] for o in outs], row0, rows)
    torch.cuda.synchronize()
    for n_, r_ in outs:
        assert torch.equal(n_.view(torch.int16), on.view(torch.int16))
        assert torch.equal(r_.view(torch.int16), orr.view(torch.int16))


def _tp_world1(q):
    import os
    import torch
    import torch.distributed as dist
    import deterministic_expert_b200 as moe
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(q.get()))
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        P, T, D = 8, 129, 1024
        tp = moe.TPAllReduceNorm(T, D, per_rank=P, device="cuda")
        gen = torch.Generator().manual_seed(5)
        parts = [(torch.randn((T, D), generator=gen) / 8).to(torch.bfloat16).cuda() for _ in range(P)]
        for j in range(P):
            tp.partial[j].copy_(parts[j])
        res = torch.randn((T, D), generator=gen).to(torch.bfloat16).cuda()
        g = torch.ones(D, dtype=torch.bfloat16, device="cuda")
        on, orr = tp(res, g)
        ref_n, ref_r = torch.empty_like(res), torch.empty_like(res)
        moe.reduce_partials(parts, res, g, ref_n, ref_r)
        torch.cuda.synchronize()
        ok = bool(torch.equal(on.view(torch.int16), ref_n.view(torch.int16)) and
                  torch.equal(orr.view(torch.int16), ref_r.view(torch.int16)))
        # A second step over new partials: the barriers' epochs advance.
        for j in range(P):
            parts[j] = (torch.randn((T, D), generator=gen) / 8).to(torch.bfloat16).cuda()
            tp.partial[j].copy_(parts[j])
        on, orr = tp(res, g)
        moe.reduce_partials(parts, res, g, ref_n, ref_r)
        torch.cuda.synchronize()
        tp.check()
        ok = ok and bool(torch.equal(on.view(torch.int16), ref_n.view(torch.int16)) and
                         torch.equal(orr.view(torch.int16), ref_r.view(torch.int16)))
        tp.close()
        q.put(ok)
    finally:
        dist.destroy_process_group()


def test_tp_epilogue_one_rank(torch_cuda):
    """TPAllReduceNorm on one rank (exported peer allocation, device-side
    barriers, the row-slice kernel) equals moe_reduce_partials bit for bit,
    over two steps."""
    import socket
    import torch.multiprocessing as mp
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    q.put(port)
    p = ctx.Process(target=_tp_world1, args=(q,))
    p.start()
    p.join(timeout=300)
    assert p.exitcode == 0
    assert q.get(timeout=5) is True


def test_peer_barrier_times_out(torch_cuda):
    """A two-rank barrier on one GPU whose second rank never signals (both flag
    arrays are this process's memory and nothing writes slot 1): the wait gives
    up after its limit, records the timeout in the error word, and the context
    keeps working."""
    import time

    import deterministic_expert_b200 as moe
    torch = torch_cuda
    flags = torch.zeros((2, 64), dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    moe.peer_barrier([flags[0].data_ptr(), flags[1].data_ptr()], 0, 1, err, 200000)
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert int(err.item()) == 1
    assert 0.15 < dt < 30.0
    # Rank 0 signalled both arrays in slot 0 and saw its own signal.
    assert int(flags[0, 0].item()) == 1 and int(flags[1, 0].item()) == 1 and int(flags[0, 1].item()) == 0
    # The context is usable: a one-rank barrier passes and leaves no error.
    err.zero_()
    own = torch.zeros(64, dtype=torch.int32, device="cuda")
    moe.peer_barrier([own.data_ptr()], 0, 1, err, 200000)
    torch.cuda.synchronize()
    assert int(err.item()) == 0 and int(own[0].item()) == 1
